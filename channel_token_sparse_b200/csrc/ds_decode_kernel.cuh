// ds_decode_kernel.cuh -- fused Double Sparsity decode step for sm_100a.
//
// One thread-block cluster of N CTAs handles one (batch b, kv head g) row.
// CTA `rank` owns the contiguous token range [rank*chunk, rank*chunk + chunk).
// The steps of "大模型稀疏化技术原理：Double Sparsity" (joto.ai), section
// 在线前向计算, run back to back without leaving the chip:
//
//   step 1  qL[j] = sum over the group's query heads of q[h, idx[g, j]]
//   step 2  stream the label-cache rows of the chunk (128-bit loads), score
//           every token in fp32, keep the upper 16 bits of its order-preserving
//           key in shared memory and histogram their top byte
//   step 3a exact top-k on the fp32 scores by radix selection across the
//           cluster: two 8-bit passes over the 16-bit keys (histograms summed
//           through distributed shared memory); if the k-th key's 16-bit
//           bucket is only partly selected, the bucket's tokens are re-scored
//           (same arithmetic, bit-identical) and two more passes resolve the
//           low 16 bits; exact ties go to the lower token index
//   compaction: the selected tokens, in ascending order, are dealt out evenly
//           to the cluster's CTAs (DSMEM stores into each CTA's list)
//   step 3b exact attention over the full K/V rows of the selected tokens,
//           online softmax per warp, then merged per CTA, then across the
//           cluster through DSMEM; each CTA writes a slice of the output.
//
// Nothing is written to global memory except the output (and the optional
// score / selection debug outputs).
#pragma once

#include <cooperative_groups.h>

#include "ds_common.cuh"

namespace ds {
namespace cg = cooperative_groups;

constexpr int kNT = 256;             // threads per CTA
constexpr int kNW = kNT / 32;        // warps per CTA
constexpr int kMaxChunk = 32768;     // tokens per CTA (16-bit keys -> 64 KiB)
constexpr int kLabelInt4 = 1;
constexpr int kLabelFp = 0;

struct DecodeParams {
    const void* q;
    const void* k;
    const void* v;
    const void* label;
    const uint16_t* lscale;
    const uint16_t* lzero;
    const int32_t* idx;
    const int32_t* seq_lens;  // [nb] tokens per batch entry, or null (all rows have s)
    void* out;
    int32_t* sel_out;
    float* score_out;
    int hkv, G, s, s_cap, topk;  // s: tokens per row (the maximum when seq_lens is given)
    int chunk;     // tokens per CTA, multiple of 32
    int lay_chunk; // chunk used to size shared memory (0 in dense mode)
    int per;       // selected tokens attended per CTA (ceil(min(topk,s) / N))
    int append;    // 1: first build the label row of token s-1 from the key cache (decode step)
    int att_stages; // attention ring stages per warp (bf16: 2 or 3; fp32: kAttStagesF32)
    int lab_ring;  // 1: fp label rows stream through a shared-memory ring behind the keys
    int keep_low;  // 1: the low 16 key bits are kept in shared memory too (no re-scoring)
    float qscale;  // sm_scale * log2(e)
    int out_bf16;
    int dense;     // 1: attend every token, no label / scores / selection
    // with seq_lens: entries shorter than `threshold` attend all their tokens;
    // batch_rule = 1 applies the rule to the whole batch instead (every entry
    // attends all its tokens when the longest is shorter than `threshold` or
    // the shortest is shorter than topk)
    int nb, threshold, batch_rule;
    // paged K/V (null block_table: K/V are [b, hkv, s_cap, d]): K/V pools are
    // [num_blocks, hkv, 1 << page_shift, d] and token t of batch entry b is
    // row t & (page - 1) of block block_table[b * max_blocks + (t >> page_shift)]
    const int32_t* block_table;
    int max_blocks, page_shift, num_blocks;
    // decode step with the new token's rows given ([b, hkv, d] each, or null):
    // the kernel writes them into the K/V caches at position s-1 itself
    const void* k_new;
    const void* v_new;
    // label rounds pulled into L2 ahead of the register-path scan (0: none)
    int scan_prefetch;
    // byte offset in the region of the selection scratch (bucket flags, mask
    // cache, bucket list): behind the 16-bit keys and kept low bits, over the
    // label ring, which is dead by the time the selection starts
    int sel_off;
};

// Row (in units of d elements) of token t of (b, g) in the K/V caches, dense
// or paged; block ids are clamped into the pool.
template <bool PAGED>
__device__ __forceinline__ size_t kv_row_of(const DecodeParams& p, int b, int g, size_t row_tok, int t) {
    if constexpr (!PAGED) return row_tok + (size_t)t;
    int blk = __ldg(p.block_table + (size_t)b * p.max_blocks + (t >> p.page_shift));
    blk = min(max(blk, 0), p.num_blocks - 1);
    return (((size_t)blk * p.hkv + g) << p.page_shift) + (size_t)(t & ((1 << p.page_shift) - 1));
}

// Shared-memory carve-up (bytes), identical on host and device.
struct DecodeSmem {
    int qs, qa, qL, ql4, idx, histA, histB, ctl, scan, cm, cl, co, krow, app, sel, region, total;
};

__host__ __device__ inline int align16(int x) { return (x + 15) & ~15; }

// Selection scratch in the region (see DecodeParams::sel_off): bucket flags
// (a byte per 8 tokens), the per-group selected / tie mask cache (2 bytes per
// 8 tokens) and the bucket list (kBucketCap words).
__host__ __device__ inline int sel_scratch_bytes(int chunk);

// Attention-phase staging: each warp owns a ring of shared-memory stages; a
// stage holds the K rows then the V rows of att_stage_tokens() tokens. With
// bf16 K/V a stage is 8 tokens (one 8-token tensor-core tile; 2 or 3 stages,
// chosen by the host from the shared-memory budget); with fp32 K/V, ~1 KiB
// of rows per stage and kAttStagesF32 stages. A warp's partial softmax state
// (at most 8 * (128 + 2) floats) is later written into its own ring.
constexpr int kAttStagesF32 = 4;
// Label-streaming ring (fp labels): stages of one row per thread.
// Stages of the label ring: 8 for fp rows; 6 for 4-bit rows, whose ring
// then fits beside the kept low key bits on the 32-channel layer (12 stages
// were measured no faster than 8, 6 slightly faster).
__host__ __device__ constexpr int lab_stages(bool int4) { return int4 ? 6 : 8; }
// ring bytes for label rows of `label_row_bytes` (a 4-bit row adds its fp16
// scale and zero, 4 bytes, kept in two arrays of the stage)
__host__ __device__ constexpr int lab_ring_bytes(int label_row_bytes, bool int4) {
    return lab_stages(int4) * 256 * label_row_bytes;
}
__host__ __device__ constexpr int att_stage_tokens(int row_bytes, int elem_bytes) {
    return elem_bytes == 2 ? 8 : (row_bytes >= 1024 ? 1 : 1024 / row_bytes);
}
__host__ __device__ constexpr int att_ring_bytes(int row_bytes, int elem_bytes, int stages) {
    return stages * att_stage_tokens(row_bytes, elem_bytes) * 2 * row_bytes;
}
// Tokens of the k-th key's 16-bit bucket kept in a list for the last radix
// pass (a CTA whose bucket is larger falls back to sweeping its keys).
constexpr int kBucketCap = 1024;
constexpr int kMaxCluster = 16;  // CTAs per row at most (portable 8, non-portable 16)
__host__ __device__ inline int sel_scratch_bytes(int chunk) {
    return align16(chunk / 8) + align16(chunk / 8 * 2) + kBucketCap * 4;
}

// region_min: room the selection phase wants for the label ring and the
// low key bits beyond the keys and the attention ring (host plans only).
__host__ __device__ inline DecodeSmem decode_smem_layout(int GT, int D, int C, int chunk, int per,
                                                         int elem_bytes, int att_stages, int region_min = 0) {
    DecodeSmem L;
    int o = 0;
    L.qs = o;     o += align16(GT * D * 4);
    L.qa = o;     o += elem_bytes == 2 ? (D / 16) * 32 * 8 : 0;  // packed bf16 Q fragments
    L.qL = o;     o += align16(C * 4);
    L.ql4 = o;    o += align16(C * 3 + 4);                  // 4-bit scoring: qL as byte limbs, 2^-E
    L.idx = o;    o += align16(C * 4);
    L.histA = o;  o += 256 * 4;
    L.histB = o;  o += 256 * 4;
    L.ctl = o;    o += 64 * 4;
    L.scan = o;   o += align16((kNW + 1) * 4);
    L.cm = o;     o += align16(kMaxCluster * GT * 4);        // cluster merge: (m, l) of every CTA
    L.cl = o;     o += align16(kMaxCluster * GT * 4);
    L.co = o;     o += align16((GT * D + kMaxCluster) * 4);  // cluster merge: partial o received
    L.krow = o;   o += align16(D * elem_bytes);            // the appended token's key row
    L.app = o;    o += align16(C * 4) + 16;  // appended token's label row (+ fp16 scale, zero)
    L.sel = o;    o += align16(per * 4);
    L.region = o;
    const int keys = chunk * 2;
    const int ring = kNW * att_ring_bytes(D * elem_bytes, elem_bytes, att_stages);
    int region = keys > ring ? keys : ring;
    if (region_min > region) region = region_min;
    o += align16(region);
    L.total = o;
    return L;
}

// ctl[] slots
enum { kCtlBin = 0, kCtlNeed = 1, kCtlCnt = 2, kCtlCS = 4, kCtlCT = 5, kCtlP = 6, kCtlTP = 7, kCtlBL = 8,
       kCtlTlo = 9, kCtlTie = 10, kCtlWarp = 16 /* kNW per-warp packed counts */,
       kCtlGather = 32 /* 16 per-CTA bucket-list offsets, then the total */ };

// Row geometry of the label cache.
template <typename TKV, int LK, int C>
struct LabelGeom {
    static constexpr int kBytes = (LK == kLabelInt4) ? C / 2 : C * Elem<TKV>::kBytes;
    static constexpr int kWords = kBytes / 4;
    // tokens in flight per thread in the scoring loop (~128 B per thread)
    static constexpr int kU = (128 / kBytes) < 1 ? 1 : ((128 / kBytes) > 8 ? 8 : (128 / kBytes));
};

// 4-bit rows: the dot product sum_j qL[j] n_j in integer arithmetic. qL is
// held in fixed point, Q_j = rint(qL[j] * 2^E) with E chosen per row so that
// |Q_j| <= 2^21 (22 significant bits, as fine as the fp32 sum needs), split
// into bytes Q = q2 * 2^16 + q1 * 2^8 + q0 (q0, q1 unsigned, q2 signed). One
// 32-bit label word holds 8 channels: its low nibbles (channels 2j) and high
// nibbles (2j + 1) are two vectors of 4 bytes, so each limb costs two dp4a
// per word and every product is exact; the three limb sums meet in fp32.
// lim[(2k + h) * C/8 + i] holds limb k of channels 8i + 2b + h in byte b.
template <int C>
__device__ __forceinline__ float i4_dot(const uint32_t (&w)[C / 8], const uint32_t* lim, float s_e) {
    uint32_t s0 = 0u, s1 = 0u;
    int s2 = 0;
#pragma unroll
    for (int i = 0; i < C / 8; ++i) {
        const uint32_t lo = w[i] & 0x0F0F0F0Fu, hi = (w[i] >> 4) & 0x0F0F0F0Fu;
        s0 = __dp4a(lim[0 * (C / 8) + i], lo, s0);
        s0 = __dp4a(lim[1 * (C / 8) + i], hi, s0);
        s1 = __dp4a(lim[2 * (C / 8) + i], lo, s1);
        s1 = __dp4a(lim[3 * (C / 8) + i], hi, s1);
        s2 = __dp4a((int)lim[4 * (C / 8) + i], (int)lo, s2);
        s2 = __dp4a((int)lim[5 * (C / 8) + i], (int)hi, s2);
    }
    const float f = __fmaf_rn((float)s2, 65536.f, __fmaf_rn((float)s1, 256.f, (float)s0));
    return __fmul_rn(f, s_e);
}

// Byte limbs of qL for i4_dot (word `wi` of the 6 * C/8), and the scale 2^-E.
__device__ __forceinline__ float i4_scale_exp(float qmax, float* two_e) {
    int e = qmax > 0.f ? (int)((__float_as_uint(qmax) >> 23) & 255u) - 127 : 0;
    int E = 21 - e;
    E = E < -126 ? -126 : (E > 126 ? 126 : E);
    *two_e = __uint_as_float((uint32_t)(127 + E) << 23);
    return __uint_as_float((uint32_t)(127 - E) << 23);
}
template <int C>
__device__ __forceinline__ uint32_t i4_limb_word(const float* qL, float two_e, int wi) {
    const int k = wi / (2 * (C / 8)), h = (wi / (C / 8)) & 1, i = wi % (C / 8);
    uint32_t word = 0u;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        const int q = __float2int_rn(__fmul_rn(qL[8 * i + 2 * b + h], two_e));
        word |= ((uint32_t)(q >> (8 * k)) & 255u) << (8 * b);
    }
    return word;
}

// fp32 score of one token from its label row (step 2). The arithmetic is a
// fixed chain of fused multiply-adds in channel order, so scoring the same
// row twice gives bit-identical results.
// 4-bit rows use i4_dot with the limbs `lim` and scale `s_e` (the fp qL
// arguments are unused); fp rows use qreg (C <= 32) or qsm.
template <typename TKV, int LK, int C>
__device__ __forceinline__ float label_score(const uint32_t (&w)[LabelGeom<TKV, LK, C>::kWords],
                                             const float* qreg, const float* qsm, float sc, float z,
                                             float qsum, const uint32_t* lim, float s_e) {
    constexpr bool kReg = C <= 32;
    auto ql = [&](int j) -> float { return kReg ? qreg[j] : qsm[j]; };
    float acc = 0.f;
    if constexpr (LK == kLabelInt4) {
        // sum_j qL[j] * (sc * n_j + z) = sc * sum_j qL[j] n_j + z * sum_j qL[j]
        return __fmaf_rn(sc, i4_dot<C>(w, lim, s_e), __fmul_rn(z, qsum));
    } else if constexpr (Elem<TKV>::kBytes == 2) {
#pragma unroll
        for (int i = 0; i < C / 2; ++i) {
            acc = __fmaf_rn(ql(2 * i), bf16lo(w[i]), acc);
            acc = __fmaf_rn(ql(2 * i + 1), bf16hi(w[i]), acc);
        }
        return acc;
    } else {
#pragma unroll
        for (int i = 0; i < C; ++i) acc = __fmaf_rn(ql(i), __uint_as_float(w[i]), acc);
        return acc;
    }
}

// Barrier and shared-memory mapping across the CTAs of a row: a single-CTA
// cluster (N == 1, uniform per launch) uses the CTA barrier and plain
// shared-memory pointers instead of the cluster barrier and DSMEM windows.
__device__ __forceinline__ void row_sync(cg::cluster_group& cluster, int nblocks) {
    if (nblocks == 1) __syncthreads();
    else cluster.sync();
}
template <typename T>
__device__ __forceinline__ T* row_smem(cg::cluster_group& cluster, int nblocks, T* p, int rank) {
    return nblocks == 1 ? p : cluster.map_shared_rank(p, rank);
}

// Sum a 256-bin histogram over the cluster (DSMEM) and find the bin holding
// the `need`-th largest key. Writes ctl[kCtlBin], ctl[kCtlNeed] (how many to
// take from that bin) and ctl[kCtlCnt] (the bin's size). Requires a cluster
// barrier before (histograms complete); ends with __syncthreads().
// `zero_next` (may be null) is the other histogram buffer: no CTA reads it
// any more once every CTA has passed the barrier before this call, so it is
// cleared here for the next pass.
__device__ __forceinline__ void cluster_select_bin(cg::cluster_group& cluster, uint32_t* hist,
                                                   int nblocks, uint32_t need, int* ctl,
                                                   uint32_t* scan, uint32_t* zero_next) {
    const int tid = threadIdx.x;
    const int bin = 255 - tid;  // thread 0 holds the largest bin
    uint32_t cnt = 0;
    if (nblocks == 1) {
        cnt = hist[bin];
    } else {
        // all remote loads in flight together, then the sum
        uint32_t v[kMaxCluster];
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r) v[r] = r < nblocks ? cluster.map_shared_rank(hist, r)[bin] : 0u;
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r) cnt += v[r];
    }
    if (zero_next) zero_next[tid] = 0u;
    // prefix over bins (largest first): warp scans, then every warp adds the
    // totals of the warps before it (one barrier, no second scan)
    const uint32_t incl = warp_incl_scan(cnt);
    if (lane_id() == 31) scan[warp_id()] = incl;
    __syncthreads();
    uint32_t excl = incl - cnt;
#pragma unroll
    for (int w = 0; w < kNW; ++w) excl += w < warp_id() ? scan[w] : 0u;
    if (excl < need && need <= excl + cnt) {
        ctl[kCtlBin] = bin;
        ctl[kCtlNeed] = (int)(need - excl);
        ctl[kCtlCnt] = (int)cnt;
    }
    __syncthreads();
}

// PAGED: K/V are paged pools addressed through p.block_table (a separate
// instantiation, so the dense layout's copy loops carry no lookup).
template <typename TKV, int LK, int D, int C, int GT, bool PAGED>
__global__ void __launch_bounds__(kNT, 2) ds_decode_kernel(const DecodeParams p) {
    using E = Elem<TKV>;
    using LG = LabelGeom<TKV, LK, C>;
    constexpr int EPL = D / 32;                       // elements of a K/V row per lane
    constexpr int RBL = EPL * E::kBytes;              // bytes of a K/V row per lane
    static_assert(EPL * 32 == D, "D must be a multiple of 32");

    cg::cluster_group cluster = cg::this_cluster();
    const int N = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    const int row = blockIdx.x / N;  // = b * hkv + g
    const int g = row % p.hkv;
    const int G = p.G;
    const int tid = threadIdx.x, lane = lane_id(), wid = warp_id();

    extern __shared__ __align__(16) uint8_t smem[];
    const DecodeSmem L = decode_smem_layout(GT, D, C, p.lay_chunk, p.per, E::kBytes, p.att_stages);
    float* qs = reinterpret_cast<float*>(smem + L.qs);
    float* qLs = reinterpret_cast<float*>(smem + L.qL);
    int* idx_s = reinterpret_cast<int*>(smem + L.idx);
    uint32_t* histA = reinterpret_cast<uint32_t*>(smem + L.histA);
    uint32_t* histB = reinterpret_cast<uint32_t*>(smem + L.histB);
    int* ctl = reinterpret_cast<int*>(smem + L.ctl);
    uint32_t* scan = reinterpret_cast<uint32_t*>(smem + L.scan);
    float* cm = reinterpret_cast<float*>(smem + L.cm);
    float* cl = reinterpret_cast<float*>(smem + L.cl);
    float* co = reinterpret_cast<float*>(smem + L.co);
    uint8_t* bits8 = smem + L.region + p.sel_off;       // bucket flags, one byte per 8 tokens
    uint16_t* mcache = reinterpret_cast<uint16_t*>(bits8 + align16(p.lay_chunk / 8));
    uint32_t* blist = reinterpret_cast<uint32_t*>(bits8 + align16(p.lay_chunk / 8) + align16(p.lay_chunk / 8 * 2));
    int* sel_list = reinterpret_cast<int*>(smem + L.sel);
    uint16_t* keys = reinterpret_cast<uint16_t*>(smem + L.region);

    // tokens of this row: one length for all rows, or per batch entry
    // (clamped into [1, s]) when the caller gives seq_lens
    const int s = p.seq_lens ? min(max(p.seq_lens[row / p.hkv], 1), p.s) : p.s;
    const int t0 = rank * p.chunk;
    const int n_loc = max(0, min(s, t0 + p.chunk) - t0);
    const size_t row_tok = (size_t)row * (size_t)p.s_cap;  // first token of this row in the caches
    const TKV* qrow = reinterpret_cast<const TKV*>(p.q) + (size_t)row * G * D;
    const int k_eff = min(p.topk, s);
    bool select_all = p.dense || p.topk >= s;
    if (p.seq_lens) {  // the fallback rule for short entries
        if (p.batch_rule) {
            int any_short = 0, any_long = 0;
            for (int j = threadIdx.x; j < p.nb; j += kNT) {
                const int len = min(max(p.seq_lens[j], 1), p.s);
                any_short |= len < p.topk;
                any_long |= len >= p.threshold;
            }
            any_short = __syncthreads_or(any_short);
            any_long = __syncthreads_or(any_long);
            select_all = select_all || any_short || !any_long;
        } else {
            select_all = select_all || s < p.threshold;
        }
    }

    // [phase] 0
    const uint8_t* lab = reinterpret_cast<const uint8_t*>(p.label) + row_tok * LG::kBytes;
    const uint16_t* lsc = (LK == kLabelInt4) ? p.lscale + row_tok : nullptr;
    const uint16_t* lze = (LK == kLabelInt4) ? p.lzero + row_tok : nullptr;
    const bool need_scores = !p.dense && (!select_all || p.score_out != nullptr);
    constexpr int U = LG::kU;
    constexpr int kRound = kNT * U;  // tokens per scoring round

    const int app_i = (p.append && !p.dense && s - 1 >= t0 && s - 1 < t0 + n_loc) ? s - 1 - t0 : -1;

    // ---------------------------------------------------------- setup, step 1
    // The independent global loads go out first -- q, the channel indices and
    // (decode step) the newest token's key row -- then the label stream's
    // first copies; the loads are consumed afterwards, so the set-up costs a
    // single memory round trip.
    constexpr int kQPer = (GT * D + kNT - 1) / kNT;
    float qv[kQPer];
#pragma unroll
    for (int e = 0; e < kQPer; ++e) {
        const int x = tid + kNT * e;
        qv[e] = x < G * D ? E::to_f32(qrow[x]) : 0.f;
    }
    const int iv = (!p.dense && tid < C) ? p.idx[(size_t)g * C + tid] : 0;
    constexpr int kKRowVecs = D * E::kBytes / 16;   // 16-byte pieces of a key row
    uint4 kv_app = make_uint4(0u, 0u, 0u, 0u), vv_app = make_uint4(0u, 0u, 0u, 0u);
    if (app_i >= 0 && tid < kKRowVecs) {
        if (p.k_new) {
            kv_app = ldg_stream16(reinterpret_cast<const uint8_t*>(p.k_new) + ((size_t)row * D) * E::kBytes + tid * 16);
            vv_app = ldg_stream16(reinterpret_cast<const uint8_t*>(p.v_new) + ((size_t)row * D) * E::kBytes + tid * 16);
        } else {
            kv_app = ldg_stream16(reinterpret_cast<const uint8_t*>(p.k) +
                                  (kv_row_of<PAGED>(p, row / p.hkv, g, row_tok, s - 1) * D) * E::kBytes + tid * 16);
        }
    }

    // fp label rows stream through a kLabStages-deep shared-memory ring with
    // cp.async (no registers held while in flight): in stage j, thread tid
    // copies and then scores local token j * kNT + tid, so it only ever reads
    // its own copies (no block barrier needed).
    // A 4-bit stage is [256 payloads][256 scales][256 zeros]; the scales and
    // zeros of warp w's 32 tokens are 4 + 4 16-byte chunks, copied by lanes
    // 0..7 of that warp (so a __syncwarp makes them visible to its lanes).
    constexpr bool kI4 = LK == kLabelInt4;
    constexpr int kLabStages = lab_stages(kI4);
    static_assert(kLabStages % 2 == 0 && kLabStages >= 4, "the scan takes two stages per iteration");
    constexpr bool kRingable = kI4 ? (LG::kBytes == 4 || LG::kBytes == 8 || LG::kBytes % 16 == 0)
                                   : LG::kBytes % 16 == 0;
    const bool use_ring = kRingable && need_scores && p.lab_ring;
    uint16_t* low16 = reinterpret_cast<uint16_t*>(smem + L.region + align16(p.lay_chunk * 2));
    uint8_t* lring = smem + L.region + align16(p.lay_chunk * 2) * (p.keep_low ? 2 : 1);
    constexpr int kSlot = LG::kBytes;               // payload bytes per token
    constexpr int kStage = kNT * (kSlot + (kI4 ? 4 : 0));
    const int nst = (n_loc + kNT - 1) / kNT;
    // stage j goes to ring slot `slot` (= j mod kLabStages, kept by the
    // caller); i < n_loc implies j < nst. The appended token's row is copied
    // too (stale, never read: stage_row takes it from shared memory).
    // per-thread bases of the copies; stage j adds j * kNT tokens
    const uint8_t* lab_t = lab + (size_t)(t0 + tid) * kSlot;
    uint8_t* ring_t = lring + tid * kSlot;
    const int c8 = wid * 32 + (lane & 3) * 8;   // 4-bit: first token of this lane's scale / zero chunk
    const uint16_t* sz_t = kI4 ? (lane < 4 ? lsc : lze) + t0 + c8 : nullptr;
    const int sz_off = kNT * kSlot + (lane < 4 ? 0 : kNT * 2) + c8 * 2;
    auto issue = [&](int j, int slot) {
        const int jr = j * kNT;
        if (jr + tid < n_loc) {
            uint8_t* dst = ring_t + slot * kStage;
            const uint8_t* src = lab_t + (size_t)jr * kSlot;
            if constexpr (kSlot % 16 == 0) {
#pragma unroll
                for (int o = 0; o < kSlot; o += 16) cp_async16(dst + o, src + o);
            } else if constexpr (kSlot == 8) {
                cp_async8(dst, src);
            } else {
                cp_async4(dst, src);
            }
        }
        if constexpr (kI4) {
            if (lane < 8 && jr + c8 < n_loc) cp_async16(lring + slot * kStage + sz_off, sz_t + jr);
        }
    };
    if (use_ring) {
#pragma unroll 1
        for (int j = 0; j < kLabStages - 2; ++j) { issue(j, j); cp_async_commit(); }
    }

#pragma unroll
    for (int e = 0; e < kQPer; ++e)
        if (tid + kNT * e < G * D) qs[tid + kNT * e] = qv[e];
    // the newest token's key row is staged in shared memory
    uint8_t* krow_s = smem + L.krow;
    if (app_i >= 0 && tid < kKRowVecs) {
        reinterpret_cast<uint4*>(krow_s)[tid] = kv_app;
        if (p.k_new) {  // the new token's K/V rows into the caches (read back by the attention)
            const size_t r = kv_row_of<PAGED>(p, row / p.hkv, g, row_tok, s - 1) * D * E::kBytes;
            reinterpret_cast<uint4*>(const_cast<uint8_t*>(reinterpret_cast<const uint8_t*>(p.k)) + r)[tid] = kv_app;
            reinterpret_cast<uint4*>(const_cast<uint8_t*>(reinterpret_cast<const uint8_t*>(p.v)) + r)[tid] = vv_app;
            __threadfence();
        }
    }
    if (!p.dense) {
        if (tid < C) idx_s[tid] = min(max(iv, 0), D - 1);
        histA[tid] = 0u;
        histB[tid] = 0u;
        if (tid == 0) { ctl[kCtlBL] = 0; ctl[kCtlTie] = 0; }
    }
    __syncthreads();
    if (!p.dense) {
        for (int j = tid; j < C; j += kNT) {
            float a = 0.f;
            for (int e = 0; e < G; ++e) a += qs[e * D + idx_s[j]];
            qLs[j] = a;
        }
        if constexpr (LK == kLabelInt4 && C <= 32) {
            // warp 0 already holds qL (lane j has channel j): it forms the
            // fixed-point limbs for i4_dot once, for every thread to load
            if (wid == 0) {
                float qv = 0.f;
                if (lane < C) {
                    for (int e = 0; e < G; ++e) qv += qs[e * D + idx_s[lane]];
                }
                float qmax = fabsf(qv);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) qmax = fmaxf(qmax, __shfl_xor_sync(0xffffffffu, qmax, o));
                float two_e;
                const float s_e = i4_scale_exp(qmax, &two_e);
                const int q = __float2int_rn(__fmul_rn(qv, two_e));
                // word wi = (k, h, i): byte b is limb k of channel 8i + 2b + h
                const int wi = lane, k = wi / (2 * (C / 8)), h = (wi / (C / 8)) & 1, i = wi % (C / 8);
                uint32_t word = 0u;
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const int qc = __shfl_sync(0xffffffffu, q, (8 * i + 2 * b + h) & 31);
                    word |= ((uint32_t)(qc >> (8 * (k < 3 ? k : 0))) & 255u) << (8 * b);
                }
                if (wi < 6 * C / 8) reinterpret_cast<uint32_t*>(smem + L.ql4)[wi] = word;
                if (lane == 0) reinterpret_cast<float*>(smem + L.ql4)[6 * C / 8] = s_e;
            }
        }
    }
    if constexpr (E::kBytes == 2) {
        // tensor-core A fragments of q for the attention phase (see step 3b)
        uint2* qa_w = reinterpret_cast<uint2*>(smem + L.qa);
        for (int e = tid; e < (D / 16) * 32; e += kNT) {
            const int c = e >> 5, ln = e & 31, h = ln >> 2, col = 16 * c + (ln & 3) * 2;
            const float* qh = qs + h * D + col;
            qa_w[e] = h < G ? make_uint2(pack_bf16x2(qh[0], qh[1]), pack_bf16x2(qh[8], qh[9])) : make_uint2(0u, 0u);
        }
    }
    // decode step: the CTA holding token s-1 builds its label row (the same
    // copy / 4-bit pack as ds_append_label), keeps it in shared memory and
    // stores it to the label cache; 4-bit rows use warp 1, so the pack runs
    // beside warp 0's fixed-point limbs
    if (app_i >= 0 && wid == (LK == kLabelInt4 ? 1 : 0)) {
        const TKV* krow = reinterpret_cast<const TKV*>(krow_s);
        uint8_t* grow = const_cast<uint8_t*>(lab) + (size_t)(s - 1) * LG::kBytes;
        if constexpr (LK == kLabelFp) {
            TKV* srow = reinterpret_cast<TKV*>(smem + L.app);
            for (int j = lane; j < C; j += 32) {
                const TKV x = krow[idx_s[j]];
                srow[j] = x;
                reinterpret_cast<TKV*>(grow)[j] = x;
            }
        } else {
            // pack_int4_row's arithmetic with a lane per channel: mn / mx by a
            // butterfly over the lanes (fminf / fmaxf do not depend on the
            // order), then lane j divides for channel j and the even lanes
            // pack pairs
            uint16_t* ssz = reinterpret_cast<uint16_t*>(smem + L.app + align16(C * 4));
            float mn = Elem<TKV>::to_f32(krow[idx_s[lane % C]]), mx = mn;
            for (int j = lane + 32; j < C; j += 32) {
                const float v = Elem<TKV>::to_f32(krow[idx_s[j]]);
                mn = fminf(mn, v);
                mx = fmaxf(mx, v);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            }
            const float step = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
            const uint16_t sh = __half_as_ushort(__float2half_rn(step));
            const uint16_t zh = __half_as_ushort(__float2half_rn(mn));
            const float sc = fp16_bits_to_f32(sh), z = fp16_bits_to_f32(zh);
#pragma unroll
            for (int j0 = 0; j0 < C; j0 += 32) {
                const int j = j0 + lane;
                uint32_t code = 0;
                if (j < C && sc > 0.f) {
                    float qv = rintf(__fdiv_rn(__fsub_rn(Elem<TKV>::to_f32(krow[idx_s[j]]), z), sc));
                    qv = fminf(fmaxf(qv, 0.f), 15.f);
                    code = (uint32_t)qv;
                }
                const uint32_t hi = __shfl_down_sync(0xffffffffu, code, 1);
                if (j < C && !(j & 1)) {
                    const uint8_t byte = (uint8_t)(code | (hi << 4));
                    smem[L.app + j / 2] = byte;
                    grow[j / 2] = byte;
                }
            }
            if (lane == 0) {
                ssz[0] = sh;
                ssz[1] = zh;
                const_cast<uint16_t*>(lsc)[s - 1] = sh;
                const_cast<uint16_t*>(lze)[s - 1] = zh;
            }
        }
    }
    __syncthreads();

    constexpr bool kI4Score = LK == kLabelInt4;
    float qreg[(C <= 32 && !kI4Score) ? C : 1];
    uint32_t qlim[(C <= 32 && kI4Score) ? 6 * C / 8 : 1];   // 4-bit: limbs in registers
    const uint32_t* lim = (C <= 32) ? qlim : reinterpret_cast<const uint32_t*>(smem + L.ql4);
    float qsum = 0.f, s_e = 0.f;

    // The label row of the appended token (local index app_i, -1 if none) is
    // read from shared memory: this kernel writes it to the label cache and
    // must not read it back through the read-only path.
    const uint8_t* app_row = smem + L.app;
    const uint16_t* app_sz = reinterpret_cast<const uint16_t*>(smem + L.app + align16(C * 4));
    auto load_label = [&](int i, uint32_t (&w)[LG::kWords], float& sc, float& z) {
        if (i == app_i) {
            lds_row<LG::kBytes>(w, app_row);
            if constexpr (LK == kLabelInt4) { sc = fp16_bits_to_f32(app_sz[0]); z = fp16_bits_to_f32(app_sz[1]); }
        } else {
            load_words<LG::kBytes>(w, lab + (size_t)(t0 + i) * LG::kBytes);
            if constexpr (LK == kLabelInt4) {
                sc = fp16_bits_to_f32(ldg_u16(lsc + t0 + i));
                z = fp16_bits_to_f32(ldg_u16(lze + t0 + i));
            }
        }
    };
    // Score of local token i straight from memory; same arithmetic as the
    // streaming loop below.
    auto rescore = [&](int i) -> float {
        uint32_t w[LG::kWords];
        float sc = 0.f, z = 0.f;
        load_label(i, w, sc, z);
        return label_score<TKV, LK, C>(w, qreg, qLs, sc, z, qsum, lim, s_e);
    };

    if (need_scores) {
        if constexpr (C <= 32 && !kI4Score) {
#pragma unroll
            for (int j = 0; j < C; ++j) qreg[j] = qLs[j];
        }
        for (int j = 0; j < C; ++j) qsum += qLs[j];
        if constexpr (kI4Score) {
            if constexpr (C <= 32) {
                // formed by warp 0 before the barrier above
                const uint32_t* lw = reinterpret_cast<const uint32_t*>(smem + L.ql4);
#pragma unroll
                for (int wi = 0; wi < 6 * C / 8; ++wi) qlim[wi] = lw[wi];
                s_e = reinterpret_cast<const float*>(smem + L.ql4)[6 * C / 8];
            } else {
                float qmax = 0.f;
                for (int j = 0; j < C; ++j) qmax = fmaxf(qmax, fabsf(qLs[j]));
                float two_e;
                s_e = i4_scale_exp(qmax, &two_e);
                for (int wi = tid; wi < 6 * C / 8; wi += kNT)
                    reinterpret_cast<uint32_t*>(smem + L.ql4)[wi] = i4_limb_word<C>(qLs, two_e, wi);
            }
        }
    }
    if constexpr (kI4Score && C > 32) __syncthreads();  // limbs in shared memory

    // [phase] 1
    // ---------------------------------------------------------------- step 2
    // Score one token (local index i) from its label row, store its 16-bit
    // key and count its top byte.
    auto record_token = [&](int i, float sv) {
        const uint32_t key = score_key(sv);
        if (!select_all) {
            keys[i] = (uint16_t)(key >> 16);
            if (p.keep_low) low16[i] = (uint16_t)key;
            atomicAdd(&histA[key >> 24], 1u);
        }
        if (p.score_out) p.score_out[(size_t)row * p.s + t0 + i] = sv;
    };
    auto score_token = [&](int i, const uint32_t (&w)[LG::kWords], float ss, float zz) {
        record_token(i, label_score<TKV, LK, C>(w, qreg, qLs, ss, zz, qsum, lim, s_e));
    };
    if (use_ring) {
        // two stages per iteration: each thread scores two tokens (j and
        // j + 1 stages apart) whose arithmetic chains are independent
        // the row of local token i from ring slot `slot` (the appended token's
        // from shared memory): pointers picked, no branch
        auto stage_row = [&](int slot, int i, uint32_t (&w)[LG::kWords], float& ss, float& zz) {
            const uint8_t* stg = lring + slot * kStage;
            const bool app = i == app_i;
            lds_row<LG::kBytes>(w, app ? app_row : stg + tid * kSlot);
            if constexpr (kI4) {
                const uint16_t* sp = app ? app_sz : reinterpret_cast<const uint16_t*>(stg + kNT * kSlot) + tid;
                ss = fp16_bits_to_f32(sp[0]);
                zz = fp16_bits_to_f32(sp[app ? 1 : kNT]);
            }
        };
        int sj = 0;  // ring slot of stage j (j even; kLabStages is even)
#pragma unroll 1
        for (int j = 0; j < nst; j += 2) {
            if constexpr (kI4) __syncwarp();   // every lane is done with the slots refilled next
            const int sr = sj == 0 ? kLabStages - 2 : sj - 2;   // slot of stage j + kLabStages - 2
            issue(j + kLabStages - 2, sr);
            cp_async_commit();
            issue(j + kLabStages - 1, sr + 1);
            cp_async_commit();
            cp_async_wait<kLabStages - 2>();   // stages j and j + 1 have landed
            if constexpr (kI4) __syncwarp();   // the warp's scale / zero chunks
            const int i0 = j * kNT + tid, i1 = i0 + kNT;
            uint32_t w0[LG::kWords], w1[LG::kWords];
            float ss0 = 0.f, zz0 = 0.f, ss1 = 0.f, zz1 = 0.f;
            stage_row(sj, i0, w0, ss0, zz0);
            stage_row(sj + 1, i1, w1, ss1, zz1);
            sj = sj + 2 == kLabStages ? 0 : sj + 2;
            // rows past the chunk hold stale ring bytes: scored, not recorded
            const float sv0 = label_score<TKV, LK, C>(w0, qreg, qLs, ss0, zz0, qsum, lim, s_e);
            const float sv1 = label_score<TKV, LK, C>(w1, qreg, qLs, ss1, zz1, qsum, lim, s_e);
            if (i0 < n_loc) record_token(i0, sv0);
            if (i1 < n_loc) record_token(i1, sv1);
        }
        cp_async_wait<0>();
    } else if (need_scores) {
        // rounds `scan_prefetch` ahead are pulled into L2 (128-byte lines of
        // the payload and, for 4-bit rows, of the scales and zeros), so the
        // register loads of a round mostly hit L2
        auto prefetch_round = [&](int base) {
            const int n = min(kRound, n_loc - base);
            if (n <= 0) return;
            const uint8_t* p0 = lab + (size_t)(t0 + base) * LG::kBytes;
            const int lines = (n * LG::kBytes + 127) >> 7;
            for (int l = tid; l < lines; l += kNT) prefetch_line_l2(p0 + (l << 7));
            if constexpr (LK == kLabelInt4) {
                const int zl = (n * 2 + 127) >> 7;
                for (int l = tid; l < 2 * zl; l += kNT)
                    prefetch_line_l2(reinterpret_cast<const uint8_t*>((l < zl ? lsc : lze) + t0 + base) +
                                     ((l < zl ? l : l - zl) << 7));
            }
        };
        for (int r = 1; r <= p.scan_prefetch; ++r) prefetch_round(r * kRound);
        for (int base = 0; base < n_loc; base += kRound) {
            if (p.scan_prefetch > 0) prefetch_round(base + (p.scan_prefetch + 1) * kRound);
            uint32_t w[U][LG::kWords];
            float sc[U], z[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = base + u * kNT + tid;
                if (i < n_loc) load_label(i, w[u], sc[u], z[u]);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = base + u * kNT + tid;
                if (i < n_loc) {
                    float zz = 0.f, ss = 0.f;
                    if constexpr (LK == kLabelInt4) { ss = sc[u]; zz = z[u]; }
                    score_token(i, w[u], ss, zz);
                }
            }
        }
    }

    // [phase] 2
    // --------------------------------------------------------------- step 3a
    const TKV* kb = reinterpret_cast<const TKV*>(p.k);   // rows addressed by att_row()
    const TKV* vb = reinterpret_cast<const TKV*>(p.v);
    constexpr int RB = D * E::kBytes;              // bytes of one K or V row
    int T16 = 0, Tlo = 0, r_tie = 0;
    bool refine = false;
    if (!select_all) {
        row_sync(cluster, N);                                        // histograms A complete
        cluster_select_bin(cluster, histA, N, (uint32_t)k_eff, ctl, scan, nullptr);
        const int bA = ctl[kCtlBin];
        const int needA = ctl[kCtlNeed];
        // [phase] 3
        // Key sweeps read 8 keys (16 bytes) per thread per step; group g holds
        // local tokens [8g, 8g + 8). Keys past n_loc in the last group are masked.
        const uint8_t* kbytes = reinterpret_cast<const uint8_t*>(keys);
        const int ngrp = (n_loc + 7) >> 3;
        auto key8 = [&](int grp, uint32_t (&w)[4]) { lds_words<16>(w, kbytes + grp * 16); };
        auto kat = [](const uint32_t (&w)[4], int e) -> int { return (int)((w[e >> 1] >> ((e & 1) * 16)) & 0xFFFFu); };
        for (int grp = tid; grp < ngrp; grp += kNT) {
            uint32_t w[4];
            key8(grp, w);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int k16 = kat(w, e);
                if (grp * 8 + e < n_loc && (k16 >> 8) == bA) atomicAdd(&histB[k16 & 255], 1u);
            }
        }
        // [phase] 10
        row_sync(cluster, N);                                        // histograms B complete
        // [phase] 11
        cluster_select_bin(cluster, histB, N, (uint32_t)needA, ctl, scan, histA);
        T16 = (bA << 8) | ctl[kCtlBin];
        const int needB = ctl[kCtlNeed];
        refine = needB < ctl[kCtlCnt];
        // a split bucket of at most kNT tokens (over the cluster) is ranked
        // exactly instead of running two more radix passes
        const bool rank_mode = ctl[kCtlCnt] <= kNT;
        // Warp w owns the contiguous key groups [wg0, wg1) for the refine
        // sweep and the compaction; in each step lane l reads group
        // wg0 + 32*step + l (conflict-free), so lane order is index order.
        const int gpw = (((ngrp + kNW - 1) / kNW) + 63) & ~63;   // groups per warp
        const int wg0 = wid * gpw, wg1 = min(ngrp, wg0 + gpw);
        // [phase] 4
        if (refine) {
            // The k-th key's 16-bit bucket is split: take the low 16 key bits
            // of its tokens (kept, or re-scored with bit-identical arithmetic)
            // in place of the high ones, flag and list them; count each warp's
            // keys above the bucket (selected outright) on the way.
            uint32_t above_cnt = 0;
            for (int grp = wg0 + lane; grp - lane < wg1; grp += 32) {
                if (grp >= wg1) continue;
                uint32_t w[4];
                key8(grp, w);
                uint32_t flags = 0, above = 0;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const bool ok = grp * 8 + e < n_loc;
                    if (ok && kat(w, e) == T16) flags |= 1u << e;
                    if (ok && kat(w, e) > T16) above |= 1u << e;
                }
                above_cnt += __popc(above);
                bits8[grp] = (uint8_t)flags;
                mcache[grp] = (uint16_t)above;   // keys selected outright, for the write pass
                for (uint32_t m = flags; m; m &= m - 1) {
                    const int i = grp * 8 + __ffs(m) - 1;
                    const int slot = atomicAdd(&ctl[kCtlBL], 1);
                    if (p.keep_low || slot >= kBucketCap) {
                        // low bits at hand, or no list slot left: take them here
                        const uint32_t low = p.keep_low ? (uint32_t)low16[i] : score_key(rescore(i)) & 0xFFFFu;
                        keys[i] = (uint16_t)low;
                        if (!rank_mode) atomicAdd(&histA[low >> 8], 1u);
                        if (slot < kBucketCap) blist[slot] = low | ((uint32_t)i << 16);
                    } else {
                        blist[slot] = (uint32_t)i << 16;  // re-scored below
                    }
                }
            }
            above_cnt = __reduce_add_sync(0xffffffffu, above_cnt);
            if (lane == 0) ctl[kCtlWarp + wid] = (int)(above_cnt << 16);
            if (!p.keep_low) {
                // the listed bucket tokens are re-scored all at once (one
                // label-row load per thread in flight, not one per lane in turn)
                __syncthreads();
                const int nbl = min(ctl[kCtlBL], kBucketCap);
                for (int j = tid; j < nbl; j += kNT) {
                    const uint32_t e = blist[j];
                    const int i = (int)(e >> 16);
                    const uint32_t low = score_key(rescore(i)) & 0xFFFFu;
                    keys[i] = (uint16_t)low;
                    blist[j] = e | low;
                    if (!rank_mode) atomicAdd(&histA[low >> 8], 1u);
                }
            }
        }
        if (refine && rank_mode) {
            // rank of each bucket token by (low key bits desc, index asc); the
            // needB-th gives the low threshold, and the tokens equal to it that
            // rank inside are the ties to take. A cluster first gathers every
            // CTA's bucket list (low key in histB, token index in the row in
            // histA; both free by now), so all its CTAs rank the same list.
            int nbl, my_low = -1, my_rank = 0;
            if (N == 1) {
                __syncthreads();
                nbl = ctl[kCtlBL];
                if (tid < nbl) {
                    const uint32_t e = blist[tid];
                    my_low = (int)(e & 0xFFFFu);
                    const int my_idx = (int)(e >> 16);
                    for (int j = 0; j < nbl; ++j) {
                        const uint32_t f = blist[j];
                        const int lo = (int)(f & 0xFFFFu), ix = (int)(f >> 16);
                        my_rank += (lo > my_low) || (lo == my_low && ix < my_idx);
                    }
                }
            } else {
                row_sync(cluster, N);                                // bucket lists complete
                if (wid == 0) {
                    const int c = lane < N ? row_smem(cluster, N, ctl, lane)[kCtlBL] : 0;
                    const int incl = (int)warp_incl_scan((uint32_t)c);
                    if (lane < N) ctl[kCtlGather + lane] = incl - c;
                    if (lane == N - 1) ctl[kCtlGather + 16] = incl;
                }
                __syncthreads();
                nbl = min(ctl[kCtlGather + 16], kNT);
                if (tid < nbl) {
                    int r = 0;
                    while (r + 1 < N && ctl[kCtlGather + r + 1] <= tid) ++r;
                    const uint32_t e = row_smem(cluster, N, blist, r)[tid - ctl[kCtlGather + r]];
                    histB[tid] = e & 0xFFFFu;
                    histA[tid] = (uint32_t)(r * p.chunk) + (e >> 16);
                }
                __syncthreads();
                if (tid < nbl) {
                    my_low = (int)histB[tid];
                    const int my_idx = (int)histA[tid];
                    for (int j = 0; j < nbl; ++j) {
                        const int lo = (int)histB[j], ix = (int)histA[j];
                        my_rank += (lo > my_low) || (lo == my_low && ix < my_idx);
                    }
                }
            }
            if (tid < nbl && my_rank == needB - 1) ctl[kCtlTlo] = my_low;
            __syncthreads();
            Tlo = ctl[kCtlTlo];
            if (tid < nbl && my_low == Tlo && my_rank < needB) atomicAdd(&ctl[kCtlTie], 1);
            __syncthreads();
            r_tie = ctl[kCtlTie];
        } else if (refine) {
            // [phase] 12
            row_sync(cluster, N);                                    // histograms C complete
            // [phase] 13
            cluster_select_bin(cluster, histA, N, (uint32_t)needB, ctl, scan, histB);
            const int bC = ctl[kCtlBin];
            const int needC = ctl[kCtlNeed];
            const int nbl = ctl[kCtlBL];
            if (nbl <= kBucketCap) {
                for (int j = tid; j < nbl; j += kNT) {
                    const uint32_t low = blist[j] & 0xFFFFu;
                    if ((int)(low >> 8) == bC) atomicAdd(&histB[low & 255u], 1u);
                }
            } else {
                for (int grp = tid; grp < ngrp; grp += kNT) {
                    const uint32_t fl = bits8[grp];
                    if (!fl) continue;
                    uint32_t w[4];
                    key8(grp, w);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int low = kat(w, e);
                        if (((fl >> e) & 1u) && (low >> 8) == bC) atomicAdd(&histB[low & 255], 1u);
                    }
                }
            }
            // [phase] 14
            row_sync(cluster, N);                                    // histograms D complete
            // [phase] 15
            cluster_select_bin(cluster, histB, N, (uint32_t)needC, ctl, scan, nullptr);
            Tlo = (bC << 8) | ctl[kCtlBin];
            r_tie = ctl[kCtlNeed];
        }

        // [phase] 5
        // ----------------------------------------------------- compaction
        // classes: 1 = selected outright, 2 = exact tie with the k-th key.
        // Warp w owns a contiguous segment of key groups; in each step lane l
        // reads group seg + 32*step + l (conflict-free 16-byte loads), so lane
        // order is index order and warp scans rank the selected tokens.
        // Per key group: bit e of the low byte marks a key selected outright,
        // bit e of the second byte an exact tie with the k-th key.
        auto masks8 = [&](int grp) -> uint32_t {
            uint32_t w[4];
            key8(grp, w);
            const uint32_t fl = refine ? bits8[grp] : 0u;
            const int lim = n_loc - grp * 8;
            uint32_t sm = 0, tm = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int k16 = kat(w, e);
                const bool inb = (fl >> e) & 1u;
                const bool strict = refine ? k16 > (inb ? Tlo : T16) : k16 >= T16;
                const bool tie = inb && k16 == Tlo;
                sm |= (uint32_t)(e < lim && strict) << e;
                tm |= (uint32_t)(e < lim && tie) << e;
            }
            return sm | (tm << 8);
        };
        // Per-warp (selected, tie) counts. With a split bucket that is fully
        // listed they follow from the refine sweep's counts plus the listed
        // bucket tokens; otherwise a count pass classifies every key (and
        // keeps each group's masks, 2 bytes, for the write pass).
        const bool counts_known = refine && ctl[kCtlBL] <= kBucketCap;
        // With the counts known, a group's masks are the refine sweep's
        // "above" bits plus its bucket tokens classified by their low bits.
        auto masks_swept = [&](int grp) -> uint32_t {
            uint32_t m = mcache[grp];
            const uint32_t fl = bits8[grp];
            if (fl) {
                uint32_t w[4];
                key8(grp, w);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if ((fl >> e) & 1u) {
                        const int low = kat(w, e);
                        m |= low > Tlo ? (1u << e) : (low == Tlo ? (1u << (8 + e)) : 0u);
                    }
            }
            return m;
        };
        if (counts_known) {
            const int nbl = ctl[kCtlBL];
            for (int j = tid; j < nbl; j += kNT) {
                const uint32_t e = blist[j];
                const int low = (int)(e & 0xFFFFu), i = (int)(e >> 16);
                const int w = (i >> 3) / gpw;
                if (low > Tlo) atomicAdd(&ctl[kCtlWarp + w], 1 << 16);
                else if (low == Tlo) atomicAdd(&ctl[kCtlWarp + w], 1);
            }
            __syncthreads();
            if (lane == 0) scan[wid] = (uint32_t)ctl[kCtlWarp + wid];
        } else {
            uint32_t ns = 0, nt = 0;
            for (int grp = wg0 + lane; grp - lane < wg1; grp += 32) {
                const uint32_t m = grp < wg1 ? masks8(grp) : 0u;
                if (grp < wg1) mcache[grp] = (uint16_t)m;
                ns += __popc(m & 255u);
                nt += __popc(m >> 8);
            }
            ns = (uint32_t)__reduce_add_sync(0xffffffffu, ns);
            nt = (uint32_t)__reduce_add_sync(0xffffffffu, nt);
            if (lane == 0) scan[wid] = (ns << 16) | nt;
        }
        __syncthreads();
        // each warp's (selected, tie) counts before it and the CTA's totals,
        // from the kNW per-warp counts
        uint32_t before = 0, all = 0;
#pragma unroll
        for (int w = 0; w < kNW; ++w) {
            const uint32_t x = scan[w];
            before += w < wid ? x : 0u;
            all += x;
        }
        // [phase] 16
        int P = 0, TP = 0;  // selections and ties of the cluster's CTAs before this one
        if (N > 1) {
            if (tid == 0) { ctl[kCtlCS] = (int)(all >> 16); ctl[kCtlCT] = (int)(all & 0xFFFFu); }
            // [phase] 17
            row_sync(cluster, N);                                    // per-CTA counts visible
            // [phase] 18
            if (wid == 0) {
                int cs = 0, ct = 0;
                if (lane < N) {
                    const int* rc = row_smem(cluster, N, ctl, lane);
                    cs = rc[kCtlCS];
                    ct = rc[kCtlCT];
                }
                const int tp_incl = (int)warp_incl_scan((uint32_t)ct);
                const int tp = tp_incl - ct;  // ties in CTAs before `lane`
                const int ntake = refine ? max(0, min(ct, r_tie - tp)) : 0;
                const int cnt = cs + ntake;
                const int p_incl = (int)warp_incl_scan((uint32_t)cnt);
                if (lane == rank) { ctl[kCtlP] = p_incl - cnt; ctl[kCtlTP] = tp; }
            }
            __syncthreads();
            P = ctl[kCtlP];
            TP = ctl[kCtlTP];
        }
        // [phase] 19
        const int tie_quota = max(0, r_tie - TP);  // ties this CTA may still take
        int sb = (int)(before >> 16), tb = (int)(before & 0xFFFFu);  // before this step
        const uint32_t per = (uint32_t)p.per;
        const uint32_t per_inv = 0xFFFFFFFFu / per;  // q = umulhi(pos, per_inv) is q or q-1
        int cur_dst = -1;
        int* rl = nullptr;
        // two key groups (16 tokens) per lane and step: lane l takes groups
        // g0 = wg0 + 64*step + 2l and g0 + 1, so lane order is still index order
        auto gmask = [&](int grp) -> uint32_t {
            return grp < wg1 ? (counts_known ? masks_swept(grp) : (uint32_t)mcache[grp]) : 0u;
        };
        for (int g0 = wg0 + 2 * lane; g0 - 2 * lane < wg1; g0 += 64) {
            const uint32_t m0 = gmask(g0), m1 = gmask(g0 + 1);
            const uint32_t smk = (m0 & 255u) | ((m1 & 255u) << 8), tmk = (m0 >> 8) | ((m1 >> 8) << 8);
            const uint32_t pk = ((uint32_t)__popc(smk) << 16) | (uint32_t)__popc(tmk);
            const uint32_t incl = warp_incl_scan(pk);
            const int my_sb = sb + (int)((incl - pk) >> 16), my_tb = tb + (int)((incl - pk) & 0xFFFFu);
            const uint32_t tot_step = __shfl_sync(0xffffffffu, incl, 31);
            sb += (int)(tot_step >> 16);
            tb += (int)(tot_step & 0xFFFFu);
            for (uint32_t mm = smk | tmk; mm; mm &= mm - 1u) {
                const int e = __ffs(mm) - 1;
                const uint32_t below = (1u << e) - 1u;
                const int s_before = my_sb + __popc(smk & below);
                const int t_before = my_tb + __popc(tmk & below);
                if (((tmk >> e) & 1u) && t_before >= tie_quota) continue;  // tie beyond the quota
                const uint32_t pos = (uint32_t)(P + s_before + min(t_before, tie_quota));
                const int t = t0 + g0 * 8 + e;
                if (N == 1) {
                    sel_list[pos] = t;
                } else {
                    uint32_t dst = __umulhi(pos, per_inv);
                    if ((dst + 1u) * per <= pos) ++dst;
                    if ((int)dst != cur_dst) { cur_dst = (int)dst; rl = row_smem(cluster, N, sel_list, (int)dst); }
                    rl[pos - dst * per] = t;
                }
                if (p.sel_out) p.sel_out[(size_t)row * p.topk + pos] = t;
            }
        }
        // [phase] 20
        row_sync(cluster, N);                                        // selection lists complete
    } else if (p.sel_out) {
        // every token is attended: listed when they fit, else the row is all -1
        if (s <= p.topk) {
            for (int i = tid; i < n_loc; i += kNT) p.sel_out[(size_t)row * p.topk + t0 + i] = t0 + i;
            if (rank == 0)
                for (int j = s + tid; j < p.topk; j += kNT) p.sel_out[(size_t)row * p.topk + j] = -1;
        } else if (rank == 0) {
            for (int j = tid; j < p.topk; j += kNT) p.sel_out[(size_t)row * p.topk + j] = -1;
        }
    }

    // [phase] 6
    // --------------------------------------------------------------- step 3b
    const int n_att = select_all ? n_loc : max(0, min(p.per, k_eff - rank * p.per));
    // paged K/V: this CTA's selected tokens become pool rows first (one
    // table lookup per token, all in flight together)
    uint32_t* sel_rows = reinterpret_cast<uint32_t*>(sel_list);
    if (PAGED && !select_all) {
        for (int j = tid; j < n_att; j += kNT)
            sel_rows[j] = (uint32_t)kv_row_of<PAGED>(p, row / p.hkv, g, row_tok, sel_list[j]);
        __syncthreads();
    }
    float* wp_out = nullptr;  // this warp's partial (m, l, o) per head, [GT][D + 2]
    auto write_out = [&](int h, int d, float res) {
        const size_t oidx = (size_t)row * G * D + (size_t)h * D + d;
        if (p.out_bf16) reinterpret_cast<uint16_t*>(p.out)[oidx] = f32_to_bf16_bits(res);
        else reinterpret_cast<float*>(p.out)[oidx] = res;
    };
    // K/V row (units of d elements) of the j-th token this CTA attends
    auto att_row = [&](int j) -> size_t {
        if constexpr (PAGED)
            return select_all ? kv_row_of<PAGED>(p, row / p.hkv, g, row_tok, t0 + j) : (size_t)sel_rows[j];
        else
            return row_tok + (size_t)(select_all ? t0 + j : sel_list[j]);
    };
    {
        if constexpr (E::kBytes == 2) {
            // bf16 K/V: tensor cores (mma.sync, fp32 accumulate) on 8-token tiles.
            //   Z  = Q K^T   m16n8k16: rows = the group's heads (padded to 16),
            //                cols = 8 tokens, k = 16 dims per step
            //   O^T += V^T P^T  m16n8k8: rows = 16 dims, cols = heads, k = 8 tokens
            // so the softmax probabilities of a head (a row of Z's accumulator)
            // are already laid out as the B operand of the second product. P is
            // split into bf16 hi + lo parts (two products), keeping ~2^-17 of
            // relative precision. Rows are staged with cp.async into a per-warp
            // ring; 16-byte chunks are XOR-swizzled by token so that ldmatrix reads
            // are bank-conflict free.
            constexpr int TB8 = 8;
            constexpr int kChunks = RB / 16;           // 16-byte chunks per row
            constexpr int kStageBytes = 2 * TB8 * RB;
            const int stages = p.att_stages;
            uint8_t* ring = smem + L.region + wid * att_ring_bytes(RB, 2, stages);
            const int nb = n_att > wid * TB8 ? (n_att - wid * TB8 + kNW * TB8 - 1) / (kNW * TB8) : 0;
            // lane l copies 16-byte chunk l % kChunks of token rows l / kChunks,
            // l / kChunks + 32 / kChunks, ... of the tile, the K and the V row of
            // each token together (one row lookup per token)
            static_assert(32 % kChunks == 0 && TB8 % (32 / kChunks) == 0, "chunk layout");
            constexpr int kRowsPerPass = 32 / kChunks;
            const int cl = lane % kChunks, ul = lane / kChunks;
            // tile bi of this warp goes to ring slot `slot` (= bi mod stages,
            // kept by the caller: stages is a launch parameter)
            auto issue_stage = [&](int bi, int slot) {
                const int bt0 = (wid + bi * kNW) * TB8;
                uint8_t* st = ring + slot * kStageBytes;
    #pragma unroll
                for (int u0 = 0; u0 < TB8; u0 += kRowsPerPass) {
                    const int u = u0 + ul;
                    const bool ok = bt0 + u < n_att;
                    const size_t off = ok ? att_row(bt0 + u) * D : 0;
                    const uint8_t* ks = reinterpret_cast<const uint8_t*>(kb + off) + (cl << 4);
                    const uint8_t* vs = reinterpret_cast<const uint8_t*>(vb + off) + (cl << 4);
                    // rows of tokens past the end are zero-filled (their p is 0, and 0 * garbage could be NaN)
                    cp_async16_zfill(st + u * RB + ((cl ^ u) << 4), ks, ok);
                    cp_async16_zfill(st + (TB8 + u) * RB + ((cl ^ u) << 4), vs, ok);
                }
            };
            for (int bi = 0; bi < stages - 1; ++bi) {
                if (bi < nb) issue_stage(bi, bi);
                cp_async_commit();
            }
            // Q fragments (A operand, rows = heads): bf16 pairs, exact (q is bf16),
            // kept in shared memory ([D/16 steps][32 lanes][2 words]) to spare registers
            const int hr = lane >> 2, kc = (lane & 3) * 2;
            const uint2* qa = reinterpret_cast<const uint2*>(smem + L.qa);
            float o[D / 16][4];
    #pragma unroll
            for (int i = 0; i < D / 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
            float m_run = -INFINITY, l_run = 0.f;  // for head hr (row of Z)
            // [phase] 21
            int cs = 0;  // ring slot of tile bi
    #pragma unroll 1
            for (int bi = 0; bi < nb; ++bi) {
                if (bi + stages - 1 < nb) issue_stage(bi + stages - 1, cs == 0 ? stages - 1 : cs - 1);
                cp_async_commit();
                if (stages == 3) cp_async_wait<2>();
                else cp_async_wait<1>();
                __syncwarp();
                const uint8_t* st = ring + cs * kStageBytes;
                cs = cs + 1 == stages ? 0 : cs + 1;
                const int bt0 = (wid + bi * kNW) * TB8;
                // Z = Q K^T over D in 16-dim steps; one ldmatrix.x4 covers 32 dims
                float z[4] = {0.f, 0.f, 0.f, 0.f};
                const int mr = lane & 7, mi = lane >> 3;  // ldmatrix: row (token) and matrix index
    #pragma unroll
                for (int c4 = 0; c4 < D / 32; ++c4) {
                    uint32_t b[4];
                    ldmatrix_x4(b, st + mr * RB + (((4 * c4 + mi) ^ mr) << 4));
                    const uint2 q0 = qa[(2 * c4) * 32 + lane], q1 = qa[(2 * c4 + 1) * 32 + lane];
                    mma_bf16_16816(z, q0.x, 0u, q0.y, 0u, b[0], b[1]);
                    mma_bf16_16816(z, q1.x, 0u, q1.y, 0u, b[2], b[3]);
                }
                // online softmax for head hr over tokens kc, kc + 1 of the tile
                const bool ok0 = bt0 + kc < n_att, ok1 = bt0 + kc + 1 < n_att;
                const float z0 = ok0 ? z[0] * p.qscale : -INFINITY;
                const float z1 = ok1 ? z[1] * p.qscale : -INFINITY;
                float mx = fmaxf(z0, z1);
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                // The running max moves only when the tile's max exceeds it by
                // more than 2^kSlack (probabilities then stay below 2^kSlack): most
                // tiles leave it, and the rescale of O, alone. O and l share the
                // same max, so O / l is unchanged.
                constexpr float kSlack = 8.f;
                const bool move = mx > m_run + kSlack;
                const float m_new = move ? mx : m_run;
                const float corr = move ? exp2f(m_run - m_new) : 1.f;
                const float p0 = exp2f(z0 - m_new), p1 = exp2f(z1 - m_new);
                float rs = p0 + p1;
                rs += __shfl_xor_sync(0xffffffffu, rs, 1);
                rs += __shfl_xor_sync(0xffffffffu, rs, 2);
                l_run = l_run * corr + rs;
                m_run = m_new;
                if (__any_sync(0xffffffffu, move)) {
                    // O^T columns are heads kc, kc + 1: fetch their corrections
                    const float ca = __shfl_sync(0xffffffffu, corr, 4 * kc);
                    const float cb = __shfl_sync(0xffffffffu, corr, 4 * kc + 4);
    #pragma unroll
                    for (int i = 0; i < D / 16; ++i) { o[i][0] *= ca; o[i][1] *= cb; o[i][2] *= ca; o[i][3] *= cb; }
                }
                const uint32_t ph = pack_bf16x2(p0, p1);
                const uint32_t pl = pack_bf16x2(p0 - bf16lo(ph), p1 - bf16hi(ph));
                // O^T += V^T P^T; one ldmatrix.x4.trans covers two 16-dim row tiles
    #pragma unroll
                for (int m2 = 0; m2 < D / 32; ++m2) {
                    uint32_t a[4];
                    ldmatrix_x4_trans(a, st + (TB8 + mr) * RB + (((4 * m2 + mi) ^ mr) << 4));
                    mma_bf16_1688(o[2 * m2], a[0], a[1], ph);
                    mma_bf16_1688(o[2 * m2], a[0], a[1], pl);
                    mma_bf16_1688(o[2 * m2 + 1], a[2], a[3], ph);
                    mma_bf16_1688(o[2 * m2 + 1], a[2], a[3], pl);
                }
                __syncwarp();
            }
            cp_async_wait<0>();
            __syncwarp();
            // [phase] 7
            // per-warp partials -> the warp's own ring (its copies have all landed)
            wp_out = reinterpret_cast<float*>(ring);
    #pragma unroll
            for (int i = 0; i < D / 16; ++i) {
    #pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int h = kc + (e & 1), d = 16 * i + hr + ((e & 2) ? 8 : 0);
                    if (h < G) wp_out[h * (D + 2) + d] = o[i][e];
                }
            }
            if ((lane & 3) == 0 && hr < G) { wp_out[hr * (D + 2) + D] = m_run; wp_out[hr * (D + 2) + D + 1] = l_run; }
        } else {
            // fp32 K/V: CUDA cores. Each warp streams the K and V rows of its tokens
            // through a ring of kAttStagesF32 shared-memory stages with cp.async
            // (16-byte LDGSTS, no registers held while in flight), kAttStagesF32-1
            // stages ahead of compute; lane l holds dims [l*EPL, l*EPL + EPL).
            constexpr int kAttStages = kAttStagesF32;
            constexpr int TBS = att_stage_tokens(RB, E::kBytes);      // tokens per stage
            constexpr int kStageBytes = 2 * TBS * RB;
            constexpr int kPiecesPerRow = RB / 16;
            uint8_t* ring = smem + L.region + wid * att_ring_bytes(RB, E::kBytes, kAttStages);
            const int nb = n_att > wid * TBS ? (n_att - wid * TBS + kNW * TBS - 1) / (kNW * TBS) : 0;
            auto issue_stage = [&](int bi) {
                const int bt0 = (wid + bi * kNW) * TBS;
                uint8_t* st = ring + (bi % kAttStages) * kStageBytes;
                for (int pc = lane; pc < 2 * TBS * kPiecesPerRow; pc += 32) {
                    const int r = pc / kPiecesPerRow, off = (pc - r * kPiecesPerRow) * 16;
                    const int u = r < TBS ? r : r - TBS;
                    if (bt0 + u < n_att) {
                        const TKV* src = (r < TBS ? kb : vb) + att_row(bt0 + u) * D;
                        cp_async16(st + r * RB + off, reinterpret_cast<const uint8_t*>(src) + off);
                    }
                }
            };
    #pragma unroll 1
            for (int bi = 0; bi < kAttStages - 1; ++bi) {
                if (bi < nb) issue_stage(bi);
                cp_async_commit();
            }

            float qf[GT][EPL];
    #pragma unroll
            for (int h = 0; h < GT; ++h)
    #pragma unroll
                for (int e = 0; e < EPL; ++e)
                    qf[h][e] = h < G ? qs[h * D + lane * EPL + e] * p.qscale : 0.f;

            float m_run[GT], l_run[GT], o_run[GT][EPL];  // per query head of the group
    #pragma unroll
            for (int h = 0; h < GT; ++h) {
                m_run[h] = -INFINITY;
                l_run[h] = 0.f;
    #pragma unroll
                for (int e = 0; e < EPL; ++e) o_run[h][e] = 0.f;
            }

            // [phase] 21
    #pragma unroll 1
            for (int bi = 0; bi < nb; ++bi) {
                if (bi + kAttStages - 1 < nb) issue_stage(bi + kAttStages - 1);
                cp_async_commit();
                cp_async_wait<kAttStages - 1>();
                __syncwarp();
                const uint8_t* st = ring + (bi % kAttStages) * kStageBytes;
                const int bt0 = (wid + bi * kNW) * TBS;
                bool ok[TBS];
                float zt[TBS * GT];  // index u * GT + h
    #pragma unroll
                for (int u = 0; u < TBS; ++u) {
                    ok[u] = bt0 + u < n_att;
                    uint32_t kw[RBL / 4 > 0 ? RBL / 4 : 1];
                    lds_words<RBL>(kw, st + u * RB + lane * RBL);
                    float kf[EPL];
    #pragma unroll
                    for (int e = 0; e < EPL; ++e) {
                        if constexpr (E::kBytes == 2) kf[e] = (e & 1) ? bf16hi(kw[e >> 1]) : bf16lo(kw[e >> 1]);
                        else kf[e] = __uint_as_float(kw[e]);
                    }
    #pragma unroll
                    for (int h = 0; h < GT; ++h) {
                        float a = 0.f;
    #pragma unroll
                        for (int e = 0; e < EPL; ++e) a = fmaf(qf[h][e], kf[e], a);
                        zt[u * GT + h] = a;
                    }
                }
                warp_allreduce_n<TBS * GT>(zt);
    #pragma unroll
                for (int h = 0; h < GT; ++h) {
                    if (h >= G) break;
                    float mx = -INFINITY;
    #pragma unroll
                    for (int u = 0; u < TBS; ++u) if (ok[u]) mx = fmaxf(mx, zt[u * GT + h]);
                    const float m_new = fmaxf(m_run[h], mx);
                    const float corr = exp2f(m_run[h] - m_new);
                    float l = l_run[h] * corr;
    #pragma unroll
                    for (int e = 0; e < EPL; ++e) o_run[h][e] *= corr;
    #pragma unroll
                    for (int u = 0; u < TBS; ++u) {
                        if (!ok[u]) continue;
                        const float pr = exp2f(zt[u * GT + h] - m_new);
                        l += pr;
                        uint32_t vw[RBL / 4 > 0 ? RBL / 4 : 1];
                        lds_words<RBL>(vw, st + (TBS + u) * RB + lane * RBL);
    #pragma unroll
                        for (int e = 0; e < EPL; ++e) {
                            float vf;
                            if constexpr (E::kBytes == 2) vf = (e & 1) ? bf16hi(vw[e >> 1]) : bf16lo(vw[e >> 1]);
                            else vf = __uint_as_float(vw[e]);
                            o_run[h][e] = fmaf(pr, vf, o_run[h][e]);
                        }
                    }
                    m_run[h] = m_new;
                    l_run[h] = l;
                }
                __syncwarp();
            }
            cp_async_wait<0>();
            __syncwarp();

            // [phase] 7
            // per-warp partials -> the warp's own ring (its copies have all landed)
            wp_out = reinterpret_cast<float*>(ring);
            {
            float* wp = wp_out;
    #pragma unroll
            for (int h = 0; h < GT; ++h) {
                if (h >= G) break;
    #pragma unroll
                for (int e = 0; e < EPL; ++e) wp[h * (D + 2) + lane * EPL + e] = o_run[h][e];
                if (lane == 0) { wp[h * (D + 2) + D] = m_run[h]; wp[h * (D + 2) + D + 1] = l_run[h]; }
            }
        }
        }
    }
    __syncthreads();
    // merge the warps' states per head; a single-CTA row writes its output
    // here. In a cluster, CTA o owns the output elements [o*slice, ...): every
    // CTA pushes its partial o of those elements, and its (m, l) per head, into
    // the owner's shared memory (remote stores, no waiting), and after one
    // cluster barrier each owner merges its slice from local memory.
    const int slice = (G * D + N - 1) / N;
    // remote shared memory may only be written once every CTA of the cluster
    // is running: rows that skipped the selection have had no cluster barrier yet
    if (N > 1 && select_all) row_sync(cluster, N);
    for (int e = tid; e < G * D; e += kNT) {
        const int h = e / D, d = e - h * D;
        float M = -INFINITY;
        auto wpart = [&](int w) -> const float* {
            return reinterpret_cast<const float*>(smem + L.region + w * att_ring_bytes(RB, E::kBytes, p.att_stages)) +
                   h * (D + 2);
        };
        for (int w = 0; w < kNW; ++w) M = fmaxf(M, wpart(w)[D]);
        float O = 0.f, Lsum = 0.f;
        if (M != -INFINITY) {
            for (int w = 0; w < kNW; ++w) {
                const float* wp = wpart(w);
                const float f = exp2f(wp[D] - M);
                O = fmaf(f, wp[d], O);
                Lsum = fmaf(f, wp[D + 1], Lsum);
            }
        }
        if (N == 1) {
            write_out(h, d, O / Lsum);
        } else {
            const int own = e / slice;
            row_smem(cluster, N, co, own)[rank * slice + (e - own * slice)] = O;
            if (d == 0)
                for (int r = 0; r < N; ++r) {
                    row_smem(cluster, N, cm, r)[rank * GT + h] = M;
                    row_smem(cluster, N, cl, r)[rank * GT + h] = Lsum;
                }
        }
    }
    if (N > 1) {
        // [phase] 8
        row_sync(cluster, N);                                        // all partials delivered
        const int e0 = rank * slice, e1 = min(G * D, e0 + slice);
        for (int e = e0 + tid; e < e1; e += kNT) {
            const int h = e / D, d = e - h * D;
            float M = -INFINITY;
            for (int r = 0; r < N; ++r) M = fmaxf(M, cm[r * GT + h]);
            float O = 0.f, Lsum = 0.f;
            for (int r = 0; r < N; ++r) {
                const float mr = cm[r * GT + h];
                if (mr == -INFINITY) continue;
                const float f = exp2f(mr - M);
                O = fmaf(f, co[r * slice + (e - e0)], O);
                Lsum = fmaf(f, cl[r * GT + h], Lsum);
            }
            write_out(h, d, O / Lsum);
        }
    }
    // [phase] 9
}

}  // namespace ds
