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
    void* out;
    int32_t* sel_out;
    float* score_out;
    int hkv, G, s, s_cap, topk;
    int chunk;     // tokens per CTA, multiple of 32
    int lay_chunk; // chunk used to size shared memory (0 in dense mode)
    int per;       // selected tokens attended per CTA (ceil(min(topk,s) / N))
    float qscale;  // sm_scale * log2(e)
    int out_bf16;
    int dense;     // 1: attend every token, no label / scores / selection
};

// Shared-memory carve-up (bytes), identical on host and device.
struct DecodeSmem {
    int qs, qL, idx, histA, histB, ctl, scan, cm, cl, co, bits, sel, region, total;
};

__host__ __device__ inline int align16(int x) { return (x + 15) & ~15; }

__host__ __device__ inline DecodeSmem decode_smem_layout(int GT, int D, int C, int chunk, int per) {
    DecodeSmem L;
    int o = 0;
    L.qs = o;     o += align16(GT * D * 4);
    L.qL = o;     o += align16(C * 4);
    L.idx = o;    o += align16(C * 4);
    L.histA = o;  o += 256 * 4;
    L.histB = o;  o += 256 * 4;
    L.ctl = o;    o += 64 * 4;
    L.scan = o;   o += align16((kNW + 1) * 4);
    L.cm = o;     o += align16(GT * 4);
    L.cl = o;     o += align16(GT * 4);
    L.co = o;     o += align16(GT * D * 4);
    L.bits = o;   o += align16((chunk / 32) * 4);
    L.sel = o;    o += align16(per * 4);
    L.region = o;
    const int keys = chunk * 2;
    const int parts = kNW * GT * (D + 2) * 4;
    o += align16(keys > parts ? keys : parts);
    L.total = o;
    return L;
}

// ctl[] slots
enum { kCtlBin = 0, kCtlNeed = 1, kCtlCnt = 2, kCtlCS = 4, kCtlCT = 5, kCtlP = 6, kCtlTP = 7 };

// Row geometry of the label cache.
template <typename TKV, int LK, int C>
struct LabelGeom {
    static constexpr int kBytes = (LK == kLabelInt4) ? C / 2 : C * Elem<TKV>::kBytes;
    static constexpr int kWords = kBytes / 4;
    // tokens in flight per thread in the scoring loop (~128 B per thread)
    static constexpr int kU = (128 / kBytes) < 1 ? 1 : ((128 / kBytes) > 8 ? 8 : (128 / kBytes));
};

// fp32 score of one token from its label row (step 2). The arithmetic is a
// fixed chain of fused multiply-adds in channel order, so scoring the same
// row twice gives bit-identical results.
template <typename TKV, int LK, int C>
__device__ __forceinline__ float label_score(const uint32_t (&w)[LabelGeom<TKV, LK, C>::kWords],
                                             const float* qreg, const float* qsm, float sc, float z,
                                             float qsum) {
    constexpr bool kReg = C <= 32;
    auto ql = [&](int j) -> float { return kReg ? qreg[j] : qsm[j]; };
    float acc = 0.f;
    if constexpr (LK == kLabelInt4) {
#pragma unroll
        for (int i = 0; i < C / 8; ++i) {
            const uint32_t x = w[i];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                // nibble -> float exactly: 2^23 + n has n in its low mantissa bits
                const float n = __uint_as_float(0x4B000000u | ((x >> (4 * e)) & 15u)) - 8388608.0f;
                acc = __fmaf_rn(ql(8 * i + e), n, acc);
            }
        }
        // sum_j qL[j] * (sc * n_j + z) = sc * sum_j qL[j] n_j + z * sum_j qL[j]
        return __fmaf_rn(sc, acc, __fmul_rn(z, qsum));
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

// Warp-aggregated histogram increment; bin >= 256 means "no count". Must be
// called by all 32 lanes.
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin) {
    const uint32_t peers = __match_any_sync(0xffffffffu, bin);
    const int leader = __ffs(peers) - 1;
    if (lane_id() == leader && bin < 256u) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
}

// Sum a 256-bin histogram over the cluster (DSMEM) and find the bin holding
// the `need`-th largest key. Writes ctl[kCtlBin], ctl[kCtlNeed] (how many to
// take from that bin) and ctl[kCtlCnt] (the bin's size). Requires a cluster
// barrier before (histograms complete); ends with __syncthreads().
__device__ __forceinline__ void cluster_select_bin(cg::cluster_group& cluster, uint32_t* hist,
                                                   int nblocks, uint32_t need, int* ctl,
                                                   uint32_t* scan) {
    const int tid = threadIdx.x;
    const int bin = 255 - tid;  // thread 0 holds the largest bin
    uint32_t cnt = 0;
    for (int r = 0; r < nblocks; ++r) cnt += cluster.map_shared_rank(hist, r)[bin];
    uint32_t total;
    const uint32_t excl = block_excl_scan<kNT>(cnt, scan, &total);
    if (excl < need && need <= excl + cnt) {
        ctl[kCtlBin] = bin;
        ctl[kCtlNeed] = (int)(need - excl);
        ctl[kCtlCnt] = (int)cnt;
    }
    __syncthreads();
}

template <typename TKV, int LK, int D, int C, int GT>
__global__ void __launch_bounds__(kNT, 2) ds_decode_kernel(const DecodeParams p) {
    using E = Elem<TKV>;
    using LG = LabelGeom<TKV, LK, C>;
    constexpr int EPL = D / 32;                       // elements of a K/V row per lane
    constexpr int RBL = EPL * E::kBytes;              // bytes of a K/V row per lane
    // tokens per warp batch: ~64 B of K plus 64 B of V in flight per lane,
    // fewer when several query heads share the kv head (registers)
    constexpr int TB0 = (64 / RBL) < 4 ? 4 : ((64 / RBL) > 8 ? 8 : (64 / RBL));
    constexpr int TB = GT >= 8 ? (TB0 / 4 < 2 ? 2 : TB0 / 4) : GT >= 4 ? (TB0 / 2 < 2 ? 2 : TB0 / 2) : TB0;
    static_assert(EPL * 32 == D, "D must be a multiple of 32");

    cg::cluster_group cluster = cg::this_cluster();
    const int N = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    const int row = blockIdx.x / N;  // = b * hkv + g
    const int g = row % p.hkv;
    const int G = p.G;
    const int tid = threadIdx.x, lane = lane_id(), wid = warp_id();

    extern __shared__ __align__(16) uint8_t smem[];
    const DecodeSmem L = decode_smem_layout(GT, D, C, p.lay_chunk, p.per);
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
    uint32_t* bits = reinterpret_cast<uint32_t*>(smem + L.bits);
    int* sel_list = reinterpret_cast<int*>(smem + L.sel);
    uint16_t* keys = reinterpret_cast<uint16_t*>(smem + L.region);
    float* wpart = reinterpret_cast<float*>(smem + L.region);  // after compaction

    const int s = p.s;
    const int t0 = rank * p.chunk;
    const int n_loc = max(0, min(s, t0 + p.chunk) - t0);
    const size_t row_tok = (size_t)row * (size_t)p.s_cap;  // first token of this row in the caches
    const TKV* qrow = reinterpret_cast<const TKV*>(p.q) + (size_t)row * G * D;
    const int k_eff = min(p.topk, s);
    const bool select_all = p.dense || p.topk >= s;

    // ---------------------------------------------------------- setup, step 1
    for (int e = tid; e < G * D; e += kNT) qs[e] = E::to_f32(qrow[e]);
    if (!p.dense) {
        for (int j = tid; j < C; j += kNT) idx_s[j] = min(max(p.idx[(size_t)g * C + j], 0), D - 1);
        histA[tid] = 0u;
        histB[tid] = 0u;
        for (int e = tid; e < p.lay_chunk / 32; e += kNT) bits[e] = 0u;
    }
    __syncthreads();
    if (!p.dense) {
        for (int j = tid; j < C; j += kNT) {
            float a = 0.f;
            for (int e = 0; e < G; ++e) a += qs[e * D + idx_s[j]];
            qLs[j] = a;
        }
    }
    __syncthreads();

    const uint8_t* lab = reinterpret_cast<const uint8_t*>(p.label) + row_tok * LG::kBytes;
    const uint16_t* lsc = (LK == kLabelInt4) ? p.lscale + row_tok : nullptr;
    const uint16_t* lze = (LK == kLabelInt4) ? p.lzero + row_tok : nullptr;
    float qreg[C <= 32 ? C : 1];
    float qsum = 0.f;

    // Score of token t (absolute index in the row) straight from global memory;
    // same arithmetic as the streaming loop below.
    auto rescore = [&](int t) -> float {
        uint32_t w[LG::kWords];
        load_words<LG::kBytes>(w, lab + (size_t)t * LG::kBytes);
        float sc = 0.f, z = 0.f;
        if constexpr (LK == kLabelInt4) {
            sc = fp16_bits_to_f32(ldg_u16(lsc + t));
            z = fp16_bits_to_f32(ldg_u16(lze + t));
        }
        return label_score<TKV, LK, C>(w, qreg, qLs, sc, z, qsum);
    };

    if (!select_all) {
        if constexpr (C <= 32) {
#pragma unroll
            for (int j = 0; j < C; ++j) qreg[j] = qLs[j];
        }
        for (int j = 0; j < C; ++j) qsum += qLs[j];
    }

    // ---------------------------------------------------------------- step 2
    if (!p.dense && (!select_all || p.score_out != nullptr)) {
        constexpr int U = LG::kU;
        for (int base = 0; base < n_loc; base += kNT * U) {
            uint32_t w[U][LG::kWords];
            float sc[U], z[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = base + u * kNT + tid;
                if (i < n_loc) {
                    load_words<LG::kBytes>(w[u], lab + (size_t)(t0 + i) * LG::kBytes);
                    if constexpr (LK == kLabelInt4) {
                        sc[u] = fp16_bits_to_f32(ldg_u16(lsc + t0 + i));
                        z[u] = fp16_bits_to_f32(ldg_u16(lze + t0 + i));
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = base + u * kNT + tid;
                const bool valid = i < n_loc;
                uint32_t bin = 256u;
                if (valid) {
                    float zz = 0.f, ss = 0.f;
                    if constexpr (LK == kLabelInt4) { ss = sc[u]; zz = z[u]; }
                    const float sv = label_score<TKV, LK, C>(w[u], qreg, qLs, ss, zz, qsum);
                    const uint32_t key = score_key(sv);
                    if (!select_all) {
                        keys[i] = (uint16_t)(key >> 16);
                        bin = key >> 24;
                    }
                    if (p.score_out) p.score_out[(size_t)row * s + t0 + i] = sv;
                }
                if (!select_all) hist_add(histA, bin);
            }
        }
    }

    // --------------------------------------------------------------- step 3a
    int T16 = 0, Tlo = 0, r_tie = 0;
    bool refine = false;
    if (!select_all) {
        cluster.sync();                                        // histograms A complete
        cluster_select_bin(cluster, histA, N, (uint32_t)k_eff, ctl, scan);
        const int bA = ctl[kCtlBin];
        const int needA = ctl[kCtlNeed];
        for (int base = 0; base < n_loc; base += kNT) {
            const int i = base + tid;
            uint32_t bin = 256u;
            if (i < n_loc) {
                const uint32_t k16 = keys[i];
                if ((int)(k16 >> 8) == bA) bin = k16 & 255u;
            }
            hist_add(histB, bin);
        }
        cluster.sync();                                        // histograms B complete
        cluster_select_bin(cluster, histB, N, (uint32_t)needA, ctl, scan);
        T16 = (bA << 8) | ctl[kCtlBin];
        const int needB = ctl[kCtlNeed];
        refine = needB < ctl[kCtlCnt];
        if (refine) {
            // the k-th key's 16-bit bucket is split: re-score its tokens exactly
            histA[tid] = 0u;
            __syncthreads();
            for (int base = 0; base < n_loc; base += kNT) {
                const int i = base + tid;
                bool inb = false;
                uint32_t bin = 256u;
                if (i < n_loc && (int)keys[i] == T16) {
                    inb = true;
                    const uint32_t low = score_key(rescore(t0 + i)) & 0xFFFFu;
                    keys[i] = (uint16_t)low;
                    bin = low >> 8;
                }
                const uint32_t m = __ballot_sync(0xffffffffu, inb);
                if (lane == 0 && (base + wid * 32) < n_loc) bits[(base + wid * 32) >> 5] = m;
                hist_add(histA, bin);
            }
            cluster.sync();                                    // histograms C complete
            cluster_select_bin(cluster, histA, N, (uint32_t)needB, ctl, scan);
            const int bC = ctl[kCtlBin];
            const int needC = ctl[kCtlNeed];
            histB[tid] = 0u;
            __syncthreads();
            for (int base = 0; base < n_loc; base += kNT) {
                const int i = base + tid;
                uint32_t bin = 256u;
                if (i < n_loc && ((bits[i >> 5] >> (i & 31)) & 1u)) {
                    const uint32_t low = keys[i];
                    if ((int)(low >> 8) == bC) bin = low & 255u;
                }
                hist_add(histB, bin);
            }
            cluster.sync();                                    // histograms D complete
            cluster_select_bin(cluster, histB, N, (uint32_t)needC, ctl, scan);
            Tlo = (bC << 8) | ctl[kCtlBin];
            r_tie = ctl[kCtlNeed];
        }

        // ----------------------------------------------------- compaction
        // classes: 1 = selected outright, 2 = exact tie with the k-th key
        const int run = (n_loc + kNT - 1) / kNT;
        const int i0 = min(n_loc, tid * run), i1 = min(n_loc, i0 + run);
        auto klass = [&](int i) -> int {
            const int k16 = keys[i];
            if (!refine) return k16 >= T16 ? 1 : 0;
            if ((bits[i >> 5] >> (i & 31)) & 1u) return k16 > Tlo ? 1 : (k16 == Tlo ? 2 : 0);
            return k16 > T16 ? 1 : 0;
        };
        uint32_t ns = 0, nt = 0;
        for (int i = i0; i < i1; ++i) {
            const int c = klass(i);
            ns += c == 1;
            nt += c == 2;
        }
        uint32_t tot;
        const uint32_t ex = block_excl_scan<kNT>((ns << 16) | nt, scan, &tot);
        if (tid == 0) { ctl[kCtlCS] = (int)(tot >> 16); ctl[kCtlCT] = (int)(tot & 0xFFFFu); }
        cluster.sync();                                        // per-CTA counts visible
        if (wid == 0) {
            int cs = 0, ct = 0;
            if (lane < N) {
                const int* rc = cluster.map_shared_rank(ctl, lane);
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
        const int P = ctl[kCtlP], TP = ctl[kCtlTP];
        const int ex_s = (int)(ex >> 16), ex_t = (int)(ex & 0xFFFFu);
        int pos = P + ex_s + (refine ? max(0, min(ex_t, r_tie - TP)) : 0);
        int tie_rank = TP + ex_t;
        const int per = p.per;
        for (int i = i0; i < i1; ++i) {
            const int c = klass(i);
            bool take = c == 1;
            if (c == 2) { take = tie_rank < r_tie; ++tie_rank; }
            if (take) {
                const int dst = pos / per;
                int* rl = cluster.map_shared_rank(sel_list, dst);
                rl[pos - dst * per] = t0 + i;
                if (p.sel_out) p.sel_out[(size_t)row * p.topk + pos] = t0 + i;
                ++pos;
            }
        }
        cluster.sync();                                        // selection lists complete
    } else if (p.sel_out) {
        for (int i = tid; i < n_loc; i += kNT) p.sel_out[(size_t)row * p.topk + t0 + i] = t0 + i;
        if (rank == 0)
            for (int j = s + tid; j < p.topk; j += kNT) p.sel_out[(size_t)row * p.topk + j] = -1;
    }

    // --------------------------------------------------------------- step 3b
    const int n_att = select_all ? n_loc : max(0, min(p.per, k_eff - rank * p.per));
    const TKV* kb = reinterpret_cast<const TKV*>(p.k) + row_tok * D;
    const TKV* vb = reinterpret_cast<const TKV*>(p.v) + row_tok * D;

    float qf[GT][EPL];
#pragma unroll
    for (int h = 0; h < GT; ++h)
#pragma unroll
        for (int e = 0; e < EPL; ++e)
            qf[h][e] = h < G ? qs[h * D + lane * EPL + e] * p.qscale : 0.f;

    float m_run[GT], l_run[GT], o_run[GT][EPL];
#pragma unroll
    for (int h = 0; h < GT; ++h) {
        m_run[h] = -INFINITY;
        l_run[h] = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) o_run[h][e] = 0.f;
    }

    for (int bt = wid * TB; bt < n_att; bt += kNW * TB) {
        uint32_t kw[TB][RBL / 4 > 0 ? RBL / 4 : 1], vw[TB][RBL / 4 > 0 ? RBL / 4 : 1];
        bool ok[TB];
#pragma unroll
        for (int u = 0; u < TB; ++u) {
            const int j = bt + u;
            ok[u] = j < n_att;
            if (ok[u]) {
                const int t = select_all ? t0 + j : sel_list[j];
                load_words<RBL>(kw[u], reinterpret_cast<const uint8_t*>(kb + (size_t)t * D + lane * EPL));
                load_words<RBL>(vw[u], reinterpret_cast<const uint8_t*>(vb + (size_t)t * D + lane * EPL));
            } else {
#pragma unroll
                for (int e = 0; e < RBL / 4; ++e) { kw[u][e] = 0u; vw[u][e] = 0u; }
            }
        }
        float zt[TB][GT];
#pragma unroll
        for (int u = 0; u < TB; ++u) {
            float kf[EPL];
#pragma unroll
            for (int e = 0; e < EPL; ++e) {
                if constexpr (E::kBytes == 2) kf[e] = (e & 1) ? bf16hi(kw[u][e >> 1]) : bf16lo(kw[u][e >> 1]);
                else kf[e] = __uint_as_float(kw[u][e]);
            }
#pragma unroll
            for (int h = 0; h < GT; ++h) {
                float a = 0.f;
#pragma unroll
                for (int e = 0; e < EPL; ++e) a = fmaf(qf[h][e], kf[e], a);
                zt[u][h] = warp_sum(a);
            }
        }
#pragma unroll
        for (int h = 0; h < GT; ++h) {
            if (h >= G) break;
            float mx = -INFINITY;
#pragma unroll
            for (int u = 0; u < TB; ++u) if (ok[u]) mx = fmaxf(mx, zt[u][h]);
            const float m_new = fmaxf(m_run[h], mx);
            const float corr = exp2f(m_run[h] - m_new);
            float l = l_run[h] * corr;
#pragma unroll
            for (int e = 0; e < EPL; ++e) o_run[h][e] *= corr;
#pragma unroll
            for (int u = 0; u < TB; ++u) {
                if (!ok[u]) continue;
                const float pr = exp2f(zt[u][h] - m_new);
                l += pr;
#pragma unroll
                for (int e = 0; e < EPL; ++e) {
                    float vf;
                    if constexpr (E::kBytes == 2) vf = (e & 1) ? bf16hi(vw[u][e >> 1]) : bf16lo(vw[u][e >> 1]);
                    else vf = __uint_as_float(vw[u][e]);
                    o_run[h][e] = fmaf(pr, vf, o_run[h][e]);
                }
            }
            m_run[h] = m_new;
            l_run[h] = l;
        }
    }

    // per-warp partials -> shared memory (the key region is free now)
    {
        float* wp = wpart + (size_t)wid * GT * (D + 2);
#pragma unroll
        for (int h = 0; h < GT; ++h) {
            if (h >= G) break;
#pragma unroll
            for (int e = 0; e < EPL; ++e) wp[h * (D + 2) + lane * EPL + e] = o_run[h][e];
            if (lane == 0) { wp[h * (D + 2) + D] = m_run[h]; wp[h * (D + 2) + D + 1] = l_run[h]; }
        }
    }
    __syncthreads();
    for (int e = tid; e < G * D; e += kNT) {
        const int h = e / D, d = e - h * D;
        float M = -INFINITY;
        for (int w = 0; w < kNW; ++w) M = fmaxf(M, wpart[(w * GT + h) * (D + 2) + D]);
        float O = 0.f, Lsum = 0.f;
        if (M != -INFINITY) {
            for (int w = 0; w < kNW; ++w) {
                const float* wp = wpart + (w * GT + h) * (D + 2);
                const float f = exp2f(wp[D] - M);
                O = fmaf(f, wp[d], O);
                Lsum = fmaf(f, wp[D + 1], Lsum);
            }
        }
        co[h * D + d] = O;
        if (d == 0) { cm[h] = M; cl[h] = Lsum; }
    }
    cluster.sync();                                            // CTA partials visible

    // final merge across the cluster; CTA `rank` writes its slice of [G, D]
    {
        const int E_all = G * D;
        const int slice = (E_all + N - 1) / N;
        const int e0 = rank * slice, e1 = min(E_all, e0 + slice);
        for (int e = e0 + tid; e < e1; e += kNT) {
            const int h = e / D, d = e - h * D;
            float M = -INFINITY;
            for (int r = 0; r < N; ++r) M = fmaxf(M, cluster.map_shared_rank(cm, r)[h]);
            float O = 0.f, Lsum = 0.f;
            for (int r = 0; r < N; ++r) {
                const float mr = cluster.map_shared_rank(cm, r)[h];
                if (mr == -INFINITY) continue;
                const float f = exp2f(mr - M);
                O = fmaf(f, cluster.map_shared_rank(co, r)[h * D + d], O);
                Lsum = fmaf(f, cluster.map_shared_rank(cl, r)[h], Lsum);
            }
            const float res = O / Lsum;
            const size_t oidx = (size_t)row * G * D + (size_t)h * D + d;
            if (p.out_bf16) reinterpret_cast<uint16_t*>(p.out)[oidx] = f32_to_bf16_bits(res);
            else reinterpret_cast<float*>(p.out)[oidx] = res;
        }
    }
    cluster.sync();                                            // keep smem alive for readers
}

}  // namespace ds
