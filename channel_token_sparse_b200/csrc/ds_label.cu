// ds_label.cu -- label-cache build (prefill) and append (decode) for sm_100a.
//
// "大模型稀疏化技术原理：Double Sparsity" (joto.ai), section 离线校准: at prefill
// every token's heavy key channels are copied from the key cache into the
// contiguous label cache; at each decode step only the new token's channels
// are added. The cache may be kept in 4 bits.
//
// Two kernels. Prefill builds over a dense key cache with enough work for
// every resident CTA run ds_label_bulk_kernel: persistent CTAs stream 16 KiB
// blocks of key rows through a shared-memory ring filled by 1-D bulk copies.
// Appends, paged caches and small builds run ds_label_kernel: one CTA
// handles kTokens consecutive tokens of one (b, kv head) row, staging the key
// rows in shared memory with coalesced 16-byte loads. Both then produce each
// label element (fp) or each token's 4-bit codes from shared memory.
// The key cache is dense [b, hkv, s_cap, d] or paged (a block table maps
// token t of entry b to a row of a [num_blocks, hkv, page, d] pool); the
// label cache is always dense [b, hkv, s_cap, c].
#include "ds_common.cuh"
#include "ds_internal.h"

namespace ds {

constexpr int kLabNT = 256;
constexpr int kTokens = 64;

template <typename TKV, int LK, int D>
__global__ void __launch_bounds__(kLabNT) ds_label_kernel(const TKV* __restrict__ k,
                                                          const int32_t* __restrict__ idx, int hkv,
                                                          int t_begin, int t_end, int s_cap, int c,
                                                          uint8_t* __restrict__ label,
                                                          uint16_t* __restrict__ lscale,
                                                          uint16_t* __restrict__ lzero,
                                                          const int32_t* __restrict__ block_table,
                                                          int max_blocks, int page_shift, int num_blocks) {
    using E = Elem<TKV>;
    __shared__ __align__(16) TKV rows[kTokens * D];
    __shared__ int idx_s[128];
    const int row = blockIdx.y;  // b * hkv + g
    const int g = row % hkv;
    const int tb = t_begin + blockIdx.x * kTokens;
    const int nt = min(kTokens, t_end - tb);
    if (nt <= 0) return;
    for (int j = threadIdx.x; j < c; j += kLabNT) idx_s[j] = min(max(idx[(size_t)g * c + j], 0), D - 1);

    const size_t tok0 = (size_t)row * s_cap + tb;
    constexpr int kVecPerRow = D * E::kBytes / 16;
    uint4* dst = reinterpret_cast<uint4*>(rows);
    if (!block_table) {
        const uint4* src = reinterpret_cast<const uint4*>(k + tok0 * D);
        for (int e = threadIdx.x; e < nt * kVecPerRow; e += kLabNT) dst[e] = ldg_stream16(src + e);
    } else {
        const int32_t* bt = block_table + (size_t)(row / hkv) * max_blocks;
        const int pmask = (1 << page_shift) - 1;
        for (int e = threadIdx.x; e < nt * kVecPerRow; e += kLabNT) {
            const int t = tb + e / kVecPerRow;
            const int blk = min(max(__ldg(bt + (t >> page_shift)), 0), num_blocks - 1);
            const size_t r = (((size_t)blk * hkv + g) << page_shift) + (size_t)(t & pmask);
            dst[e] = ldg_stream16(reinterpret_cast<const uint4*>(k + r * D) + e % kVecPerRow);
        }
    }
    __syncthreads();

    if constexpr (LK == 0) {
        TKV* out = reinterpret_cast<TKV*>(label) + tok0 * c;
        for (int e = threadIdx.x; e < nt * c; e += kLabNT) {
            const int t = e / c, j = e - t * c;
            out[e] = rows[t * D + idx_s[j]];
        }
    } else {
        // 4-bit: one thread per token (pack_int4_row states the arithmetic)
        for (int t = threadIdx.x; t < nt; t += kLabNT)
            pack_int4_row<TKV>(rows + t * D, idx_s, c, label + (tok0 + t) * (size_t)(c / 2), lscale + tok0 + t,
                               lzero + tok0 + t);
    }
}

// Dense key cache, many tokens (prefill): persistent CTAs stream blocks of
// consecutive key rows -- one contiguous span of kBulkStage bytes per
// (row, block) item -- through a kBulkStages-deep shared-memory ring with 1-D
// bulk copies (thread 0 issues them; an mbarrier per stage counts the bytes
// in), so the next blocks' reads are in flight while the current one is
// gathered or packed. Same results as ds_label_kernel.
constexpr int kBulkStage = 16384;  // bytes of key rows per stage
constexpr int kBulkStages = 4;
constexpr int kBulkCtasPerSm = 3;  // 3 x (4 x 16 KiB) of ring per SM; <= 85 registers
constexpr int kBulkNT = 256;
// packing threads per token (4-bit): each takes c / kPackLanes channels
constexpr int kPackLanes = 4;

__host__ __device__ constexpr int bulk_smem_bytes() { return kBulkStages * kBulkStage + kBulkStages * 8; }

// A CTA's items are blockIdx.x, blockIdx.x + gridDim.x, ... in (row, block)
// order; the cursor steps to the next one with adds and one carry instead of
// a division per item.
struct ItemCursor {
    int row, blk, g;            // current item: row = b * hkv + g, block of the row
    int rstep, bstep, gstep;    // gridDim.x = rstep * nblk + bstep; gstep = rstep % hkv
    int nblk, hkv;
    __device__ __forceinline__ void init(int first, int grid, int nblk_, int hkv_) {
        nblk = nblk_;
        hkv = hkv_;
        row = first / nblk;
        blk = first - row * nblk;
        g = row % hkv;
        rstep = grid / nblk;
        bstep = grid - rstep * nblk;
        gstep = rstep % hkv;
    }
    __device__ __forceinline__ void next() {
        blk += bstep;
        row += rstep;
        g += gstep;
        if (blk >= nblk) {
            blk -= nblk;
            ++row;
            ++g;
        }
        if (g >= hkv) g -= hkv;
    }
};

// 4-bit codes of n values a_e = x_e - zero: the quotient a_e / scale is
// formed with the rounded reciprocal and rounded to an integer r (half to
// even); only where it lies within about 1e-5 of a half-integer (|q - r| near
// 0.5, where the product and the IEEE quotient could round differently) is it
// recomputed with the IEEE division. The code is r clamped to [0, 15] (NaN
// gives 0); the codes equal those of int4_code.
template <int N>
__device__ __forceinline__ void int4_codes(const float (&a)[N], float sc, float rcp_sc, uint32_t (&code)[N]) {
    constexpr float kNear = 0.5f - 1e-5f;
    float r[N];
    bool near = false;
#pragma unroll
    for (int e = 0; e < N; ++e) {
        const float q = __fmul_rn(a[e], rcp_sc);
        r[e] = rintf(q);
        near |= fabsf(q - r[e]) >= kNear;
    }
    if (near) {
#pragma unroll
        for (int e = 0; e < N; ++e) {
            const float q = __fmul_rn(a[e], rcp_sc);
            if (fabsf(q - rintf(q)) >= kNear) r[e] = rintf(__fdiv_rn(a[e], sc));
        }
    }
#pragma unroll
    for (int e = 0; e < N; ++e) code[e] = (uint32_t)fminf(fmaxf(r[e], 0.f), 15.f);
}

// Pick element (p - r) & 3 of a: the value a rotated thread read for output
// position p.
__device__ __forceinline__ uint32_t pick_rot(const uint32_t (&a)[4], int p, int r) {
    const int e = (p - r) & 3;
    return e == 0 ? a[0] : (e == 1 ? a[1] : (e == 2 ? a[2] : a[3]));
}

// CI: the channel count, fixed at compile time, so the per-thread channel
// lists stay in registers and the token / channel arithmetic is shifts.
//
// fp rows: a thread writes 4 consecutive label elements of one token (one
// 8-byte store for bf16, 16 bytes for fp32). The tokens a warp covers lie a
// multiple of 128 bytes apart in the ring, so one channel of each of them
// falls in the same bank: each thread reads its 4 channels rotated by its
// token index (t & 3) and rotates the values back, so at each step the
// warp's tokens read different channels.
// 4-bit rows: kPackLanes threads per token with CI / kPackLanes channels
// each, rotated the same way by the token's slot in the warp; the arithmetic
// is that of pack_int4_row, with mn / mx combined over the lanes (fminf /
// fmaxf do not depend on the order).
template <typename TKV, int LK, int D, int CI>
__global__ void __launch_bounds__(kBulkNT, kBulkCtasPerSm) ds_label_bulk_kernel(const TKV* __restrict__ k,
                                                                  const int32_t* __restrict__ idx, int hkv,
                                                                  int t_begin, int t_end, int s_cap, int rows,
                                                                  uint8_t* __restrict__ label,
                                                                  uint16_t* __restrict__ lscale,
                                                                  uint16_t* __restrict__ lzero,
                                                                  unsigned int* __restrict__ err) {
    using E = Elem<TKV>;
    constexpr int kRowBytes = D * E::kBytes;
    constexpr int kTok = kBulkStage / kRowBytes;  // tokens per stage
    extern __shared__ __align__(128) uint8_t sm[];
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + kBulkStages * kBulkStage);
    const int tid = threadIdx.x;
    const int nblk = (t_end - t_begin + kTok - 1) / kTok;  // blocks per row
    const int items = rows * nblk;                          // below 2^30 (checked by the host)
    if (tid == 0) {
        for (int i = 0; i < kBulkStages; ++i) mbar_init(&full[i], 1);
        fence_mbar_init();
    }
    __syncthreads();
    // producer (thread 0): the item kBulkStages ahead of the consumer's
    ItemCursor pc{};
    int pit = blockIdx.x;
    auto issue = [&](int slot) {
        const int tb = t_begin + pc.blk * kTok;
        const int nt = min(kTok, t_end - tb);
        const uint32_t bytes = (uint32_t)(nt * kRowBytes);
        mbar_arrive_expect_tx(&full[slot], bytes);
        bulk_g2s(sm + slot * kBulkStage, k + ((size_t)pc.row * s_cap + tb) * D, bytes, &full[slot]);
        pit += gridDim.x;
        pc.next();
    };
    if (tid == 0) {
        pc.init(blockIdx.x, gridDim.x, nblk, hkv);
        for (int i = 0; i < kBulkStages && pit < items; ++i) issue(i);
    }

    constexpr int kG = CI / 4;                  // fp: 4-element groups per label row
    const int fq = tid % kG, frot = (tid / kG) & 3;
    // fp, bf16: byte selectors that rotate 4 packed 16-bit values left by frot
    const uint32_t sel_lo = ((0u - 2 * frot) & 7) | (((1u - 2 * frot) & 7) << 4) | (((2u - 2 * frot) & 7) << 8) |
                            (((3u - 2 * frot) & 7) << 12);
    const uint32_t sel_hi = ((4u - 2 * frot) & 7) | (((5u - 2 * frot) & 7) << 4) | (((6u - 2 * frot) & 7) << 8) |
                            (((7u - 2 * frot) & 7) << 12);
    constexpr int kPer = CI / kPackLanes > 0 ? CI / kPackLanes : 1;  // 4-bit: channels per lane
    constexpr bool kRot = kPer <= 16;  // a lane's nibbles fit one 64-bit word
    const int q4 = tid % kPackLanes;
    const int rot = kRot ? (tid / kPackLanes) % kPer : 0;
    constexpr int kOff = LK == 0 ? 4 : kPer;
    int off[kOff];  // this thread's channels, in its rotated order
    int g_cur = -1;
    ItemCursor cc;
    cc.init(blockIdx.x, gridDim.x, nblk, hkv);
    for (int it = blockIdx.x, j = 0; it < items; it += gridDim.x, ++j, cc.next()) {
        const int slot = j % kBulkStages;
        const int tb = t_begin + cc.blk * kTok;
        const int nt = min(kTok, t_end - tb);
        const size_t tok0 = (size_t)cc.row * s_cap + tb;
        if (cc.g != g_cur) {
            g_cur = cc.g;
            const int32_t* ig = idx + (size_t)g_cur * CI;
#pragma unroll
            for (int e = 0; e < kOff; ++e) {
                const int ch = LK == 0 ? 4 * fq + ((e + frot) & 3) : q4 * kPer + ((e + rot) % kPer);
                off[e] = min(max(__ldg(ig + ch), 0), D - 1);
            }
        }
        const bool ok = mbar_wait_bounded(&full[slot], (uint32_t)((j / kBulkStages) & 1), err, 1);
        if (ok) {
            if constexpr (LK == 0) {
                if constexpr (E::kBytes == 2) {
                    const uint16_t* rs = reinterpret_cast<const uint16_t*>(sm + slot * kBulkStage);
                    uint16_t* out = reinterpret_cast<uint16_t*>(label) + tok0 * CI + 4 * fq;
                    for (int t = tid / kG; t < nt; t += kBulkNT / kG) {
                        const uint16_t* x = rs + t * D;
                        const uint32_t p01 = __byte_perm(x[off[0]], x[off[1]], 0x5410);
                        const uint32_t p23 = __byte_perm(x[off[2]], x[off[3]], 0x5410);
                        uint2 w;
                        w.x = __byte_perm(p01, p23, sel_lo);
                        w.y = __byte_perm(p01, p23, sel_hi);
                        *reinterpret_cast<uint2*>(out + (size_t)t * CI) = w;
                    }
                } else {
                    const uint32_t* rs = reinterpret_cast<const uint32_t*>(sm + slot * kBulkStage);
                    uint32_t* out = reinterpret_cast<uint32_t*>(label) + tok0 * CI + 4 * fq;
                    for (int t = tid / kG; t < nt; t += kBulkNT / kG) {
                        const uint32_t* x = rs + t * D;
                        const uint32_t a[4] = {x[off[0]], x[off[1]], x[off[2]], x[off[3]]};
                        *reinterpret_cast<uint4*>(out + (size_t)t * CI) =
                            make_uint4(pick_rot(a, 0, frot), pick_rot(a, 1, frot), pick_rot(a, 2, frot),
                                       pick_rot(a, 3, frot));
                    }
                }
            } else {
                const TKV* rows_s = reinterpret_cast<const TKV*>(sm + slot * kBulkStage);
                for (int t = tid / kPackLanes; t < ((nt + 7) & ~7); t += kBulkNT / kPackLanes) {
                    const bool live = t < nt;
                    const TKV* x = rows_s + (size_t)(live ? t : 0) * D;
                    float v[kPer];
#pragma unroll
                    for (int e = 0; e < kPer; ++e) v[e] = E::to_f32(x[off[e]]);
                    float mn = v[0], mx = v[0];
#pragma unroll
                    for (int e = 1; e < kPer; ++e) {
                        mn = fminf(mn, v[e]);
                        mx = fmaxf(mx, v[e]);
                    }
#pragma unroll
                    for (int o = 1; o < kPackLanes; o <<= 1) {
                        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                    }
                    const float step = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
                    const uint16_t sh = __half_as_ushort(__float2half_rn(step));
                    const uint16_t zh = __half_as_ushort(__float2half_rn(mn));
                    const float sc = fp16_bits_to_f32(sh), z = fp16_bits_to_f32(zh);
                    const float rsc = sc > 0.f ? __frcp_rn(sc) : 0.f;
                    if (live) {
                        float a[kPer];
#pragma unroll
                        for (int e = 0; e < kPer; ++e) a[e] = __fsub_rn(v[e], z);
                        uint32_t code[kPer];
                        int4_codes<kPer>(a, sc, rsc, code);
                        if (!(sc > 0.f)) {
#pragma unroll
                            for (int e = 0; e < kPer; ++e) code[e] = 0u;
                        }
                        // channel q4 * kPer + e of the row is nibble e of this
                        // lane's kPer / 2 bytes (low nibble first)
                        uint8_t* dst = label + (tok0 + t) * (size_t)(CI / 2) + q4 * kPer / 2;
                        if constexpr (kRot) {
                            // the codes in the rotated order, packed, then the
                            // word rotated left by 4 * rot bits (nibble e to
                            // nibble (e + rot) % kPer)
                            uint64_t w = 0;
#pragma unroll
                            for (int e = 0; e < kPer; ++e) w |= (uint64_t)code[e] << (4 * e);
                            const uint32_t sh = 4u * (uint32_t)rot;
                            // dst is kPer / 2-byte aligned: label is 16-byte
                            // aligned and rows are 2 * kPer bytes long
                            if constexpr (kPer == 2) {
                                const uint32_t x = (uint32_t)w * 0x101u;  // the byte twice
                                *dst = (uint8_t)(x >> (8u - sh));
                            } else if constexpr (kPer == 4) {
                                const uint32_t x = (uint32_t)w * 0x10001u;
                                *reinterpret_cast<uint16_t*>(dst) = (uint16_t)(x >> (16u - sh));
                            } else if constexpr (kPer == 8) {
                                *reinterpret_cast<uint32_t*>(dst) = __funnelshift_l((uint32_t)w, (uint32_t)w, sh);
                            } else {
                                const uint32_t lo = (uint32_t)w, hi = (uint32_t)(w >> 32);
                                const uint32_t l2 = sh >= 32u ? hi : lo, h2 = sh >= 32u ? lo : hi;
                                const uint32_t s2 = sh & 31u;
                                *reinterpret_cast<uint2*>(dst) =
                                    make_uint2(__funnelshift_l(h2, l2, s2), __funnelshift_l(l2, h2, s2));
                            }
                        } else {
#pragma unroll
                            for (int e = 0; e < kPer; e += 2) dst[e / 2] = (uint8_t)(code[e] | (code[e + 1] << 4));
                        }
                        if (q4 == 0) {
                            lscale[tok0 + t] = sh;
                            lzero[tok0 + t] = zh;
                        }
                    }
                }
            }
        }
        // every thread is done with the slot; a copy that never arrived
        // (recorded in *err) ends the CTA
        if (!__syncthreads_and(ok)) break;
        if (tid == 0 && pit < items) issue(slot);
    }
}

template <typename TKV, int LK, int D, int CI>
static cudaError_t launch_label_bulk(const LabelArgs& a, long long items, cudaStream_t st) {
    static bool attr = false;  // set once per process (the attribute is per function)
    if (!attr) {
        const cudaError_t e = cudaFuncSetAttribute(ds_label_bulk_kernel<TKV, LK, D, CI>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, bulk_smem_bytes());
        if (e != cudaSuccess) return e;
        attr = true;
    }
    const long long slots = (long long)kBulkCtasPerSm * a.sms;
    const long long grid = items < slots ? items : slots;
    ds_label_bulk_kernel<TKV, LK, D, CI><<<(unsigned)grid, kBulkNT, bulk_smem_bytes(), st>>>(
        reinterpret_cast<const TKV*>(a.k), a.idx, a.hkv, a.t_begin, a.t_end, a.s_cap, a.b * a.hkv,
        reinterpret_cast<uint8_t*>(a.label), a.lscale, a.lzero, a.err);
    return cudaGetLastError();
}

template <typename TKV, int LK, int D>
static cudaError_t launch_label_t(const LabelArgs& a, cudaStream_t st) {
    const int n = a.t_end - a.t_begin;
    constexpr int kTok = kBulkStage / (D * Elem<TKV>::kBytes);
    const long long items = (long long)a.b * a.hkv * ((n + kTok - 1) / kTok);
    if (!a.block_table && a.err && items >= (long long)kBulkCtasPerSm * a.sms && items < (1LL << 30) &&
        (LK == 0 || a.c >= 2 * kPackLanes)) {
        switch (a.c) {
        case 8: return launch_label_bulk<TKV, LK, D, 8>(a, items, st);
        case 16: return launch_label_bulk<TKV, LK, D, 16>(a, items, st);
        case 32: return launch_label_bulk<TKV, LK, D, 32>(a, items, st);
        case 64: if constexpr (D >= 64) return launch_label_bulk<TKV, LK, D, 64>(a, items, st); break;
        case 128: if constexpr (D >= 128) return launch_label_bulk<TKV, LK, D, 128>(a, items, st); break;
        }
    }
    dim3 grid((n + kTokens - 1) / kTokens, a.b * a.hkv);
    ds_label_kernel<TKV, LK, D><<<grid, kLabNT, 0, st>>>(
        reinterpret_cast<const TKV*>(a.k), a.idx, a.hkv, a.t_begin, a.t_end, a.s_cap, a.c,
        reinterpret_cast<uint8_t*>(a.label), a.lscale, a.lzero, a.block_table, a.max_blocks, a.page_shift,
        a.num_blocks);
    return cudaGetLastError();
}

cudaError_t launch_label(const LabelArgs& a, cudaStream_t st) {
    const bool i4 = a.int4;
#define DS_LAB(T, D_)                                                               \
    if (a.d == D_) return i4 ? launch_label_t<T, 1, D_>(a, st) : launch_label_t<T, 0, D_>(a, st);
    if (a.kdt_bf16) {
        DS_LAB(bf16_t, 64)
        DS_LAB(bf16_t, 128)
    } else {
        DS_LAB(float, 64)
        DS_LAB(float, 128)
    }
#undef DS_LAB
    return cudaErrorInvalidValue;
}

}  // namespace ds
