// ds_label.cu -- label-cache build (prefill) and append (decode) for sm_100a.
//
// "大模型稀疏化技术原理：Double Sparsity" (joto.ai), section 离线校准: at prefill
// every token's heavy key channels are copied from the key cache into the
// contiguous label cache; at each decode step only the new token's channels
// are added. The cache may be kept in 4 bits.
//
// One CTA handles kTokens consecutive tokens of one (b, kv head) row: the key
// rows are staged in shared memory with coalesced 16-byte loads, then each
// label element (fp) or each token (4-bit) is produced from shared memory.
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

template <typename TKV, int LK, int D>
static cudaError_t launch_label_t(const LabelArgs& a, cudaStream_t st) {
    const int n = a.t_end - a.t_begin;
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
