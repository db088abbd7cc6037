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

// Dense key cache, many tokens (prefill): persistent CTAs stream blocks of
// consecutive key rows -- one contiguous span of kBulkStage bytes per
// (row, block) item -- through a kBulkStages-deep shared-memory ring with 1-D
// bulk copies (thread 0 issues them; an mbarrier per stage counts the bytes
// in), so the next blocks' reads are in flight while the current one is
// gathered or packed. Same results as ds_label_kernel.
constexpr int kBulkStage = 16384;  // bytes of key rows per stage
constexpr int kBulkStages = 4;
constexpr int kBulkNT = 256;
// packing threads per token (4-bit): each takes c / kPackLanes channels
constexpr int kPackLanes = 4;

__host__ __device__ constexpr int bulk_smem_bytes() { return kBulkStages * kBulkStage + kBulkStages * 8; }

// CI: the channel count, fixed at compile time for 4-bit rows (each lane's
// CI / kPackLanes channel indices then stay in registers); 0 for fp rows.
template <typename TKV, int LK, int D, int CI>
__global__ void __launch_bounds__(kBulkNT, 2) ds_label_bulk_kernel(const TKV* __restrict__ k,
                                                                  const int32_t* __restrict__ idx, int hkv,
                                                                  int t_begin, int t_end, int s_cap, int c,
                                                                  int rows, uint8_t* __restrict__ label,
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
    const long long items = (long long)rows * nblk;
    if (tid == 0) {
        for (int i = 0; i < kBulkStages; ++i) mbar_init(&full[i], 1);
        fence_mbar_init();
    }
    __syncthreads();
    auto issue = [&](long long it, int slot) {
        const int row = (int)(it / nblk), blk = (int)(it - (long long)row * nblk);
        const int tb = t_begin + blk * kTok;
        const int nt = min(kTok, t_end - tb);
        const uint32_t bytes = (uint32_t)(nt * kRowBytes);
        mbar_arrive_expect_tx(&full[slot], bytes);
        bulk_g2s(sm + slot * kBulkStage, k + ((size_t)row * s_cap + tb) * D, bytes, &full[slot]);
    };
    if (tid == 0)
        for (int i = 0; i < kBulkStages; ++i) {
            const long long it = blockIdx.x + (long long)i * gridDim.x;
            if (it < items) issue(it, i);
        }
    constexpr int kPer = CI / kPackLanes > 0 ? CI / kPackLanes : 1;  // 4-bit channels per lane
    int g_cur = -1;
    int my_idx[kPer];  // 4-bit: this thread's channels
    int fp_idx = 0;    // fp: this thread's channel (tid % c)
    int j = 0;
    for (long long it = blockIdx.x; it < items; it += gridDim.x, ++j) {
        const int slot = j % kBulkStages;
        const int row = (int)(it / nblk), blk = (int)(it - (long long)row * nblk);
        const int g = row % hkv;
        const int tb = t_begin + blk * kTok;
        const int nt = min(kTok, t_end - tb);
        const size_t tok0 = (size_t)row * s_cap + tb;
        if (g != g_cur) {
            g_cur = g;
            if constexpr (LK == 0) {
                fp_idx = min(max(__ldg(idx + (size_t)g * c + tid % c), 0), D - 1);
            } else {
                const int q = tid % kPackLanes;
#pragma unroll
                for (int e = 0; e < kPer; ++e)
                    my_idx[e] = min(max(__ldg(idx + (size_t)g * CI + q * kPer + e), 0), D - 1);
            }
        }
        const bool ok = mbar_wait_bounded(&full[slot], (uint32_t)((j / kBulkStages) & 1), err, 1);
        const TKV* rows_s = reinterpret_cast<const TKV*>(sm + slot * kBulkStage);
        if (ok) {
            if constexpr (LK == 0) {
                // thread tid always handles channel tid % c (c divides the CTA size)
                TKV* out = reinterpret_cast<TKV*>(label) + tok0 * c;
                for (int e = tid; e < nt * c; e += kBulkNT) out[e] = rows_s[(e / c) * D + fp_idx];
            } else {
                // kPackLanes threads per token, c / kPackLanes channels each:
                // the arithmetic of pack_int4_row, with mn / mx combined over
                // the lanes (fminf / fmaxf do not depend on the order)
                const int q = tid % kPackLanes;
                for (int t = tid / kPackLanes; t < ((nt + 7) & ~7); t += kBulkNT / kPackLanes) {
                    const bool live = t < nt;
                    const TKV* x = rows_s + (size_t)(live ? t : 0) * D;
                    float mn = E::to_f32(x[my_idx[0]]), mx = mn;
#pragma unroll
                    for (int e = 1; e < kPer; ++e) {
                        const float v = E::to_f32(x[my_idx[e]]);
                        mn = fminf(mn, v);
                        mx = fmaxf(mx, v);
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
                        uint8_t* dst = label + (tok0 + t) * (size_t)(CI / 2) + q * kPer / 2;
#pragma unroll
                        for (int e = 0; e < kPer; e += 2) {
                            uint32_t nib[2];
#pragma unroll
                            for (int h = 0; h < 2; ++h)
                                nib[h] = sc > 0.f ? int4_code(E::to_f32(x[my_idx[e + h]]), z, sc, rsc) : 0u;
                            dst[e / 2] = (uint8_t)(nib[0] | (nib[1] << 4));
                        }
                        if (q == 0) {
                            lscale[tok0 + t] = sh;
                            lzero[tok0 + t] = zh;
                        }
                    }
                }
            }
        }
        __syncthreads();  // every thread is done with the slot
        if (!__syncthreads_and(ok)) break;  // a copy never arrived: leave (recorded in *err)
        if (tid == 0) {
            const long long nx = it + (long long)kBulkStages * gridDim.x;
            if (nx < items) issue(nx, slot);
        }
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
    const long long grid = items < 2LL * a.sms ? items : 2LL * a.sms;
    ds_label_bulk_kernel<TKV, LK, D, CI><<<(unsigned)grid, kBulkNT, bulk_smem_bytes(), st>>>(
        reinterpret_cast<const TKV*>(a.k), a.idx, a.hkv, a.t_begin, a.t_end, a.s_cap, a.c, a.b * a.hkv,
        reinterpret_cast<uint8_t*>(a.label), a.lscale, a.lzero, a.err);
    return cudaGetLastError();
}

template <typename TKV, int LK, int D>
static cudaError_t launch_label_t(const LabelArgs& a, cudaStream_t st) {
    const int n = a.t_end - a.t_begin;
    constexpr int kTok = kBulkStage / (D * Elem<TKV>::kBytes);
    const long long items = (long long)a.b * a.hkv * ((n + kTok - 1) / kTok);
    if (!a.block_table && a.err && items >= 2 * (long long)a.sms && (LK == 0 || a.c >= 2 * kPackLanes)) {
        if constexpr (LK == 0) return launch_label_bulk<TKV, 0, D, 0>(a, items, st);
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
