// ds_common.cuh -- device helpers shared by the Double Sparsity kernels (sm_100a).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ds {

constexpr int kWarp = 32;

// Storage element types. bf16 is carried as its raw 16-bit pattern; widening
// it to fp32 is the exact operation "put the bits in the upper half".
struct bf16_t { uint16_t bits; };

template <typename T> struct Elem;
template <> struct Elem<float> {
    static constexpr int kBytes = 4;
    __device__ __forceinline__ static float to_f32(float x) { return x; }
};
template <> struct Elem<bf16_t> {
    static constexpr int kBytes = 2;
    __device__ __forceinline__ static float to_f32(bf16_t x) {
        return __uint_as_float(static_cast<uint32_t>(x.bits) << 16);
    }
};

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float fp16_bits_to_f32(uint16_t b) {
    return __half2float(__ushort_as_half(b));
}

// fp32 -> bf16 bits, round to nearest even (inputs of the attention output are finite).
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7F800000u) == 0x7F800000u) return static_cast<uint16_t>((u >> 16) | ((u & 0xFFFF) ? 0x40 : 0));
    u += 0x7FFFu + ((u >> 16) & 1u);
    return static_cast<uint16_t>(u >> 16);
}

// Streaming 16/8/4-byte global loads that bypass L1 allocation (read-only data).
__device__ __forceinline__ uint4 ldg_stream16(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}
__device__ __forceinline__ uint2 ldg_stream8(const void* p) {
    uint2 r;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
    return r;
}
__device__ __forceinline__ uint32_t ldg_stream4(const void* p) {
    uint32_t r;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
    return r;
}
__device__ __forceinline__ uint16_t ldg_u16(const uint16_t* p) {
    unsigned short r;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(r) : "l"(p));
    return r;
}

// Loads of N bytes (N in {4, 8, 16, 32, ...}) into N/4 registers.
template <int N>
__device__ __forceinline__ void load_words(uint32_t (&w)[N / 4], const uint8_t* p) {
    if constexpr (N % 16 == 0) {
#pragma unroll
        for (int i = 0; i < N / 16; ++i) {
            uint4 x = ldg_stream16(p + 16 * i);
            w[4 * i + 0] = x.x; w[4 * i + 1] = x.y; w[4 * i + 2] = x.z; w[4 * i + 3] = x.w;
        }
    } else if constexpr (N == 8) {
        uint2 x = ldg_stream8(p);
        w[0] = x.x; w[1] = x.y;
    } else {
        static_assert(N == 4, "row size");
        w[0] = ldg_stream4(p);
    }
}

// Shared-memory loads of N bytes (N in {4, 8, 16}) into N/4 registers.
template <int N>
__device__ __forceinline__ void lds_words(uint32_t (&w)[N / 4], const uint8_t* p) {
    if constexpr (N == 16) {
        const uint4 x = *reinterpret_cast<const uint4*>(p);
        w[0] = x.x; w[1] = x.y; w[2] = x.z; w[3] = x.w;
    } else if constexpr (N == 8) {
        const uint2 x = *reinterpret_cast<const uint2*>(p);
        w[0] = x.x; w[1] = x.y;
    } else {
        static_assert(N == 4, "lds size");
        w[0] = *reinterpret_cast<const uint32_t*>(p);
    }
}

// 16-byte asynchronous global -> shared copy (LDGSTS, L2 only), and its
// group bookkeeping. Completion is awaited per thread with cp_async_wait;
// other lanes' copies become visible after a __syncwarp / __syncthreads.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Bulk prefetch of [p, p + bytes) into L2 (TMA unit; no registers held while
// in flight). p must be 16-byte aligned and bytes a multiple of 16.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Prefetch the byte range [base + lo, base + hi) in pieces of `piece` bytes
// (a multiple of 16), one piece per thread index `who`. The range is trimmed
// inward to 16-byte aligned ABSOLUTE addresses (row bases of small-row arrays,
// e.g. fp16 scales at row * s_cap * 2 bytes, need not be aligned), so every
// prefetch starts on a 16-byte boundary and covers a multiple of 16 bytes.
__device__ __forceinline__ void prefetch_range(const uint8_t* base, size_t lo, size_t hi, int who,
                                               uint32_t piece) {
    const uintptr_t a = (reinterpret_cast<uintptr_t>(base + lo) + 15) & ~(uintptr_t)15;
    const uintptr_t e = reinterpret_cast<uintptr_t>(base + hi) & ~(uintptr_t)15;
    const uintptr_t start = a + (uintptr_t)who * piece;
    if (start >= e) return;
    const uintptr_t n = e - start < piece ? e - start : piece;
    prefetch_l2(reinterpret_cast<const void*>(start), (uint32_t)n);
}

// Order-preserving map of an fp32 score to uint32: larger score -> larger key.
// -0 is folded onto +0 so that equal scores give equal keys.
__device__ __forceinline__ uint32_t score_key(float s) {
    uint32_t u = __float_as_uint(s);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }
__device__ __forceinline__ int warp_id() { return threadIdx.x >> 5; }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Inclusive prefix sum over the warp.
__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v) {
    const int lane = lane_id();
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

// Block-wide exclusive prefix sum (blockDim.x == NT, multiple of 32). `tmp`
// holds NT/32 + 1 words of shared memory. Returns the exclusive prefix and
// writes the block total to *total. Contains two __syncthreads().
template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* tmp, uint32_t* total) {
    const int lane = lane_id(), w = warp_id();
    uint32_t incl = warp_incl_scan(v);
    if (lane == 31) tmp[w] = incl;
    __syncthreads();
    if (w == 0) {
        uint32_t x = lane < NT / 32 ? tmp[lane] : 0u;
        uint32_t xi = warp_incl_scan(x);
        if (lane < NT / 32) tmp[lane] = xi - x;
        if (lane == NT / 32 - 1) tmp[NT / 32] = xi;
    }
    __syncthreads();
    const uint32_t excl = tmp[w] + incl - v;
    *total = tmp[NT / 32];
    return excl;
}

}  // namespace ds
