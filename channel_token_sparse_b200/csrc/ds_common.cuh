// ds_common.cuh -- device helpers shared by the Double Sparsity kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
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

// Shared-memory loads of a label row of N bytes (N a multiple of 4).
template <int N>
__device__ __forceinline__ void lds_row(uint32_t (&w)[N / 4], const uint8_t* p) {
    if constexpr (N % 16 == 0) {
#pragma unroll
        for (int i = 0; i < N / 16; ++i) {
            const uint4 x = reinterpret_cast<const uint4*>(p)[i];
            w[4 * i + 0] = x.x; w[4 * i + 1] = x.y; w[4 * i + 2] = x.z; w[4 * i + 3] = x.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < N / 4; ++i) w[i] = reinterpret_cast<const uint32_t*>(p)[i];
    }
}

// The 4-bit code of value x with zero z and scale sc > 0:
// clamp(rint((x - z) / sc), 0, 15), the quotient an IEEE single-precision
// division rounded to nearest even. The quotient is first formed as
// (x - z) * (1 / sc), within 3 * 2^-24 relative of the exact one; rint can only
// differ between the two when a half-integer lies within that distance, so
// only then (|frac - 1/2| <= 1e-5, codes < 16 keep |q| <= 16) is the division
// done exactly. The result is always that of the exact division.
__device__ __forceinline__ uint32_t int4_code(float x, float z, float sc, float rcp_sc) {
    const float a = __fsub_rn(x, z);
    float q = __fmul_rn(a, rcp_sc);
    if (fabsf(q - floorf(q) - 0.5f) <= 1e-5f) q = __fdiv_rn(a, sc);
    q = fminf(fmaxf(rintf(q), 0.f), 15.f);
    return (uint32_t)q;
}

// 4-bit label row of one token (the heavy channels idx[0..c) of key row x):
// in fp32, mn/mx over the c values, scale = fp16_rn((mx - mn) / 15),
// zero = fp16_rn(mn), code_j = scale > 0 ? clamp(rint((x_j - zero) / scale),
// 0, 15) : 0 with IEEE division and round-half-even; channel 2j goes to the
// low nibble of byte j. Used by the label kernel and by the fused decode step,
// so both produce the same bits.
template <typename T>
__device__ __forceinline__ void pack_int4_row(const T* x, const int* idx, int c, uint8_t* payload,
                                              uint16_t* scale_bits, uint16_t* zero_bits) {
    float mn = Elem<T>::to_f32(x[idx[0]]), mx = mn;
    for (int j = 1; j < c; ++j) {
        const float v = Elem<T>::to_f32(x[idx[j]]);
        mn = fminf(mn, v);
        mx = fmaxf(mx, v);
    }
    const float step = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
    const uint16_t sh = __half_as_ushort(__float2half_rn(step));
    const uint16_t zh = __half_as_ushort(__float2half_rn(mn));
    const float sc = fp16_bits_to_f32(sh);
    const float z = fp16_bits_to_f32(zh);
    for (int j = 0; j < c; j += 2) {
        uint32_t nib[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            uint32_t code = 0;
            if (sc > 0.f) {
                float qv = rintf(__fdiv_rn(__fsub_rn(Elem<T>::to_f32(x[idx[j + e]]), z), sc));
                qv = fminf(fmaxf(qv, 0.f), 15.f);
                code = (uint32_t)qv;
            }
            nib[e] = code;
        }
        payload[j / 2] = (uint8_t)(nib[0] | (nib[1] << 4));
    }
    *scale_bits = sh;
    *zero_bits = zh;
}

// Sum NV values (NV a power of two, <= 32) over the 32 lanes of a warp; on
// return every lane holds all NV sums. A transposing butterfly: at each of
// the first log2(NV) exchange steps a lane sends half of its values and keeps
// the other half, so NV - 1 + 5 - log2(NV) shuffles reduce, and NV shuffles
// broadcast (instead of 5 * NV for separate reductions).
template <int NV>
__device__ __forceinline__ void warp_allreduce_multi(float (&v)[NV]) {
    constexpr int LOGN = NV >= 32 ? 5 : NV >= 16 ? 4 : NV >= 8 ? 3 : NV >= 4 ? 2 : NV >= 2 ? 1 : 0;
    static_assert((1 << LOGN) == NV, "NV must be a power of two <= 32");
    const int lane = threadIdx.x & 31;
    float r[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) r[i] = v[i];
#pragma unroll
    for (int step = 0; step < 5; ++step) {
        const int m = 16 >> step;
        if (step < LOGN) {
            const int half = NV >> (step + 1);
            const bool up = (lane & m) != 0;
#pragma unroll
            for (int i = 0; i < half; ++i) {
                const float send = up ? r[i] : r[i + half];
                const float keep = up ? r[i + half] : r[i];
                r[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
            }
        } else {
            r[0] += __shfl_xor_sync(0xffffffffu, r[0], m);
        }
    }
    // lane l now holds the sum of value (l >> (5 - LOGN))
#pragma unroll
    for (int j = 0; j < NV; ++j) v[j] = __shfl_sync(0xffffffffu, r[0], j << (5 - LOGN));
}

// Same for any power of two NV: blocks of 32 values at a time.
template <int NV>
__device__ __forceinline__ void warp_allreduce_n(float (&v)[NV]) {
    if constexpr (NV <= 32) {
        warp_allreduce_multi<NV>(v);
    } else {
#pragma unroll
        for (int b = 0; b < NV / 32; ++b) {
            float t[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) t[i] = v[b * 32 + i];
            warp_allreduce_multi<32>(t);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[b * 32 + i] = t[i];
        }
    }
}

// 16-byte asynchronous global -> shared copy (LDGSTS, L2 only), and its
// group bookkeeping. Completion is awaited per thread with cp_async_wait;
// other lanes' copies become visible after a __syncwarp / __syncthreads.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gsrc) : "memory");
}
// 8- and 4-byte forms (L1-allocating .ca, the only one that takes them).
__device__ __forceinline__ void cp_async8(void* smem_dst, const void* gsrc) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(d), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gsrc) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(d), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
// Same copy, or 16 zero bytes when !valid (nothing is read from gsrc then).
__device__ __forceinline__ void cp_async16_zfill(void* smem_dst, const void* gsrc, bool valid) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
    const int n = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(gsrc), "r"(n) : "memory");
}

// ---------------------------------------------------------------- mbarriers
// Shared-memory transaction barriers (sm_90+) used to await 1-D bulk copies.
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
// Makes barrier initialisation visible to the async proxy (bulk copies).
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// One arrival that also announces `bytes` of bulk-copy data to come.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
                 : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}
// Device-wide record of a wait that gave up (see mbar_wait_bounded).
__device__ __forceinline__ void note_timeout(unsigned int* flag, unsigned int where) {
    if (flag) atomicOr(flag, 1u << (where & 31));
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Wait for phase `parity` of `bar` to complete, giving up after about
// `limit_ns` nanoseconds (default one second): then `where` is recorded in
// *flag and false returned, so the caller can leave instead of waiting for
// ever.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, unsigned int* flag,
                                                  unsigned int where, uint64_t limit_ns = 1000000000ull) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (;;) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > limit_ns) break;
    }
    note_timeout(flag, where);
    return false;
}
// 1-D bulk copy global -> this CTA's shared memory (no multicast); both
// addresses 16-byte aligned and `bytes` a multiple of 16. Completion is
// counted on `bar` in bytes (mbar_arrive_expect_tx by the issuing thread).
__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(smem_dst)), "l"(gsrc), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// Two floats -> packed bf16x2 (first in the low half), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// Four 8x8 b16 matrices from shared memory (lanes 8i..8i+7 give the row
// addresses of matrix i); thread t receives row t/4, columns 2(t%4), 2(t%4)+1
// of each (.trans: the transposed matrices).
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void* p) {
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(a) : "memory");
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], const void* p) {
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(a) : "memory");
}

// Warp-level tensor-core products, bf16 inputs, fp32 accumulate in place.
// m16n8k16: A 16x16 (4 regs), B 16x8 (2 regs); m16n8k8: A 16x8 (2), B 8x8 (1).
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_bf16_1688(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a0), "r"(a1), "r"(b0));
}

// Prefetch of the 128-byte line holding p into L2 (no register result).
__device__ __forceinline__ void prefetch_line_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
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
