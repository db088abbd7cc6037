// ds_calib.cu -- offline heavy-channel calibration for sm_100a.
//
// "K通道静态性量化方法解析" (aitangshan.cn) §1.1 ranks channel i of a head by
//     r_i = ||Q[i] K[i]^T|| / ||Q K^T||
// with Q the queries of an observation window at the end of the input and K
// all keys; "大模型稀疏化技术原理：Double Sparsity" (joto.ai, section 离线校准)
// fixes the heavy channels offline from a few samples.
//
// Q[i]K[i]^T has rank one, so its norm is ||Q[:,i]|| * ||K[:,i]||: the kernels
// accumulate per-channel sums of squares of Q and K and the sum of squared
// entries of Q K^T (fp32 dot products, fp64 accumulation) into the caller's
// workspace, then one CTA per kv head forms r (mean over samples) and ranks
// the channels (ties to the lower channel index).
//
// The same sums also rank channels by the outlier criteria that "大模型稀疏化
// 技术原理：Double Sparsity" lists beside its offline calibration (Q-, K- and
// QK-outlier), and by the chunked-norm collection "K通道静态性量化方法解析"
// §2.1 attributes to Double Sparsity: the per-channel score is the column
// norm ||Q[:,i]||, ||K[:,i]||, the product of both, or ||Q[:,i]|| times the sum
// over context chunks of ||K[chunk, i]||.
#include <mutex>

#include "ds_common.cuh"
#include "ds_internal.h"

namespace ds {

constexpr int kCalNT = 256;
constexpr int kCalTile = 32;  // key rows and query rows per tile

// Workspace: [n][hkv] blocks of (q_sq[d], k_sq[d], den_sq) doubles.
__host__ __device__ inline size_t calib_ws_doubles(int n, int hkv, int d) {
    return (size_t)n * hkv * (2 * (size_t)d + 1);
}

template <typename T, int D>
__global__ void __launch_bounds__(kCalNT) ds_calib_partial_kernel(const T* __restrict__ qwin,
                                                                   const T* __restrict__ k, int hq,
                                                                   int hkv, int w, int s,
                                                                   bool k_sums, bool den_sums,
                                                                   double* __restrict__ ws) {
    using E = Elem<T>;
    __shared__ float ks[kCalTile][D + 1];
    __shared__ float qt[kCalTile][D + 1];
    __shared__ double red[kCalNT / 32];
    const int G = hq / hkv;
    const int rows = G * w;
    const int n = blockIdx.z, g = blockIdx.y;
    const int t0 = blockIdx.x * kCalTile;
    const int nt = min(kCalTile, s - t0);
    double* blk = ws + ((size_t)n * hkv + g) * (2 * D + 1);
    const T* kbase = k + (((size_t)n * hkv + g) * s + t0) * D;

    for (int e = threadIdx.x; e < kCalTile * D; e += kCalNT) {
        const int t = e / D, i = e - t * D;
        ks[t][i] = t < nt ? E::to_f32(kbase[(size_t)t * D + i]) : 0.f;
    }
    __syncthreads();
    // per-channel sum of squares of this key tile
    for (int i = threadIdx.x; k_sums && i < D; i += kCalNT) {
        double a = 0.0;
        for (int t = 0; t < nt; ++t) a += (double)ks[t][i] * (double)ks[t][i];
        atomicAdd(&blk[D + i], a);
    }

    // sum over (query row, key row) of (q . k)^2
    double acc = 0.0;
    for (int r0 = 0; r0 < rows; r0 += kCalTile) {
        const int nr = min(kCalTile, rows - r0);
        __syncthreads();
        for (int e = threadIdx.x; e < kCalTile * D; e += kCalNT) {
            const int rr = e / D, i = e - rr * D;
            float x = 0.f;
            if (rr < nr) {
                const int row = r0 + rr;
                const int h = g * G + row / w, t = row % w;
                x = E::to_f32(qwin[(((size_t)n * hq + h) * w + t) * D + i]);
            }
            qt[rr][i] = x;
        }
        __syncthreads();
        if (blockIdx.x == 0) {  // query-channel sums of squares, once per (n, g)
            for (int i = threadIdx.x; i < D; i += kCalNT) {
                double a = 0.0;
                for (int rr = 0; rr < nr; ++rr) a += (double)qt[rr][i] * (double)qt[rr][i];
                atomicAdd(&blk[i], a);
            }
        }
        for (int e = threadIdx.x; den_sums && e < kCalTile * kCalTile; e += kCalNT) {
            const int rr = e / kCalTile, t = e - rr * kCalTile;
            if (rr < nr && t < nt) {
                float dot = 0.f;
#pragma unroll 8
                for (int i = 0; i < D; ++i) dot = fmaf(qt[rr][i], ks[t][i], dot);
                acc += (double)dot * (double)dot;
            }
        }
    }
    acc = warp_sum_d(acc);
    if (lane_id() == 0) red[warp_id()] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double a = 0.0;
        for (int i = 0; i < kCalNT / 32; ++i) a += red[i];
        atomicAdd(&blk[2 * D], a);
    }
}

// Sum over the context chunks [t0, t0 + chunk) of ||K[chunk, i]|| per channel,
// into the k slot of the workspace (chunked-norm criterion). One CTA per
// (chunk, kv head, sample); each of the kCalNT / D token lanes sums a strided
// part of the chunk, and the lanes are added in a fixed order.
template <typename T, int D>
__global__ void __launch_bounds__(kCalNT) ds_calib_kchunk_kernel(const T* __restrict__ k, int hkv,
                                                                  int s, int chunk,
                                                                  double* __restrict__ ws) {
    using E = Elem<T>;
    constexpr int L = kCalNT / D;
    __shared__ double part[L][D];
    const int n = blockIdx.z, g = blockIdx.y;
    const int t0 = blockIdx.x * chunk;
    const int t1 = min(s, t0 + chunk);
    const int i = threadIdx.x % D, l = threadIdx.x / D;
    const T* kb = k + ((size_t)n * hkv + g) * (size_t)s * D;
    double a = 0.0;
    for (int t = t0 + l; t < t1; t += L) {
        const double x = (double)E::to_f32(kb[(size_t)t * D + i]);
        a += x * x;
    }
    part[l][i] = a;
    __syncthreads();
    if (l == 0) {
        double sq = 0.0;
        for (int j = 0; j < L; ++j) sq += part[j][i];
        atomicAdd(&ws[((size_t)n * hkv + g) * (2 * D + 1) + D + i], sqrt(sq));
    }
}

template <int D>
__global__ void __launch_bounds__(D) ds_calib_rank_kernel(const double* __restrict__ ws, int n,
                                                          int hkv, int c, int criterion,
                                                          float* __restrict__ ratio,
                                                          int32_t* __restrict__ idx) {
    __shared__ double r[D];
    __shared__ uint32_t scan[D / 32 + 1];
    const int g = blockIdx.x, i = threadIdx.x;
    double acc = 0.0;
    for (int ns = 0; ns < n; ++ns) {
        const double* blk = ws + ((size_t)ns * hkv + g) * (2 * D + 1);
        double v;
        switch (criterion) {
        case kCritQ: v = sqrt(blk[i]); break;
        case kCritK: v = sqrt(blk[D + i]); break;
        case kCritQK: v = sqrt(blk[i]) * sqrt(blk[D + i]); break;
        case kCritQKChunked: v = sqrt(blk[i]) * blk[D + i]; break;
        default: {
            const double den = sqrt(blk[2 * D]);
            v = den > 0.0 ? sqrt(blk[i]) * sqrt(blk[D + i]) / den : 0.0;
        }
        }
        acc += v / (double)n;
    }
    r[i] = acc;
    if (ratio) ratio[(size_t)g * D + i] = (float)acc;
    __syncthreads();
    int rank = 0;
    for (int j = 0; j < D; ++j) rank += (r[j] > acc) || (r[j] == acc && j < i);
    const uint32_t picked = rank < c ? 1u : 0u;
    uint32_t total;
    const uint32_t pos = block_excl_scan<D>(picked, scan, &total);
    if (picked) idx[(size_t)g * c + pos] = i;
}

size_t calib_workspace_bytes(int n, int hkv, int d) { return calib_ws_doubles(n, hkv, d) * sizeof(double); }

template <typename T, int D>
static cudaError_t launch_calib_t(const CalibArgs& a, cudaStream_t st) {
    cudaError_t e = cudaMemsetAsync(a.ws, 0, calib_workspace_bytes(a.n, a.hkv, D), st);
    if (e != cudaSuccess) return e;
    const bool chunked = a.criterion == kCritQKChunked;
    dim3 grid((a.s + kCalTile - 1) / kCalTile, a.hkv, a.n);
    ds_calib_partial_kernel<T, D><<<grid, kCalNT, 0, st>>>(
        reinterpret_cast<const T*>(a.q_win), reinterpret_cast<const T*>(a.k), a.hq, a.hkv, a.w, a.s,
        !chunked, a.criterion == kCritLeanK, reinterpret_cast<double*>(a.ws));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (chunked) {
        dim3 cg((a.s + a.chunk - 1) / a.chunk, a.hkv, a.n);
        ds_calib_kchunk_kernel<T, D><<<cg, kCalNT, 0, st>>>(reinterpret_cast<const T*>(a.k), a.hkv,
                                                             a.s, a.chunk,
                                                             reinterpret_cast<double*>(a.ws));
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    ds_calib_rank_kernel<D><<<a.hkv, D, 0, st>>>(reinterpret_cast<const double*>(a.ws), a.n, a.hkv,
                                                  a.c, a.criterion, a.ratio, a.idx);
    return cudaGetLastError();
}

cudaError_t launch_calib(const CalibArgs& a, cudaStream_t st) {
    if (a.bf16) {
        if (a.d == 64) return launch_calib_t<bf16_t, 64>(a, st);
        if (a.d == 128) return launch_calib_t<bf16_t, 128>(a, st);
    } else {
        if (a.d == 64) return launch_calib_t<float, 64>(a, st);
        if (a.d == 128) return launch_calib_t<float, 128>(a, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace ds

// ------------------------------------------------ calibration without allocation
//
// For callers that cannot obtain device memory from cudaMalloc or a caching
// allocator: hosts that hand a plugin only fixed tensors and own every
// allocation, or runtimes with a preallocated device budget. The scratch then lives in this fixed
// file-scope array, which every GPU that loads the library keeps until exit.
// All calls share it and each call first clears the part it uses; calls that
// overlap on the GPU (different streams, no ordering between them) race on it.
namespace {

constexpr size_t kStaticCalibDoubles = 131072;  // 1 MiB
static __device__ __align__(256) double g_calib_static_scratch[kStaticCalibDoubles];

std::mutex g_static_mu;
struct StaticAddr { unsigned long long ctx; void* ptr; };
StaticAddr g_static_addr[16];  // most recent contexts first-come
int g_static_used = 0, g_static_next = 0;

// Device address of the scratch array in the current context. Host code sees
// the array's name as a host-side stand-in, not a device address, so the
// address is asked of the runtime with the device current and cached per
// context (keyed by the context's process-unique id: after a device reset the
// new context's copy of the array is looked up afresh).
cudaError_t static_scratch(void** out) {
    unsigned long long ctx = 0;
    const bool keyed = ds::current_context_id(&ctx);
    std::lock_guard<std::mutex> lk(g_static_mu);
    if (keyed)
        for (int i = 0; i < g_static_used; ++i)
            if (g_static_addr[i].ctx == ctx) { *out = g_static_addr[i].ptr; return cudaSuccess; }
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_calib_static_scratch);
    if (e != cudaSuccess) return e;
    // the lookup makes the device's primary context current when none was
    if (keyed || ds::current_context_id(&ctx)) {
        g_static_addr[g_static_next] = StaticAddr{ctx, p};
        g_static_next = (g_static_next + 1) % 16;
        if (g_static_used < 16) ++g_static_used;
    }
    *out = p;
    return cudaSuccess;
}

}  // namespace

namespace ds {

size_t calib_static_scratch_bytes() { return kStaticCalibDoubles * sizeof(double); }

cudaError_t launch_calib_static(CalibArgs a, cudaStream_t st) {
    void* p = nullptr;
    const cudaError_t e = static_scratch(&p);
    if (e != cudaSuccess) return e;
    a.ws = p;
    return launch_calib(a, st);
}

}  // namespace ds
