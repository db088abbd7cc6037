// ds_api.cu -- C ABI of libds.so: argument validation, launch planning and
// kernel dispatch. Declarations and the full contract are in include/ds.h.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>

#include <atomic>
#include <mutex>
#include <string>
#include <unordered_map>

#include "ds.h"
#include "ds_decode_kernel.cuh"
#include "ds_internal.h"

namespace {

thread_local char g_err[256] = "";
std::atomic<int> g_cluster_override{0};
// Tuning knob (ds_sparse_decode_tune)
std::atomic<int> g_scan_prefetch{2};  // label scan without the ring: rounds prefetched into L2 ahead
std::atomic<int> g_i4_ring{1};        // 4-bit rows: 1 = the label ring before the kept low key bits

// The library's status word on each device: a kernel records there a
// bounded wait that gave up (bit = where); ds_check_device reads and clears it.
static __device__ __align__(16) unsigned int g_status_word[4];

std::mutex g_status_mu;
struct StatusAddr { unsigned long long ctx; unsigned int* ptr; };
StatusAddr g_status_addr[16];
int g_status_used = 0, g_status_next = 0;

ds_status fail(ds_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return st;
}

ds_status cuda_fail(cudaError_t e, const char* what) {
    return fail(DS_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool kv_dtype_ok(ds_dtype t) { return t == DS_F32 || t == DS_BF16; }
bool c_ok(int c, int d) { return (c == 8 || c == 16 || c == 32 || c == 64 || c == 128) && c <= d; }
bool d_ok(int d) { return d == 64 || d == 128; }

int group_tier(int G) { return G <= 1 ? 1 : G <= 2 ? 2 : G <= 4 ? 4 : 8; }

// Number of SMs of the current device (148 on B200); queried once per process.
int sm_count() {
    static int n = [] {
        int dev = 0, v = 0;
        if (cudaGetDevice(&dev) != cudaSuccess) return 148;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
        return v > 0 ? v : 148;
    }();
    return n;
}

// L2 size of the current device (126 MB on B200); queried once per process.
int l2_bytes() {
    static int n = [] {
        int dev = 0, v = 0;
        if (cudaGetDevice(&dev) != cudaSuccess) return 126 << 20;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrL2CacheSize, dev) != cudaSuccess) return 126 << 20;
        return v > 0 ? v : 126 << 20;
    }();
    return n;
}

constexpr int kMaxSmem = 227 * 1024;
constexpr int kCtasPerSm = 2;  // __launch_bounds__(256, 2) -> <= 128 registers

struct Plan {
    int N, chunk, lay_chunk, per, smem, att_stages, lab_ring, keep_low, sel_off;
};

// Two CTAs of 256 threads per SM: each may use up to (228 KiB - 2 KiB) / 2.
constexpr int kSmemFor2 = (228 * 1024 - 2 * 1024) / 2;

int round_up(int x, int m) { return (x + m - 1) / m * m; }

// Cluster size N (CTAs per (b, kv head) row): the largest power of two whose
// grid (rows * N CTAs) still fits in one wave of resident CTAs, keeping at
// least 256 tokens per CTA; rows beyond one wave use N = 1. A forced N
// (ds_sparse_decode_set_cluster) overrides the choice when feasible.
bool make_plan(int rows, int G, int s, int d, int c, int topk, bool dense, bool int4, int esz, int slots,
               int forced, Plan* out, int s_cap = 0) {
    const int GT = group_tier(G);
    const bool select_all = dense || topk >= s;
    const int k_eff = topk < s ? topk : s;
    Plan best{0, 0, 0, 0, 0, 0, 0, 0, 0};
    for (int N = 1; N <= 16; N *= 2) {
        Plan p;
        p.N = N;
        p.chunk = round_up((s + N - 1) / N, 32);
        if (p.chunk > ds::kMaxChunk) continue;
        p.lay_chunk = dense ? 0 : p.chunk;
        p.per = select_all ? 0 : (k_eff + N - 1) / N;
        // bf16 K/V: 3 attention stages per warp when two CTAs still fit per SM
        // (with the selection's needs below), else 2
        p.att_stages = esz == 2 ? 3 : ds::kAttStagesF32;
        p.smem = ds::decode_smem_layout(GT, d, c, p.lay_chunk, p.per, esz, p.att_stages).total;
        const int sel_need = dense ? 0 : ds::align16(p.lay_chunk * 2) + ds::sel_scratch_bytes(p.lay_chunk);
        if (esz == 2) {
            const ds::DecodeSmem L3 = ds::decode_smem_layout(GT, d, c, p.lay_chunk, p.per, esz, 3, sel_need);
            if (L3.total > kSmemFor2) p.att_stages = 2;
            p.smem = ds::decode_smem_layout(GT, d, c, p.lay_chunk, p.per, esz, p.att_stages).total;
        }
        if (p.smem > kMaxSmem) continue;
        // fp labels of 16-byte multiples stream through a shared-memory ring
        // placed behind the 16-bit keys when the region has room for it
        // and the low 16 key bits are kept beside the high ones when they fit too
        p.lab_ring = 0;
        p.keep_low = 0;
        if (!dense) {
            // The selection phase keeps the 16-bit keys, optionally the low
            // 16 key bits, and the label ring in the region the attention
            // ring uses later; the region may grow beyond the attention ring
            // for them, as long as the CTAs per SM the plan has stay resident.
            const ds::DecodeSmem L = ds::decode_smem_layout(GT, d, c, p.lay_chunk, p.per, esz, p.att_stages);
            const int region_att = L.total - L.region;
            const int cap = (L.total <= kSmemFor2 ? kSmemFor2 : kMaxSmem) - L.region;
            const int keys = ds::align16(p.lay_chunk * 2);
            // 4-bit rows also stream their fp16 scale and zero in 16-byte
            // chunks of 8 tokens, which needs rows of a multiple of 8 tokens
            const int pay = c / 2;
            const bool i4_ring = int4 && s_cap > 0 && s_cap % 8 == 0 && (pay == 4 || pay == 8 || pay % 16 == 0);
            const int ring = int4 ? (i4_ring ? ds::lab_ring_bytes(pay + 4, true) : -1)
                                  : ((c * esz) % 16 == 0 ? ds::lab_ring_bytes(c * esz, false) : -1);
            // options in order of preference: {bytes, ring, low}; for 4-bit
            // rows, whose re-scoring costs more, the kept low bits come before
            // the ring when only one of them fits
            struct Opt { int need, ring, low; };
            const bool ring_first = !int4 || g_i4_ring.load();
            const Opt opts[] = {
                {ring >= 0 ? 2 * keys + ring : -1, 1, 1},
                {ring >= 0 && ring_first ? keys + ring : -1, 1, 0},
                {2 * keys, 0, 1},
                {ring >= 0 ? keys + ring : -1, 1, 0},
            };
            // the selection scratch sits behind the keys (and kept low bits),
            // over the label ring, which is dead by then
            const int scratch = ds::sel_scratch_bytes(p.lay_chunk);
            int used = keys + scratch;
            for (const Opt& o : opts) {
                if (o.need < 0) continue;
                const int need_o = o.need > (o.low ? 2 : 1) * keys + scratch ? o.need : (o.low ? 2 : 1) * keys + scratch;
                if (need_o > cap) continue;
                p.lab_ring = o.ring;
                p.keep_low = o.low;
                used = need_o;
                break;
            }
            p.sel_off = keys * (p.keep_low ? 2 : 1);
            // without the label ring the scan's register loads live in L1,
            // which shares the SM's storage with shared memory: such rows
            // keep 2 attention stages (3 cost the 256K layer 11 us)
            if (!p.lab_ring && p.att_stages == 3 && esz == 2) {
                p.att_stages = 2;
                const ds::DecodeSmem L2s = ds::decode_smem_layout(GT, d, c, p.lay_chunk, p.per, esz, 2);
                p.smem = L2s.total;
                if (used > L2s.total - L2s.region)
                    p.smem = ds::decode_smem_layout(GT, d, c, p.lay_chunk, p.per, esz, 2, used).total;
            }
            if (used > region_att)
                p.smem = ds::decode_smem_layout(GT, d, c, p.lay_chunk, p.per, esz, p.att_stages, used).total;
        }
        if (forced) {
            if (N == forced) { *out = p; return true; }
            continue;
        }
        if (best.N == 0) best = p;  // smallest feasible
        if ((long long)rows * N <= slots && (N == 1 || p.chunk >= 256)) best = p;
    }
    if (best.N == 0) return false;
    *out = best;
    return true;
}

std::mutex g_attr_mu;
std::unordered_map<const void*, int> g_attr_smem;

cudaError_t prepare_kernel(ds::DecodeKernel kern, int smem, int N) {
    std::lock_guard<std::mutex> lk(g_attr_mu);
    auto it = g_attr_smem.find(reinterpret_cast<const void*>(kern));
    if (it != g_attr_smem.end() && it->second >= smem) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    (void)N;
    g_attr_smem[reinterpret_cast<const void*>(kern)] = kMaxSmem;
    return cudaSuccess;
}

ds::DecodeKernel pick_kernel(ds_dtype kvdt, bool int4, int d, int c, int GT, bool paged = false) {
    if (paged) {
        if (kvdt == DS_F32)
            return int4 ? ds::decode_kernel_f32_i4_paged(d, c, GT) : ds::decode_kernel_f32_fp_paged(d, c, GT);
        return int4 ? ds::decode_kernel_bf16_i4_paged(d, c, GT) : ds::decode_kernel_bf16_fp_paged(d, c, GT);
    }
    if (kvdt == DS_F32) return int4 ? ds::decode_kernel_f32_i4(d, c, GT) : ds::decode_kernel_f32_fp(d, c, GT);
    return int4 ? ds::decode_kernel_bf16_i4(d, c, GT) : ds::decode_kernel_bf16_fp(d, c, GT);
}

ds_status launch_decode(ds::DecodeKernel kern, const ds::DecodeParams& p, int rows, const Plan& pl,
                        cudaStream_t st) {
    cudaError_t e = prepare_kernel(kern, pl.smem, pl.N);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(rows * pl.N), 1, 1);
    cfg.blockDim = dim3(ds::kNT, 1, 1);
    cfg.dynamicSmemBytes = (size_t)pl.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)pl.N;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, p);
    if (e != cudaSuccess) return cuda_fail(e, "decode launch");
    return DS_OK;
}

}  // namespace

namespace ds {

// Process-unique id of the calling thread's current CUDA context (0 and
// false when there is none or the driver does not provide one). Caches of
// device addresses are keyed by it: a context created after a device reset
// gets a new id, and its modules (and their __device__ variables) may sit
// elsewhere. The driver functions are fetched through the runtime, so the
// library does not link the driver library itself.
bool current_context_id(unsigned long long* id) {
    using GetCurrent = int (*)(void**);
    using GetId = int (*)(void*, unsigned long long*);
    static GetCurrent get_current = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            f = nullptr;
        return reinterpret_cast<GetCurrent>(f);
    }();
    static GetId get_id = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &f, 12000, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            f = nullptr;
        return reinterpret_cast<GetId>(f);
    }();
    void* ctx = nullptr;
    *id = 0;
    return get_current && get_id && get_current(&ctx) == 0 && ctx && get_id(ctx, id) == 0;
}

}  // namespace ds

namespace {

// A barrier that nothing completes: the bounded wait runs out after
// `limit_ns` and records site bit 0 (ds_selftest_bounded_wait).
__global__ void ds_selftest_wait_kernel(unsigned int* err, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        ds::mbar_init(&bar, 1);
        ds::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) ds::mbar_wait_bounded(&bar, 0, err, 0, limit_ns);
}

// Device address of g_status_word in the current context, cached per
// context (host code only has the array's name as a host-side stand-in).
cudaError_t status_word(unsigned int** out) {
    unsigned long long ctx = 0;
    const bool keyed = ds::current_context_id(&ctx);
    std::lock_guard<std::mutex> lk(g_status_mu);
    if (keyed)
        for (int i = 0; i < g_status_used; ++i)
            if (g_status_addr[i].ctx == ctx) { *out = g_status_addr[i].ptr; return cudaSuccess; }
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_status_word);
    if (e != cudaSuccess) return e;
    if (keyed || ds::current_context_id(&ctx)) {
        g_status_addr[g_status_next] = StatusAddr{ctx, static_cast<unsigned int*>(p)};
        g_status_next = (g_status_next + 1) % 16;
        if (g_status_used < 16) ++g_status_used;
    }
    *out = static_cast<unsigned int*>(p);
    return cudaSuccess;
}

ds_status check_common(int b, int hq, int hkv, int s, int s_cap, int d, ds_dtype kvdt) {
    if (b < 1 || hkv < 1 || hq < 1) return fail(DS_ERR_INVALID_ARG, "b, hq and hkv must be >= 1");
    if (hq % hkv) return fail(DS_ERR_INVALID_ARG, "hq (%d) must be a multiple of hkv (%d)", hq, hkv);
    if (hq / hkv > 8) return fail(DS_ERR_UNSUPPORTED, "hq/hkv = %d > 8", hq / hkv);
    if (s < 1 || s > s_cap) return fail(DS_ERR_INVALID_ARG, "need 1 <= s (%d) <= s_cap (%d)", s, s_cap);
    if (!d_ok(d)) return fail(DS_ERR_UNSUPPORTED, "head_dim %d (supported: 64, 128)", d);
    if (!kv_dtype_ok(kvdt)) return fail(DS_ERR_UNSUPPORTED, "k/v dtype %d (supported: f32, bf16)", (int)kvdt);
    if ((long long)b * hkv * (long long)s_cap * d >= (1ll << 40))
        return fail(DS_ERR_UNSUPPORTED, "cache too large");
    if ((long long)b * hkv > (1ll << 26)) return fail(DS_ERR_UNSUPPORTED, "too many rows");
    return DS_OK;
}

ds_status check_label(ds_dtype kdt, ds_dtype label_dt, int c, int d, const void* label,
                      const uint16_t* lscale, const uint16_t* lzero) {
    if (!c_ok(c, d)) return fail(DS_ERR_UNSUPPORTED, "heavy channels c=%d (supported: 8,16,32,64,128; c <= d)", c);
    if (!label) return fail(DS_ERR_INVALID_ARG, "label is NULL");
    if (!aligned16(label)) return fail(DS_ERR_INVALID_ARG, "label not 16-byte aligned");
    if (label_dt == DS_INT4) {
        if (!lscale || !lzero) return fail(DS_ERR_INVALID_ARG, "4-bit label needs lscale and lzero");
        if (!aligned16(lscale) || !aligned16(lzero)) return fail(DS_ERR_INVALID_ARG, "lscale/lzero not 16-byte aligned");
    } else if (label_dt != kdt) {
        return fail(DS_ERR_INVALID_ARG, "label dtype must equal the key dtype or be DS_INT4");
    }
    return DS_OK;
}

// Paged K/V: a block table [b, max_blocks] of block ids into pools
// [num_blocks, hkv, page_size, d].
struct Paged {
    const int32_t* bt = nullptr;
    int max_blocks = 0, page_size = 0, num_blocks = 0;
};

int log2_exact(int x) {
    int l = 0;
    while ((1 << l) < x) ++l;
    return (1 << l) == x ? l : -1;
}

ds_status check_paged(const Paged& pg, int s_max, int hkv, int d) {
    if (!pg.bt) return fail(DS_ERR_INVALID_ARG, "block_table is NULL");
    if (reinterpret_cast<uintptr_t>(pg.bt) % 4) return fail(DS_ERR_INVALID_ARG, "block_table not 4-byte aligned");
    if (pg.page_size < 1 || pg.page_size > (1 << 16) || log2_exact(pg.page_size) < 0)
        return fail(DS_ERR_INVALID_ARG, "page_size %d must be a power of two in [1, 65536]", pg.page_size);
    if (pg.num_blocks < 1 || pg.max_blocks < 1) return fail(DS_ERR_INVALID_ARG, "num_blocks and max_blocks must be >= 1");
    if ((long long)pg.max_blocks * pg.page_size < s_max)
        return fail(DS_ERR_INVALID_ARG, "max_blocks * page_size (%lld) < tokens (%d)",
                    (long long)pg.max_blocks * pg.page_size, s_max);
    if ((long long)pg.num_blocks * hkv * pg.page_size >= (1ll << 32))
        return fail(DS_ERR_UNSUPPORTED, "pool too large (rows must fit 32 bits)");
    if ((long long)pg.num_blocks * hkv * pg.page_size * d >= (1ll << 40))
        return fail(DS_ERR_UNSUPPORTED, "pool too large");
    return DS_OK;
}

ds_status run_label(const void* k, ds_dtype kdt, const int32_t* idx, int b, int hkv, int t_begin,
                    int t_end, int s_cap, int d, int c, void* label, ds_dtype label_dt,
                    uint16_t* lscale, uint16_t* lzero, cudaStream_t st, const Paged* pg = nullptr) {
    ds_status r = check_common(b, hkv, hkv, t_end, s_cap, d, kdt);
    if (r != DS_OK) return r;
    if (pg && (r = check_paged(*pg, t_end, hkv, d)) != DS_OK) return r;
    if ((r = check_label(kdt, label_dt, c, d, label, lscale, lzero)) != DS_OK) return r;
    if (!k || !idx) return fail(DS_ERR_INVALID_ARG, "k or idx is NULL");
    if (!aligned16(k) || !aligned16(idx)) return fail(DS_ERR_INVALID_ARG, "k/idx not 16-byte aligned");
    ds::LabelArgs a{k, kdt == DS_BF16, label_dt == DS_INT4, idx, b, hkv, t_begin, t_end, s_cap, d, c,
                    label, lscale, lzero};
    unsigned int* words = nullptr;
    if (!pg && t_end - t_begin > 1) {
        cudaError_t e = status_word(&words);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
        a.err = words;
        a.sms = sm_count();
    }
    if (pg) {
        a.block_table = pg->bt;
        a.max_blocks = pg->max_blocks;
        a.page_shift = log2_exact(pg->page_size);
        a.num_blocks = pg->num_blocks;
    }
    cudaError_t e = ds::launch_label(a, st);
    if (e != cudaSuccess) return cuda_fail(e, "label launch");
    return DS_OK;
}

}  // namespace

extern "C" {

const char* ds_status_string(ds_status st) {
    switch (st) {
    case DS_OK: return "DS_OK";
    case DS_ERR_INVALID_ARG: return "DS_ERR_INVALID_ARG";
    case DS_ERR_UNSUPPORTED: return "DS_ERR_UNSUPPORTED";
    case DS_ERR_CUDA: return "DS_ERR_CUDA";
    case DS_ERR_WORKSPACE: return "DS_ERR_WORKSPACE";
    case DS_ERR_TIMEOUT: return "DS_ERR_TIMEOUT";
    }
    return "DS_ERR_UNKNOWN";
}

const char* ds_last_error(void) { return g_err; }

void ds_sparse_decode_set_cluster(int n) { g_cluster_override.store(n); }

ds_status ds_sparse_decode_tune(const char* name, int value) {
    if (!name) return fail(DS_ERR_INVALID_ARG, "name is NULL");
    const std::string n(name);
    if (n == "scan_prefetch") {
        if (value > 8) return fail(DS_ERR_INVALID_ARG, "scan_prefetch: 0..8 rounds (<0 default)");
        g_scan_prefetch.store(value < 0 ? 2 : value);
    } else if (n == "i4_ring") {
        if (value > 1) return fail(DS_ERR_INVALID_ARG, "i4_ring: 0 or 1 (<0 default)");
        g_i4_ring.store(value < 0 ? 1 : value);
    } else {
        return fail(DS_ERR_INVALID_ARG, "unknown tuning knob '%s'", name);
    }
    return DS_OK;
}

ds_status ds_selftest_bounded_wait(int polls, cudaStream_t stream) {
    if (polls < 1 || polls > 1000000) return fail(DS_ERR_INVALID_ARG, "polls must be in [1, 1000000]");
    unsigned int* words = nullptr;
    cudaError_t e = status_word(&words);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
    ds_selftest_wait_kernel<<<1, 32, 0, stream>>>(words, (unsigned long long)polls * 1000ull);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
    return DS_OK;
}

ds_status ds_check_device(cudaStream_t stream) {
    unsigned int* words = nullptr;
    cudaError_t e = status_word(&words);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
    unsigned int w = 0;
    e = cudaMemcpyAsync(&w, words, sizeof w, cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device status");
    if (!w) return DS_OK;
    const unsigned int zero = 0;
    e = cudaMemcpyAsync(words, &zero, sizeof zero, cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device status");
    return fail(DS_ERR_TIMEOUT, "a kernel gave up a bounded wait (sites 0x%x: bit 0 self-test, "
                "bit 1 label build stage, bit 2 decode stage)", w);
}

ds_status ds_calibrate_workspace_size(int n_samples, int hq, int hkv, int w, int s, int d,
                                      size_t* bytes) {
    if (!bytes) return fail(DS_ERR_INVALID_ARG, "bytes is NULL");
    if (n_samples < 1 || hkv < 1 || hq < 1 || w < 1 || s < 1)
        return fail(DS_ERR_INVALID_ARG, "sizes must be >= 1");
    if (hq % hkv) return fail(DS_ERR_INVALID_ARG, "hq must be a multiple of hkv");
    if (!d_ok(d)) return fail(DS_ERR_UNSUPPORTED, "head_dim %d (supported: 64, 128)", d);
    *bytes = ds::calib_workspace_bytes(n_samples, hkv, d);
    return DS_OK;
}

ds_status ds_calibrate_channels(const void* q_win, const void* k, ds_dtype dt, int n_samples,
                                int hq, int hkv, int w, int s, int d, int c, float* ratio_out,
                                int32_t* idx_out, void* ws, size_t ws_bytes, cudaStream_t stream) {
    size_t need = 0;
    ds_status r = ds_calibrate_workspace_size(n_samples, hq, hkv, w, s, d, &need);
    if (r != DS_OK) return r;
    if (!kv_dtype_ok(dt)) return fail(DS_ERR_UNSUPPORTED, "dtype %d (supported: f32, bf16)", (int)dt);
    if (c < 1 || c > d) return fail(DS_ERR_INVALID_ARG, "need 1 <= c (%d) <= d (%d)", c, d);
    if (hq / hkv * (long long)w > (1 << 20)) return fail(DS_ERR_UNSUPPORTED, "window too large");
    if (!q_win || !k || !idx_out || !ws) return fail(DS_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(q_win) || !aligned16(k) || !aligned16(idx_out) || !aligned16(ws) ||
        (ratio_out && !aligned16(ratio_out)))
        return fail(DS_ERR_INVALID_ARG, "pointer not 16-byte aligned");
    if (ws_bytes < need) return fail(DS_ERR_WORKSPACE, "workspace %zu B < required %zu B", ws_bytes, need);
    ds::CalibArgs a{q_win, k, dt == DS_BF16, n_samples, hq, hkv, w, s, d, c, ratio_out, idx_out, ws};
    cudaError_t e = ds::launch_calib(a, stream);
    if (e != cudaSuccess) return cuda_fail(e, "calibration launch");
    return DS_OK;
}

ds_status ds_calibrate_channels_criterion(const void* q_win, const void* k, ds_dtype dt, int n_samples,
                                          int hq, int hkv, int w, int s, int d, int c,
                                          ds_calib_criterion criterion, int chunk, float* score_out,
                                          int32_t* idx_out, void* ws, size_t ws_bytes,
                                          cudaStream_t stream) {
    size_t need = 0;
    ds_status r = ds_calibrate_workspace_size(n_samples, hq, hkv, w, s, d, &need);
    if (r != DS_OK) return r;
    if (!kv_dtype_ok(dt)) return fail(DS_ERR_UNSUPPORTED, "dtype %d (supported: f32, bf16)", (int)dt);
    if (c < 1 || c > d) return fail(DS_ERR_INVALID_ARG, "need 1 <= c (%d) <= d (%d)", c, d);
    if ((int)criterion < DS_CRIT_LEANK_RATIO || (int)criterion > DS_CRIT_QK_CHUNKED)
        return fail(DS_ERR_INVALID_ARG, "unknown criterion %d", (int)criterion);
    if (criterion == DS_CRIT_QK_CHUNKED && chunk < 1)
        return fail(DS_ERR_INVALID_ARG, "chunk (%d) must be >= 1", chunk);
    if (hq / hkv * (long long)w > (1 << 20)) return fail(DS_ERR_UNSUPPORTED, "window too large");
    if (!q_win || !k || !idx_out || !ws) return fail(DS_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(q_win) || !aligned16(k) || !aligned16(idx_out) || !aligned16(ws) ||
        (score_out && !aligned16(score_out)))
        return fail(DS_ERR_INVALID_ARG, "pointer not 16-byte aligned");
    if (ws_bytes < need) return fail(DS_ERR_WORKSPACE, "workspace %zu B < required %zu B", ws_bytes, need);
    ds::CalibArgs a{q_win, k, dt == DS_BF16, n_samples, hq, hkv, w, s, d, c, score_out, idx_out, ws};
    a.criterion = (int)criterion;
    a.chunk = criterion == DS_CRIT_QK_CHUNKED ? chunk : 0;
    cudaError_t e = ds::launch_calib(a, stream);
    if (e != cudaSuccess) return cuda_fail(e, "calibration launch");
    return DS_OK;
}

ds_status ds_calibrate_channels_noalloc(const void* q_win, const void* k, ds_dtype dt, int n_samples,
                                        int hq, int hkv, int w, int s, int d, int c, float* ratio_out,
                                        int32_t* idx_out, cudaStream_t stream) {
    size_t need = 0;
    ds_status r = ds_calibrate_workspace_size(n_samples, hq, hkv, w, s, d, &need);
    if (r != DS_OK) return r;
    if (!kv_dtype_ok(dt)) return fail(DS_ERR_UNSUPPORTED, "dtype %d (supported: f32, bf16)", (int)dt);
    if (c < 1 || c > d) return fail(DS_ERR_INVALID_ARG, "need 1 <= c (%d) <= d (%d)", c, d);
    if (hq / hkv * (long long)w > (1 << 20)) return fail(DS_ERR_UNSUPPORTED, "window too large");
    if (!q_win || !k || !idx_out) return fail(DS_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(q_win) || !aligned16(k) || !aligned16(idx_out) || (ratio_out && !aligned16(ratio_out)))
        return fail(DS_ERR_INVALID_ARG, "pointer not 16-byte aligned");
    const size_t cap = ds::calib_static_scratch_bytes();
    if (need > cap)
        return fail(DS_ERR_WORKSPACE,
                    "calibration needs %zu B of scratch (n_samples * hkv * (2d + 1) doubles); the fixed "
                    "scratch holds %zu B: use ds_calibrate_channels with a workspace", need, cap);
    ds::CalibArgs a{q_win, k, dt == DS_BF16, n_samples, hq, hkv, w, s, d, c, ratio_out, idx_out, nullptr};
    cudaError_t e = ds::launch_calib_static(a, stream);
    if (e != cudaSuccess) return cuda_fail(e, "calibration launch (fixed scratch)");
    return DS_OK;
}

ds_status ds_build_label_cache(const void* k, ds_dtype kdt, const int32_t* idx, int b, int hkv,
                               int s, int s_cap, int d, int c, void* label, ds_dtype label_dt,
                               uint16_t* lscale, uint16_t* lzero, cudaStream_t stream) {
    return run_label(k, kdt, idx, b, hkv, 0, s, s_cap, d, c, label, label_dt, lscale, lzero, stream);
}

ds_status ds_append_label(const void* k, ds_dtype kdt, const int32_t* idx, int b, int hkv, int pos,
                          int s_cap, int d, int c, void* label, ds_dtype label_dt, uint16_t* lscale,
                          uint16_t* lzero, cudaStream_t stream) {
    if (pos < 0 || pos >= s_cap) return fail(DS_ERR_INVALID_ARG, "need 0 <= pos (%d) < s_cap (%d)", pos, s_cap);
    return run_label(k, kdt, idx, b, hkv, pos, pos + 1, s_cap, d, c, label, label_dt, lscale, lzero,
                     stream);
}

ds_status ds_sparse_decode_workspace(int b, int hq, int hkv, int s, int d, int c, int topk,
                                     size_t* bytes) {
    if (!bytes) return fail(DS_ERR_INVALID_ARG, "bytes is NULL");
    ds_status r = check_common(b, hq, hkv, s, s, d, DS_BF16);
    if (r != DS_OK) return r;
    if (!c_ok(c, d)) return fail(DS_ERR_UNSUPPORTED, "heavy channels c=%d (supported: 8,16,32,64,128; c <= d)", c);
    if (topk < 1) return fail(DS_ERR_INVALID_ARG, "topk must be >= 1");
    // scores, the selection and the softmax partials of a step stay on chip
    *bytes = 0;
    return DS_OK;
}

ds_status ds_sparse_decode_plan(int b, int hq, int hkv, int s, int d, int c, int topk, ds_dtype kvdt,
                                ds_dtype label_dt, int* cluster_out, int* chunk_out, int* smem_out) {
    ds_status r = check_common(b, hq, hkv, s, s, d, kvdt);
    if (r != DS_OK) return r;
    if (!c_ok(c, d)) return fail(DS_ERR_UNSUPPORTED, "heavy channels c=%d", c);
    if (label_dt != DS_INT4 && label_dt != kvdt) return fail(DS_ERR_INVALID_ARG, "label dtype");
    if (topk < 1) return fail(DS_ERR_INVALID_ARG, "topk must be >= 1");
    Plan pl;
    if (!make_plan(b * hkv, hq / hkv, s, d, c, topk, false, label_dt == DS_INT4, kvdt == DS_F32 ? 4 : 2,
                   kCtasPerSm * 148,
                   g_cluster_override.load(), &pl, s))
        return fail(DS_ERR_UNSUPPORTED, "no feasible launch plan (s too long for 16 CTAs per row)");
    if (cluster_out) *cluster_out = pl.N;
    if (chunk_out) *chunk_out = pl.chunk;
    if (smem_out) *smem_out = pl.smem;
    return DS_OK;
}

}  // extern "C"

namespace {

ds_status sparse_decode_impl(const void* q, const void* k, const void* v, ds_dtype kvdt, const void* label,
                             ds_dtype label_dt, const uint16_t* lscale, const uint16_t* lzero,
                             const int32_t* idx, int b, int hq, int hkv, int s, int s_cap, int d, int c,
                             int topk, float sm_scale, void* out, ds_dtype out_dt, int32_t* sel_out,
                             float* score_out, bool append, const int32_t* seq_lens, int threshold,
                             int batch_rule, cudaStream_t stream, const Paged* pg = nullptr,
                             const void* k_new = nullptr, const void* v_new = nullptr) {
    ds_status r = check_common(b, hq, hkv, s, s_cap, d, kvdt);
    if (r != DS_OK) return r;
    if (pg && (r = check_paged(*pg, s, hkv, d)) != DS_OK) return r;
    if ((k_new == nullptr) != (v_new == nullptr)) return fail(DS_ERR_INVALID_ARG, "give both k_new and v_new or neither");
    if (k_new && (!aligned16(k_new) || !aligned16(v_new))) return fail(DS_ERR_INVALID_ARG, "k_new/v_new not 16-byte aligned");
    if ((r = check_label(kvdt, label_dt, c, d, label, lscale, lzero)) != DS_OK) return r;
    if (topk < 1) return fail(DS_ERR_INVALID_ARG, "topk must be >= 1");
    if (!q || !k || !v || !idx || !out) return fail(DS_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(out) ||
        (sel_out && !aligned16(sel_out)) || (score_out && !aligned16(score_out)))
        return fail(DS_ERR_INVALID_ARG, "pointer not 16-byte aligned");
    if (!(out_dt == DS_F32 || (out_dt == DS_BF16 && kvdt == DS_BF16)))
        return fail(DS_ERR_INVALID_ARG, "out dtype must be DS_F32 or (with bf16 k/v) DS_BF16");
    if (!(sm_scale == sm_scale)) return fail(DS_ERR_INVALID_ARG, "sm_scale is NaN");
    const int G = hq / hkv, GT = group_tier(G);
    const int rows = b * hkv;
    Plan pl;
    if (!make_plan(rows, G, s, d, c, topk, false, label_dt == DS_INT4, kvdt == DS_F32 ? 4 : 2,
                   kCtasPerSm * sm_count(),
                   g_cluster_override.load(), &pl, s_cap))
        return fail(DS_ERR_UNSUPPORTED, "no feasible launch plan (s too long for 16 CTAs per row)");
    ds::DecodeKernel kern = pick_kernel(kvdt, label_dt == DS_INT4, d, c, GT, pg != nullptr);
    if (!kern) return fail(DS_ERR_UNSUPPORTED, "no kernel for d=%d c=%d G=%d", d, c, G);
    ds::DecodeParams p{};
    if (seq_lens && !aligned16(seq_lens)) return fail(DS_ERR_INVALID_ARG, "seq_lens not 16-byte aligned");
    p.q = q; p.k = k; p.v = v; p.label = label; p.lscale = lscale; p.lzero = lzero; p.idx = idx;
    p.seq_lens = seq_lens;
    p.nb = b;
    p.threshold = threshold;
    p.batch_rule = batch_rule;
    p.k_new = k_new;
    p.v_new = v_new;
    if (pg) {
        p.block_table = pg->bt;
        p.max_blocks = pg->max_blocks;
        p.page_shift = log2_exact(pg->page_size);
        p.num_blocks = pg->num_blocks;
    }
    p.out = out; p.sel_out = sel_out; p.score_out = score_out;
    p.hkv = hkv; p.G = G; p.s = s; p.s_cap = s_cap; p.topk = topk;
    p.chunk = pl.chunk; p.lay_chunk = pl.lay_chunk; p.per = pl.per;
    p.append = append ? 1 : 0;
    p.att_stages = pl.att_stages;
    p.lab_ring = pl.lab_ring;
    p.keep_low = pl.keep_low;
    const float scale = sm_scale > 0.f ? sm_scale : 1.0f / sqrtf((float)d);
    p.qscale = scale * 1.4426950408889634f;
    p.out_bf16 = out_dt == DS_BF16;
    p.dense = 0;
    p.scan_prefetch = g_scan_prefetch.load();
    p.sel_off = pl.sel_off;
    return launch_decode(kern, p, rows, pl, stream);
}

}  // namespace

extern "C" {

ds_status ds_sparse_decode(const void* q, const void* k, const void* v, ds_dtype kvdt,
                           const void* label, ds_dtype label_dt, const uint16_t* lscale,
                           const uint16_t* lzero, const int32_t* idx, int b, int hq, int hkv, int s,
                           int s_cap, int d, int c, int topk, float sm_scale, void* out,
                           ds_dtype out_dt, int32_t* sel_out, float* score_out, cudaStream_t stream) {
    return sparse_decode_impl(q, k, v, kvdt, label, label_dt, lscale, lzero, idx, b, hq, hkv, s, s_cap, d, c,
                              topk, sm_scale, out, out_dt, sel_out, score_out, false, nullptr, 0, 0, stream);
}

ds_status ds_decode_step(const void* q, const void* k, const void* v, ds_dtype kvdt, void* label,
                         ds_dtype label_dt, uint16_t* lscale, uint16_t* lzero, const int32_t* idx, int b,
                         int hq, int hkv, int s, int s_cap, int d, int c, int topk, float sm_scale,
                         void* out, ds_dtype out_dt, int32_t* sel_out, float* score_out,
                         cudaStream_t stream) {
    return sparse_decode_impl(q, k, v, kvdt, label, label_dt, lscale, lzero, idx, b, hq, hkv, s, s_cap, d, c,
                              topk, sm_scale, out, out_dt, sel_out, score_out, true, nullptr, 0, 0, stream);
}

ds_status ds_decode_step_kv(const void* q, const void* k_new, const void* v_new, void* k, void* v, ds_dtype kvdt,
                            void* label, ds_dtype label_dt, uint16_t* lscale, uint16_t* lzero, const int32_t* idx,
                            int b, int hq, int hkv, int s, int s_cap, int d, int c, int topk, float sm_scale,
                            void* out, ds_dtype out_dt, int32_t* sel_out, float* score_out, cudaStream_t stream) {
    if (!k_new || !v_new) return fail(DS_ERR_INVALID_ARG, "k_new or v_new is NULL");
    return sparse_decode_impl(q, k, v, kvdt, label, label_dt, lscale, lzero, idx, b, hq, hkv, s, s_cap, d, c,
                              topk, sm_scale, out, out_dt, sel_out, score_out, true, nullptr, 0, 0, stream, nullptr,
                              k_new, v_new);
}

ds_status ds_decode_step_varlen(const void* q, const void* k, const void* v, ds_dtype kvdt, void* label,
                                ds_dtype label_dt, uint16_t* lscale, uint16_t* lzero, const int32_t* idx,
                                const int32_t* seq_lens, int sparse_threshold, ds_fallback fallback, int b,
                                int hq, int hkv, int s_max, int s_cap, int d, int c, int topk, float sm_scale,
                                void* out, ds_dtype out_dt, int32_t* sel_out, float* score_out,
                                cudaStream_t stream) {
    if (!seq_lens) return fail(DS_ERR_INVALID_ARG, "seq_lens is NULL");
    if (sparse_threshold < 0) return fail(DS_ERR_INVALID_ARG, "sparse_threshold (%d) < 0", sparse_threshold);
    if (fallback != DS_FALLBACK_PER_ENTRY && fallback != DS_FALLBACK_BATCH)
        return fail(DS_ERR_INVALID_ARG, "unknown fallback rule %d", (int)fallback);
    return sparse_decode_impl(q, k, v, kvdt, label, label_dt, lscale, lzero, idx, b, hq, hkv, s_max, s_cap, d, c,
                              topk, sm_scale, out, out_dt, sel_out, score_out, true, seq_lens, sparse_threshold,
                              fallback == DS_FALLBACK_BATCH ? 1 : 0, stream);
}

ds_status ds_build_label_cache_paged(const void* k_pool, ds_dtype kdt, const int32_t* idx,
                                     const int32_t* block_table, int max_blocks, int page_size, int num_blocks,
                                     int b, int hkv, int s, int s_cap, int d, int c, void* label,
                                     ds_dtype label_dt, uint16_t* lscale, uint16_t* lzero, cudaStream_t stream) {
    Paged pg;
    pg.bt = block_table; pg.max_blocks = max_blocks; pg.page_size = page_size; pg.num_blocks = num_blocks;
    return run_label(k_pool, kdt, idx, b, hkv, 0, s, s_cap, d, c, label, label_dt, lscale, lzero, stream, &pg);
}

ds_status ds_decode_step_paged(const void* q, const void* k_pool, const void* v_pool, ds_dtype kvdt, void* label,
                               ds_dtype label_dt, uint16_t* lscale, uint16_t* lzero, const int32_t* idx,
                               const int32_t* block_table, int max_blocks, int page_size, int num_blocks,
                               const int32_t* seq_lens, int sparse_threshold, ds_fallback fallback, int b,
                               int hq, int hkv, int s_max, int s_cap, int d, int c, int topk, float sm_scale,
                               void* out, ds_dtype out_dt, int32_t* sel_out, float* score_out,
                               cudaStream_t stream) {
    if (sparse_threshold < 0) return fail(DS_ERR_INVALID_ARG, "sparse_threshold (%d) < 0", sparse_threshold);
    if (fallback != DS_FALLBACK_PER_ENTRY && fallback != DS_FALLBACK_BATCH)
        return fail(DS_ERR_INVALID_ARG, "unknown fallback rule %d", (int)fallback);
    Paged pg;
    pg.bt = block_table; pg.max_blocks = max_blocks; pg.page_size = page_size; pg.num_blocks = num_blocks;
    return sparse_decode_impl(q, k_pool, v_pool, kvdt, label, label_dt, lscale, lzero, idx, b, hq, hkv, s_max, s_cap,
                              d, c, topk, sm_scale, out, out_dt, sel_out, score_out, true, seq_lens,
                              sparse_threshold, fallback == DS_FALLBACK_BATCH ? 1 : 0, stream, &pg);
}

ds_status ds_dense_decode(const void* q, const void* k, const void* v, ds_dtype kvdt, int b, int hq,
                          int hkv, int s, int s_cap, int d, float sm_scale, void* out,
                          ds_dtype out_dt, cudaStream_t stream) {
    ds_status r = check_common(b, hq, hkv, s, s_cap, d, kvdt);
    if (r != DS_OK) return r;
    if (!q || !k || !v || !out) return fail(DS_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return fail(DS_ERR_INVALID_ARG, "pointer not 16-byte aligned");
    if (!(out_dt == DS_F32 || (out_dt == DS_BF16 && kvdt == DS_BF16)))
        return fail(DS_ERR_INVALID_ARG, "out dtype must be DS_F32 or (with bf16 k/v) DS_BF16");
    const int G = hq / hkv, GT = group_tier(G);
    const int rows = b * hkv;
    Plan pl;
    if (!make_plan(rows, G, s, d, 8, s, true, false, kvdt == DS_F32 ? 4 : 2, kCtasPerSm * sm_count(),
                   g_cluster_override.load(), &pl))
        return fail(DS_ERR_UNSUPPORTED, "no feasible launch plan");
    ds::DecodeKernel kern = pick_kernel(kvdt, false, d, 8, GT);
    if (!kern) return fail(DS_ERR_UNSUPPORTED, "no kernel for d=%d G=%d", d, G);
    ds::DecodeParams p{};
    p.q = q; p.k = k; p.v = v; p.out = out;
    p.hkv = hkv; p.G = G; p.s = s; p.s_cap = s_cap; p.topk = s;
    p.chunk = pl.chunk; p.lay_chunk = 0; p.per = 0;
    p.att_stages = pl.att_stages;
    p.lab_ring = pl.lab_ring;
    p.keep_low = pl.keep_low;
    const float scale = sm_scale > 0.f ? sm_scale : 1.0f / sqrtf((float)d);
    p.qscale = scale * 1.4426950408889634f;
    p.out_bf16 = out_dt == DS_BF16;
    p.dense = 1;
    return launch_decode(kern, p, rows, pl, stream);
}

}  // extern "C"
