/*
 * ds.h -- C ABI of the B200 (sm_100a) Double Sparsity decode-attention library
 * (libds.so).
 *
 * Double Sparsity ("大模型稀疏化技术原理：Double Sparsity", joto.ai blog) speeds up
 * decode attention in two stages. Offline, a few samples fix the heavy key
 * channels of each head (section 离线校准). At run time:
 *   step 1  gather the query's heavy channels,
 *   step 2  score every cached token approximately against a contiguous "label
 *           cache" holding only those channels of K (optionally 4-bit),
 *   step 3  keep the top-k tokens and run exact softmax attention over their
 *           full K/V rows (section 在线前向计算).
 * The channel criterion is the importance ratio of "K通道静态性量化方法解析"
 * (aitangshan.cn) §1.1: r_i = ||Q[i]K[i]^T|| / ||QK^T||.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Pointers are DEVICE pointers owned by the caller, unless stated. The
 *    library allocates nothing, frees nothing and does not synchronise: work is
 *    enqueued on `stream` (0 = legacy default stream) and runs asynchronously.
 *  - Tensors are dense, row-major, with these layouts:
 *      q        [b, hq, d]                  query of the current decode token
 *      k, v     [b, hkv, s_cap, d]          key / value cache; tokens [0, s) valid
 *      idx      [hkv, c]    int32           heavy channels per kv head, each in [0, d)
 *                                           (kernels clamp out-of-range values into
 *                                           [0, d); the host does not read idx)
 *      label    [b, hkv, s_cap, c]          fp label cache (dtype of k), or
 *               [b, hkv, s_cap, c/2] bytes  4-bit label cache: channel 2j in the
 *                                           low nibble of byte j, 2j+1 in the high
 *      lscale, lzero [b, hkv, s_cap]        fp16 bit patterns (4-bit cache only)
 *      out      [b, hq, d]                  attention output
 *    Query head h belongs to kv head h / (hq / hkv).
 *  - Every device pointer must be 16-byte aligned.
 *  - Arguments are validated before anything is launched. A failed check
 *    returns DS_ERR_INVALID_ARG (or DS_ERR_UNSUPPORTED for a valid but
 *    unimplemented shape) and enqueues nothing. A CUDA launch error returns
 *    DS_ERR_CUDA. ds_last_error() gives a one-line reason for the last
 *    failure on the calling thread. No exception or exit crosses this ABI.
 *  - Supported: d in {64, 128}; c in {8, 16, 32, 64, 128} with c <= d;
 *    hq / hkv <= 8; k/v dtype DS_F32 or DS_BF16; label dtype equal to the k
 *    dtype or DS_INT4; 1 <= s <= s_cap.
 */
#ifndef DS_H
#define DS_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define DS_API __attribute__((visibility("default")))
#else
#define DS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DS_OK = 0,
    DS_ERR_INVALID_ARG = 1,
    DS_ERR_UNSUPPORTED = 2,
    DS_ERR_CUDA = 3,
    DS_ERR_WORKSPACE = 4,
    DS_ERR_TIMEOUT = 5
} ds_status;

typedef enum { DS_F32 = 0, DS_BF16 = 1, DS_F16 = 2, DS_INT4 = 3 } ds_dtype;

/* Human-readable name of a status code (static string). */
DS_API const char* ds_status_string(ds_status st);

/* One-line reason for the last non-DS_OK status returned on this thread
 * (static thread-local buffer; empty string if none). */
DS_API const char* ds_last_error(void);

/* ------------------------------------------------------------ calibration
 * Offline channel selection ("K通道静态性量化方法解析" §1.1; Double Sparsity
 * 离线校准). For every calibration sample n and kv head g, Q_g stacks the
 * observation windows of the group's query heads ((hq/hkv)*w rows) and K_g
 * holds the s keys:
 *     r[g, i] = mean_n ||Q_g[:, i] K_g[:, i]^T||_F / ||Q_g K_g^T||_F
 * (a head with Q_g K_g^T == 0 contributes 0). idx_out[g] receives the c
 * channels with the largest r (ties to the lower channel), ascending.
 *
 *   q_win      [n_samples, hq, w, d]   dtype `dt` (DS_F32 or DS_BF16)
 *   k          [n_samples, hkv, s, d]  dtype `dt`
 *   ratio_out  [hkv, d] float32, or NULL
 *   idx_out    [hkv, c] int32
 *   ws         caller-owned device scratch of at least
 *              ds_calibrate_workspace_size() bytes (16-byte aligned); its
 *              contents on entry do not matter. DS_ERR_WORKSPACE if too small.
 */
DS_API ds_status ds_calibrate_workspace_size(int n_samples, int hq, int hkv, int w, int s, int d,
                                      size_t* bytes);
DS_API ds_status ds_calibrate_channels(const void* q_win, const void* k, ds_dtype dt,
                                int n_samples, int hq, int hkv, int w, int s, int d, int c,
                                float* ratio_out, int32_t* idx_out,
                                void* ws, size_t ws_bytes, cudaStream_t stream);

/* Channel ranking criteria for ds_calibrate_channels_criterion. The
 * Double Sparsity page ("大模型稀疏化技术原理：Double Sparsity", 离线校准)
 * lists outlier strategies by query, key and query*key; "K通道静态性量化方法
 * 解析" §2.1 says Double Sparsity's offline collection takes norms of the QK
 * product chunked along the context. Per sample n and kv head g (Q_g, K_g as
 * for ds_calibrate_channels), channel i scores
 *   DS_CRIT_LEANK_RATIO  ||Q_g[:,i] K_g[:,i]^T||_F / ||Q_g K_g^T||_F  (= ds_calibrate_channels)
 *   DS_CRIT_Q_OUTLIER    ||Q_g[:,i]||_2
 *   DS_CRIT_K_OUTLIER    ||K_g[:,i]||_2
 *   DS_CRIT_QK_OUTLIER   ||Q_g[:,i] K_g[:,i]^T||_F  (= ||Q_g[:,i]|| ||K_g[:,i]||)
 *   DS_CRIT_QK_CHUNKED   sum over chunks [j*chunk, min(s, (j+1)*chunk)) of
 *                        ||Q_g[:,i] K_g[chunk,i]^T||_F
 * and the score is the mean over samples. The activation-outlier strategy
 * ranks channels of the layer input, before the projections, and is not
 * offered: this library starts from Q and K. */
typedef enum {
    DS_CRIT_LEANK_RATIO = 0,
    DS_CRIT_Q_OUTLIER = 1,
    DS_CRIT_K_OUTLIER = 2,
    DS_CRIT_QK_OUTLIER = 3,
    DS_CRIT_QK_CHUNKED = 4
} ds_calib_criterion;

/* ds_calibrate_channels with a choice of criterion. `chunk` (>= 1) is the
 * context chunk length of DS_CRIT_QK_CHUNKED and is ignored otherwise.
 * score_out [hkv, d] float32 (or NULL) receives the mean score; idx_out and
 * the workspace are as for ds_calibrate_channels (same size). Ties go to the
 * lower channel. DS_ERR_INVALID_ARG for an unknown criterion or chunk < 1. */
DS_API ds_status ds_calibrate_channels_criterion(const void* q_win, const void* k, ds_dtype dt,
                                                 int n_samples, int hq, int hkv, int w, int s,
                                                 int d, int c, ds_calib_criterion criterion,
                                                 int chunk, float* score_out, int32_t* idx_out,
                                                 void* ws, size_t ws_bytes, cudaStream_t stream);

/* Calibration for callers that cannot allocate device memory: plugins whose
 * host framework owns every allocation and hands them only fixed tensors, or
 * runtimes that work inside a device budget fixed up front, so that a call
 * to cudaMalloc (or to an allocator that may call it) is not open to them.
 * It has no
 * counterpart on the pages; it computes exactly what ds_calibrate_channels
 * computes, with the same arguments minus the workspace. Its scratch is a
 * fixed 1 MiB device array inside the library (held by every GPU that loads
 * the library until the process exits), so it needs
 * n_samples * hkv * (2*d + 1) * 8 <= 1048576 bytes (ds_calibrate_workspace_size
 * gives the figure); larger problems get DS_ERR_WORKSPACE with the numbers.
 * It allocates nothing and calls no allocating routine. The first call in a
 * CUDA context looks up the array's device address (with that device current)
 * and caches it for the context; a context created later, e.g. after a device
 * reset, is looked up afresh on its first call. Make that first call before
 * any stream capture. All calls
 * share the array and each clears the part it uses: calls that may run
 * concurrently on the GPU (different streams without ordering) race on it. */
DS_API ds_status ds_calibrate_channels_noalloc(const void* q_win, const void* k, ds_dtype dt,
                                               int n_samples, int hq, int hkv, int w, int s, int d,
                                               int c, float* ratio_out, int32_t* idx_out,
                                               cudaStream_t stream);

/* ----------------------------------------------------------- label cache
 * Prefill (Double Sparsity 离线校准, label cache paragraph): copy the heavy
 * channels of tokens [0, s) of the key cache into the label cache.
 *   fp label  : label[b,g,t,j] = k[b,g,t,idx[g,j]]  (bit-exact copy; label_dt == kdt)
 *   4-bit     : per (b, g, t), in fp32: mn/mx over the c values,
 *               scale = fp16_rn((mx-mn)/15), zero = fp16_rn(mn),
 *               code_j = scale > 0 ? clamp(rint((x_j - zero)/scale), 0, 15) : 0
 *               (IEEE division, round half to even); lscale/lzero receive the
 *               fp16 bits. Requires c even. Dequantised value: scale*code + zero.
 * Rows t >= s are not touched.
 */
DS_API ds_status ds_build_label_cache(const void* k, ds_dtype kdt, const int32_t* idx,
                               int b, int hkv, int s, int s_cap, int d, int c,
                               void* label, ds_dtype label_dt,
                               uint16_t* lscale, uint16_t* lzero, cudaStream_t stream);

/* Decode-time append: the same copy/pack for the single token at position
 * `pos` (0 <= pos < s_cap), after the caller has written k[:, :, pos, :]. */
DS_API ds_status ds_append_label(const void* k, ds_dtype kdt, const int32_t* idx,
                          int b, int hkv, int pos, int s_cap, int d, int c,
                          void* label, ds_dtype label_dt,
                          uint16_t* lscale, uint16_t* lzero, cudaStream_t stream);

/* ------------------------------------------------------ sparse decode step
 * One decode step of Double Sparsity (在线前向计算 steps 1-3), fused in one
 * launch. Per batch b and kv head g:
 *   qL[j]  = sum_{h in group g} q[b, h, idx[g, j]]                  (step 1)
 *   s_t    = sum_j qL[j] * label[b, g, t, j]        for t < s        (step 2)
 *            (4-bit: label value scale_t*code + zero_t; fp32 arithmetic)
 *   sel    = the min(topk, s) tokens with the largest s_t, ties to the
 *            lower token index (exact on the fp32 scores)             (step 3)
 *   out[b,h] = softmax_{t in sel}(sm_scale * q[b,h].k[b,g,t]) . v[b,g,t]
 * topk >= s selects every token (dense attention over the cache).
 *
 *   q, k, v    dtype kvdt (DS_F32 or DS_BF16)
 *   sm_scale   <= 0 selects 1/sqrt(d)
 *   out        dtype out_dt (DS_F32, or DS_BF16 when kvdt is DS_BF16)
 *   sel_out    [b, hkv, topk] int32 or NULL: the selected tokens in ascending
 *              order; entries past min(topk, s) are -1
 *   score_out  [b, hkv, s] float32 or NULL: the approximate scores s_t
 * No workspace: scores, the selection and the partial softmax states stay in
 * on-chip memory of one thread-block cluster per (b, g).
 */
DS_API ds_status ds_sparse_decode(const void* q, const void* k, const void* v, ds_dtype kvdt,
                           const void* label, ds_dtype label_dt,
                           const uint16_t* lscale, const uint16_t* lzero, const int32_t* idx,
                           int b, int hq, int hkv, int s, int s_cap, int d, int c, int topk,
                           float sm_scale, void* out, ds_dtype out_dt,
                           int32_t* sel_out, float* score_out, cudaStream_t stream);

/* Device scratch ds_sparse_decode needs for a shape, in bytes (host only,
 * launches nothing). The decode step of 在线前向计算 keeps its per-step
 * intermediates -- the approximate scores of step 2, the top-k selection of
 * step 3 and the partial softmax states -- in shared memory of the thread-block
 * cluster serving each (b, g), so the answer is 0 for every supported shape and
 * ds_sparse_decode takes no workspace argument. Validates the shape like
 * ds_sparse_decode (DS_ERR_INVALID_ARG / DS_ERR_UNSUPPORTED, *bytes untouched). */
DS_API ds_status ds_sparse_decode_workspace(int b, int hq, int hkv, int s, int d, int c, int topk,
                                            size_t* bytes);

/* One decode step in one launch (Double Sparsity 离线校准 + 在线前向计算):
 * the label row of the newest token, position s-1, whose K/V the caller has
 * already written, is built exactly as ds_append_label builds it and stored
 * to label (and lscale/lzero for 4-bit); then the step runs exactly as
 * ds_sparse_decode over tokens [0, s). Same arguments and rules as
 * ds_sparse_decode; only row s-1 of the label cache is written. */
DS_API ds_status ds_decode_step(const void* q, const void* k, const void* v, ds_dtype kvdt,
                                void* label, ds_dtype label_dt,
                                uint16_t* lscale, uint16_t* lzero, const int32_t* idx,
                                int b, int hq, int hkv, int s, int s_cap, int d, int c, int topk,
                                float sm_scale, void* out, ds_dtype out_dt,
                                int32_t* sel_out, float* score_out, cudaStream_t stream);

/* ds_decode_step that also takes the new token's key and value rows,
 * k_new and v_new [b, hkv, d] (dtype kvdt, device or device-mapped, 16-byte
 * aligned), and writes them into k and v at position s-1 itself before using
 * them: the serving loop then needs one host-to-device copy (q, k_new, v_new
 * side by side) and this one launch per layer and step. Otherwise the same
 * arguments and results as ds_decode_step with those rows already in the
 * caches. DS_ERR_INVALID_ARG if k_new or v_new is NULL. */
DS_API ds_status ds_decode_step_kv(const void* q, const void* k_new, const void* v_new,
                                   void* k, void* v, ds_dtype kvdt,
                                   void* label, ds_dtype label_dt,
                                   uint16_t* lscale, uint16_t* lzero, const int32_t* idx,
                                   int b, int hq, int hkv, int s, int s_cap, int d, int c, int topk,
                                   float sm_scale, void* out, ds_dtype out_dt,
                                   int32_t* sel_out, float* score_out, cudaStream_t stream);

/* When a batch entry is decoded with every one of its tokens instead of its
 * top-k (the pages' SGLang section: --ds-sparse-decode-threshold and the
 * heavy-token count decide when Double Sparsity is not used).
 *   DS_FALLBACK_PER_ENTRY  entry b attends all its tokens when
 *                          s_b <= topk or s_b < sparse_threshold; the other
 *                          entries of the batch still select topk tokens.
 *   DS_FALLBACK_BATCH      the rule as SGLang states it, for the whole batch:
 *                          every entry attends all its tokens when
 *                          max_b s_b < sparse_threshold or min_b s_b < topk. */
typedef enum { DS_FALLBACK_PER_ENTRY = 0, DS_FALLBACK_BATCH = 1 } ds_fallback;

/* ds_decode_step for a batch of sequences of different lengths (serving):
 * seq_lens [b] (device, int32) gives each batch entry's token count s_b, and
 * kernels clamp it into [1, s_max]. Row (b, g) appends its token s_b - 1 and
 * attends over its own top-min(topk, s_b) of tokens [0, s_b), or over all of
 * [0, s_b) when the fallback rule says so (sparse_threshold >= 0; 0 disables
 * the threshold part). score_out is laid out [b, hkv, s_max] with entries
 * t >= s_b untouched. sel_out: the selected tokens, ascending, padded with
 * -1; a row that attends all its tokens lists them when s_b <= topk and is
 * all -1 otherwise. The launch is planned for s_max.
 * DS_ERR_INVALID_ARG for seq_lens == NULL, a negative threshold or an
 * unknown rule. */
DS_API ds_status ds_decode_step_varlen(const void* q, const void* k, const void* v, ds_dtype kvdt,
                                       void* label, ds_dtype label_dt,
                                       uint16_t* lscale, uint16_t* lzero, const int32_t* idx,
                                       const int32_t* seq_lens, int sparse_threshold,
                                       ds_fallback fallback,
                                       int b, int hq, int hkv, int s_max, int s_cap, int d, int c,
                                       int topk, float sm_scale, void* out, ds_dtype out_dt,
                                       int32_t* sel_out, float* score_out, cudaStream_t stream);

/* ------------------------------------------------------------ paged K/V
 * The serving layout the pages' SGLang section implies (a shared pool of
 * fixed-size pages instead of one contiguous cache per sequence). The key and
 * value pools are [num_blocks, hkv, page_size, d] (dtype kdt / kvdt) and
 * block_table [b, max_blocks] (int32, device) names, for batch entry b, the
 * block that holds its tokens [j * page_size, (j + 1) * page_size): token t
 * is row t % page_size of block block_table[b * max_blocks + t / page_size].
 * Block ids are clamped into [0, num_blocks). page_size is a power of two in
 * [1, 65536], max_blocks * page_size >= the token count, and
 * num_blocks * hkv * page_size < 2^32. The label cache stays dense
 * [b, hkv, s_cap, c] (s_cap is its capacity). block_table needs 4-byte
 * alignment, the pools 16. Same results as the dense-layout calls on the
 * same values. */

/* ds_build_label_cache for a paged key pool: label rows [0, s). */
DS_API ds_status ds_build_label_cache_paged(const void* k_pool, ds_dtype kdt, const int32_t* idx,
                                            const int32_t* block_table, int max_blocks,
                                            int page_size, int num_blocks, int b, int hkv, int s,
                                            int s_cap, int d, int c, void* label, ds_dtype label_dt,
                                            uint16_t* lscale, uint16_t* lzero, cudaStream_t stream);

/* ds_decode_step_varlen over paged K/V pools. seq_lens may be NULL (every
 * entry has s_max tokens). */
DS_API ds_status ds_decode_step_paged(const void* q, const void* k_pool, const void* v_pool,
                                      ds_dtype kvdt, void* label, ds_dtype label_dt,
                                      uint16_t* lscale, uint16_t* lzero, const int32_t* idx,
                                      const int32_t* block_table, int max_blocks, int page_size,
                                      int num_blocks, const int32_t* seq_lens,
                                      int sparse_threshold, ds_fallback fallback,
                                      int b, int hq, int hkv, int s_max, int s_cap, int d, int c,
                                      int topk, float sm_scale, void* out, ds_dtype out_dt,
                                      int32_t* sel_out, float* score_out, cudaStream_t stream);

/* Launch plan of ds_sparse_decode for a shape (host only, launches nothing),
 * for caches of capacity s on a 148-SM B200: CTAs per thread-block cluster
 * (one cluster per (b, kv head)), tokens per CTA and dynamic shared memory
 * per CTA in bytes. Any output may be NULL. */
DS_API ds_status ds_sparse_decode_plan(int b, int hq, int hkv, int s, int d, int c, int topk,
                                ds_dtype kvdt, ds_dtype label_dt,
                                int* cluster_out, int* chunk_out, int* smem_out);

/* Force the cluster size (1, 2, 4, 8 or 16 CTAs per (b, kv head) row) used
 * by ds_sparse_decode, ds_dense_decode and ds_sparse_decode_plan in this
 * process; 0 restores the automatic choice. A forced size that does not fit
 * a shape makes those calls return DS_ERR_UNSUPPORTED. Tuning/testing knob. */
DS_API void ds_sparse_decode_set_cluster(int n);

/* Process-wide tuning/testing knobs of ds_sparse_decode and the decode steps
 * (prefetch and staging choices; results never depend on them). A negative value restores
 * the default. DS_ERR_INVALID_ARG for an unknown name or a value out of
 * range.
 *   "scan_prefetch" (0..8, default 2) label scan through registers (when the
 *                   shared-memory ring does not fit): rounds of label rows
 *                   prefetched into L2 ahead.
 *   "i4_ring"       (0 or 1, default 1) 4-bit label rows: when the label ring
 *                   and the kept low key bits do not both fit, 1 takes the
 *                   ring (bucket tokens are then re-scored), 0 the low bits. */
DS_API ds_status ds_sparse_decode_tune(const char* name, int value);

/* Every wait of a kernel on a transaction barrier (a bulk copy landing in
 * shared memory) polls a bounded number of times. A wait that gives up
 * records where in a status word inside the library and the kernel leaves
 * instead of hanging the GPU; the results of that launch are then undefined.
 * ds_check_device synchronises `stream`, reads the word and clears it:
 * DS_OK if no wait gave up since the last check, else DS_ERR_TIMEOUT
 * (ds_last_error names the sites). Not a hot-path call. */
DS_API ds_status ds_check_device(cudaStream_t stream);

/* Self-test of that mechanism: launches one thread that waits on a
 * transaction barrier nothing completes, for about `polls` microseconds, so
 * the wait runs out and is recorded (site bit 0); the next ds_check_device
 * returns DS_ERR_TIMEOUT. DS_ERR_INVALID_ARG unless 1 <= polls <= 1000000. */
DS_API ds_status ds_selftest_bounded_wait(int polls, cudaStream_t stream);

/* ------------------------------------------------------------- baseline
 * Dense decode attention over tokens [0, s) of the same cache (no label,
 * no selection): the measurement baseline the sparse step is compared with.
 * Same layouts and rules as ds_sparse_decode. */
DS_API ds_status ds_dense_decode(const void* q, const void* k, const void* v, ds_dtype kvdt,
                          int b, int hq, int hkv, int s, int s_cap, int d,
                          float sm_scale, void* out, ds_dtype out_dt, cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* DS_H */
