/*
 * ds_oracle.c -- plain, slow CPU reference for Double Sparsity decode attention.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the oracle the CUDA path is checked
 * against. Only the test-suite, the smoke check and the benchmark's CPU-baseline
 * leg may load it. It shares no code, header, table or helper with the CUDA
 * library, and the CUDA library never calls it.
 *
 * Sources (web pages, cited by title and section):
 *   [DS]    "大模型稀疏化技术原理：Double Sparsity" (joto.ai blog), sections
 *           "离线校准" (offline calibration, label cache, 4-bit label cache) and
 *           "在线前向计算" (online decode: steps 1-3).
 *   [LeanK] "K通道静态性量化方法解析" (aitangshan.cn), §1.1 "通道重要性比率计算"
 *           (the channel importance ratio r_i) and §2.1 "与Double Sparsity的对比分析"
 *           (Double Sparsity's chunked norm collection).
 *
 * Floating point is fp64 except the int4 quantiser, whose integer codes are a
 * decision taken in fp32 by the kernel; the oracle takes it in fp32 too.
 * Readings of what the pages leave open are stated beside each function.
 *
 * Element storage codes (for reading caller arrays): 0 = float32,
 * 1 = bfloat16, 2 = float16. Reading converts each element exactly to double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------ storage reads */

static double f16_bits_to_double(uint16_t h) {
    _Float16 v;
    memcpy(&v, &h, sizeof v);
    return (double)v;
}

static double bf16_bits_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double elem(const void* base, int dtype, size_t i) {
    switch (dtype) {
    case 0: return (double)((const float*)base)[i];
    case 1: return bf16_bits_to_double(((const uint16_t*)base)[i]);
    case 2: return f16_bits_to_double(((const uint16_t*)base)[i]);
    default: return NAN;
    }
}

static size_t elem_size(int dtype) { return dtype == 0 ? 4 : 2; }

/* ------------------------------------------------- calibration  ([LeanK] §1.1)
 *
 * For a head with query window Q (rows x d) and full keys K (s x d):
 *     r_i = ||Q[i] K[i]^T||_2 / ||Q K^T||_2
 * where Q[i], K[i] are the i-th channel columns. Readings:
 *   - "L2 norm of a matrix" is taken entrywise (Frobenius). Q[i]K[i]^T has rank
 *     one, so its spectral and Frobenius norms coincide; the denominator is
 *     common to all channels of a head, so the channel ranking does not depend
 *     on this reading.
 *   - Q of kv head g stacks the observation windows of every query head of the
 *     group (h = g*G .. g*G+G-1), so grouped heads share one channel set.
 *   - r is averaged (arithmetic mean) over the calibration samples.
 *   - a head whose QK^T is identically zero contributes r_i = 0.
 *   - the heavy channels are the c largest r_i (ties to the lower index),
 *     stored in ascending channel order.
 * Both norms are written out as sums of squared entries of the product
 * matrices, exactly as defined.
 */
typedef struct { double r; int i; } ranked_t;

static int cmp_ranked(const void* pa, const void* pb) {
    const ranked_t* a = (const ranked_t*)pa;
    const ranked_t* b = (const ranked_t*)pb;
    if (a->r > b->r) return -1;
    if (a->r < b->r) return 1;
    return (a->i < b->i) ? -1 : (a->i > b->i);
}

static int cmp_int(const void* pa, const void* pb) {
    int a = *(const int*)pa, b = *(const int*)pb;
    return (a > b) - (a < b);
}

int oracle_calibrate(const void* q_win, const void* k, int dtype,
                     int n, int hq, int hkv, int w, int s, int d, int c,
                     double* ratio /* [hkv, d] */, int32_t* idx /* [hkv, c] */) {
    if (n < 1 || hkv < 1 || hq % hkv || w < 1 || s < 1 || d < 1 || c < 1 || c > d)
        return 1;
    const int G = hq / hkv;
    const int rows = G * w;
    double* Q = (double*)malloc(sizeof(double) * (size_t)rows * d);
    double* K = (double*)malloc(sizeof(double) * (size_t)s * d);
    ranked_t* rk = (ranked_t*)malloc(sizeof(ranked_t) * (size_t)d);
    int* pick = (int*)malloc(sizeof(int) * (size_t)c);
    if (!Q || !K || !rk || !pick) { free(Q); free(K); free(rk); free(pick); return 2; }

    for (int g = 0; g < hkv; ++g)
        for (int i = 0; i < d; ++i) ratio[(size_t)g * d + i] = 0.0;

    for (int ns = 0; ns < n; ++ns) {
        for (int g = 0; g < hkv; ++g) {
            /* stack the group's observation windows */
            for (int j = 0; j < G; ++j)
                for (int t = 0; t < w; ++t)
                    for (int i = 0; i < d; ++i) {
                        size_t src = (((size_t)ns * hq + (size_t)g * G + j) * w + t) * d + i;
                        Q[((size_t)j * w + t) * d + i] = elem(q_win, dtype, src);
                    }
            for (int t = 0; t < s; ++t)
                for (int i = 0; i < d; ++i)
                    K[(size_t)t * d + i] = elem(k, dtype, (((size_t)ns * hkv + g) * s + t) * d + i);

            /* denominator: ||Q K^T||_F^2 = sum over (row, t) of (sum_i Q[row,i] K[t,i])^2 */
            double den2 = 0.0;
            for (int row = 0; row < rows; ++row)
                for (int t = 0; t < s; ++t) {
                    double e = 0.0;
                    for (int i = 0; i < d; ++i) e += Q[(size_t)row * d + i] * K[(size_t)t * d + i];
                    den2 += e * e;
                }
            const double den = sqrt(den2);

            /* numerator per channel: ||Q[i] K[i]^T||_F^2 = sum over (row, t) of (Q[row,i] K[t,i])^2 */
            for (int i = 0; i < d; ++i) {
                double num2 = 0.0;
                for (int row = 0; row < rows; ++row)
                    for (int t = 0; t < s; ++t) {
                        double e = Q[(size_t)row * d + i] * K[(size_t)t * d + i];
                        num2 += e * e;
                    }
                double r = den > 0.0 ? sqrt(num2) / den : 0.0;
                ratio[(size_t)g * d + i] += r / (double)n;
            }
        }
    }

    for (int g = 0; g < hkv; ++g) {
        for (int i = 0; i < d; ++i) { rk[i].r = ratio[(size_t)g * d + i]; rk[i].i = i; }
        qsort(rk, (size_t)d, sizeof(ranked_t), cmp_ranked);
        for (int j = 0; j < c; ++j) pick[j] = rk[j].i;
        qsort(pick, (size_t)c, sizeof(int), cmp_int);
        for (int j = 0; j < c; ++j) idx[(size_t)g * c + j] = pick[j];
    }
    free(Q); free(K); free(rk); free(pick);
    return 0;
}

/* ------------------------------------- outlier criteria  ([DS] 离线校准;
 *                                         [LeanK] §2.1 "与Double Sparsity的对比分析")
 *
 * [DS] lists channel strategies by outliers of the query, of the key and of
 * query * key; [LeanK] §2.1 says DS collects norms of the QK product chunked
 * along the context. Readings, for Q (the group's stacked windows, rows x d)
 * and K (s x d) of one sample and kv head:
 *   criterion 1 (Q-outlier):  score_i = L2 norm of the channel column Q[:, i]
 *   criterion 2 (K-outlier):  score_i = L2 norm of K[:, i]
 *   criterion 3 (QK-outlier): score_i = Frobenius norm of the channel's part
 *                             of the product, Q[:, i] K[:, i]^T
 *   criterion 4 (chunked):    the same norm taken over each context chunk
 *                             [j*chunk, min(s, (j+1)*chunk)) and summed over j
 *   criterion 0:              the LeanK ratio of oracle_calibrate.
 * Each is averaged over the samples and ranked like oracle_calibrate. The
 * norms are written out entrywise as defined (no closed form).
 */
int oracle_calibrate_criterion(const void* q_win, const void* k, int dtype,
                               int n, int hq, int hkv, int w, int s, int d, int c,
                               int criterion, int chunk,
                               double* score /* [hkv, d] */, int32_t* idx /* [hkv, c] */) {
    if (criterion == 0)
        return oracle_calibrate(q_win, k, dtype, n, hq, hkv, w, s, d, c, score, idx);
    if (criterion < 0 || criterion > 4 || (criterion == 4 && chunk < 1)) return 1;
    if (n < 1 || hkv < 1 || hq % hkv || w < 1 || s < 1 || d < 1 || c < 1 || c > d)
        return 1;
    const int G = hq / hkv;
    const int rows = G * w;
    double* Q = (double*)malloc(sizeof(double) * (size_t)rows * d);
    double* K = (double*)malloc(sizeof(double) * (size_t)s * d);
    ranked_t* rk = (ranked_t*)malloc(sizeof(ranked_t) * (size_t)d);
    int* pick = (int*)malloc(sizeof(int) * (size_t)c);
    if (!Q || !K || !rk || !pick) { free(Q); free(K); free(rk); free(pick); return 2; }

    for (int g = 0; g < hkv; ++g)
        for (int i = 0; i < d; ++i) score[(size_t)g * d + i] = 0.0;

    for (int ns = 0; ns < n; ++ns) {
        for (int g = 0; g < hkv; ++g) {
            for (int j = 0; j < G; ++j)
                for (int t = 0; t < w; ++t)
                    for (int i = 0; i < d; ++i) {
                        size_t src = (((size_t)ns * hq + (size_t)g * G + j) * w + t) * d + i;
                        Q[((size_t)j * w + t) * d + i] = elem(q_win, dtype, src);
                    }
            for (int t = 0; t < s; ++t)
                for (int i = 0; i < d; ++i)
                    K[(size_t)t * d + i] = elem(k, dtype, (((size_t)ns * hkv + g) * s + t) * d + i);

            for (int i = 0; i < d; ++i) {
                double v = 0.0;
                if (criterion == 1) {
                    double a = 0.0;
                    for (int row = 0; row < rows; ++row) a += Q[(size_t)row * d + i] * Q[(size_t)row * d + i];
                    v = sqrt(a);
                } else if (criterion == 2) {
                    double a = 0.0;
                    for (int t = 0; t < s; ++t) a += K[(size_t)t * d + i] * K[(size_t)t * d + i];
                    v = sqrt(a);
                } else {
                    const int len = criterion == 3 ? s : chunk;
                    for (int t0 = 0; t0 < s; t0 += len) {
                        const int t1 = t0 + len < s ? t0 + len : s;
                        double a = 0.0;
                        for (int row = 0; row < rows; ++row)
                            for (int t = t0; t < t1; ++t) {
                                double e = Q[(size_t)row * d + i] * K[(size_t)t * d + i];
                                a += e * e;
                            }
                        v += sqrt(a);
                    }
                }
                score[(size_t)g * d + i] += v / (double)n;
            }
        }
    }

    for (int g = 0; g < hkv; ++g) {
        for (int i = 0; i < d; ++i) { rk[i].r = score[(size_t)g * d + i]; rk[i].i = i; }
        qsort(rk, (size_t)d, sizeof(ranked_t), cmp_ranked);
        for (int j = 0; j < c; ++j) pick[j] = rk[j].i;
        qsort(pick, (size_t)c, sizeof(int), cmp_int);
        for (int j = 0; j < c; ++j) idx[(size_t)g * c + j] = pick[j];
    }
    free(Q); free(K); free(rk); free(pick);
    return 0;
}

/* ------------------------------------------------ label cache  ([DS] 离线校准)
 *
 * The label cache is a contiguous copy of the heavy K channels of every token:
 *     label[b, g, t, j] = K[b, g, t, idx[g, j]]      for t < s
 * laid out [b, hkv, s_cap, c]. Copying raw element bytes makes it bit-exact.
 * Appending one decode token is the same copy for t = pos only.
 */
int oracle_label_copy(const void* k, int dtype, const int32_t* idx,
                      int b, int hkv, int t_begin, int t_end, int s_cap, int d, int c,
                      void* label) {
    const size_t es = elem_size(dtype);
    for (int bb = 0; bb < b; ++bb)
        for (int g = 0; g < hkv; ++g)
            for (int t = t_begin; t < t_end; ++t)
                for (int j = 0; j < c; ++j) {
                    int ch = idx[(size_t)g * c + j];
                    if (ch < 0 || ch >= d) return 1;
                    size_t src = (((size_t)bb * hkv + g) * s_cap + t) * d + (size_t)ch;
                    size_t dst = (((size_t)bb * hkv + g) * s_cap + t) * c + (size_t)j;
                    memcpy((char*)label + dst * es, (const char*)k + src * es, es);
                }
    return 0;
}

/* ------------------------------------------ 4-bit label cache  ([DS] 离线校准)
 *
 * The pages store the label cache in 4 bits because approximate attention is
 * insensitive to precision; they fix nothing else. Reading (per token and kv
 * head, asymmetric min/max, fp16 scale and zero), in fp32 arithmetic:
 *   x_j = K[idx[j]],  mn = min x_j,  mx = max x_j
 *   scale = fp16_rn((mx - mn) / 15),  zero = fp16_rn(mn)      (IEEE division)
 *   n_j   = scale > 0 ? clamp(rint_even((x_j - zero) / scale), 0, 15) : 0
 *   byte m of the payload = n_{2m} | n_{2m+1} << 4
 * Dequantised value: scale * n_j + zero.
 */
static uint16_t f32_to_f16_bits(float x) {
    _Float16 h = (_Float16)x; /* IEEE round to nearest even */
    uint16_t b;
    memcpy(&b, &h, sizeof b);
    return b;
}

static float f16_bits_to_f32(uint16_t b) {
    _Float16 h;
    memcpy(&h, &b, sizeof h);
    return (float)h;
}

int oracle_label_int4(const void* k, int dtype, const int32_t* idx,
                      int b, int hkv, int t_begin, int t_end, int s_cap, int d, int c,
                      uint8_t* label /* [b,hkv,s_cap,c/2] */,
                      uint16_t* lscale, uint16_t* lzero /* [b,hkv,s_cap] fp16 bits */) {
    if (c % 2) return 1;
    float* x = (float*)malloc(sizeof(float) * (size_t)c);
    if (!x) return 2;
    for (int bb = 0; bb < b; ++bb)
        for (int g = 0; g < hkv; ++g)
            for (int t = t_begin; t < t_end; ++t) {
                const size_t tok = ((size_t)bb * hkv + g) * s_cap + t;
                for (int j = 0; j < c; ++j) {
                    int ch = idx[(size_t)g * c + j];
                    if (ch < 0 || ch >= d) { free(x); return 1; }
                    x[j] = (float)elem(k, dtype, tok * d + (size_t)ch); /* exact */
                }
                float mn = x[0], mx = x[0];
                for (int j = 1; j < c; ++j) {
                    if (x[j] < mn) mn = x[j];
                    if (x[j] > mx) mx = x[j];
                }
                float range = mx - mn;
                float step = range / 15.0f;
                uint16_t sh = f32_to_f16_bits(step);
                uint16_t zh = f32_to_f16_bits(mn);
                float sc = f16_bits_to_f32(sh);
                float z = f16_bits_to_f32(zh);
                lscale[tok] = sh;
                lzero[tok] = zh;
                for (int j = 0; j < c; j += 2) {
                    int nib[2];
                    for (int e = 0; e < 2; ++e) {
                        int code = 0;
                        if (sc > 0.0f) {
                            float diff = x[j + e] - z;
                            float qv = rintf(diff / sc);
                            if (qv < 0.0f) qv = 0.0f;
                            if (qv > 15.0f) qv = 15.0f;
                            code = (int)qv;
                        }
                        nib[e] = code;
                    }
                    label[tok * (size_t)(c / 2) + (size_t)(j / 2)] = (uint8_t)(nib[0] | (nib[1] << 4));
                }
            }
    free(x);
    return 0;
}

/* Dequantise a 4-bit label cache to double: value = scale * n + zero (exact in fp64). */
int oracle_label_int4_values(const uint8_t* label, const uint16_t* lscale, const uint16_t* lzero,
                             int rows, int s, int s_cap, int c, double* out /* [rows, s, c] */) {
    for (int r = 0; r < rows; ++r)
        for (int t = 0; t < s; ++t) {
            const size_t tok = (size_t)r * s_cap + t;
            const double sc = f16_bits_to_double(lscale[tok]);
            const double z = f16_bits_to_double(lzero[tok]);
            for (int j = 0; j < c; ++j) {
                uint8_t byte = label[tok * (size_t)(c / 2) + (size_t)(j / 2)];
                int n = (j & 1) ? (byte >> 4) : (byte & 15);
                out[((size_t)r * s + t) * c + j] = sc * (double)n + z;
            }
        }
    return 0;
}

/* ----------------------------------------- approximate scores  ([DS] steps 1-2)
 *
 * Step 1 gathers the query's heavy channels into a contiguous vector; step 2
 * takes its dot product with every label-cache row. For grouped-query
 * attention the group's query heads are summed into one channel vector
 * (the kv head's channel set is shared by its query heads):
 *     qL[j]   = sum_{h in group g} q[b, h, idx[g, j]]
 *     s[b,g,t] = sum_j qL[j] * label[b, g, t, j]          for t < s
 * No 1/sqrt(d) factor and no softmax: neither changes the ranking.
 * `lab` holds label values as doubles, [b*hkv, s, c].
 */
int oracle_scores(const void* q, int qdtype, const double* lab, const int32_t* idx,
                  int b, int hq, int hkv, int s, int d, int c, double* scores /* [b,hkv,s] */) {
    if (hq % hkv) return 1;
    const int G = hq / hkv;
    double* qL = (double*)malloc(sizeof(double) * (size_t)c);
    if (!qL) return 2;
    for (int bb = 0; bb < b; ++bb)
        for (int g = 0; g < hkv; ++g) {
            for (int j = 0; j < c; ++j) {
                double acc = 0.0;
                for (int e = 0; e < G; ++e) {
                    int h = g * G + e;
                    acc += elem(q, qdtype, ((size_t)bb * hq + h) * d + (size_t)idx[(size_t)g * c + j]);
                }
                qL[j] = acc;
            }
            const size_t r = (size_t)bb * hkv + g;
            for (int t = 0; t < s; ++t) {
                double acc = 0.0;
                for (int j = 0; j < c; ++j) acc += qL[j] * lab[(r * s + t) * c + j];
                scores[r * s + t] = acc;
            }
        }
    free(qL);
    return 0;
}

/* ---------------------------------------------------- top-k  ([DS] step 3)
 *
 * Per (b, kv head) row: the min(k, s) tokens with the largest approximate
 * score. Ties go to the lower token index (a total order, so the selected set
 * is unique). The set is written in ascending token order and padded with -1
 * up to k.
 */
typedef struct { double v; int t; } scored_t;

static int cmp_scored(const void* pa, const void* pb) {
    const scored_t* a = (const scored_t*)pa;
    const scored_t* b = (const scored_t*)pb;
    if (a->v > b->v) return -1;
    if (a->v < b->v) return 1;
    return (a->t < b->t) ? -1 : (a->t > b->t);
}

int oracle_topk(const double* scores, int rows, int s, int k, int32_t* sel /* [rows, k] */) {
    scored_t* buf = (scored_t*)malloc(sizeof(scored_t) * (size_t)s);
    int* pick = (int*)malloc(sizeof(int) * (size_t)(s < k ? s : k));
    if (!buf || !pick) { free(buf); free(pick); return 2; }
    const int m = s < k ? s : k;
    for (int r = 0; r < rows; ++r) {
        for (int t = 0; t < s; ++t) { buf[t].v = scores[(size_t)r * s + t]; buf[t].t = t; }
        qsort(buf, (size_t)s, sizeof(scored_t), cmp_scored);
        for (int j = 0; j < m; ++j) pick[j] = buf[j].t;
        qsort(pick, (size_t)m, sizeof(int), cmp_int);
        for (int j = 0; j < k; ++j) sel[(size_t)r * k + j] = j < m ? pick[j] : -1;
    }
    free(buf); free(pick);
    return 0;
}

/* --------------------------------- exact attention over the selected tokens
 *                                                         ([DS] step 3)
 * Full-channel q, K and V, over the selected tokens only:
 *     z_t = sm_scale * sum_d q[b,h,d] K[b,g,t,d]
 *     out[b,h,:] = sum_t softmax(z)_t V[b,g,t,:]
 * with g = h / G. Entries of `sel` equal to -1 are skipped.
 */
int oracle_attention(const void* q, const void* k, const void* v, int dtype,
                     const int32_t* sel, int kk, int b, int hq, int hkv, int s_cap, int d,
                     double sm_scale, double* out /* [b,hq,d] */) {
    if (hq % hkv) return 1;
    const int G = hq / hkv;
    double* z = (double*)malloc(sizeof(double) * (size_t)kk);
    if (!z) return 2;
    for (int bb = 0; bb < b; ++bb)
        for (int h = 0; h < hq; ++h) {
            const int g = h / G;
            const size_t r = (size_t)bb * hkv + g;
            const int32_t* st = sel + r * (size_t)kk;
            double zmax = -INFINITY;
            for (int j = 0; j < kk; ++j) {
                if (st[j] < 0) { z[j] = -INFINITY; continue; }
                double acc = 0.0;
                for (int e = 0; e < d; ++e)
                    acc += elem(q, dtype, ((size_t)bb * hq + h) * d + e) *
                           elem(k, dtype, (r * s_cap + (size_t)st[j]) * d + e);
                z[j] = acc * sm_scale;
                if (z[j] > zmax) zmax = z[j];
            }
            double l = 0.0;
            for (int j = 0; j < kk; ++j) {
                z[j] = (st[j] < 0) ? 0.0 : exp(z[j] - zmax);
                l += z[j];
            }
            for (int e = 0; e < d; ++e) {
                double acc = 0.0;
                for (int j = 0; j < kk; ++j)
                    if (st[j] >= 0) acc += z[j] * elem(v, dtype, (r * s_cap + (size_t)st[j]) * d + e);
                out[((size_t)bb * hq + h) * d + e] = acc / l;
            }
        }
    free(z);
    return 0;
}
