/*
 * flint_oracle.c -- plain, slow, float64 CPU reference for one decode step of
 * Flint attention.  TEST INFRASTRUCTURE ONLY: it is used by tests/, by the
 * smoke check in __graft_entry__.py and by bench.py's CPU-baseline leg, never
 * by the product path.  It shares no code, header or constant table with the
 * CUDA library.
 *
 * What it computes (sources are the pages' titles and sections):
 *   - "Day-0 Support for Flint on vLLM" (hnkhoi.com/news/1467), "Model
 *     architecture": grouped-query attention with 32 query heads over 4 KV
 *     heads, learned attention sinks, per-head Q/K RMSNorm, 35 layers with a
 *     513-token sliding window and RoPE, 14 full-context layers with no
 *     positional encoding; only the full layers keep KV for the whole sequence.
 *   - "Recursive Flint" model JSON (studiotvai.com/api/models/flint.json),
 *     `architecture` ("GQA 4 KV x 128") and `kvCacheGiBPerRequest`.
 *   - "Day-0 Support for Flint on vLLM" (newruntime.com), "What happened":
 *     BF16 KV cache, fused normalization / rotary-position / cache operations.
 *   - "Recursive Flint" model JSON, the "fp8" column of kvCacheGiBPerRequest:
 *     a one-byte cache variant (format reading in the FP8 section below).
 * The pages print no formula.  The numeric definitions this library adopts
 * are: softmax over [q.k_j / sqrt(d) for j in window, sink_h], where the sink
 * logit carries no value; window at position t = max(0, t-512) .. t; RMSNorm
 * y = x * w / sqrt(mean(x^2) + eps), eps = 1e-6; RoPE in rotate-half form over
 * all d dims, pairs (i, i + d/2), angle t * theta^(-2i/d), theta = 10000.
 *
 * Every function works on general shapes (nq, nkv, d) so that the pins in
 * tests/ can use special cases (e.g. nkv == nq for the GQA check).
 * bf16 values travel as their uint16 bit patterns; arithmetic is float64.
 * Parity status: every function here is pinned by a -m "not gpu" test.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- bf16 <-> float64 -------------------------------------------------- */

/* bf16 is the top half of an IEEE binary32; the widening is exact. */
double fo_bf16_to_f64(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a float64 to the nearest bf16 (8 significant bits), ties to even.
 * The quantum is 2^(e-7) for a normal result with exponent e and 2^-133 in
 * the subnormal range; nearbyint() rounds half to even in the default mode. */
uint16_t fo_f64_to_bf16(double x)
{
    if (isnan(x)) return 0x7fc0;
    if (x == 0.0) return signbit(x) ? 0x8000 : 0x0000;
    if (isinf(x)) return signbit(x) ? 0xff80 : 0x7f80;
    int e = ilogb(x);
    if (e < -126) e = -126;
    double q = ldexp(1.0, e - 7);
    double r = nearbyint(x / q) * q;
    if (fabs(r) >= ldexp(1.0, 128)) return signbit(x) ? 0xff80 : 0x7f80;
    float f = (float)r; /* exact: r has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

void fo_bf16_to_f64_array(const uint16_t* src, double* dst, long n)
{
    for (long i = 0; i < n; ++i) dst[i] = fo_bf16_to_f64(src[i]);
}

void fo_f64_to_bf16_array(const double* src, uint16_t* dst, long n)
{
    for (long i = 0; i < n; ++i) dst[i] = fo_f64_to_bf16(src[i]);
}

/* ---- per-head RMSNorm ("per-head Q/K RMSNorm", Model architecture) ------ */

/* y[r][i] = x[r][i] * w[i] / sqrt(mean_i x[r][i]^2 + eps); w == NULL means
 * all-ones.  The weight is used as given (no 1 + w form) and is shared by all
 * heads of the tensor. */
void fo_rmsnorm_rows(const double* x, int rows, int d, const double* w,
                     double eps, double* y)
{
    for (int r = 0; r < rows; ++r) {
        const double* xr = x + (long)r * d;
        double ss = 0.0;
        for (int i = 0; i < d; ++i) ss += xr[i] * xr[i];
        double inv = 1.0 / sqrt(ss / d + eps);
        for (int i = 0; i < d; ++i)
            y[(long)r * d + i] = xr[i] * inv * (w ? w[i] : 1.0);
    }
}

/* ---- RoPE on the sliding-window layers (Model architecture) ------------- */

/* Rotate-half form: for i < d/2 the pair (x_i, x_{i+d/2}) is turned by the
 * angle pos * theta^(-2i/d).  Done in place, in float64 throughout. */
void fo_rope_rows(double* x, int rows, int d, long pos, double theta)
{
    int half = d / 2;
    for (int r = 0; r < rows; ++r) {
        double* xr = x + (long)r * d;
        for (int i = 0; i < half; ++i) {
            double a = (double)pos * pow(theta, -2.0 * i / d);
            double c = cos(a), s = sin(a);
            double x0 = xr[i], x1 = xr[i + half];
            xr[i] = x0 * c - x1 * s;
            xr[i + half] = x1 * c + x0 * s;
        }
    }
}

/* ---- fused per-head norm (+ RoPE) of q and k for one token -------------- */

/* q_raw [nq][d], k_raw [nkv][d] bf16 bits; w_q, w_k [d] bf16 bits or NULL
 * (NULL skips the norm).  Outputs q_out [nq][d], k_out [nkv][d] in float64
 * and, if k_bf16 != NULL, the bf16 (round-to-nearest-even) of k_out: the
 * value appended to the cache. */
void fo_qk_norm_rope(const uint16_t* q_raw, const uint16_t* k_raw,
                     const uint16_t* w_q, const uint16_t* w_k,
                     int nq, int nkv, int d, long pos, double eps,
                     double theta, int apply_rope, double* q_out,
                     double* k_out, uint16_t* k_bf16)
{
    double* xq = (double*)malloc(sizeof(double) * (size_t)nq * d);
    double* xk = (double*)malloc(sizeof(double) * (size_t)nkv * d);
    double* wq = (double*)malloc(sizeof(double) * (size_t)d);
    double* wk = (double*)malloc(sizeof(double) * (size_t)d);
    fo_bf16_to_f64_array(q_raw, xq, (long)nq * d);
    fo_bf16_to_f64_array(k_raw, xk, (long)nkv * d);
    if (w_q) {
        fo_bf16_to_f64_array(w_q, wq, d);
        fo_rmsnorm_rows(xq, nq, d, wq, eps, q_out);
    } else {
        memcpy(q_out, xq, sizeof(double) * (size_t)nq * d);
    }
    if (w_k) {
        fo_bf16_to_f64_array(w_k, wk, d);
        fo_rmsnorm_rows(xk, nkv, d, wk, eps, k_out);
    } else {
        memcpy(k_out, xk, sizeof(double) * (size_t)nkv * d);
    }
    if (apply_rope) {
        fo_rope_rows(q_out, nq, d, pos, theta);
        fo_rope_rows(k_out, nkv, d, pos, theta);
    }
    if (k_bf16) fo_f64_to_bf16_array(k_out, k_bf16, (long)nkv * d);
    free(xq); free(xk); free(wq); free(wk);
}

/* ---- where a logical position lives in the cache ------------------------ */

/* Cache layouts (all bf16, rows of [nkv][d]):
 *   0 contiguous: row = pos                   (cache [capacity][nkv][d])
 *   1 ring:       row = pos mod capacity      (sliding layers keep only the
 *                                              window: capacity 513)
 *   2 paged:      row = table[pos / bs] * bs + pos mod bs
 *                                             (cache [num_blocks][bs][nkv][d])
 * The ring reading follows "Only those 14 keep KV for the whole sequence"
 * (Model architecture) and the per-request KV sizes of the model JSON. */
long fo_storage_row(int layout, long pos, int capacity,
                    const int32_t* block_table, int block_size)
{
    switch (layout) {
    case 0: return pos;
    case 1: return pos % capacity;
    case 2: return (long)block_table[pos / block_size] * block_size + pos % block_size;
    default: return -1;
    }
}

/* Write k, v ([nkv][d] bf16 bits, already final) at position pos. */
void fo_kv_append(uint16_t* k_cache, uint16_t* v_cache, int layout,
                  int capacity, const int32_t* block_table, int block_size,
                  int nkv, int d, long pos, const uint16_t* k,
                  const uint16_t* v)
{
    long row = fo_storage_row(layout, pos, capacity, block_table, block_size);
    memcpy(k_cache + row * nkv * d, k, sizeof(uint16_t) * (size_t)nkv * d);
    memcpy(v_cache + row * nkv * d, v, sizeof(uint16_t) * (size_t)nkv * d);
}

/* ---- decode attention with a per-head sink logit ------------------------ */

/* One request, query position t = L - 1.  Head h reads KV head h / (nq/nkv)
 * (contiguous GQA groups).  The window is {max(0, t-(window-1)) .. t} for
 * window > 0, else {0 .. t}.  With s_j = q_h . K[j] / sqrt(d):
 *     M     = max(max_j s_j, sink_h)
 *     out_h = sum_j e^(s_j - M) V[j] / (sum_j e^(s_j - M) + e^(sink_h - M))
 * sinks[h] may be -INFINITY (then the sink drops out).
 * q [nq][d], out [nq][d] float64.  Returns 0, or -1 on bad arguments. */
int fo_attn_decode(const double* q, int nq, int nkv, int d,
                   const uint16_t* k_cache, const uint16_t* v_cache,
                   int layout, int capacity, const int32_t* block_table,
                   int block_size, long L, int window, const double* sinks,
                   double* out, int nthreads)
{
    if (L < 1 || nq <= 0 || nkv <= 0 || nq % nkv != 0 || d <= 0) return -1;
    long t = L - 1;
    long lo = (window > 0 && t - (window - 1) > 0) ? t - (window - 1) : 0;
    long n = t - lo + 1;
    int group = nq / nkv;
    double scale = 1.0 / sqrt((double)d);
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel for schedule(static)
    for (int h = 0; h < nq; ++h) {
        int g = h / group;
        const double* qh = q + (long)h * d;
        double* s = (double*)malloc(sizeof(double) * (size_t)n);
        double mx = sinks[h];
        for (long j = 0; j < n; ++j) {
            long row = fo_storage_row(layout, lo + j, capacity, block_table, block_size);
            const uint16_t* kr = k_cache + (row * nkv + g) * d;
            double dot = 0.0;
            for (int i = 0; i < d; ++i) dot += qh[i] * fo_bf16_to_f64(kr[i]);
            s[j] = dot * scale;
            if (s[j] > mx) mx = s[j];
        }
        double den = exp(sinks[h] - mx);
        double* o = out + (long)h * d;
        for (int i = 0; i < d; ++i) o[i] = 0.0;
        for (long j = 0; j < n; ++j) {
            long row = fo_storage_row(layout, lo + j, capacity, block_table, block_size);
            const uint16_t* vr = v_cache + (row * nkv + g) * d;
            double p = exp(s[j] - mx);
            den += p;
            for (int i = 0; i < d; ++i) o[i] += p * fo_bf16_to_f64(vr[i]);
        }
        for (int i = 0; i < d; ++i) o[i] /= den;
        free(s);
    }
    return 0;
}

/* ---- one layer of one decode step: norm (+RoPE) -> append -> attend ----- */

/* The new token sits at t = L - 1: its k (normed, roped on window layers,
 * rounded to bf16) and v_raw are appended at t, then q attends the window.
 * k_cache / v_cache are modified in place.  out [nq][d] float64. */
int fo_decode_layer(const uint16_t* q_raw, const uint16_t* k_raw,
                    const uint16_t* v_raw, const uint16_t* w_q,
                    const uint16_t* w_k, const double* sinks, int nq, int nkv,
                    int d, uint16_t* k_cache, uint16_t* v_cache, int layout,
                    int capacity, const int32_t* block_table, int block_size,
                    long L, int window, int apply_rope, double eps,
                    double theta, double* out, int nthreads)
{
    if (L < 1) return -1;
    double* q = (double*)malloc(sizeof(double) * (size_t)nq * d);
    double* k = (double*)malloc(sizeof(double) * (size_t)nkv * d);
    uint16_t* kb = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)nkv * d);
    fo_qk_norm_rope(q_raw, k_raw, w_q, w_k, nq, nkv, d, L - 1, eps, theta,
                    apply_rope, q, k, kb);
    fo_kv_append(k_cache, v_cache, layout, capacity, block_table, block_size,
                 nkv, d, L - 1, kb, v_raw);
    int rc = fo_attn_decode(q, nq, nkv, d, k_cache, v_cache, layout, capacity,
                            block_table, block_size, L, window, sinks, out,
                            nthreads);
    free(q); free(k); free(kb);
    return rc;
}

/* ---- FP8 (e4m3) KV cache ------------------------------------------------ */

/* The "fp8" column of kvCacheGiBPerRequest ("Recursive Flint" model JSON)
 * stores one byte per cached value, half of bf16; the pages give no format.
 * Reading adopted: OCP 8-bit floating point E4M3 -- 1 sign bit, 4 exponent
 * bits with bias 7, 3 mantissa bits; exponent field 0 holds subnormals
 * m * 2^-9; the code S.1111.111 is NaN; no infinities; largest magnitude
 * 448 (S.1111.110).  Each (layer, KV head) has one float32 scale for K and
 * one for V: the cache holds e4m3(x / scale), read back as value * scale.
 * The division and the rounding decision are taken in float32 (the
 * precision the GPU takes them in): code = rne_satfinite(float(x) / scale). */

double fo_e4m3_to_f64(uint8_t c)
{
    int sgn = c >> 7, e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    double mag = e == 0 ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
    return sgn ? -mag : mag;
}

/* Nearest e4m3 code to x, ties to even; magnitudes at or above 448 (and
 * infinities) saturate to +-448; NaN gives 0x7f. */
uint8_t fo_f64_to_e4m3(double x)
{
    if (isnan(x)) return 0x7f;
    uint8_t sgn = signbit(x) ? 0x80 : 0x00;
    double a = fabs(x);
    if (a >= 448.0) return sgn | 0x7e;
    /* quantum: 2^(e-3) for a in [2^e, 2^(e+1)), e >= -6; 2^-9 below 2^-6 */
    int e2;
    frexp(a, &e2);               /* a = f * 2^e2, f in [0.5, 1) */
    int e = e2 - 1;
    if (e < -6) e = -6;
    double q = ldexp(1.0, e - 3);
    double r = nearbyint(a / q) * q;   /* round half to even (default mode) */
    if (r == 0.0) return sgn;
    frexp(r, &e2);
    e = e2 - 1;                  /* r may have moved up one binade */
    if (e < -6) return sgn | (uint8_t)(r / ldexp(1.0, -9));       /* subnormal */
    int mant = (int)(r / ldexp(1.0, e - 3)) - 8;                  /* 0..7 */
    return sgn | (uint8_t)(((e + 7) << 3) | mant);
}

/* The cache code of x with the given scale: float32 division, then e4m3. */
uint8_t fo_quantize_e4m3(double x, float scale)
{
    float t = (float)x / scale;
    return fo_f64_to_e4m3((double)t);
}

/* Write k ([nkv][d] float64, the normed/roped values) and v ([nkv][d] bf16
 * bits) at position pos of byte caches laid out like the bf16 ones. */
void fo_kv_append_fp8(uint8_t* k_cache, uint8_t* v_cache, int layout,
                      int capacity, const int32_t* block_table, int block_size,
                      int nkv, int d, long pos, const double* k,
                      const uint16_t* v, const float* k_scale,
                      const float* v_scale)
{
    long row = fo_storage_row(layout, pos, capacity, block_table, block_size);
    for (int g = 0; g < nkv; ++g)
        for (int i = 0; i < d; ++i) {
            k_cache[(row * nkv + g) * d + i] = fo_quantize_e4m3(k[g * d + i], k_scale[g]);
            v_cache[(row * nkv + g) * d + i] =
                fo_quantize_e4m3(fo_bf16_to_f64(v[g * d + i]), v_scale[g]);
        }
}

/* fo_attn_decode over e4m3 caches: K[j] = decode(code) * k_scale[g],
 * V[j] = decode(code) * v_scale[g], everything else as there. */
int fo_attn_decode_fp8(const double* q, int nq, int nkv, int d,
                       const uint8_t* k_cache, const uint8_t* v_cache,
                       const float* k_scale, const float* v_scale,
                       int layout, int capacity, const int32_t* block_table,
                       int block_size, long L, int window, const double* sinks,
                       double* out, int nthreads)
{
    if (L < 1 || nq <= 0 || nkv <= 0 || nq % nkv != 0 || d <= 0) return -1;
    long t = L - 1;
    long lo = (window > 0 && t - (window - 1) > 0) ? t - (window - 1) : 0;
    long n = t - lo + 1;
    int group = nq / nkv;
    double scale = 1.0 / sqrt((double)d);
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel for schedule(static)
    for (int h = 0; h < nq; ++h) {
        int g = h / group;
        const double* qh = q + (long)h * d;
        double* s = (double*)malloc(sizeof(double) * (size_t)n);
        double mx = sinks[h];
        for (long j = 0; j < n; ++j) {
            long row = fo_storage_row(layout, lo + j, capacity, block_table, block_size);
            const uint8_t* kr = k_cache + (row * nkv + g) * d;
            double dot = 0.0;
            for (int i = 0; i < d; ++i) dot += qh[i] * (fo_e4m3_to_f64(kr[i]) * (double)k_scale[g]);
            s[j] = dot * scale;
            if (s[j] > mx) mx = s[j];
        }
        double den = exp(sinks[h] - mx);
        double* o = out + (long)h * d;
        for (int i = 0; i < d; ++i) o[i] = 0.0;
        for (long j = 0; j < n; ++j) {
            long row = fo_storage_row(layout, lo + j, capacity, block_table, block_size);
            const uint8_t* vr = v_cache + (row * nkv + g) * d;
            double p = exp(s[j] - mx);
            den += p;
            for (int i = 0; i < d; ++i) o[i] += p * (fo_e4m3_to_f64(vr[i]) * (double)v_scale[g]);
        }
        for (int i = 0; i < d; ++i) o[i] /= den;
        free(s);
    }
    return 0;
}

/* fo_decode_layer with e4m3 caches: norm (+RoPE) -> quantized append -> attend. */
int fo_decode_layer_fp8(const uint16_t* q_raw, const uint16_t* k_raw,
                        const uint16_t* v_raw, const uint16_t* w_q,
                        const uint16_t* w_k, const double* sinks, int nq,
                        int nkv, int d, uint8_t* k_cache, uint8_t* v_cache,
                        const float* k_scale, const float* v_scale, int layout,
                        int capacity, const int32_t* block_table,
                        int block_size, long L, int window, int apply_rope,
                        double eps, double theta, double* out, int nthreads)
{
    if (L < 1) return -1;
    double* q = (double*)malloc(sizeof(double) * (size_t)nq * d);
    double* k = (double*)malloc(sizeof(double) * (size_t)nkv * d);
    fo_qk_norm_rope(q_raw, k_raw, w_q, w_k, nq, nkv, d, L - 1, eps, theta,
                    apply_rope, q, k, NULL);
    fo_kv_append_fp8(k_cache, v_cache, layout, capacity, block_table,
                     block_size, nkv, d, L - 1, k, v_raw, k_scale, v_scale);
    int rc = fo_attn_decode_fp8(q, nq, nkv, d, k_cache, v_cache, k_scale,
                                v_scale, layout, capacity, block_table,
                                block_size, L, window, sinks, out, nthreads);
    free(q); free(k);
    return rc;
}

/* ---- KV bytes per request ("Recursive Flint" JSON, kvCacheGiBPerRequest) */

/* Full layers keep every token, window layers keep min(ctx, window) tokens;
 * each token costs nkv * d values for K and again for V. */
double fo_kv_bytes(long ctx, int n_full, int n_window, int window, int nkv,
                   int d, int elem_bytes)
{
    double per_tok = 2.0 * nkv * d * elem_bytes;
    long kept = ctx < window ? ctx : window;
    return per_tok * ((double)n_full * ctx + (double)n_window * kept);
}

int fo_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
