/*
 * gqa_oracle.c -- plain fp64 CPU reference for the grouped-query-attention forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark may load this file's library.  The product path
 * (the CUDA library and its Python binding) never calls it and shares no code
 * with it.
 *
 * What it computes (the plain definition; no tiling, no online rescaling):
 *
 *   for every batch b, query head h, query row i:
 *     g  = floor(h / G),  G = Hq / Hkv
 *          -- G query heads share one KV head, contiguous grouping
 *             (AstrAI commit log, head-packing commit: "pack HB = min(G, WARPS)
 *             q heads per block"; nvfp4-megamoe-kernel dsv4/kernels/attention
 *             commit log, multi-head decode commit: MQA by a zero KV head stride)
 *     n  = kv_len[b] (logical length; padded capacity rows are never visible --
 *          dsv4 attention commit log, "logical vs padded N" commit)
 *     visible keys V_i = { j : 0 <= j < n  and  (not causal  or  j <= n - Tq + i) }
 *          -- causal masks are aligned bottom-right against the logical length
 *     s_j = scale * sum_c q[b,h,i,c] * k[b,g,j,c]
 *     M   = max( max_{j in V_i} s_j , sink[h] )      (sink term only when given)
 *     Z   = sum_{j in V_i} exp(s_j - M)  +  exp(sink[h] - M)
 *     O[b,h,i,:] = sum_{j in V_i} exp(s_j - M) * v[b,g,j,:] / Z
 *     lse[b,h,i] = M + ln Z
 *   The sink is one extra logit with a zero value row, already in the scaled
 *   domain, so it is never multiplied by scale (dsv4 attention commit log, sink
 *   commit).  With no visible key and no sink, O = 0 and lse = -inf.
 *
 * The LSE combine (oracle_combine) is the plain definition of merging softmax
 * partials over disjoint key sets (kernbench2 benches commit log, the (m, l, O)
 * merge / chain-reduce commits):
 *     lse = ln( sum_s exp(lse_s) + exp(sink_h) ),   O = sum_s exp(lse_s - lse) * O_s
 *
 * Inputs are bf16 bit patterns (uint16); each is widened exactly to double.
 * Layouts: q/out [B, Hq, Tq, d], k/v [B, Hkv, Tkv, d], lse [B, Hq, Tq], all
 * contiguous; Tkv is the buffer capacity.
 *
 * FP8 K/V (the *_fp8kv entry points): K and V are stored as OCP FP8 E4M3 bytes
 * with one scale per tensor, the format of the AstrAI commit log's fp8 family
 * (e4m3 quantize with a per-tensor scale; the consumer multiplies back by the
 * scale).  The value of a byte (sign s, exponent field e, mantissa field m,
 * exponent bias 7):
 *     e = 0            (-1)^s * 2^-6 * m/8          (subnormal)
 *     e = 15, m = 7    NaN                          (the format has no infinities)
 *     otherwise        (-1)^s * 2^(e-7) * (1 + m/8)
 * and the attention above is computed on K = value(k) * k_scale and
 * V = value(v) * v_scale, in double.
 *
 * Every function here is pinned by the CPU tests (closed forms, invariants,
 * brute force at high precision), none by this code itself.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_bits_to_double(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP FP8 E4M3 byte -> double (the table in the header comment). */
static double e4m3_to_double(uint8_t x) {
    const int s = x >> 7, e = (x >> 3) & 15, m = x & 7;
    double v;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else if (e == 15 && m == 7)
        return NAN;
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* K and V elements: bf16 bit patterns (kv_fmt 0) or E4M3 bytes times a
 * per-tensor scale (kv_fmt 1). */
typedef struct {
    const void *k, *v;
    int fmt;
    double k_scale, v_scale;
} kv_src;

static double kv_k(const kv_src *s, long idx) {
    return s->fmt ? e4m3_to_double(((const uint8_t *)s->k)[idx]) * s->k_scale
                  : bf16_bits_to_double(((const uint16_t *)s->k)[idx]);
}
static double kv_v(const kv_src *s, long idx) {
    return s->fmt ? e4m3_to_double(((const uint8_t *)s->v)[idx]) * s->v_scale
                  : bf16_bits_to_double(((const uint16_t *)s->v)[idx]);
}

/* One output row (b, h, i) over the visible keys restricted to [kv_begin, kv_end).
 * s_buf must hold at least Tkv doubles. */
static void attend_row(const uint16_t *q, const kv_src *kv,
                       const int32_t *kv_lens, const float *sink,
                       int B, int Hq, int Hkv, int Tq, int Tkv, int d,
                       double scale, int causal, long kv_begin, long kv_end,
                       int b, int h, int i, double *o_row, double *lse_out,
                       double *s_buf) {
    (void)B;
    const int G = Hq / Hkv;
    const int g = h / G;
    long n = kv_lens ? (long)kv_lens[b] : (long)Tkv;
    if (n > Tkv) n = Tkv;
    if (n < 0) n = 0;
    long last = causal ? (n - Tq + i) : (n - 1);
    if (last > n - 1) last = n - 1;
    long first = 0;
    if (kv_begin > first) first = kv_begin;
    if (kv_end - 1 < last) last = kv_end - 1;

    const uint16_t *qr = q + (((long)b * Hq + h) * Tq + i) * (long)d;
    const long kb = ((long)b * Hkv + g) * (long)Tkv * d;  /* first element of the head's K / V rows */
    const long vb = kb;

    double M = -INFINITY;
    for (long j = first; j <= last; ++j) {
        const long kr = kb + j * (long)d;
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += bf16_bits_to_double(qr[c]) * kv_k(kv, kr + c);
        double s = scale * acc;
        s_buf[j] = s;
        if (s > M) M = s;
    }
    const int has_sink = sink != NULL;
    const double sk = has_sink ? (double)sink[h] : -INFINITY;
    if (sk > M) M = sk;

    for (int c = 0; c < d; ++c) o_row[c] = 0.0;
    if (M == -INFINITY) {   /* nothing visible and no finite sink */
        *lse_out = -INFINITY;
        return;
    }
    double Z = 0.0;
    for (long j = first; j <= last; ++j) {
        double p = exp(s_buf[j] - M);
        Z += p;
        const long vr = vb + j * (long)d;
        for (int c = 0; c < d; ++c) o_row[c] += p * kv_v(kv, vr + c);
    }
    if (has_sink) Z += exp(sk - M);
    for (int c = 0; c < d; ++c) o_row[c] /= Z;
    *lse_out = M + log(Z);
}

static int check_shape(int B, int Hq, int Hkv, int Tq, int Tkv, int d) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Tq < 0 || Tkv < 0 || d <= 0) return -2;
    if (Hq % Hkv != 0) return -2;
    return 0;
}

/* Attention over the key window [kv_begin, kv_end) intersected with each row's
 * visible set: the partial result of one split of the keys.  kv_begin = 0 and
 * kv_end >= Tkv gives the full attention.  out: double [B,Hq,Tq,d]; lse: double
 * [B,Hq,Tq].  nthreads <= 0 uses the OpenMP default. */
static int attention_window(const uint16_t *q, const kv_src *kv,
                            const int32_t *kv_lens, const float *sink,
                            double *out, double *lse,
                            int B, int Hq, int Hkv, int Tq, int Tkv, int d,
                            double scale, int causal, long kv_begin, long kv_end,
                            int nthreads) {
    int rc = check_shape(B, Hq, Hkv, Tq, Tkv, d);
    if (rc) return rc;
    const long rows = (long)B * Hq * Tq;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int fail = 0;
#pragma omp parallel
    {
        double *s_buf = (double *)malloc(sizeof(double) * (size_t)(Tkv > 0 ? Tkv : 1));
        if (!s_buf) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (long r = 0; r < rows; ++r) {
                int i = (int)(r % Tq);
                int h = (int)((r / Tq) % Hq);
                int b = (int)(r / ((long)Tq * Hq));
                attend_row(q, kv, kv_lens, sink, B, Hq, Hkv, Tq, Tkv, d, scale, causal,
                           kv_begin, kv_end, b, h, i, out + r * d, lse + r, s_buf);
            }
            free(s_buf);
        }
    }
    return fail ? -7 : 0;
}

int oracle_attention_window(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                            const int32_t *kv_lens, const float *sink,
                            double *out, double *lse,
                            int B, int Hq, int Hkv, int Tq, int Tkv, int d,
                            double scale, int causal, long kv_begin, long kv_end,
                            int nthreads) {
    const kv_src kv = {k, v, 0, 1.0, 1.0};
    return attention_window(q, &kv, kv_lens, sink, out, lse, B, Hq, Hkv, Tq, Tkv, d, scale, causal,
                            kv_begin, kv_end, nthreads);
}

/* The same with E4M3 K / V bytes and their per-tensor scales. */
int oracle_attention_window_fp8kv(const uint16_t *q, const uint8_t *k, const uint8_t *v,
                                  double k_scale, double v_scale,
                                  const int32_t *kv_lens, const float *sink,
                                  double *out, double *lse,
                                  int B, int Hq, int Hkv, int Tq, int Tkv, int d,
                                  double scale, int causal, long kv_begin, long kv_end,
                                  int nthreads) {
    const kv_src kv = {k, v, 1, k_scale, v_scale};
    return attention_window(q, &kv, kv_lens, sink, out, lse, B, Hq, Hkv, Tq, Tkv, d, scale, causal,
                            kv_begin, kv_end, nthreads);
}

/* The full attention. */
int oracle_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                     const int32_t *kv_lens, const float *sink,
                     double *out, double *lse,
                     int B, int Hq, int Hkv, int Tq, int Tkv, int d,
                     double scale, int causal, int nthreads) {
    return oracle_attention_window(q, k, v, kv_lens, sink, out, lse, B, Hq, Hkv, Tq, Tkv, d,
                                   scale, causal, 0, (long)Tkv, nthreads);
}

/* The full attention for a list of rows only: rows[r] = (b*Hq + h)*Tq + i.
 * out: double [nrows, d]; lse: double [nrows]. */
static int attention_rows(const uint16_t *q, const kv_src *kv,
                          const int32_t *kv_lens, const float *sink,
                          const int64_t *rows, long nrows, double *out, double *lse,
                          int B, int Hq, int Hkv, int Tq, int Tkv, int d,
                          double scale, int causal, int nthreads) {
    int rc = check_shape(B, Hq, Hkv, Tq, Tkv, d);
    if (rc) return rc;
    const long total = (long)B * Hq * Tq;
    for (long r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= total) return -2;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int fail = 0;
#pragma omp parallel
    {
        double *s_buf = (double *)malloc(sizeof(double) * (size_t)(Tkv > 0 ? Tkv : 1));
        if (!s_buf) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long r = 0; r < nrows; ++r) {
                long fr = (long)rows[r];
                int i = (int)(fr % Tq);
                int h = (int)((fr / Tq) % Hq);
                int b = (int)(fr / ((long)Tq * Hq));
                attend_row(q, kv, kv_lens, sink, B, Hq, Hkv, Tq, Tkv, d, scale, causal,
                           0, (long)Tkv, b, h, i, out + r * d, lse + r, s_buf);
            }
            free(s_buf);
        }
    }
    return fail ? -7 : 0;
}

int oracle_attention_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                          const int32_t *kv_lens, const float *sink,
                          const int64_t *rows, long nrows, double *out, double *lse,
                          int B, int Hq, int Hkv, int Tq, int Tkv, int d,
                          double scale, int causal, int nthreads) {
    const kv_src kv = {k, v, 0, 1.0, 1.0};
    return attention_rows(q, &kv, kv_lens, sink, rows, nrows, out, lse, B, Hq, Hkv, Tq, Tkv, d,
                          scale, causal, nthreads);
}

int oracle_attention_rows_fp8kv(const uint16_t *q, const uint8_t *k, const uint8_t *v,
                                double k_scale, double v_scale,
                                const int32_t *kv_lens, const float *sink,
                                const int64_t *rows, long nrows, double *out, double *lse,
                                int B, int Hq, int Hkv, int Tq, int Tkv, int d,
                                double scale, int causal, int nthreads) {
    const kv_src kv = {k, v, 1, k_scale, v_scale};
    return attention_rows(q, &kv, kv_lens, sink, rows, nrows, out, lse, B, Hq, Hkv, Tq, Tkv, d,
                          scale, causal, nthreads);
}

/* E4M3 bytes -> doubles (for the pins of the decoder). */
void oracle_e4m3_decode(const uint8_t *in, double *out, long n) {
    for (long i = 0; i < n; ++i) out[i] = e4m3_to_double(in[i]);
}

/* Merge S partial results per row.  o_part: float [rows, S, d] (each partial
 * normalized over its own keys); lse_part: float [rows, S] (natural log, -inf for
 * a partial with no keys); rows = B*Hq*Tq; sink: float [Hq] or NULL.
 * out: double [rows, d]; lse: double [rows]. */
int oracle_combine(const float *o_part, const float *lse_part, int S, const float *sink,
                   double *out, double *lse, int B, int Hq, int Tq, int d) {
    if (B < 0 || Hq <= 0 || Tq < 0 || d <= 0 || S <= 0) return -2;
    const long rows = (long)B * Hq * Tq;
    for (long r = 0; r < rows; ++r) {
        const int h = (int)((r / Tq) % Hq);
        double L = -INFINITY;
        for (int s = 0; s < S; ++s) {
            double l = (double)lse_part[r * S + s];
            if (l > L) L = l;
        }
        double sk = sink ? (double)sink[h] : -INFINITY;
        if (sk > L) L = sk;
        double *o = out + r * d;
        for (int c = 0; c < d; ++c) o[c] = 0.0;
        if (L == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        double Z = 0.0;
        for (int s = 0; s < S; ++s) Z += exp((double)lse_part[r * S + s] - L);
        if (sink) Z += exp(sk - L);
        const double total_lse = L + log(Z);
        for (int s = 0; s < S; ++s) {
            double w = exp((double)lse_part[r * S + s] - total_lse);
            if (w == 0.0) continue;
            const float *os = o_part + (r * S + s) * (long)d;
            for (int c = 0; c < d; ++c) o[c] += w * (double)os[c];
        }
        lse[r] = total_lse;
    }
    return 0;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
