/*
 * arkattn_oracle.c -- plain, slow, fp64 CPU oracle for GQA attention over a
 * static, sequence-major KV cache (the ARK-ASR-3B decoder attention).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library.  The CUDA product
 * path never calls it, and the two share no code: this file has its own bf16
 * conversion, its own RoPE table and its own softmax.
 *
 * What it computes, and where the pages state it:
 *   - Shapes: 16 query heads, 2 KV heads (grouped-query attention), head dim
 *     128, static cache cache_{key,value}_i of shape [1, max_total_len, 2, 128],
 *     sequence-major.  "ARK-ASR-3B -- INT8 ONNX" model card, section Shapes.
 *   - Each call produces key_delta/value_delta rows for the positions it
 *     writes, and those rows land in the cache at cache_position.  Same
 *     card, section Shapes.
 *   - The decoder is a Qwen2 language model (SGLang-Omni cookbook page
 *     "ARK-ASR-3B", introduction), so RoPE is applied to the new query and key
 *     rows in the Qwen2 rotate-half form.  The pages do not print the RoPE
 *     formula; the reading used here (pairs i and i+D/2, inverse frequency
 *     theta^(-2i/D), absolute position cache_position + t) is the plain Qwen2
 *     convention.
 *   - The static graph attends over ALL max_total_len positions with the
 *     positions past the valid length masked ("ARK-ASR-3B -- INT8 ONNX",
 *     section Shapes).  Masking gives those positions weight exactly zero, so
 *     the result is softmax attention over the valid prefix; ora_attend_one is
 *     that definition and ora_attend_one_static is the literal masked form.
 *   - Precision: bf16 is the serving dtype (SGLang-Omni "ARK-ASR-3B", section
 *     dtype).  Inputs are bf16; this oracle decodes them exactly to double and
 *     computes everything in double.
 *
 * Rounding reading for the RoPE outputs (the pages say nothing): the cos/sin
 * table is cos/sin of the fp64 angle rounded once to fp32; each rotated value
 * x[i]*c - x[i+64]*s (or x[i+64]*c + x[i]*s) is formed in fp64 and rounded once
 * to bf16, round-to-nearest-even.  With bf16 inputs and fp32 table entries the
 * products are exact in fp64.
 *
 * Two neighbours of the decoder attention, for the tests of their kernels:
 *   - ora_attention_bidir: the audio encoder's bidirectional multi-head
 *     attention ("Inside ARK-ASR-3B's Whisper and Qwen architecture",
 *     components; reading: 20 heads of 64, every frame of a clip attends to
 *     every frame of the same clip, q and k already rotated).
 *   - ora_qkv_proj: the Q/K/V projections in front of the attention ("ARK-ASR-3B
 *     -- INT8 ONNX" model card, Qwen2 decoder, hidden 2048) as one Linear over
 *     the concatenated weight, the sum in double and one rounding to bf16.
 *
 * Every function here is a direct, unblocked statement of its definition.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Threads the OpenMP loops of this library use (1 without OpenMP). */
int ora_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---------------------------------------------------------------- bf16 ---- */

/* bf16 is the upper half of an IEEE-754 binary32 value; widening is exact. */
double ora_bf16_to_f64(uint16_t h) {
    uint32_t bits = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/*
 * Round a double to the nearest bf16 value, ties to even, by the IEEE-754
 * definition: find the two neighbouring bf16 values and pick the closer one.
 * Written out on the binary64 encoding: sign, exponent and a 52-bit fraction.
 * bf16 keeps 8 significant bits (7 stored), the binary32 exponent range, and
 * binary32's subnormals (2^-133 .. 2^-126).
 */
uint16_t ora_f64_to_bf16_rne(double x) {
    uint64_t b;
    memcpy(&b, &x, sizeof b);
    uint16_t sign = (uint16_t)((b >> 48) & 0x8000u);
    int e = (int)((b >> 52) & 0x7ff);
    uint64_t frac = b & 0xFFFFFFFFFFFFFull;
    if (e == 0x7ff) {                       /* inf or nan */
        if (frac) return (uint16_t)(sign | 0x7FC0u);
        return (uint16_t)(sign | 0x7F80u);
    }
    if (e == 0 && frac == 0) return sign;   /* signed zero */
    double a = fabs(x);
    /* unbiased exponent of a: a = m * 2^E with m in [1,2) */
    int E;
    double m = frexp(a, &E);                /* a = m * 2^E, m in [0.5,1) */
    E -= 1;                                 /* now m*2 in [1,2) */
    (void)m;
    /* spacing of bf16 values around a: normal range E >= -126 has 2^(E-7);
       below that the spacing is fixed at the subnormal step 2^-133. */
    int q = (E >= -126) ? (E - 7) : -133;
    double step = ldexp(1.0, q);
    double n = floor(a / step);             /* a/step is exact: power-of-2 scale */
    double lo = n * step;
    double rem = a - lo;                    /* exact */
    double half = step * 0.5;
    double r;
    if (rem > half) r = lo + step;
    else if (rem < half) r = lo;
    else r = (fmod(n, 2.0) == 0.0) ? lo : lo + step;
    /* r is now a bf16 value or 2^128 (overflow) */
    if (r >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80u);
    float rf = (float)r;                    /* exact: r has <= 8 significant bits */
    uint32_t rb;
    memcpy(&rb, &rf, sizeof rb);
    return (uint16_t)(sign | (uint16_t)(rb >> 16));
}

/* ---------------------------------------------------------------- RoPE ---- */

/*
 * Qwen2-style rotary table for positions 0..T-1 and pair index i < D/2:
 * inv_freq_i = theta^(-2i/D), angle = p * inv_freq_i (fp64), entries rounded to
 * fp32.  Layout: cos_tab[p*(D/2) + i], sin_tab[p*(D/2) + i].
 */
void ora_rope_table(int T, int D, double theta, float* cos_tab, float* sin_tab) {
    int half = D / 2;
    for (int p = 0; p < T; ++p) {
        for (int i = 0; i < half; ++i) {
            double inv_freq = pow(theta, -(2.0 * (double)i) / (double)D);
            double angle = (double)p * inv_freq;
            cos_tab[(size_t)p * half + i] = (float)cos(angle);
            sin_tab[(size_t)p * half + i] = (float)sin(angle);
        }
    }
}

/*
 * Rotate one head row x[0..D) by the rotate-half rule with per-pair cos c[i]
 * and sin s[i] (i < D/2):
 *   out[i]       = x[i]       * c[i] - x[i + D/2] * s[i]
 *   out[i + D/2] = x[i + D/2] * c[i] + x[i]       * s[i]
 * All in double, no rounding beyond double's own.
 */
void ora_rope_rotate(const double* x, const double* c, const double* s, int D, double* out) {
    int half = D / 2;
    for (int i = 0; i < half; ++i) {
        double lo = x[i];
        double hi = x[i + half];
        out[i] = lo * c[i] - hi * s[i];
        out[i + half] = hi * c[i] + lo * s[i];
    }
}

/* rotate one bf16 head row at absolute position p, result rounded to bf16 */
static void rope_row_bf16(const uint16_t* in, uint16_t* out, int p, int D,
                          const float* cos_tab, const float* sin_tab) {
    int half = D / 2;
    double x[512], c[256], s[256], y[512];
    for (int d = 0; d < D; ++d) x[d] = ora_bf16_to_f64(in[d]);
    for (int i = 0; i < half; ++i) {
        c[i] = (double)cos_tab[(size_t)p * half + i];
        s[i] = (double)sin_tab[(size_t)p * half + i];
    }
    ora_rope_rotate(x, c, s, D, y);
    for (int d = 0; d < D; ++d) out[d] = ora_f64_to_bf16_rne(y[d]);
}

/*
 * RoPE + delta write, layouts (all contiguous, bf16 as uint16):
 *   q       [B, S, Hq,  D]   rotated in place
 *   k_new   [B, S, Hkv, D]   rotated, then written to cache_k
 *   v_new   [B, S, Hkv, D]   copied unchanged to cache_v
 *   cache_k [B, T, Hkv, D], cache_v [B, T, Hkv, D]
 * For request b and new row t < n_new[b] the absolute position is
 * p = pos0[b] + t (pos0 = cache_position).  Rows t >= n_new[b] and rows with
 * p >= T are left untouched.  Returns the number of skipped rows with p >= T.
 */
int ora_append_rope(uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                    uint16_t* cache_k, uint16_t* cache_v,
                    const int32_t* pos0, const int32_t* n_new,
                    int B, int S, int T, int Hq, int Hkv, int D,
                    const float* cos_tab, const float* sin_tab) {
    int skipped = 0;
    for (int b = 0; b < B; ++b) {
        for (int t = 0; t < S && t < n_new[b]; ++t) {
            int p = pos0[b] + t;
            if (p < 0 || p >= T) { ++skipped; continue; }
            for (int h = 0; h < Hq; ++h) {
                uint16_t* row = q + (((size_t)b * S + t) * Hq + h) * D;
                uint16_t tmp[512];
                rope_row_bf16(row, tmp, p, D, cos_tab, sin_tab);
                memcpy(row, tmp, sizeof(uint16_t) * (size_t)D);
            }
            for (int g = 0; g < Hkv; ++g) {
                const uint16_t* krow = k_new + (((size_t)b * S + t) * Hkv + g) * D;
                const uint16_t* vrow = v_new + (((size_t)b * S + t) * Hkv + g) * D;
                uint16_t* kdst = cache_k + (((size_t)b * T + p) * Hkv + g) * D;
                uint16_t* vdst = cache_v + (((size_t)b * T + p) * Hkv + g) * D;
                rope_row_bf16(krow, kdst, p, D, cos_tab, sin_tab);
                memcpy(vdst, vrow, sizeof(uint16_t) * (size_t)D);
            }
        }
    }
    return skipped;
}

/* ----------------------------------------------------------- attention ---- */

/*
 * Softmax attention of one query row over key/value rows j in [j0, j1):
 *   s_j   = scale * sum_d q[d] * k_j[d]
 *   m     = max_j s_j
 *   l     = sum_j exp(s_j - m)
 *   o[d]  = sum_j exp(s_j - m) * v_j[d] / l
 *   lse   = m + ln(l)
 * Two plain passes in double.  Row j of K sits at krows + j*row_stride (same
 * for V).  An empty range gives o = 0 and lse = -inf.
 */
void ora_attend_one(const uint16_t* qrow, const uint16_t* krows, const uint16_t* vrows,
                    long row_stride, int j0, int j1, int D, double scale,
                    double* o, double* lse) {
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    if (j1 <= j0) { *lse = -INFINITY; return; }
    double m = -INFINITY;
    for (int j = j0; j < j1; ++j) {
        double dot = 0.0;
        const uint16_t* k = krows + (size_t)j * row_stride;
        for (int d = 0; d < D; ++d) dot += ora_bf16_to_f64(qrow[d]) * ora_bf16_to_f64(k[d]);
        double s = scale * dot;
        if (s > m) m = s;
    }
    double l = 0.0;
    for (int j = j0; j < j1; ++j) {
        double dot = 0.0;
        const uint16_t* k = krows + (size_t)j * row_stride;
        const uint16_t* v = vrows + (size_t)j * row_stride;
        for (int d = 0; d < D; ++d) dot += ora_bf16_to_f64(qrow[d]) * ora_bf16_to_f64(k[d]);
        double w = exp(scale * dot - m);
        l += w;
        for (int d = 0; d < D; ++d) o[d] += w * ora_bf16_to_f64(v[d]);
    }
    for (int d = 0; d < D; ++d) o[d] /= l;
    *lse = m + log(l);
}

/*
 * The static-cache form: score every one of the T rows and give the rows at or
 * past n_valid a score of -inf, then take the softmax over all T.  A masked row
 * contributes exp(-inf) = 0 times its V row, which is 0 only when that V row is
 * finite; so this form needs finite values past the valid length.
 */
void ora_attend_one_static(const uint16_t* qrow, const uint16_t* krows, const uint16_t* vrows,
                           long row_stride, int T, int n_valid, int D, double scale,
                           double* o, double* lse) {
    double* sc = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    double m = -INFINITY;
    for (int j = 0; j < T; ++j) {
        double dot = 0.0;
        const uint16_t* k = krows + (size_t)j * row_stride;
        for (int d = 0; d < D; ++d) dot += ora_bf16_to_f64(qrow[d]) * ora_bf16_to_f64(k[d]);
        sc[j] = (j < n_valid) ? scale * dot : -INFINITY;
        if (sc[j] > m) m = sc[j];
    }
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    if (m == -INFINITY) { *lse = -INFINITY; free(sc); return; }
    double l = 0.0;
    for (int j = 0; j < T; ++j) {
        double w = exp(sc[j] - m);
        const uint16_t* v = vrows + (size_t)j * row_stride;
        l += w;
        for (int d = 0; d < D; ++d) o[d] += w * ora_bf16_to_f64(v[d]);
    }
    for (int d = 0; d < D; ++d) o[d] /= l;
    *lse = m + log(l);
    free(sc);
}

/*
 * Causal GQA attention over the cache, for decode and prefill alike.
 *   q       [B, S, Hq, D] (already rotated), cache_k/cache_v [B, T, Hkv, D]
 *   query row t < n_rows[b] of request b sees keys j < first_vis[b] + t
 *   (decode: first_vis = kv_len, n_rows = 1; prefill: first_vis = pos0 + 1,
 *   n_rows = n_new, so row t at position pos0+t sees j <= pos0+t).
 *   Query head h reads KV head g = h / (Hq/Hkv).
 *   o [B, S, Hq, D] (double), lse [B, Hq, S] (double).  Rows t >= n_rows[b]
 *   are not written.  Visible counts are clamped to [0, T].
 * static_mode != 0 uses ora_attend_one_static over all T rows.
 * The outer loop over (b, h) is spread over OpenMP threads when the library
 * is built with OpenMP; each (b, h, t) is computed by exactly one thread.
 */
void ora_attention(const uint16_t* q, const uint16_t* cache_k, const uint16_t* cache_v,
                   const int32_t* first_vis, const int32_t* n_rows,
                   int B, int S, int T, int Hq, int Hkv, int D, double scale, int static_mode,
                   double* o, double* lse) {
    int group = Hq / Hkv;
    long row_stride = (long)Hkv * D;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < Hq; ++h) {
            int g = h / group;
            const uint16_t* kb = cache_k + ((size_t)b * T * Hkv + g) * D;
            const uint16_t* vb = cache_v + ((size_t)b * T * Hkv + g) * D;
            for (int t = 0; t < S && t < n_rows[b]; ++t) {
                int vis = first_vis[b] + t;
                if (vis < 0) vis = 0;
                if (vis > T) vis = T;
                const uint16_t* qrow = q + (((size_t)b * S + t) * Hq + h) * D;
                double* orow = o + (((size_t)b * S + t) * Hq + h) * D;
                double* l = lse + ((size_t)b * Hq + h) * S + t;
                if (static_mode)
                    ora_attend_one_static(qrow, kb, vb, row_stride, T, vis, D, scale, orow, l);
                else
                    ora_attend_one(qrow, kb, vb, row_stride, 0, vis, D, scale, orow, l);
            }
        }
    }
}

/*
 * Merge of n partial results of the same query over disjoint key ranges, each
 * given as its normalised output o_c[D] and its log-sum-exp lse_c:
 *   M = max_c lse_c,  w_c = exp(lse_c - M),
 *   o = sum_c w_c o_c / sum_c w_c,  lse = M + ln(sum_c w_c).
 * A part with lse_c = -inf (no keys) has weight 0 and its o_c is not read.
 * All parts empty: o = 0, lse = -inf.
 */
void ora_combine(const double* o_part, const double* lse_part, int n, int D,
                 double* o, double* lse) {
    double M = -INFINITY;
    for (int c = 0; c < n; ++c) if (lse_part[c] > M) M = lse_part[c];
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    if (M == -INFINITY) { *lse = -INFINITY; return; }
    double wsum = 0.0;
    for (int c = 0; c < n; ++c) {
        if (lse_part[c] == -INFINITY) continue;
        double w = exp(lse_part[c] - M);
        wsum += w;
        for (int d = 0; d < D; ++d) o[d] += w * o_part[(size_t)c * D + d];
    }
    for (int d = 0; d < D; ++d) o[d] /= wsum;
    *lse = M + log(wsum);
}

/* ------------------------------------------------------- fp8 KV cache ---- */
/*
 * An fp8 variant of the cache format.  The pages quantise weights only (the
 * int8/int4 tiers of the "ARK-ASR-3B -- INT8 ONNX" model card); keeping the
 * cache itself in 8 bits is not on them.  Reading taken for it:
 *   - element format: OCP FP8 E4M3 ("fn"): 1 sign bit, 4 exponent bits (bias
 *     7), 3 mantissa bits, no infinities, S.1111.111 is NaN, largest finite
 *     value 448, subnormals down to 2^-9;
 *   - one fp32 scale per (layer, KV head) for K and one for V, given by the
 *     caller; the stored code of a value x is e4m3(fp32(x / scale)): the
 *     quotient formed in fp64, rounded to fp32 (nearest even), then to e4m3
 *     (nearest even, finite values beyond +-448 and infinities saturate to
 *     +-448, NaN stays NaN);
 *   - x is the rotated key (formed in fp64 as for the bf16 cache, not rounded
 *     to bf16 first) or the bf16 value row;
 *   - attention reads code * scale.
 */

/* e4m3 code -> its exact value (as double); NaN for S.1111.111. */
double ora_e4m3_to_f64(uint8_t code) {
    int sign = code >> 7;
    int e = (code >> 3) & 15;
    int m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);                 /* subnormal: m/8 * 2^-6 */
    else
        v = ldexp(8.0 + m, e - 10);               /* (1 + m/8) * 2^(e-7) */
    return sign ? -v : v;
}

/*
 * fp32 value -> e4m3 code, nearest-even, saturating: the plain definition,
 * a search over the 127 non-negative finite codes for the nearest value, a
 * tie going to the code with an even mantissa (its low bit clear).
 */
uint8_t ora_f32_to_e4m3(float f) {
    double x = (double)f;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    if (isnan(x)) return (uint8_t)(sign | 0x7F);
    double a = fabs(x);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);   /* saturate, infinities included */
    int best = 0;
    double best_err = a;                               /* code 0 is +0 */
    for (int c = 1; c <= 0x7E; ++c) {
        double err = fabs(ora_e4m3_to_f64((uint8_t)c) - a);
        if (err < best_err || (err == best_err && (c & 1) == 0)) {
            best = c;
            best_err = err;
        }
    }
    return (uint8_t)(sign | best);
}

/* x (fp64) quantised with `scale`: e4m3(fp32(x / scale)) */
uint8_t ora_quantize_e4m3(double x, float scale) {
    float y = (float)(x / (double)scale);
    return ora_f32_to_e4m3(y);
}

/*
 * RoPE + delta write into an fp8 cache (same rows, positions and skipping as
 * ora_append_rope): q is rotated in place to bf16 as before; the rotated key
 * (fp64) and the value row are quantised with the scales of their KV head,
 * k_scale[g] and v_scale[g] (this layer's).
 */
int ora_append_rope_fp8(uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                        uint8_t* cache_k, uint8_t* cache_v, const float* k_scale, const float* v_scale,
                        const int32_t* pos0, const int32_t* n_new,
                        int B, int S, int T, int Hq, int Hkv, int D,
                        const float* cos_tab, const float* sin_tab) {
    int skipped = 0;
    int half = D / 2;
    for (int b = 0; b < B; ++b) {
        for (int t = 0; t < S && t < n_new[b]; ++t) {
            int p = pos0[b] + t;
            if (p < 0 || p >= T) { ++skipped; continue; }
            for (int h = 0; h < Hq; ++h) {
                uint16_t* row = q + (((size_t)b * S + t) * Hq + h) * D;
                uint16_t tmp[512];
                rope_row_bf16(row, tmp, p, D, cos_tab, sin_tab);
                memcpy(row, tmp, sizeof(uint16_t) * (size_t)D);
            }
            for (int g = 0; g < Hkv; ++g) {
                const uint16_t* krow = k_new + (((size_t)b * S + t) * Hkv + g) * D;
                const uint16_t* vrow = v_new + (((size_t)b * S + t) * Hkv + g) * D;
                uint8_t* kdst = cache_k + (((size_t)b * T + p) * Hkv + g) * D;
                uint8_t* vdst = cache_v + (((size_t)b * T + p) * Hkv + g) * D;
                double x[512], c[256], s[256], y[512];
                for (int d = 0; d < D; ++d) x[d] = ora_bf16_to_f64(krow[d]);
                for (int i = 0; i < half; ++i) {
                    c[i] = (double)cos_tab[(size_t)p * half + i];
                    s[i] = (double)sin_tab[(size_t)p * half + i];
                }
                ora_rope_rotate(x, c, s, D, y);
                for (int d = 0; d < D; ++d) kdst[d] = ora_quantize_e4m3(y[d], k_scale[g]);
                for (int d = 0; d < D; ++d) vdst[d] = ora_quantize_e4m3(ora_bf16_to_f64(vrow[d]), v_scale[g]);
            }
        }
    }
    return skipped;
}

/*
 * Attention over an fp8 cache: the definition of ora_attention with key row j
 * read as code * k_scale[g] and value row j as code * v_scale[g] (exact in
 * double).  Each (b, h) dequantises its KV head's rows into double arrays and
 * takes the same two-pass softmax (or the masked static form).
 */
static void attend_rows_f64(const double* q, const double* k, const double* v, int n_rows_total,
                            int n_valid, int static_form, int D, double scale, double* o, double* lse) {
    int n = static_form ? n_rows_total : n_valid;
    double m = -INFINITY;
    double* sc = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    for (int j = 0; j < n; ++j) {
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += q[d] * k[(size_t)j * D + d];
        sc[j] = (j < n_valid) ? scale * dot : -INFINITY;
        if (sc[j] > m) m = sc[j];
    }
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    if (m == -INFINITY) { *lse = -INFINITY; free(sc); return; }
    double l = 0.0;
    for (int j = 0; j < n; ++j) {
        double w = exp(sc[j] - m);
        l += w;
        for (int d = 0; d < D; ++d) o[d] += w * v[(size_t)j * D + d];
    }
    for (int d = 0; d < D; ++d) o[d] /= l;
    *lse = m + log(l);
    free(sc);
}

void ora_attention_fp8(const uint16_t* q, const uint8_t* cache_k, const uint8_t* cache_v,
                       const float* k_scale, const float* v_scale,
                       const int32_t* first_vis, const int32_t* n_rows,
                       int B, int S, int T, int Hq, int Hkv, int D, double scale, int static_mode,
                       double* o, double* lse) {
    int group = Hq / Hkv;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < Hq; ++h) {
            int g = h / group;
            double* kd = (double*)malloc(sizeof(double) * (size_t)T * D);
            double* vd = (double*)malloc(sizeof(double) * (size_t)T * D);
            for (int j = 0; j < T; ++j)
                for (int d = 0; d < D; ++d) {
                    size_t idx = (((size_t)b * T + j) * Hkv + g) * D + d;
                    kd[(size_t)j * D + d] = ora_e4m3_to_f64(cache_k[idx]) * (double)k_scale[g];
                    vd[(size_t)j * D + d] = ora_e4m3_to_f64(cache_v[idx]) * (double)v_scale[g];
                }
            for (int t = 0; t < S && t < n_rows[b]; ++t) {
                int vis = first_vis[b] + t;
                if (vis < 0) vis = 0;
                if (vis > T) vis = T;
                double qd[512];
                const uint16_t* qrow = q + (((size_t)b * S + t) * Hq + h) * D;
                for (int d = 0; d < D; ++d) qd[d] = ora_bf16_to_f64(qrow[d]);
                attend_rows_f64(qd, kd, vd, T, vis, static_mode, D, scale,
                                o + (((size_t)b * S + t) * Hq + h) * D, lse + ((size_t)b * Hq + h) * S + t);
            }
            free(kd);
            free(vd);
        }
    }
}

/* ------------------------------------------------- encoder attention ---- */
/*
 * Bidirectional multi-head self-attention of the audio encoder (the pages
 * give a Whisper-style encoder with rotary self-attention and a 1280-wide
 * output; reading: every frame of a clip attends to every frame of the same
 * clip, q and k already rotated).  Layouts: q, k, v [B, S, H, D] (bf16 bits),
 * len[B] valid frames per clip; o [B, S, H, D] double, lse [B, H, S] double;
 * rows i >= len[b] are not written.  Each (b, h, i) is ora_attend_one over the
 * clip's rows [0, len[b]) of head h.
 */
void ora_attention_bidir(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* len,
                         int B, int S, int H, int D, double scale, double* o, double* lse) {
    long row_stride = (long)H * D;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            int n = len[b];
            if (n < 0) n = 0;
            if (n > S) n = S;
            const uint16_t* kb = k + ((size_t)b * S * H + h) * D;
            const uint16_t* vb = v + ((size_t)b * S * H + h) * D;
            for (int i = 0; i < n; ++i) {
                const uint16_t* qrow = q + (((size_t)b * S + i) * H + h) * D;
                ora_attend_one(qrow, kb, vb, row_stride, 0, n, D, scale,
                               o + (((size_t)b * S + i) * H + h) * D, lse + ((size_t)b * H + h) * S + i);
            }
        }
    }
}

/* ------------------------------------------- Q/K/V projection (Linear) ---- */
/*
 * The Q/K/V projections of a Qwen2 decoder layer, the step in front of the
 * attention: three dense layers hidden -> Hq*D, Hkv*D, Hkv*D
 * ("ARK-ASR-3B -- INT8 ONNX", model card: Q/K/V projections of the Qwen2
 * decoder, hidden 2048).  Written as one Linear over the concatenated weight
 * W = [Wq; Wk; Wv] of shape [N, K] (N = (Hq + 2 Hkv) * D, K = hidden):
 *   out[m, n] = bf16_rne( sum_k x[m, k] * W[n, k] + bias[n] )
 * Reading for precision (the pages give bf16 serving, nothing finer): the
 * products of two bf16 values are exact in double; the sum is taken in double
 * in k order, the bias (bf16, may be absent) added in double, and the result
 * rounded once to bf16 -- the bf16 value of the exact Linear output up to the
 * double rounding of the sum.
 * Layouts: x [M, K], W [N, K], bias [N] or NULL (bf16 bits); out [M, N].
 */
void ora_qkv_proj(const uint16_t* x, const uint16_t* w, const uint16_t* bias, int M, int K, int N,
                  uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int m = 0; m < M; ++m) {
        for (int n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int k = 0; k < K; ++k)
                acc += ora_bf16_to_f64(x[(size_t)m * K + k]) * ora_bf16_to_f64(w[(size_t)n * K + k]);
            if (bias) acc += ora_bf16_to_f64(bias[n]);
            out[(size_t)m * N + n] = ora_f64_to_bf16_rne(acc);
        }
    }
}
