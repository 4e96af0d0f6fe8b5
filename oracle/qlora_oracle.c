/*
 * qlora_oracle.c -- plain, slow CPU oracle for the int8-frozen-kernel LoRA
 * Dense layer (forward, backward, lossy merge).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link,
 * load or call this file.  It is used by the test suite, by the package's
 * smoke check and by the benchmark's timed CPU baseline, and nothing else.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * Every routine is a direct restatement of what the pages define, written
 * as scalar loops with no blocking, fusion or reordering:
 *   - frozen int8 kernel: "Introduce QLoRA-like technique" (Keras PR 19356),
 *     Highlights ("training with frozen int8 weights for Dense") and the
 *     "How to fine-tune the 4-bit model?" thread (most weights are integers,
 *     non-differentiable, not changed during gradient descent);
 *   - LoRA branch: "Parameter-efficient fine-tuning of GPT-2 with LoRA",
 *     section "LoRA equation" (output = W0 x + b0 + B A x) and section
 *     "Create LoRA layer" (scale = alpha / rank, applied to B(A(x)));
 *   - lossy merge: Keras PR 19356, Results table footnote (merging into int8
 *     kernels is lossy) and the "How to fine-tune the 4-bit model?" thread
 *     (de-quantize, add the LoRA, re-quantize); the float merge adds
 *     einsum(A, B) * alpha / rank to the kernel ("Merge weights and generate
 *     text!" section of the GPT-2 LoRA notebook).
 *
 * Readings where the pages are silent (stated once here, used throughout):
 *   - quantization is symmetric abs-max: s = amax / 127, q = clamp(
 *     round_half_even(v * (127 / amax)), -127, 127), per output channel for
 *     the kernel and per row for the layer input; all of it in IEEE fp32,
 *     one rounding per operation (no fused multiply-add);
 *   - amax == 0 gives inv = 0, hence q = 0 and s = 0;
 *   - the LoRA branch sees the unquantized input x;
 *   - the backward treats the input quantizer as the identity
 *     (straight-through): dX uses the dequantized kernel Wq * s_w, formed
 *     in fp32 and, for bf16 activations, stored as bf16 like every other
 *     operand of that layer's products (the de-quantized tile is a bf16
 *     operand of the input-gradient product);
 *   - floating-point sums are taken in fp64, integer sums in int64.
 *
 * Layouts (row-major, contiguous):
 *   W  [K,N]  float kernel as the pages store it (in_features x out_features)
 *   Wq [N,K]  int8 frozen kernel, one row per output channel
 *   sw [N]    per-output-channel kernel scale
 *   X  [M,K], Xq [M,K], sx [M], acc [M,N], Y [M,N], dY [M,N], dX [M,K]
 *   A  [K,r], B [r,N], xA [M,r], G [M,r], dA [K,r], dB [r,N], dbias [N]
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fPIC -shared.  OpenMP only
 * splits independent output rows across threads; the order of every sum is
 * fixed by the loops below, so results do not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* Threads                                                                    */
/* ------------------------------------------------------------------------ */

void orc_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int orc_get_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* Symmetric abs-max int8 quantization of one vector (fp32 semantics).        */
/* v[i * stride] for i in [0, n).  Writes q[i] and returns the scale.         */
/* ------------------------------------------------------------------------ */
static float quantize_vector(const float* v, long n, long stride, int8_t* q) {
    float amax = 0.0f;
    for (long i = 0; i < n; ++i) {
        float a = fabsf(v[i * stride]);
        if (a > amax) amax = a;
    }
    float inv = (amax > 0.0f) ? 127.0f / amax : 0.0f;
    for (long i = 0; i < n; ++i) {
        float t = v[i * stride] * inv;      /* one fp32 rounding */
        float r = rintf(t);                 /* round half to even */
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        q[i] = (int8_t)r;
    }
    return amax / 127.0f;
}

/*
 * a0 -- frozen-kernel quantization, per output channel n (column of W).
 * W [K,N] fp32 -> Wq [N,K] int8 (one row per output channel), sw [N].
 */
void orc_quantize_weight(const float* W, long K, long N, int8_t* Wq, float* sw) {
    #pragma omp parallel for schedule(static)
    for (long n = 0; n < N; ++n) {
        sw[n] = quantize_vector(W + n, K, N, Wq + n * K);
    }
}

/*
 * a1 (first half) -- per-row quantization of the layer input.
 * X [M,K] fp32 (bf16 inputs are widened exactly first) -> Xq [M,K], sx [M].
 */
void orc_quantize_rows(const float* X, long M, long K, int8_t* Xq, float* sx) {
    #pragma omp parallel for schedule(static)
    for (long m = 0; m < M; ++m) {
        sx[m] = quantize_vector(X + m * K, K, 1, Xq + m * K);
    }
}

/*
 * a2 (integer part) -- acc[m,n] = sum_k Xq[m,k] * Wq[n,k], summed in int64.
 * Returns the number of entries that do not fit in int32 (0 when all fit);
 * such entries are written saturated.
 */
long orc_int8_matmul(const int8_t* Xq, const int8_t* Wq, long M, long N, long K,
                     int32_t* acc) {
    long overflow = 0;
    #pragma omp parallel for schedule(static) reduction(+ : overflow)
    for (long m = 0; m < M; ++m) {
        for (long n = 0; n < N; ++n) {
            int64_t s = 0;
            for (long k = 0; k < K; ++k)
                s += (int64_t)Xq[m * K + k] * (int64_t)Wq[n * K + k];
            if (s > INT32_MAX) { s = INT32_MAX; ++overflow; }
            if (s < INT32_MIN) { s = INT32_MIN; ++overflow; }
            acc[m * N + n] = (int32_t)s;
        }
    }
    return overflow;
}

/*
 * a1 (second half) -- the LoRA down-projection of the unquantized input:
 * xA[m,j] = sum_k X[m,k] * A[k,j] (fp64).
 */
void orc_lora_down(const double* X, const double* A, long M, long K, long r,
                   double* xA) {
    #pragma omp parallel for schedule(static)
    for (long m = 0; m < M; ++m) {
        for (long j = 0; j < r; ++j) {
            double s = 0.0;
            for (long k = 0; k < K; ++k) s += X[m * K + k] * A[k * r + j];
            xA[m * r + j] = s;
        }
    }
}

/*
 * a2 (floating part) -- the layer output (fp64):
 * Y[m,n] = acc[m,n] * sx[m] * sw[n] + bias[n] + c * sum_j xA[m,j] * B[j,n]
 * where c = alpha / rank.  bias may be NULL (no bias).
 */
void orc_forward(long M, long N, long r, double c, const int32_t* acc,
                 const float* sx, const float* sw, const double* bias,
                 const double* xA, const double* B, double* Y) {
    #pragma omp parallel for schedule(static)
    for (long m = 0; m < M; ++m) {
        for (long n = 0; n < N; ++n) {
            double base = (double)acc[m * N + n] * (double)sx[m] * (double)sw[n];
            double lora = 0.0;
            for (long j = 0; j < r; ++j) lora += xA[m * r + j] * B[j * N + n];
            double b = bias ? bias[n] : 0.0;
            Y[m * N + n] = base + b + c * lora;
        }
    }
}

/*
 * a3..a5 -- the backward pass (fp64), gradients of L = sum(Y * dY):
 *   G[m,j]  = sum_n dY[m,n] * B[j,n]
 *   dX[m,k] = sum_n dY[m,n] * Wd[n,k] + c * sum_j G[m,j] * A[k,j]
 * where Wd is the de-quantized kernel as the activation dtype stores it:
 * Wd = fl32(Wq * sw) (one fp32 rounding), further rounded to bfloat16 when
 * wdq_bf16 is set (bf16 activations: the de-quantized kernel tile is a bf16
 * operand of the input-gradient product).
 *   dA[k,j] = c * sum_m X[m,k] * G[m,j]
 *   dB[j,n] = c * sum_m xA[m,j] * dY[m,n]     (xA recomputed from X)
 *   dbias[n] = sum_m dY[m,n]
 * Any output pointer may be NULL to skip it.
 */
double orc_round_bf16(double x);

void orc_backward(long M, long K, long N, long r, double c, const double* X,
                  const double* dY, const int8_t* Wq, const float* sw,
                  const double* A, const double* B, int wdq_bf16, double* G,
                  double* dX, double* dA, double* dB, double* dbias) {
    double* g = (double*)malloc(sizeof(double) * (size_t)(M * r));
    double* xa = (double*)malloc(sizeof(double) * (size_t)(M * r));
    orc_lora_down(X, A, M, K, r, xa);

    #pragma omp parallel for schedule(static)
    for (long m = 0; m < M; ++m) {
        for (long j = 0; j < r; ++j) {
            double s = 0.0;
            for (long n = 0; n < N; ++n) s += dY[m * N + n] * B[j * N + n];
            g[m * r + j] = s;
        }
    }
    if (G) memcpy(G, g, sizeof(double) * (size_t)(M * r));

    if (dX) {
        /* the de-quantized kernel, one row per output channel n */
        double* wd = (double*)malloc(sizeof(double) * (size_t)(N * K));
        #pragma omp parallel for schedule(static)
        for (long n = 0; n < N; ++n) {
            for (long k = 0; k < K; ++k) {
                float w = (float)Wq[n * K + k] * sw[n];   /* one fp32 rounding */
                wd[n * K + k] = wdq_bf16 ? orc_round_bf16((double)w) : (double)w;
            }
        }
        #pragma omp parallel for schedule(static)
        for (long m = 0; m < M; ++m) {
            double* row = dX + m * K;
            for (long k = 0; k < K; ++k) row[k] = 0.0;
            for (long n = 0; n < N; ++n) {
                double d = dY[m * N + n];
                const double* w = wd + n * K;
                for (long k = 0; k < K; ++k) row[k] += d * w[k];
            }
            for (long k = 0; k < K; ++k) {
                double l = 0.0;
                for (long j = 0; j < r; ++j) l += g[m * r + j] * A[k * r + j];
                row[k] += c * l;
            }
        }
        free(wd);
    }

    if (dA) {
        #pragma omp parallel for schedule(static)
        for (long k = 0; k < K; ++k) {
            for (long j = 0; j < r; ++j) {
                double s = 0.0;
                for (long m = 0; m < M; ++m) s += X[m * K + k] * g[m * r + j];
                dA[k * r + j] = c * s;
            }
        }
    }

    if (dB) {
        #pragma omp parallel for schedule(static)
        for (long j = 0; j < r; ++j) {
            for (long n = 0; n < N; ++n) {
                double s = 0.0;
                for (long m = 0; m < M; ++m) s += xa[m * r + j] * dY[m * N + n];
                dB[j * N + n] = c * s;
            }
        }
    }

    if (dbias) {
        for (long n = 0; n < N; ++n) {
            double s = 0.0;
            for (long m = 0; m < M; ++m) s += dY[m * N + n];
            dbias[n] = s;
        }
    }
    free(g);
    free(xa);
}

/*
 * a6 -- lossy merge, in fp32 with a fixed operation order:
 *   w  = (float)Wq[n,k] * sw[n]
 *   d  = sum_{j = 0..r-1} A[k,j] * B[j,n]  (each product and sum rounded,
 *        ascending j, starting from the first product)
 *   w' = w + c * d                          (multiply, then add)
 * then the per-output-channel quantization of a0 applied to W'.
 * Wq_out/sw_out must not alias Wq/sw.
 */
static float merged_entry(const int8_t* Wq, const float* sw, const float* A,
                          const float* B, long K, long N, long r, float c,
                          long k, long n) {
    float w = (float)Wq[n * K + k] * sw[n];
    float d = 0.0f;
    for (long j = 0; j < r; ++j) {
        float p = A[k * r + j] * B[j * N + n];
        d = (j == 0) ? p : d + p;
    }
    float cd = c * d;
    return w + cd;
}

void orc_merge(const int8_t* Wq, const float* sw, const float* A, const float* B,
               long K, long N, long r, float c, int8_t* Wq_out, float* sw_out) {
    #pragma omp parallel for schedule(static)
    for (long n = 0; n < N; ++n) {
        float* col = (float*)malloc(sizeof(float) * (size_t)K);
        for (long k = 0; k < K; ++k)
            col[k] = merged_entry(Wq, sw, A, B, K, N, r, c, k, n);
        sw_out[n] = quantize_vector(col, K, 1, Wq_out + n * K);
        free(col);
    }
}

/* ------------------------------------------------------------------------ */
/* Packed int4 kernels ("Simplified Int4Variable quantization" in the         */
/* keras-llm-light description: two int4 values stored in one int8 byte;     */
/* "How to fine-tune the 4-bit model?": a 4-bit integer kernel, frozen, with  */
/* an fp32 LoRA, de-quantized in place; merge = de-quantize, add the LoRA,    */
/* re-quantize).  Readings where the pages are silent:                        */
/*   - the int4 quantizer is the int8 one with 7 in place of 127: per output  */
/*     channel, s = amax / 7, q = clamp(round_half_even(v * (7 / amax)),      */
/*     -7, 7), fp32, one rounding per operation (15 levels, symmetric);       */
/*   - packing runs along K: byte j of channel n holds code 2j in its low     */
/*     nibble and code 2j+1 in its high nibble, each as a two's-complement    */
/*     nibble; K is even;                                                     */
/*   - an int4 layer computes exactly what the int8 layer computes with the   */
/*     unpacked codes in place of the int8 codes (forward, backward), and its */
/*     merge re-quantizes the merged kernel to int4.                          */
/* ------------------------------------------------------------------------ */
static float quantize_vector_int4(const float* v, long n, long stride, int8_t* q) {
    float amax = 0.0f;
    for (long i = 0; i < n; ++i) {
        float a = fabsf(v[i * stride]);
        if (a > amax) amax = a;
    }
    float inv = (amax > 0.0f) ? 7.0f / amax : 0.0f;
    for (long i = 0; i < n; ++i) {
        float t = v[i * stride] * inv;      /* one fp32 rounding */
        float r = rintf(t);                 /* round half to even */
        if (r > 7.0f) r = 7.0f;
        if (r < -7.0f) r = -7.0f;
        q[i] = (int8_t)r;
    }
    return amax / 7.0f;
}

static void pack_int4_row(const int8_t* q, long K, uint8_t* out) {
    for (long j = 0; j < K / 2; ++j) {
        unsigned lo = (unsigned)q[2 * j] & 0xFu;
        unsigned hi = (unsigned)q[2 * j + 1] & 0xFu;
        out[j] = (uint8_t)(lo | (hi << 4));
    }
}

/* W [K,N] fp32 -> Wp [N, K/2] packed codes, sw [N]. */
void orc_quantize_weight_int4(const float* W, long K, long N, uint8_t* Wp, float* sw) {
    #pragma omp parallel for schedule(static)
    for (long n = 0; n < N; ++n) {
        int8_t* q = (int8_t*)malloc((size_t)K);
        sw[n] = quantize_vector_int4(W + n, K, N, q);
        pack_int4_row(q, K, Wp + n * (K / 2));
        free(q);
    }
}

/* Wp [N, K/2] -> Wq [N,K] int8 codes in [-8, 7]. */
void orc_unpack_int4(const uint8_t* Wp, long N, long K, int8_t* Wq) {
    for (long n = 0; n < N; ++n) {
        for (long j = 0; j < K / 2; ++j) {
            int lo = Wp[n * (K / 2) + j] & 0xF;
            int hi = (Wp[n * (K / 2) + j] >> 4) & 0xF;
            Wq[n * K + 2 * j] = (int8_t)(lo >= 8 ? lo - 16 : lo);
            Wq[n * K + 2 * j + 1] = (int8_t)(hi >= 8 ? hi - 16 : hi);
        }
    }
}

/* Lossy merge of an int4 layer (given its unpacked codes): the merged entries
 * of the int8 merge, re-quantized per channel to int4 and packed. */
void orc_merge_int4(const int8_t* Wq, const float* sw, const float* A, const float* B,
                    long K, long N, long r, float c, uint8_t* Wp_out, float* sw_out) {
    #pragma omp parallel for schedule(static)
    for (long n = 0; n < N; ++n) {
        float* col = (float*)malloc(sizeof(float) * (size_t)K);
        int8_t* q = (int8_t*)malloc((size_t)K);
        for (long k = 0; k < K; ++k)
            col[k] = merged_entry(Wq, sw, A, B, K, N, r, c, k, n);
        sw_out[n] = quantize_vector_int4(col, K, 1, q);
        pack_int4_row(q, K, Wp_out + n * (K / 2));
        free(q);
        free(col);
    }
}

/* ------------------------------------------------------------------------ */
/* Outlier-compensated int8 kernels (keras-llm-light, "Weights               */
/* quantization" and "Simplified Int8Variable quantization": a simplified    */
/* LLM.int8(); the weights are quantized after removing outliers with a 99.9 */
/* percentile cutoff, the outliers are kept in a sparse (row, col, value)    */
/* list in fp16, and the kernel is rebuilt as bias + value * scale with the  */
/* outliers written back; the block summary stores such kernels as uint8).   */
/* Readings where the pages are silent:                                      */
/*   - one affine code per tensor: lo and hi are the 0.1th and 99.9th        */
/*     percentiles of all entries (linear interpolation between order        */
/*     statistics, in fp64, then stored as fp32);                            */
/*   - outliers are the entries strictly below lo or strictly above hi;     */
/*     they are stored as fp16 (round to nearest even);                      */
/*   - scale = fl32((hi - lo) / 255), bias = lo, and every other entry gets  */
/*     value = clamp(rne(fl32(fl32(w - bias) / scale)), 0, 255) (0 when      */
/*     scale == 0);                                                          */
/*   - rebuilt entry = fl32(bias + fl32(value * scale)), or the outlier's    */
/*     fp16 value widened to fp32.                                           */
/* ------------------------------------------------------------------------ */
static int cmp_float(const void* a, const void* b) {
    float x = *(const float*)a, y = *(const float*)b;
    return (x > y) - (x < y);
}

/* Percentile p (in [0, 100]) of n floats, linear interpolation between the
 * order statistics at position (n - 1) * p / 100. */
double orc_percentile(const float* v, long n, double p) {
    float* s = (float*)malloc(sizeof(float) * (size_t)n);
    memcpy(s, v, sizeof(float) * (size_t)n);
    qsort(s, (size_t)n, sizeof(float), cmp_float);
    double h = (double)(n - 1) * p / 100.0;
    long i = (long)floor(h);
    if (i >= n - 1) i = n - 1;
    double frac = h - (double)i;
    double q = (double)s[i];
    if (i + 1 < n && frac > 0.0) q += frac * ((double)s[i + 1] - (double)s[i]);
    free(s);
    return q;
}

/*
 * Round an fp64 value to the nearest IEEE half (11-bit significand, normal
 * range from 2^-14, subnormal quantum 2^-24), ties to even, as fp64.
 */
double orc_round_fp16(double x) {
    if (x == 0.0 || !isfinite(x)) return x;
    int e;
    frexp(x, &e);                 /* |x| in [2^(e-1), 2^e) */
    if (e - 1 < -14) e = -13;     /* subnormal range: fixed quantum 2^-24 */
    double ulp = ldexp(1.0, e - 11);
    double q = rint(x / ulp) * ulp;
    if (fabs(q) > 65504.0) q = copysign(INFINITY, x);
    return q;
}

/*
 * W [n] fp32 -> codes [n] uint8, outlier flags [n] (0, or 1 for an outlier),
 * outlier values [n] (fp16 values as fp32, 0 elsewhere), and
 * par = {lo, hi, scale, bias}.  Returns the number of outliers.
 */
long orc_quantize_outlier_int8(const float* W, long n, uint8_t* codes, uint8_t* is_out,
                               float* out_val, float* par) {
    float lo = (float)orc_percentile(W, n, 0.1);
    float hi = (float)orc_percentile(W, n, 99.9);
    float scale = (hi - lo) / 255.0f;
    float bias = lo;
    long count = 0;
    for (long i = 0; i < n; ++i) {
        float w = W[i];
        if (w < lo || w > hi) {
            is_out[i] = 1;
            out_val[i] = (float)orc_round_fp16((double)w);
            codes[i] = 0;
            ++count;
            continue;
        }
        is_out[i] = 0;
        out_val[i] = 0.0f;
        float r = 0.0f;
        if (scale > 0.0f) {
            float d = w - bias;           /* one fp32 rounding */
            float t = d / scale;          /* one fp32 rounding */
            r = rintf(t);
            if (r < 0.0f) r = 0.0f;
            if (r > 255.0f) r = 255.0f;
        }
        codes[i] = (uint8_t)r;
    }
    par[0] = lo;
    par[1] = hi;
    par[2] = scale;
    par[3] = bias;
    return count;
}

/* Rebuilds the kernel: bias + value * scale, outliers written back. */
void orc_dequantize_outlier_int8(const uint8_t* codes, const uint8_t* is_out, const float* out_val,
                                 long n, float scale, float bias, float* W) {
    for (long i = 0; i < n; ++i) {
        float v = (float)codes[i] * scale;   /* one fp32 rounding */
        W[i] = is_out[i] ? out_val[i] : bias + v;
    }
}

/*
 * Round an fp64 value to the nearest bfloat16 (8-bit significand, the fp32
 * exponent range), ties to even, returned as fp64.  Used where a layer's
 * output is stored in bf16 before it feeds the next layer.
 */
double orc_round_bf16(double x) {
    if (x == 0.0 || !isfinite(x)) return x;
    int e;
    frexp(x, &e);                 /* |x| in [2^(e-1), 2^e) */
    if (e - 1 < -126) e = -125;   /* subnormal range: fixed quantum 2^-133 */
    double ulp = ldexp(1.0, e - 8);
    double q = rint(x / ulp) * ulp;   /* x / ulp is exact (power of two) */
    if (fabs(q) > 3.3895313892515355e38) q = copysign(INFINITY, x);
    return q;
}

void orc_round_bf16_array(const double* x, long n, double* y) {
    for (long i = 0; i < n; ++i) y[i] = orc_round_bf16(x[i]);
}
