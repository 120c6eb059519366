/*
 * oracle.c -- slow, plain fp64 CPU restatement of the fused row-normalisation ops.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or call
 * this file.  Only the tests, the smoke check and the benchmark's CPU-baseline leg
 * use it.  It shares no code, header, table or constant with the CUDA library
 * (rope_add_rms_b200/csrc); the only thing both sides share is the seeded input
 * generator, which holds none of the arithmetic below.
 *
 * Sources (docs.rs nuvec-core 0.5.0, "Enum FastOp", Variants section; docs.rs
 * nuvec-nn 0.4.0 src/layers.rs, RmsNorm / LayerNorm / Rope; miniVLLM docs "Layers",
 * LayerNorm section):
 *   RmsNorm     (x, w): x / sqrt(mean(x^2) + eps) * w over the last axis,
 *               w is 1-D or the scalar 1.
 *   AddRmsNorm  (x, r, w): h = x + r, then RmsNorm of h; the updated residual h is
 *               returned next to the normalised row (miniVLLM LayerNorm.forward,
 *               steps 1-3: x_new = x + residual, normalise x_new, return both).
 *   LayerNorm   (x, w, b): (x - mean) / sqrt(var + eps) * w + b over the last axis;
 *               w and b are length-D vectors, or absent (1 and 0).
 *   Rope        rotary embedding of the first dims features (dims even), as the two
 *               halves or as interleaved pairs ("traditional"); base and a position
 *               scale; forward = false is the inverse rotation.
 *   NormRope    each [b, h, l] row RMS-normalised (when eps is given) and then
 *               rotated as Rope at position offset + l.
 *
 * Readings taken where the pages leave a step open (each one is listed with its
 * reason in the design notes):
 *   - eps, base and scale are fp32 values (FastOp stores them as f32::to_bits);
 *     they enter here widened exactly to fp64.
 *   - AddRmsNorm normalises the h that is returned, i.e. h after rounding to the
 *     I/O type; h itself is the fp32 sum x + r rounded once to the I/O type.
 *   - var is the population variance (divide by D).
 *   - Rope frequencies: theta_i = base^(-2 i / dims), angle (offset + l) * scale *
 *     theta_i, rotation [[cos, -sin], [sin, cos]] on the pair (p, q); halves pair
 *     (i, i + dims/2), traditional pairs (2i, 2i + 1); features j >= dims pass
 *     through unrotated.
 *   - In NormRope the row is normalised (times w) over all D features first and
 *     then rotated; normalize = 0 is plain Rope (no w).
 *
 * Arithmetic: every input element is widened exactly to double; sums are plain
 * left-to-right loops in double; sqrt, pow, sin and cos are the host libm's double
 * routines.  Build with -O2 -ffp-contract=off and without fast-math.
 * All row functions work on a row range [r0, r1) so that a caller can spread
 * rows over threads; they allocate a scratch row with malloc and return 0, or -1
 * when that allocation fails.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* element types of the oracle's own: 0 = IEEE binary32, 1 = bfloat16 (raw bits) */
#define ORACLE_F32 0
#define ORACLE_BF16 1

/* ---- widening and rounding -------------------------------------------------- */

static float f32_from_bits(uint32_t u) {
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static uint32_t bits_from_f32(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return u;
}

/* A bfloat16 is the upper half of a binary32: widening is exact. */
static double widen(const void* base, int dt, int64_t i) {
    if (dt == ORACLE_F32) return (double)((const float*)base)[i];
    uint16_t b = ((const uint16_t*)base)[i];
    return (double)f32_from_bits((uint32_t)b << 16);
}

/*
 * Round a double to the nearest bfloat16, ties to even, in ONE rounding (no detour
 * through binary32).  bfloat16 has 8 significant bits, exponents -126..127 and
 * subnormals spaced 2^-133.  The value is scaled by the quantum of its binade so
 * that the rounding is rint() of a double in [128, 256), which is exact.
 */
uint16_t oracle_bf16_from_f64(double v) {
    if (isnan(v)) return signbit(v) ? 0xFFC0u : 0x7FC0u;
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    double a = fabs(v);
    if (isinf(a)) return sign | 0x7F80u;
    if (a == 0.0) return sign;
    int e;
    (void)frexp(a, &e);            /* a = f * 2^e, f in [0.5, 1) */
    int qexp = (e < -125 ? -125 : e) - 8;
    double n = rint(ldexp(a, -qexp));   /* default rounding mode: nearest, ties even */
    double r = ldexp(n, qexp);          /* exact: n has at most 9 bits */
    if (r > 3.3895313892515355e38) return sign | 0x7F80u;   /* beyond max finite */
    /* r is a bfloat16 value, hence exactly a binary32 whose low 16 bits are zero */
    return sign | (uint16_t)(bits_from_f32((float)r) >> 16);
}

void oracle_round_bf16(const double* v, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_from_f64(v[i]);
}

static void store_io(void* base, int dt, int64_t i, float v) {
    if (dt == ORACLE_F32)
        ((float*)base)[i] = v;
    else
        ((uint16_t*)base)[i] = oracle_bf16_from_f64((double)v);
}

/* ---- one-row definitions ------------------------------------------------------ */

/* RmsNorm of one row held in double: y_j = x_j / sqrt(mean(x^2) + eps) * w_j. */
static void rms_row(const double* x, const void* w, int dt, int64_t D, double eps, double* y) {
    double sumsq = 0.0;
    for (int64_t j = 0; j < D; ++j) sumsq += x[j] * x[j];
    double denom = sqrt(sumsq / (double)D + eps);
    for (int64_t j = 0; j < D; ++j) {
        double wj = w ? widen(w, dt, j) : 1.0;
        y[j] = x[j] / denom * wj;
    }
}

/* LayerNorm of one row: y_j = (x_j - mean) / sqrt(var + eps) * w_j + b_j. */
static void layer_row(const double* x, const void* w, const void* b, int dt, int64_t D,
                      double eps, double* y) {
    double sum = 0.0;
    for (int64_t j = 0; j < D; ++j) sum += x[j];
    double mean = sum / (double)D;
    double sqdev = 0.0;
    for (int64_t j = 0; j < D; ++j) sqdev += (x[j] - mean) * (x[j] - mean);
    double var = sqdev / (double)D;
    double denom = sqrt(var + eps);
    for (int64_t j = 0; j < D; ++j) {
        double wj = w ? widen(w, dt, j) : 1.0;
        double bj = b ? widen(b, dt, j) : 0.0;
        y[j] = (x[j] - mean) / denom * wj + bj;
    }
}

/*
 * Rope of one row at position pos: pair i (0 <= i < dims/2) turns by
 * phi_i = pos * scale * theta_i, theta_i = base^(-2 i / dims), or theta_i = freqs[i]
 * when a frequency vector is given (FastOp::Rope: "base ... unused with freqs");
 * forward = 0 turns by -phi_i.  Features from dims on are copied unchanged.
 */
static void rope_row_freqs(const double* x, int64_t D, int64_t dims, int traditional, double base,
                           const double* freqs, double scale, double pos, int forward, double* y) {
    int64_t half = dims / 2;
    for (int64_t j = 0; j < D; ++j) y[j] = x[j];
    for (int64_t i = 0; i < half; ++i) {
        double theta = freqs ? freqs[i] : pow(base, -2.0 * (double)i / (double)dims);
        double phi = pos * scale * theta;
        if (!forward) phi = -phi;
        int64_t p = traditional ? 2 * i : i;
        int64_t q = traditional ? 2 * i + 1 : i + half;
        double c = cos(phi), s = sin(phi);
        y[p] = x[p] * c - x[q] * s;
        y[q] = x[p] * s + x[q] * c;
    }
}

static void rope_row(const double* x, int64_t D, int64_t dims, int traditional, double base,
                     double scale, double pos, int forward, double* y) {
    rope_row_freqs(x, D, dims, traditional, base, NULL, scale, pos, forward, y);
}

static void load_row(const void* src, int dt, int64_t row, int64_t D, double* dst) {
    for (int64_t j = 0; j < D; ++j) dst[j] = widen(src, dt, row * D + j);
}

/* ---- exported ops: rows [r0, r1) of [rows, D] row-major arrays -------------- */

int oracle_rms_norm(const void* x, const void* w, double* y, int64_t r0, int64_t r1, int64_t D,
                    float eps, int dt) {
    double* row = (double*)malloc((size_t)D * sizeof(double));
    if (!row) return -1;
    for (int64_t k = r0; k < r1; ++k) {
        load_row(x, dt, k, D, row);
        rms_row(row, w, dt, D, (double)eps, y + k * D);
    }
    free(row);
    return 0;
}

/* h = x + r added in binary32 and rounded once to the I/O type; y = RmsNorm(h). */
int oracle_add_rms_norm(const void* x, const void* r, const void* w, double* y, void* h,
                        int64_t r0, int64_t r1, int64_t D, float eps, int dt) {
    double* row = (double*)malloc((size_t)D * sizeof(double));
    if (!row) return -1;
    for (int64_t k = r0; k < r1; ++k) {
        for (int64_t j = 0; j < D; ++j) {
            int64_t i = k * D + j;
            float sum = (float)widen(x, dt, i) + (float)widen(r, dt, i);
            store_io(h, dt, i, sum);
            row[j] = widen(h, dt, i);    /* the rounded h, as returned */
        }
        rms_row(row, w, dt, D, (double)eps, y + k * D);
    }
    free(row);
    return 0;
}

/*
 * AllReduce + AddRmsNorm: the step a tensor-parallel decoder takes after a row-parallel
 * linear layer (miniVLLM Layers page, section Linear layers, RowParallelLinear: the
 * forward pass sums the ranks' partial outputs with an all_reduce), followed by the fused
 * residual add + RMSNorm (same page, section LayerNorm, forward with a residual; docs.rs
 * nuvec-core 0.5.0, Enum FastOp, variant AddRmsNorm).
 *   x = the sum over the nparts partial tensors, taken in part order in double and rounded
 *       once to the I/O type (written to x_out when it is not NULL);
 *   then add_rms_norm(x, r): h = x + r rounded to the I/O type, y = RmsNorm(h) * w.
 * parts: nparts pointers to [rows, D] arrays of the I/O type.
 */
int oracle_allreduce_add_rms_norm(const void* const* parts, int nparts, const void* r,
                                  const void* w, double* y, void* x_out, void* h, int64_t r0,
                                  int64_t r1, int64_t D, float eps, int dt) {
    if (nparts < 1) return -1;
    void* xb = malloc((size_t)(r1 - r0) * (size_t)D * (dt == ORACLE_BF16 ? 2 : 4));
    if (!xb) return -1;
    for (int64_t k = r0; k < r1; ++k)
        for (int64_t j = 0; j < D; ++j) {
            const int64_t i = k * D + j;
            double s = 0.0;
            for (int p = 0; p < nparts; ++p) s += widen(parts[p], dt, i);
            const int64_t o = (k - r0) * D + j;
            if (dt == ORACLE_BF16)
                ((uint16_t*)xb)[o] = oracle_bf16_from_f64(s);
            else
                ((float*)xb)[o] = (float)s;
            if (x_out) {
                if (dt == ORACLE_BF16)
                    ((uint16_t*)x_out)[i] = ((uint16_t*)xb)[o];
                else
                    ((float*)x_out)[i] = ((float*)xb)[o];
            }
        }
    /* add_rms_norm on the rounded x, rows r0..r1 (xb holds only those rows) */
    const size_t off = (size_t)r0 * (size_t)D;
    const size_t esz = dt == ORACLE_BF16 ? 2 : 4;
    int rc = oracle_add_rms_norm(xb, (const char*)r + off * esz, w, y + off, (char*)h + off * esz,
                                 0, r1 - r0, D, eps, dt);
    free(xb);
    return rc;
}

int oracle_layer_norm(const void* x, const void* w, const void* b, double* y, int64_t r0,
                      int64_t r1, int64_t D, float eps, int dt) {
    double* row = (double*)malloc((size_t)D * sizeof(double));
    if (!row) return -1;
    for (int64_t k = r0; k < r1; ++k) {
        load_row(x, dt, k, D, row);
        layer_row(row, w, b, dt, D, (double)eps, y + k * D);
    }
    free(row);
    return 0;
}

/* Rope on rows already in double (rows of [.., L, D], row k at l = k mod L). */
int oracle_rope_f64(const double* x, double* y, int64_t r0, int64_t r1, int64_t L, int64_t D,
                    int64_t dims, int traditional, float base, float scale, int64_t offset,
                    int forward) {
    for (int64_t k = r0; k < r1; ++k) {
        double pos = (double)offset + (double)(k % L);
        rope_row(x + k * D, D, dims, traditional, (double)base, (double)scale, pos, forward,
                 y + k * D);
    }
    return 0;
}

/*
 * NormRope on rows of x [B, H, L, D] flattened to [rows, D]: row k sits at
 * l = k mod L and position offset + l.  normalize != 0: RmsNorm(x, w, eps) over all
 * D features, then Rope.  normalize == 0: Rope of x alone (w unused).
 */
int oracle_norm_rope(const void* x, const void* w, double* y, int64_t r0, int64_t r1, int64_t L,
                     int64_t D, int64_t dims, int traditional, float base, float scale,
                     int64_t offset, int normalize, float eps, int dt) {
    double* row = (double*)malloc((size_t)D * sizeof(double));
    double* nrm = (double*)malloc((size_t)D * sizeof(double));
    if (!row || !nrm) {
        free(row);
        free(nrm);
        return -1;
    }
    for (int64_t k = r0; k < r1; ++k) {
        load_row(x, dt, k, D, row);
        if (normalize)
            rms_row(row, w, dt, D, (double)eps, nrm);
        else
            memcpy(nrm, row, (size_t)D * sizeof(double));
        double pos = (double)offset + (double)(k % L);
        rope_row(nrm, D, dims, traditional, (double)base, (double)scale, pos, 1, y + k * D);
    }
    free(row);
    free(nrm);
    return 0;
}

/*
 * Llama 3 long-context frequency scaling ("NTK-by-parts"): miniVLLM Layers page, section
 * RotaryEmbedding, constructor parameters llama3_rope_factor, llama3_rope_high_freq_factor,
 * llama3_rope_low_freq_factor and llama3_rope_original_max_position_embeddings; docs.rs
 * nuvec-core 0.5.0, Enum FastOp, variant Rope (frequency scaling by mlx-lm's Llama3RoPE).
 * The pages give the parameters: `factor` scales the low-frequency components; the two
 * other factors set wavelength thresholds (orig / low_freq_factor and orig / high_freq_factor)
 * beyond which the scaling is full or absent.  Reading (the pages print no formula): with
 * theta_i = base^(-2i/dims) and wavelength 2 pi / theta_i,
 *   wavelength < orig / high_freq_factor  ->  theta_i unchanged            (high frequency)
 *   wavelength > orig / low_freq_factor   ->  theta_i / factor             (low frequency)
 *   otherwise, with s = (orig / wavelength - low_freq_factor)
 *                       / (high_freq_factor - low_freq_factor) in [0, 1],
 *                                         ->  (1 - s) theta_i / factor + s theta_i
 * out: dims / 2 doubles.  Returns -1 for arguments outside the reading's domain.
 */
int oracle_llama3_freqs(int64_t dims, double base, double factor, double low_freq_factor,
                        double high_freq_factor, double orig, double* out) {
    if (dims < 2 || dims % 2 || !(base > 0.0) || !(factor >= 1.0) || !(low_freq_factor > 0.0) ||
        !(high_freq_factor > low_freq_factor) || !(orig > 0.0))
        return -1;
    const double two_pi = 2.0 * acos(-1.0);
    for (int64_t i = 0; i < dims / 2; ++i) {
        const double theta = pow(base, -(double)(2 * i) / (double)dims);
        const double wavelen = two_pi / theta;
        if (wavelen < orig / high_freq_factor) {
            out[i] = theta;
        } else if (wavelen > orig / low_freq_factor) {
            out[i] = theta / factor;
        } else {
            const double s = (orig / wavelen - low_freq_factor) / (high_freq_factor - low_freq_factor);
            out[i] = (1.0 - s) * theta / factor + s * theta;
        }
    }
    return 0;
}

/*
 * YaRN frequency scaling: named on docs.rs nuvec-core 0.5.0, Enum FastOp, variant Rope
 * (frequency scaling by mlx-lm's YarnRoPE); the pages give neither parameters nor formula.
 * Reading: the published YaRN method (Peng, Quesnelle, Fan and Shippole, "YaRN: Efficient
 * Context Window Extension of Large Language Models", 2023), its "NTK-by-parts"
 * interpolation and its attention temperature, in the paper's notation.  For pair d,
 * theta_d = base^(-2d/dims), wavelength lambda_d = 2 pi / theta_d, and r_d = L / lambda_d
 * the turns pair d makes over the original context length L.  With the ramp
 *   gamma(r) = 0 (r < alpha),  1 (r > beta),  (r - alpha) / (beta - alpha) otherwise,
 * the scaled frequency is h(theta_d) = (1 - gamma(r_d)) theta_d / s + gamma(r_d) theta_d
 * (s the extension factor): pairs turning many times keep theta_d, pairs turning less than
 * once are interpolated to theta_d / s.  The temperature scales q and k each by
 * sqrt(1/t) = 0.1 ln(s) + 1.  out: dims / 2 doubles; *mscale: sqrt(1/t).  Returns -1
 * outside the method's domain (dims even >= 2, base > 0, s >= 1, L > 0, 0 < alpha < beta).
 */
int oracle_yarn_freqs(int64_t dims, double base, double s, double L, double alpha, double beta,
                      double* out, double* mscale) {
    if (dims < 2 || dims % 2 || !(base > 0.0) || !(s >= 1.0) || !(L > 0.0) || !(alpha > 0.0) ||
        !(beta > alpha))
        return -1;
    const double pi = acos(-1.0);
    for (int64_t d = 0; d < dims / 2; ++d) {
        const double theta_d = pow(base, -2.0 * (double)d / (double)dims);
        const double lambda_d = 2.0 * pi / theta_d;
        const double r = L / lambda_d;
        double gamma;
        if (r < alpha)
            gamma = 0.0;
        else if (r > beta)
            gamma = 1.0;
        else
            gamma = (r - alpha) / (beta - alpha);
        out[d] = (1.0 - gamma) * theta_d / s + gamma * theta_d;
    }
    *mscale = 0.1 * log(s) + 1.0;
    return 0;
}

/*
 * SuScaled (LongRoPE) frequency scaling: named on docs.rs nuvec-core 0.5.0, Enum FastOp,
 * variant Rope (frequency scaling by mlx-lm's SuScaledRoPE); the pages give neither
 * parameters nor formula.  Reading: the published LongRoPE method (Ding, Zhang, Zhang, Xu,
 * Shang, Xu, Yang and Yang, "LongRoPE: Extending LLM Context Window Beyond 2 Million
 * Tokens", 2024) in the form the Phi-3 models use it (Abdin et al., "Phi-3 Technical
 * Report", 2024): every pair i has its own rescale factor lambda_i and turns at
 * theta_i / lambda_i, theta_i = base^(-2i/dims).  Two factor sets are searched, a short
 * one for sequences within the original context L and a long one beyond it:
 * lambda = long_factors when seq_len > L, else short_factors.  Extending L to the model's
 * maximum context L' (s = L' / L) also scales q and k by the attention factor
 * sqrt(1 + ln s / ln L) when s > 1 (1 otherwise).
 * out: dims / 2 doubles; *mscale: the attention factor.  Returns -1 outside the method's
 * domain (dims even >= 2, base > 0, every factor > 0, L > 1, L' > 0, seq_len >= 0).
 */
int oracle_suscaled_freqs(int64_t dims, double base, const double* short_factors,
                          const double* long_factors, double seq_len, double max_pos,
                          double orig, double* out, double* mscale) {
    if (dims < 2 || dims % 2 || !(base > 0.0) || !(orig > 1.0) || !(max_pos > 0.0) ||
        !(seq_len >= 0.0))
        return -1;
    const double* lambda = seq_len > orig ? long_factors : short_factors;
    for (int64_t i = 0; i < dims / 2; ++i)
        if (!(lambda[i] > 0.0)) return -1;
    for (int64_t i = 0; i < dims / 2; ++i) {
        const double theta_i = 1.0 / pow(base, 2.0 * (double)i / (double)dims);
        out[i] = theta_i / lambda[i];
    }
    const double s = max_pos / orig;
    *mscale = s > 1.0 ? sqrt(1.0 + log(s) / log(orig)) : 1.0;
    return 0;
}

/*
 * The general NormRope / Rope (FastOp::NormRope with its cache form, FastOp::Rope with
 * freqs and forward): rows of x [B, H, L, D] (rows = B*H*L) are normalised when
 * normalize != 0 and rotated at position offset + l (by -phi when forward == 0), with
 * theta_i from freqs (dims/2 doubles) when freqs != NULL.  y_len == 0: y is
 * [rows, D] like x.  y_len > 0: y is a cache [B*H, y_len, D] and row (bh, l) of x is
 * written to cache row (bh, offset + l); no other cache row is touched.
 */
int oracle_rope_ex(const void* x, const void* w, const double* freqs, double* y, int64_t r0,
                   int64_t r1, int64_t L, int64_t y_len, int64_t D, int64_t dims, int traditional,
                   float base, float scale, int64_t offset, int forward, int normalize, float eps,
                   int dt) {
    double* row = (double*)malloc((size_t)D * sizeof(double));
    double* nrm = (double*)malloc((size_t)D * sizeof(double));
    if (!row || !nrm) {
        free(row);
        free(nrm);
        return -1;
    }
    for (int64_t k = r0; k < r1; ++k) {
        load_row(x, dt, k, D, row);
        if (normalize)
            rms_row(row, w, dt, D, (double)eps, nrm);
        else
            memcpy(nrm, row, (size_t)D * sizeof(double));
        int64_t l = k % L;
        int64_t out = y_len > 0 ? (k / L) * y_len + offset + l : k;
        rope_row_freqs(nrm, D, dims, traditional, (double)base, freqs, (double)scale,
                       (double)offset + (double)l, forward, y + out * D);
    }
    free(row);
    free(nrm);
    return 0;
}

/*
 * RmsNormVjp (x, w, g): gradients of rms_norm with respect to x and w (docs.rs nuvec-core 0.5.0,
 * Enum FastOp, variant RmsNormVjp).  With r = 1 / sqrt(mean(x^2) + eps) and
 * y_j = x_j r w_j:
 *   dx_j = r w_j g_j - x_j r^3 (sum_k g_k w_k x_k) / D
 *   dw_j = sum over rows of g_j x_j r            (accumulated into dw, rows r0..r1)
 * mag_dx / mag_dw receive the same expressions with every term replaced by its
 * magnitude (the scale of the rounding error of a float32 evaluation).
 */
int oracle_rms_norm_vjp(const void* x, const void* w, const void* g, double* dx, double* dw,
                        double* mag_dx, double* mag_dw, int64_t r0, int64_t r1, int64_t D,
                        float eps, int dt) {
    for (int64_t k = r0; k < r1; ++k) {
        double sumsq = 0.0, c = 0.0, cmag = 0.0;
        for (int64_t j = 0; j < D; ++j) {
            double xj = widen(x, dt, k * D + j);
            double wj = w ? widen(w, dt, j) : 1.0;
            double gj = widen(g, dt, k * D + j);
            sumsq += xj * xj;
            c += gj * wj * xj;
            cmag += fabs(gj * wj * xj);
        }
        double r = 1.0 / sqrt(sumsq / (double)D + (double)eps);
        for (int64_t j = 0; j < D; ++j) {
            double xj = widen(x, dt, k * D + j);
            double wj = w ? widen(w, dt, j) : 1.0;
            double gj = widen(g, dt, k * D + j);
            dx[k * D + j] = r * wj * gj - xj * r * r * r * c / (double)D;
            mag_dx[k * D + j] = fabs(r * wj * gj) + fabs(xj) * r * r * r * cmag / (double)D;
            dw[j] += gj * xj * r;
            mag_dw[j] += fabs(gj * xj * r);
        }
    }
    return 0;
}

/*
 * LayerNormVjp (x, w, b, g): gradients of layer_norm with respect to x, w and b (docs.rs
 * nuvec-core 0.5.0, Enum FastOp, variant LayerNormVjp).  With mean, var (population),
 * r = 1 / sqrt(var + eps), xh_j = (x_j - mean) r, a_j = w_j g_j:
 *   dx_j = r (a_j - mean_k(a_k) - xh_j mean_k(a_k xh_k))
 *   dw_j = sum over rows of g_j xh_j,   db_j = sum over rows of g_j
 * (accumulated into dw and db for rows r0..r1); mag_* as for RmsNormVjp.
 */
int oracle_layer_norm_vjp(const void* x, const void* w, const void* g, double* dx, double* dw,
                          double* db, double* mag_dx, double* mag_dw, double* mag_db, int64_t r0,
                          int64_t r1, int64_t D, float eps, int dt) {
    for (int64_t k = r0; k < r1; ++k) {
        double sum = 0.0;
        for (int64_t j = 0; j < D; ++j) sum += widen(x, dt, k * D + j);
        double mean = sum / (double)D;
        double sqdev = 0.0;
        for (int64_t j = 0; j < D; ++j) {
            double d = widen(x, dt, k * D + j) - mean;
            sqdev += d * d;
        }
        double r = 1.0 / sqrt(sqdev / (double)D + (double)eps);
        double sa = 0.0, sax = 0.0, sa_mag = 0.0, sax_mag = 0.0;
        for (int64_t j = 0; j < D; ++j) {
            double xh = (widen(x, dt, k * D + j) - mean) * r;
            double a = (w ? widen(w, dt, j) : 1.0) * widen(g, dt, k * D + j);
            sa += a;
            sax += a * xh;
            sa_mag += fabs(a);
            sax_mag += fabs(a * xh);
        }
        for (int64_t j = 0; j < D; ++j) {
            double gj = widen(g, dt, k * D + j);
            double xh = (widen(x, dt, k * D + j) - mean) * r;
            double a = (w ? widen(w, dt, j) : 1.0) * gj;
            dx[k * D + j] = r * (a - sa / (double)D - xh * sax / (double)D);
            mag_dx[k * D + j] =
                r * (fabs(a) + sa_mag / (double)D + fabs(xh) * sax_mag / (double)D);
            dw[j] += gj * xh;
            db[j] += gj;
            mag_dw[j] += fabs(gj * xh);
            mag_db[j] += fabs(gj);
        }
    }
    return 0;
}
