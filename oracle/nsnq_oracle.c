/*
 * nsnq_oracle.c -- plain, slow CPU oracle for NSNQuant KV-cache vector
 * quantization and decode attention over the quantized cache.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or call
 * this file; only the test-suite, the smoke check and the benchmark's CPU
 * baseline leg do. It shares no code, headers, tables or constants with the
 * CUDA library: it is written from the method's description alone.
 *
 * Single-threaded, fp64 throughout, no blocking, fusion or reordering beyond
 * the definitions. Sources (gist.science "NSNQuant: A Double Normalization
 * Approach for Calibration-Free Low-Bit Vector Quantization of KV Cache",
 * Technical Summary):
 *   - Methodology §1 "Normalize-Shift-Normalize": token-wise normalize to
 *     norm sqrt(d), channel-wise mean shift, token-wise re-normalize to
 *     sqrt(d); byproducts (s1, o, s2) reconstruct the tensor.
 *   - Methodology §2 "Hadamard Transform": the naive (non-randomized)
 *     Hadamard transform is the one used in the implementation.
 *   - Methodology §3 "Vector Quantization and Codebook": one global codebook
 *     built by K-Means on synthetic standard-normal data; each sub-vector is
 *     replaced by its nearest codeword.
 *   - Methodology §4 "Implementation Details": attention scores are computed
 *     from the quantized cache and the NSN byproducts.
 * Readings where the text is silent (stated once, used everywhere):
 *   s = ||v|| / sqrt(d) so that v / s has norm sqrt(d); a zero-norm token maps
 *   to the zero vector and keeps s = 0, and a shift residual at or below
 *   2^-20 of the token/shift magnitude counts as zero; H is the orthonormal Sylvester
 *   Hadamard matrix in natural order, H[i][j] = (-1)^popcount(i & j) / sqrt(d);
 *   sub-vector j covers coordinates [j*g, (j+1)*g); argmin ties go to the
 *   lowest index; k-means starts from the first k samples, runs a fixed
 *   number of Lloyd iterations and an empty cluster keeps its centroid.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_MEM 2

static int parity_of_and(unsigned i, unsigned j) {
    unsigned v = i & j;
    int p = 0;
    while (v) {
        p ^= (int)(v & 1u);
        v >>= 1;
    }
    return p;
}

/* Orthonormal Sylvester Hadamard matrix, natural order (Methodology §2). */
int oracle_hadamard(int d, double* H) {
    if (d <= 0 || (d & (d - 1)) != 0 || !H) return ORACLE_ERR_ARG;
    double s = 1.0 / sqrt((double)d);
    for (int i = 0; i < d; ++i)
        for (int j = 0; j < d; ++j)
            H[(size_t)i * d + j] = parity_of_and((unsigned)i, (unsigned)j) ? -s : s;
    return ORACLE_OK;
}

/* out = H v, explicit dense product (not a butterfly). */
static void hadamard_apply(const double* H, int d, const double* v, double* out) {
    for (int i = 0; i < d; ++i) {
        double acc = 0.0;
        const double* row = H + (size_t)i * d;
        for (int k = 0; k < d; ++k) acc += row[k] * v[k];
        out[i] = acc;
    }
}

static double sqdist(const double* a, const double* b, int g) {
    double s = 0.0;
    for (int r = 0; r < g; ++r) {
        double e = a[r] - b[r];
        s += e * e;
    }
    return s;
}

/*
 * Codebook construction (Methodology §3): Lloyd's k-means on n samples of
 * dimension g. Start: the first k samples. Each iteration assigns every
 * sample to its nearest centroid (lowest index on ties) and moves each
 * centroid to the mean of its samples; an empty cluster keeps its centroid.
 * C receives k*g values; counts (optional) the final cluster sizes from the
 * last assignment step.
 */
int oracle_kmeans(const double* X, int64_t n, int g, int k, int iters, double* C,
                  int64_t* counts) {
    if (!X || !C || n < k || g <= 0 || k <= 0 || iters < 0) return ORACLE_ERR_ARG;
    double* sums = (double*)calloc((size_t)k * g, sizeof(double));
    int64_t* cnt = (int64_t*)calloc((size_t)k, sizeof(int64_t));
    if (!sums || !cnt) {
        free(sums);
        free(cnt);
        return ORACLE_ERR_MEM;
    }
    memcpy(C, X, (size_t)k * g * sizeof(double));
    for (int it = 0; it < iters; ++it) {
        memset(sums, 0, (size_t)k * g * sizeof(double));
        memset(cnt, 0, (size_t)k * sizeof(int64_t));
        for (int64_t i = 0; i < n; ++i) {
            const double* x = X + (size_t)i * g;
            int best = 0;
            double bd = sqdist(x, C, g);
            for (int c = 1; c < k; ++c) {
                double dd = sqdist(x, C + (size_t)c * g, g);
                if (dd < bd) {
                    bd = dd;
                    best = c;
                }
            }
            cnt[best] += 1;
            for (int r = 0; r < g; ++r) sums[(size_t)best * g + r] += x[r];
        }
        for (int c = 0; c < k; ++c)
            if (cnt[c] > 0)
                for (int r = 0; r < g; ++r)
                    C[(size_t)c * g + r] = sums[(size_t)c * g + r] / (double)cnt[c];
    }
    if (counts) {
        for (int c = 0; c < k; ++c) counts[c] = iters > 0 ? cnt[c] : 0;
    }
    free(sums);
    free(cnt);
    return ORACLE_OK;
}

/* Nearest codeword of one g-dimensional sub-vector (full squared distance,
 * lowest index on exact ties). */
static int nearest_codeword(const double* w, const float* C, int K, int g) {
    double cw[64];
    int best = 0;
    double bd = INFINITY;
    for (int c = 0; c < K; ++c) {
        for (int r = 0; r < g; ++r) cw[r] = (double)C[(size_t)c * g + r];
        double dd = sqdist(w, cw, g);
        if (dd < bd) {
            bd = dd;
            best = c;
        }
    }
    return best;
}

/*
 * Encode one (batch, kv-head) slice of T tokens (Methodology §1-§3).
 *   x       [T][d] input activations (exact values of the I/O type)
 *   C       [K][g] fp32 codebook
 *   shift_given = 0: o is the channel mean of the normalized tokens;
 *               = 1: o is taken from o_in (tokens appended to a cache whose
 *                    shift was computed over the prompt)
 *   adaptive_scale = 1: s2 is multiplied by ||w||^2 / (w . w_hat), the
 *               scale adjustment of Methodology §3 (see below).
 * Outputs: codes [T][d/g], s1 [T], s2 [T], o_out [d], and optionally
 * w_out [T][d] (the transformed tokens that were quantized).
 */
/*
 * Double quantization (Methodology §3, Double Quantization: the NSN
 * parameters o and s1 and the codebook entries are quantized to 4 bits).
 * Reading (the pages give no scheme): 4-bit asymmetric uniform quantization,
 * 16 levels from the minimum to the maximum of the values (step = range/15,
 * level = round((x - min) / step), half away from zero); a constant input
 * keeps its value.
 */
int oracle_quantize4(const double* x, int64_t n, double* xq) {
    if (n < 0 || (n > 0 && (!x || !xq))) return ORACLE_ERR_ARG;
    if (n == 0) return ORACLE_OK;
    double lo = x[0], hi = x[0];
    for (int64_t i = 1; i < n; ++i) {
        if (x[i] < lo) lo = x[i];
        if (x[i] > hi) hi = x[i];
    }
    const double step = (hi - lo) / 15.0;
    for (int64_t i = 0; i < n; ++i) {
        const double q = step > 0.0 ? round((x[i] - lo) / step) : 0.0;
        xq[i] = lo + q * step;
    }
    return ORACLE_OK;
}

/*
 * The 4-bit scale grid of one head: s1 is quantized on a grid uniform in
 * log2 (s1 is a positive scale spanning orders of magnitude), from the
 * least to the largest log2 s1 of the head's non-zero tokens. The grid
 * (lo, step) is stored in fp32 and used in that rounding everywhere, so a
 * later append reproduces the prompt's levels. A zero token keeps s1 = 0.
 */
static double s1_level_value(double s1, double lo, double step) {
    if (!(s1 > 0.0)) return 0.0;
    double k = step > 0.0 ? round((log2(s1) - lo) / step) : 0.0;
    if (k < 0.0) k = 0.0;
    if (k > 15.0) k = 15.0;
    return exp2(lo + k * step);
}

int oracle_encode_head(const double* x, int64_t T, int d, int g, const float* C, int K,
                       int shift_given, const double* o_in, int adaptive_scale, int double_quant,
                       double* s1_grid, uint8_t* codes, double* s1, double* s2, double* o_out,
                       double* w_out) {
    if (d <= 0 || (d & (d - 1)) != 0 || g <= 0 || d % g != 0 || g > 64 || K <= 0 || K > 256 ||
        T < 0 || (shift_given && !o_in) || !C || !o_out || (double_quant && !s1_grid))
        return ORACLE_ERR_ARG;
    const int J = d / g;
    const double sqrt_d = sqrt((double)d);
    double* H = (double*)malloc((size_t)d * d * sizeof(double));
    double* y = (double*)malloc((size_t)(T > 0 ? T : 1) * d * sizeof(double));
    double* u = (double*)malloc((size_t)d * sizeof(double));
    double* w = (double*)malloc((size_t)d * sizeof(double));
    if (!H || !y || !u || !w) {
        free(H); free(y); free(u); free(w);
        return ORACLE_ERR_MEM;
    }
    oracle_hadamard(d, H);

    /* Normalize (token-wise): s1 = ||x|| / sqrt(d), y = x / s1. */
    for (int64_t t = 0; t < T; ++t) {
        const double* xt = x + (size_t)t * d;
        double ss = 0.0;
        for (int c = 0; c < d; ++c) ss += xt[c] * xt[c];
        s1[t] = sqrt(ss) / sqrt_d;
    }
    if (double_quant) {  /* s1 on the head's 4-bit log2 grid (given, or from these tokens) */
        if (!shift_given) {
            double lo = 0.0, hi = 0.0;
            int any = 0;
            for (int64_t t = 0; t < T; ++t) {
                if (!(s1[t] > 0.0)) continue;
                const double l = log2(s1[t]);
                if (!any || l < lo) lo = l;
                if (!any || l > hi) hi = l;
                any = 1;
            }
            s1_grid[0] = (double)(float)lo;
            s1_grid[1] = (double)(float)((hi - lo) / 15.0);
        }
        for (int64_t t = 0; t < T; ++t) s1[t] = s1_level_value(s1[t], s1_grid[0], s1_grid[1]);
    }
    for (int64_t t = 0; t < T; ++t) {
        const double* xt = x + (size_t)t * d;
        const double s = s1[t];
        for (int c = 0; c < d; ++c) y[(size_t)t * d + c] = s > 0.0 ? xt[c] / s : 0.0;
    }
    /* Shift (channel-wise): o = mean over the T tokens, or the given o. */
    for (int c = 0; c < d; ++c) {
        if (shift_given) {
            o_out[c] = o_in[c];
        } else {
            double acc = 0.0;
            for (int64_t t = 0; t < T; ++t) acc += y[(size_t)t * d + c];
            o_out[c] = T > 0 ? acc / (double)T : 0.0;
        }
    }
    if (double_quant && !shift_given) oracle_quantize4(o_out, d, o_out);  /* o on 16 levels */
    for (int64_t t = 0; t < T; ++t) {
        double* yt = y + (size_t)t * d;
        /* z = y - o; Normalize again: s2 = ||z|| / sqrt(d), u = z / s2.
         * A residual at or below 2^-20 of sqrt(||y||^2 + ||o||^2) counts as
         * zero (s2 = 0, u = 0): fp32-stored byproducts cannot resolve it, and
         * it is exactly what a one-token prompt (o = y) produces. */
        double ss = 0.0, yy = 0.0, oo = 0.0;
        for (int c = 0; c < d; ++c) {
            yy += yt[c] * yt[c];
            oo += o_out[c] * o_out[c];
            yt[c] -= o_out[c];
            ss += yt[c] * yt[c];
        }
        double s = ss <= 0x1p-40 * (yy + oo) ? 0.0 : sqrt(ss) / sqrt_d;
        s2[t] = s;
        for (int c = 0; c < d; ++c) u[c] = s > 0.0 ? yt[c] / s : 0.0;
        /* Hadamard (Methodology §2), then nearest codeword per sub-vector. */
        hadamard_apply(H, d, u, w);
        if (w_out) memcpy(w_out + (size_t)t * d, w, (size_t)d * sizeof(double));
        for (int j = 0; j < J; ++j)
            codes[(size_t)t * J + j] = (uint8_t)nearest_codeword(w + (size_t)j * g, C, K, g);
        /* Scale adjustment (Methodology §3): the quantized vector w_hat is
         * scaled by a = ||w||^2 / (w . w_hat) so that its component along w
         * equals w (the remaining error is orthogonal to w); a is folded into
         * the stored s2. a = 1 when w . w_hat <= 0 (nothing to align). */
        if (adaptive_scale) {
            double ww = 0.0, wq = 0.0;
            for (int j = 0; j < J; ++j) {
                const int c = codes[(size_t)t * J + j];
                for (int r = 0; r < g; ++r) {
                    const double wi = w[j * g + r];
                    ww += wi * wi;
                    wq += wi * (double)C[(size_t)c * g + r];
                }
            }
            if (wq > 0.0) s2[t] *= ww / wq;
        }
    }
    free(H); free(y); free(u); free(w);
    return ORACLE_OK;
}

/*
 * Dequantize one (batch, kv-head) slice: x_hat = s1 * (s2 * H w_hat + o),
 * w_hat the concatenated codewords (Methodology §1: the byproducts
 * reconstruct the tensor). s1, s2, o are the stored fp32 values.
 */
int oracle_dequant_head(const uint8_t* codes, const float* s1, const float* s2, const float* o,
                        int64_t T, int d, int g, const float* C, int K, double* out) {
    if (d <= 0 || (d & (d - 1)) != 0 || g <= 0 || d % g != 0 || K <= 0 || K > 256 || T < 0)
        return ORACLE_ERR_ARG;
    const int J = d / g;
    double* H = (double*)malloc((size_t)d * d * sizeof(double));
    double* wh = (double*)malloc((size_t)d * sizeof(double));
    double* v = (double*)malloc((size_t)d * sizeof(double));
    if (!H || !wh || !v) {
        free(H); free(wh); free(v);
        return ORACLE_ERR_MEM;
    }
    oracle_hadamard(d, H);
    for (int64_t t = 0; t < T; ++t) {
        for (int j = 0; j < J; ++j) {
            int c = codes[(size_t)t * J + j];
            if (c >= K) {
                free(H); free(wh); free(v);
                return ORACLE_ERR_ARG;
            }
            for (int r = 0; r < g; ++r) wh[j * g + r] = (double)C[(size_t)c * g + r];
        }
        hadamard_apply(H, d, wh, v);
        for (int c = 0; c < d; ++c)
            out[(size_t)t * d + c] =
                (double)s1[t] * ((double)s2[t] * v[c] + (double)o[c]);
    }
    free(H); free(wh); free(v);
    return ORACLE_OK;
}

/*
 * Decode attention for the G query heads that share one kv-head, computed
 * directly from the dense dequantized cache (Methodology §4 together with the
 * standard definition): l_t = scale * q . k_t, p = softmax(l) (max
 * subtracted), out = sum_t p_t v_t. T = 0 gives a zero output.
 */
int oracle_attention_head(const double* q, int G, const double* Kh, const double* Vh, int64_t T,
                          int d, double scale, double* out) {
    if (G <= 0 || d <= 0 || T < 0) return ORACLE_ERR_ARG;
    double* l = (double*)malloc((size_t)(T > 0 ? T : 1) * sizeof(double));
    if (!l) return ORACLE_ERR_MEM;
    for (int h = 0; h < G; ++h) {
        const double* qh = q + (size_t)h * d;
        double* oh = out + (size_t)h * d;
        for (int c = 0; c < d; ++c) oh[c] = 0.0;
        if (T == 0) continue;
        double m = -INFINITY;
        for (int64_t t = 0; t < T; ++t) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c) acc += qh[c] * Kh[(size_t)t * d + c];
            l[t] = scale * acc;
            if (l[t] > m) m = l[t];
        }
        double den = 0.0;
        for (int64_t t = 0; t < T; ++t) {
            double p = exp(l[t] - m);
            den += p;
            for (int c = 0; c < d; ++c) oh[c] += p * Vh[(size_t)t * d + c];
        }
        for (int c = 0; c < d; ++c) oh[c] /= den;
    }
    free(l);
    return ORACLE_OK;
}

/*
 * Rotary position embedding of T rows of dimension d (Methodology §4,
 * Implementation Details: keys are quantized before RoPE, so attention
 * rotates the dequantized keys). Reading (the pages do not define RoPE):
 * the standard rotary embedding with the half-split pairing, channel i with
 * channel i + d/2 for i < d/2, rotated by the angle pos * base^(-2i/d):
 *   x'_i       = x_i cos - x_{i+d/2} sin
 *   x'_{i+d/2} = x_i sin + x_{i+d/2} cos.
 * pos[t] is the position of row t; the rotation is done in place.
 */
int oracle_rope(double* X, int64_t T, int d, const int64_t* pos, double base) {
    if (d <= 0 || (d & 1) || T < 0 || !(base > 0.0)) return ORACLE_ERR_ARG;
    const int h = d / 2;
    for (int64_t t = 0; t < T; ++t) {
        double* x = X + (size_t)t * d;
        for (int i = 0; i < h; ++i) {
            const double theta = pow(base, -2.0 * (double)i / (double)d);
            const double ang = (double)pos[t] * theta;
            const double c = cos(ang), s = sin(ang);
            const double a = x[i], b = x[i + h];
            x[i] = a * c - b * s;
            x[i + h] = a * s + b * c;
        }
    }
    return ORACLE_OK;
}
