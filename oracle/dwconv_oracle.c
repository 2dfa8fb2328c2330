/*
 * CPU oracle for the depthwise-convolution hot path of a conformer speech encoder.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's CPU
 * baseline may load this file's library.  The CUDA library never links, includes or
 * calls it, and it shares no code with the CUDA library.
 *
 * Plain loops in IEEE double, no blocking, no fusion, no reordering beyond what the
 * definitions state.  Inputs are the stored values widened to double (bf16 values are
 * exactly representable).  OpenMP runs only over independent outputs, so every sum is
 * taken in the same serial order whatever the thread count.
 *
 * Sources of the definitions:
 *  - parakeet.cpp PR #102, "perf: faster GPU decode: one SSM_CONV for the depthwise
 *    conv, less host work per step", section "What changes": the depthwise conv is a
 *    sum over k of x[t + k, c] * w[k, c] over the input padded to T + K - 1 frames,
 *    NeMo's conv for the same left padding, causal or symmetric.
 *  - NeMo PR #16114, "Use Fused Kernels for Depthwise Striding Subsampler", section
 *    "What does this PR do ?": mel [B,T,F,1] -> conv0 [B,T/2,F/2,256] -> ReLU -> masking
 *    -> conv_dw1 [B,T/4,F/4,256]; the depthwise kernel fuses pre- and post-masking and
 *    the causal padding; backward kernels exist (data and weight gradients).
 *
 * Readings where the pages are silent (all masks use the per-item length len_b,
 * clamped to [0, T]):
 *  - a frame t >= len_b of the conv input counts as zero before the conv, and output
 *    frames t >= len_b are zero after it;
 *  - the data gradient applies the same output mask to dy before propagating it;
 *  - subsampler: mel frames t >= len_b count as zero; conv0 rows i >= ceil(len_b/2)
 *    and conv_dw1 rows i >= ceil(len_b/4) are zero; time padding 1|1 (causal 2|0) and
 *    frequency padding 1|1 for both convs; padding values are zero.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static int64_t clamp_len(const int32_t *lengths, int64_t b, int64_t T)
{
    if (lengths == NULL) return T;
    int64_t L = lengths[b];
    if (L < 0) L = 0;
    if (L > T) L = T;
    return L;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * xpad[b, j, c] for j in [0, T + K - 1): the input shifted right by pad_left frames,
 * with frames outside [0, len_b) of the original sequence reading as zero.
 */
static double xpad_at(const double *x, int64_t b, int64_t j, int64_t c,
                      int64_t T, int64_t C, int64_t pad_left, int64_t L)
{
    int64_t s = j - pad_left;          /* frame of the unpadded input */
    if (s < 0 || s >= L) return 0.0;   /* padding, or a frame at/after len_b */
    return x[(b * T + s) * C + c];
}

/*
 * Forward: y[b,t,c] = [t < len_b] * (bias[c] + sum_{k<K} xpad[b,t+k,c] * w[k,c]).
 * x, y: [B][T][C]; w: [K][C]; bias: [C] or NULL; lengths: [B] or NULL (no mask).
 */
int oracle_dwconv1d_fwd(const double *x, const double *w, const double *bias,
                        const int32_t *lengths, int64_t B, int64_t T, int64_t C,
                        int64_t K, int64_t pad_left, double *y)
{
    if (B < 0 || T < 0 || C < 1 || K < 1 || pad_left < 0 || pad_left > K - 1) return 1;
    for (int64_t b = 0; b < B; ++b) {
        const int64_t L = clamp_len(lengths, b, T);
        #pragma omp parallel for schedule(static)
        for (int64_t t = 0; t < T; ++t) {
            for (int64_t c = 0; c < C; ++c) {
                double acc = 0.0;
                if (t < L) {
                    acc = bias ? bias[c] : 0.0;
                    for (int64_t k = 0; k < K; ++k)
                        acc += xpad_at(x, b, t + k, c, T, C, pad_left, L) * w[k * C + c];
                }
                y[(b * T + t) * C + c] = acc;
            }
        }
    }
    return 0;
}

/*
 * Data gradient, as the transpose of the forward map: with dz[b,t,c] = [t < len_b] dy[b,t,c],
 * every term xpad[b,t+k,c] * w[k,c] of y[b,t,c] that reads the real frame s = t + k - pad_left
 * (0 <= s < len_b) sends dz[b,t,c] * w[k,c] back to dx[b,s,c].  Summation order per dx
 * element: t ascending, then k ascending.
 */
int oracle_dwconv1d_bwd_dx(const double *dy, const double *w, const int32_t *lengths,
                           int64_t B, int64_t T, int64_t C, int64_t K, int64_t pad_left,
                           double *dx)
{
    if (B < 0 || T < 0 || C < 1 || K < 1 || pad_left < 0 || pad_left > K - 1) return 1;
    const int64_t CB = 64;                         /* channels per independent task */
    const int64_t ncb = (C + CB - 1) / CB;
    memset(dx, 0, sizeof(double) * (size_t)(B * T * C));
    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t cb = 0; cb < ncb; ++cb) {
            const int64_t L = clamp_len(lengths, b, T);
            const int64_t c0 = cb * CB, c1 = (c0 + CB < C) ? c0 + CB : C;
            for (int64_t t = 0; t < L; ++t) {
                for (int64_t k = 0; k < K; ++k) {
                    const int64_t s = t + k - pad_left;
                    if (s < 0 || s >= L) continue;
                    for (int64_t c = c0; c < c1; ++c)
                        dx[(b * T + s) * C + c] += dy[(b * T + t) * C + c] * w[k * C + c];
                }
            }
        }
    }
    return 0;
}

/*
 * Weight and bias gradients: dW[k,c] = sum_{b,t} dz[b,t,c] * xpad[b,t+k,c] and
 * dbias[c] = sum_{b,t} dz[b,t,c], with dz[b,t,c] = [t < len_b] dy[b,t,c].
 * Summation order per output: b ascending, then t ascending.  dbias may be NULL.
 */
int oracle_dwconv1d_bwd_dw(const double *x, const double *dy, const int32_t *lengths,
                           int64_t B, int64_t T, int64_t C, int64_t K, int64_t pad_left,
                           double *dw, double *dbias)
{
    if (B < 0 || T < 0 || C < 1 || K < 1 || pad_left < 0 || pad_left > K - 1) return 1;
    #pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < C; ++c) {
        double db = 0.0;
        for (int64_t k = 0; k < K; ++k) dw[k * C + c] = 0.0;
        for (int64_t b = 0; b < B; ++b) {
            const int64_t L = clamp_len(lengths, b, T);
            for (int64_t t = 0; t < T; ++t) {
                const double dz = (t < L) ? dy[(b * T + t) * C + c] : 0.0;
                db += dz;
                for (int64_t k = 0; k < K; ++k)
                    dw[k * C + c] += dz * xpad_at(x, b, t + k, c, T, C, pad_left, L);
            }
        }
        if (dbias) dbias[c] = db;
    }
    return 0;
}

/* Output size of a 3-tap, stride-2 convolution over n frames padded by p0|p1. */
static int64_t s2_out(int64_t n, int64_t p0, int64_t p1)
{
    int64_t m = n + p0 + p1 - 3;
    if (m < 0) return 0;
    return m / 2 + 1;
}

static int64_t ceil_half(int64_t n) { return (n + 1) / 2; }

/*
 * Fused depthwise-striding subsampler front, computed stage by stage:
 *   melpad  = mel (frames t >= len_b zeroed) padded by Pt|Pb in time and 1|1 in frequency
 *   h       = ReLU(b0[c] + sum_{p,q<3} melpad[2i+p, 2j+q] * w0[p,q,c]); rows i >= ceil(len_b/2) -> 0
 *   hpad    = h padded by Pt|Pb in time and 1|1 in frequency, zeros
 *   out     = b1[c] + sum_{p,q<3} hpad[2i+p, 2j+q, c] * w1[p,q,c];     rows i >= ceil(len_b/4) -> 0
 * with Pt|Pb = 1|1 (symmetric) or 2|0 (causal).
 * mel: [B][T][F]; w0, w1: [3][3][C]; b0, b1: [C]; out: [B][T4][F4][C];
 * out_lengths: [B] or NULL, receives ceil(ceil(len_b/2)/2).
 */
int oracle_dw_subsample_fwd(const double *mel, const double *w0, const double *b0,
                            const double *w1, const double *b1, const int32_t *lengths,
                            int64_t B, int64_t T, int64_t F, int64_t C, int causal,
                            double *out, int32_t *out_lengths)
{
    if (B < 0 || T < 0 || F < 1 || C < 1) return 1;
    const int64_t Pt = causal ? 2 : 1, Pb = causal ? 0 : 1;
    const int64_t T2 = s2_out(T, Pt, Pb), F2 = s2_out(F, 1, 1);
    const int64_t T4 = s2_out(T2, Pt, Pb), F4 = s2_out(F2, 1, 1);
    const int64_t TP = T + Pt + Pb, FP = F + 2;          /* melpad extent */
    const int64_t HT = T2 + Pt + Pb, HF = F2 + 2;        /* hpad extent */
    double *melpad = (double *)malloc(sizeof(double) * (size_t)(TP * FP));
    double *hpad = (double *)malloc(sizeof(double) * (size_t)(HT * HF * C));
    if ((TP * FP > 0 && !melpad) || (HT * HF * C > 0 && !hpad)) {
        free(melpad);
        free(hpad);
        return 2;
    }
    for (int64_t b = 0; b < B; ++b) {
        const int64_t L = clamp_len(lengths, b, T);
        const int64_t L2 = ceil_half(L), L4 = ceil_half(L2);
        if (out_lengths) out_lengths[b] = (int32_t)L4;

        /* melpad: zero padding, and zero at frames t >= len_b */
        for (int64_t r = 0; r < TP; ++r)
            for (int64_t f = 0; f < FP; ++f) {
                const int64_t t = r - Pt, ff = f - 1;
                melpad[r * FP + f] = (t >= 0 && t < L && ff >= 0 && ff < F)
                                         ? mel[(b * T + t) * F + ff] : 0.0;
            }

        /* conv0 + bias + ReLU + row mask, written into the interior of hpad */
        memset(hpad, 0, sizeof(double) * (size_t)(HT * HF * C));
        #pragma omp parallel for schedule(static)
        for (int64_t i = 0; i < T2; ++i) {
            for (int64_t j = 0; j < F2; ++j) {
                for (int64_t c = 0; c < C; ++c) {
                    double a = b0[c];
                    for (int64_t p = 0; p < 3; ++p)
                        for (int64_t q = 0; q < 3; ++q)
                            a += melpad[(2 * i + p) * FP + (2 * j + q)] * w0[(p * 3 + q) * C + c];
                    double hv = a > 0.0 ? a : 0.0;          /* ReLU */
                    if (i >= L2) hv = 0.0;                  /* mask beyond ceil(len/2) */
                    hpad[((i + Pt) * HF + (j + 1)) * C + c] = hv;
                }
            }
        }

        /* conv_dw1 (depthwise) + bias + row mask */
        #pragma omp parallel for schedule(static)
        for (int64_t i = 0; i < T4; ++i) {
            for (int64_t j = 0; j < F4; ++j) {
                for (int64_t c = 0; c < C; ++c) {
                    double a = b1[c];
                    for (int64_t p = 0; p < 3; ++p)
                        for (int64_t q = 0; q < 3; ++q)
                            a += hpad[((2 * i + p) * HF + (2 * j + q)) * C + c] * w1[(p * 3 + q) * C + c];
                    if (i >= L4) a = 0.0;                   /* mask beyond ceil(len/4) */
                    out[((b * T4 + i) * F4 + j) * C + c] = a;
                }
            }
        }
    }
    free(melpad);
    free(hpad);
    return 0;
}

/*
 * Streaming causal forward, one chunk (parakeet.cpp PR #102, "What changes": the streaming
 * encoder keeps its own depthwise conv with a cache).  For stream b the sequence seen so far
 * ends with the K-1 cached frames, and this chunk appends its first len_b frames:
 *   xcat_b      = [cache_b frames 0..K-2 ; x_b frames 0..len_b-1]
 *   y[b,t,c]    = [t < len_b] * (bias[c] + sum_{k<K} xcat_b[t+k,c] * w[k,c])
 *   cache_out_b = xcat_b frames len_b .. len_b+K-2   (the K-1 most recent frames)
 * which is the causal conv (pad_left = K-1) of the whole stream, chunk by chunk, when the
 * cache starts at zero.  x, y: [B][T][C]; cache_in, cache_out: [B][K-1][C] (NULL if K == 1).
 */
int oracle_dwconv1d_stream_fwd(const double *x, const double *w, const double *bias,
                               const double *cache_in, const int32_t *lengths, int64_t B,
                               int64_t T, int64_t C, int64_t K, double *y, double *cache_out)
{
    if (B < 0 || T < 0 || C < 1 || K < 1) return 1;
    if (K > 1 && (cache_in == NULL || cache_out == NULL)) return 1;
    const int64_t H = K - 1;                       /* cached frames */
    for (int64_t b = 0; b < B; ++b) {
        const int64_t L = clamp_len(lengths, b, T);
        /* H + T frames: the frames after the chunk's valid ones stay zero and are never summed */
        double *xcat = (double *)calloc((size_t)((H + T) * C + 1), sizeof(double));
        if (!xcat) return 2;
        for (int64_t j = 0; j < H; ++j)
            for (int64_t c = 0; c < C; ++c) xcat[j * C + c] = cache_in[(b * H + j) * C + c];
        for (int64_t s = 0; s < L; ++s)
            for (int64_t c = 0; c < C; ++c) xcat[(H + s) * C + c] = x[(b * T + s) * C + c];
        #pragma omp parallel for schedule(static)
        for (int64_t t = 0; t < T; ++t) {
            for (int64_t c = 0; c < C; ++c) {
                double acc = 0.0;
                if (L > t) {   /* frame t of the chunk is part of the stream */
                    acc = bias ? bias[c] : 0.0;
                    for (int64_t k = 0; k < K; ++k) acc += xcat[(t + k) * C + c] * w[k * C + c];
                }
                y[(b * T + t) * C + c] = acc;
            }
        }
        for (int64_t j = 0; j < H; ++j)
            for (int64_t c = 0; c < C; ++c) cache_out[(b * H + j) * C + c] = xcat[(L + j) * C + c];
        free(xcat);
    }
    return 0;
}

/*
 * Backward of the fused subsampler front (NeMo PR #16114, "What does this PR do ?": the fused
 * kernels come with backward passes for training): given dout [B][T4][F4][C], the gradients of
 * sum(out * dout) with respect to w0, b0, w1 and b1, the forward's stages taken backward:
 *   doutm[i,j,c]         = [i < ceil(len/4)] dout[i,j,c]
 *   db1[c]              += sum_{i,j} doutm[i,j,c]
 *   dw1[p,q,c]          += sum_{i,j} doutm[i,j,c] hpad[2i+p, 2j+q, c]
 *   dhpad[2i+p,2j+q,c]  += doutm[i,j,c] w1[p,q,c]              (transpose of conv_dw1)
 *   dz[r,s,c]            = [r < ceil(len/2)] [z[r,s,c] > 0] dhpad[r+Pt, s+1, c]
 *   db0[c]              += sum_{r,s} dz[r,s,c]
 *   dw0[p,q,c]          += sum_{r,s} dz[r,s,c] melpad[2r+p, 2s+q]
 * with z = b0 + conv0(melpad) the pre-activation (ReLU' = [z > 0]) and melpad, hpad as in the
 * forward.  The mel input has no gradient (it is the network's input).  Every sum runs over
 * items, then rows, then columns, in order.  Outputs [3][3][C], [C], [3][3][C], [C].
 */
int oracle_dw_subsample_bwd(const double *mel, const double *w0, const double *b0,
                            const double *w1, const double *dout, const int32_t *lengths,
                            int64_t B, int64_t T, int64_t F, int64_t C, int causal,
                            double *dw0, double *db0, double *dw1, double *db1)
{
    if (B < 0 || T < 0 || F < 1 || C < 1) return 1;
    const int64_t Pt = causal ? 2 : 1, Pb = causal ? 0 : 1;
    const int64_t T2 = s2_out(T, Pt, Pb), F2 = s2_out(F, 1, 1);
    const int64_t T4 = s2_out(T2, Pt, Pb), F4 = s2_out(F2, 1, 1);
    const int64_t TP = T + Pt + Pb, FP = F + 2;
    const int64_t HT = T2 + Pt + Pb, HF = F2 + 2;
    memset(dw0, 0, sizeof(double) * (size_t)(9 * C));
    memset(dw1, 0, sizeof(double) * (size_t)(9 * C));
    memset(db0, 0, sizeof(double) * (size_t)C);
    memset(db1, 0, sizeof(double) * (size_t)C);
    double *melpad = (double *)malloc(sizeof(double) * (size_t)(TP * FP + 1));
    double *z = (double *)malloc(sizeof(double) * (size_t)(T2 * F2 * C + 1));
    double *hpad = (double *)malloc(sizeof(double) * (size_t)(HT * HF * C + 1));
    double *dhpad = (double *)malloc(sizeof(double) * (size_t)(HT * HF * C + 1));
    if (!melpad || !z || !hpad || !dhpad) {
        free(melpad); free(z); free(hpad); free(dhpad);
        return 2;
    }
    for (int64_t b = 0; b < B; ++b) {
        const int64_t L = clamp_len(lengths, b, T);
        const int64_t L2 = ceil_half(L), L4 = ceil_half(L2);
        for (int64_t r = 0; r < TP; ++r)
            for (int64_t f = 0; f < FP; ++f) {
                const int64_t t = r - Pt, ff = f - 1;
                melpad[r * FP + f] = (ff >= 0 && ff < F && t >= 0 && t < L)
                                         ? mel[(b * T + t) * F + ff] : 0.0;
            }
        memset(hpad, 0, sizeof(double) * (size_t)(HT * HF * C));
        memset(dhpad, 0, sizeof(double) * (size_t)(HT * HF * C));
        #pragma omp parallel for schedule(static)
        for (int64_t c = 0; c < C; ++c) {
            /* forward again: pre-activation z and the masked, ReLU'd h in hpad */
            for (int64_t r = 0; r < T2; ++r)
                for (int64_t s = 0; s < F2; ++s) {
                    double a = b0[c];
                    for (int64_t p = 0; p < 3; ++p)
                        for (int64_t q = 0; q < 3; ++q) {
                            const double tap = w0[(p * 3 + q) * C + c];
                            a += melpad[(2 * r + p) * FP + (2 * s + q)] * tap;
                        }
                    z[(r * F2 + s) * C + c] = a;
                    hpad[((r + Pt) * HF + (s + 1)) * C + c] = (r < L2 && a > 0.0) ? a : 0.0;
                }
            /* conv_dw1 backward: its weight and bias gradients, and dhpad */
            for (int64_t i = 0; i < T4; ++i)
                for (int64_t j = 0; j < F4; ++j) {
                    const double dm = (i < L4) ? dout[((b * T4 + i) * F4 + j) * C + c] : 0.0;
                    db1[c] += dm;
                    for (int64_t p = 0; p < 3; ++p)
                        for (int64_t q = 0; q < 3; ++q) {
                            const int64_t at = ((2 * i + p) * HF + (2 * j + q)) * C + c;
                            dw1[(p * 3 + q) * C + c] += dm * hpad[at];
                            dhpad[at] += dm * w1[(p * 3 + q) * C + c];
                        }
                }
            /* row mask and ReLU backward, then conv0's weight and bias gradients */
            for (int64_t r = 0; r < T2; ++r)
                for (int64_t s = 0; s < F2; ++s) {
                    const double dzv = (r < L2 && z[(r * F2 + s) * C + c] > 0.0)
                                           ? dhpad[((r + Pt) * HF + (s + 1)) * C + c] : 0.0;
                    db0[c] += dzv;
                    for (int64_t p = 0; p < 3; ++p)
                        for (int64_t q = 0; q < 3; ++q)
                            dw0[(p * 3 + q) * C + c] += dzv * melpad[(2 * r + p) * FP + (2 * s + q)];
                }
        }
    }
    free(melpad); free(z); free(hpad); free(dhpad);
    return 0;
}

/*
 * Tolerance term for the subsampler backward at the ReLU kink.  The derivative [z > 0] is a
 * decision taken on a floating-point z: where |z| is within rounding of 0, a float32 evaluation
 * and this float64 one may decide differently, and each such h pixel moves dw0 by at most
 * |dz| |melpad tap| and db0 by at most |dz|.  The rounding error of any evaluation of
 * z = b0 + sum_t melpad_t w0_t is bounded by a multiple of the sum of the magnitudes of its
 * terms, S = |b0| + sum_t |melpad_t w0_t|, so a pixel counts when |z| <= delta + delta_rel * S
 * (unmasked rows only).  This returns the bounds summed over those pixels, per tap and
 * channel: kdw0 [3][3][C], kdb0 [C].
 */
int oracle_dw_subsample_bwd_kinks(const double *mel, const double *w0, const double *b0,
                                  const double *w1, const double *dout, const int32_t *lengths,
                                  int64_t B, int64_t T, int64_t F, int64_t C, int causal,
                                  double delta, double delta_rel, double *kdw0, double *kdb0)
{
    if (B < 0 || T < 0 || F < 1 || C < 1) return 1;
    const int64_t Pt = causal ? 2 : 1, Pb = causal ? 0 : 1;
    const int64_t T2 = s2_out(T, Pt, Pb), F2 = s2_out(F, 1, 1);
    const int64_t T4 = s2_out(T2, Pt, Pb), F4 = s2_out(F2, 1, 1);
    const int64_t TP = T + Pt + Pb, FP = F + 2;
    memset(kdw0, 0, sizeof(double) * (size_t)(9 * C));
    memset(kdb0, 0, sizeof(double) * (size_t)C);
    double *melpad = (double *)malloc(sizeof(double) * (size_t)(TP * FP + 1));
    if (!melpad) return 2;
    for (int64_t b = 0; b < B; ++b) {
        const int64_t L = clamp_len(lengths, b, T);
        const int64_t L2 = ceil_half(L), L4 = ceil_half(L2);
        for (int64_t r = 0; r < TP; ++r)
            for (int64_t f = 0; f < FP; ++f) {
                const int64_t t = r - Pt, ff = f - 1;
                melpad[r * FP + f] = (t < L && t >= 0 && ff < F && ff >= 0) ? mel[(b * T + t) * F + ff] : 0.0;
            }
        #pragma omp parallel for schedule(static)
        for (int64_t c = 0; c < C; ++c) {
            for (int64_t r = 0; r < T2 && r < L2; ++r)
                for (int64_t s = 0; s < F2; ++s) {
                    double zv = b0[c], mag = fabs(b0[c]);
                    for (int64_t t = 0; t < 9; ++t) {
                        const double term = melpad[(2 * r + t / 3) * FP + (2 * s + t % 3)] * w0[t * C + c];
                        zv += term;
                        mag += fabs(term);
                    }
                    if (fabs(zv) > delta + delta_rel * mag) continue;
                    double dh = 0.0;   /* the transposed conv_dw1 at (r, s) */
                    for (int64_t p = 0; p < 3; ++p)
                        for (int64_t q = 0; q < 3; ++q) {
                            const int64_t ii = r + Pt - p, jj = s + 1 - q;
                            if (ii < 0 || jj < 0 || ii % 2 || jj % 2) continue;
                            const int64_t i = ii / 2, j = jj / 2;
                            if (i >= T4 || i >= L4 || j >= F4) continue;
                            dh += dout[((b * T4 + i) * F4 + j) * C + c] * w1[(p * 3 + q) * C + c];
                        }
                    kdb0[c] += fabs(dh);
                    for (int64_t t = 0; t < 9; ++t)
                        kdw0[t * C + c] += fabs(dh) * fabs(melpad[(2 * r + t / 3) * FP + (2 * s + t % 3)]);
                }
        }
    }
    free(melpad);
    return 0;
}

/*
 * General depthwise conv2d with fused length masking (NeMo PR #16114, "What does this PR do ?",
 * the second kernel: a depthwise conv with fused pre/post masking and causal padding, for the
 * subsampler's later stages).  Channels-last x [B][T][F][C], taps w [KT][KF][C]:
 *   xpad[b,r,s,c] = x[b, r-pt, s-pf, c] if 0 <= r-pt < len_b and 0 <= s-pf < F, else 0
 *   To = (T + pt + pb - KT) / st + 1, Fo = (F + 2 pf - KF) / sf + 1 (0 when negative inside)
 *   Lo_b = min(To, (len_b + pt + pb - KT) / st + 1), the usual conv length rule
 *   y[b,i,j,c] = [i < Lo_b] (bias[c] + sum_{p<KT,q<KF} xpad[b, st i + p, sf j + q, c] w[p,q,c])
 * The data gradient is the transpose (scatter) of this map with dy masked to rows i < Lo_b; the
 * weight and bias gradients sum dy_masked * xpad and dy_masked over (b, i, j).
 */
static int64_t conv_out(int64_t n, int64_t p0, int64_t p1, int64_t k, int64_t s)
{
    const int64_t m = n + p0 + p1 - k;
    if (m < 0) return 0;
    return m / s + 1;
}

static double xpad2(const double *x, int64_t b, int64_t r, int64_t s, int64_t c, int64_t T, int64_t F,
                    int64_t C, int64_t pt, int64_t pf, int64_t L)
{
    const int64_t t = r - pt, f = s - pf;
    if (t < 0 || t >= L || f < 0 || f >= F) return 0.0;   /* padding, or a frame at/after len_b */
    return x[((b * T + t) * F + f) * C + c];
}

static int conv2d_args_ok(int64_t B, int64_t T, int64_t F, int64_t C, int64_t KT, int64_t KF, int64_t st,
                          int64_t sf, int64_t pt, int64_t pb, int64_t pf)
{
    return B >= 0 && T >= 0 && F >= 1 && C >= 1 && KT >= 1 && KF >= 1 && st >= 1 && sf >= 1 &&
           pt >= 0 && pb >= 0 && pf >= 0;
}

int oracle_dwconv2d_fwd(const double *x, const double *w, const double *bias, const int32_t *lengths,
                        int64_t B, int64_t T, int64_t F, int64_t C, int64_t KT, int64_t KF, int64_t st,
                        int64_t sf, int64_t pt, int64_t pb, int64_t pf, double *y, int32_t *out_lengths)
{
    if (!conv2d_args_ok(B, T, F, C, KT, KF, st, sf, pt, pb, pf)) return 1;
    const int64_t To = conv_out(T, pt, pb, KT, st), Fo = conv_out(F, pf, pf, KF, sf);
    for (int64_t b = 0; b < B; ++b) {
        const int64_t L = clamp_len(lengths, b, T);
        int64_t Lo = conv_out(L, pt, pb, KT, st);
        if (Lo > To) Lo = To;
        if (out_lengths) out_lengths[b] = (int32_t)Lo;
        #pragma omp parallel for schedule(static)
        for (int64_t i = 0; i < To; ++i)
            for (int64_t j = 0; j < Fo; ++j)
                for (int64_t c = 0; c < C; ++c) {
                    double acc = 0.0;
                    if (i < Lo) {
                        acc = bias ? bias[c] : 0.0;
                        for (int64_t p = 0; p < KT; ++p)
                            for (int64_t q = 0; q < KF; ++q)
                                acc += xpad2(x, b, st * i + p, sf * j + q, c, T, F, C, pt, pf, L) *
                                       w[(p * KF + q) * C + c];
                    }
                    y[((b * To + i) * Fo + j) * C + c] = acc;
                }
    }
    return 0;
}

int oracle_dwconv2d_bwd_dx(const double *dy, const double *w, const int32_t *lengths, int64_t B, int64_t T,
                           int64_t F, int64_t C, int64_t KT, int64_t KF, int64_t st, int64_t sf, int64_t pt,
                           int64_t pb, int64_t pf, double *dx)
{
    if (!conv2d_args_ok(B, T, F, C, KT, KF, st, sf, pt, pb, pf)) return 1;
    const int64_t To = conv_out(T, pt, pb, KT, st), Fo = conv_out(F, pf, pf, KF, sf);
    memset(dx, 0, sizeof(double) * (size_t)(B * T * F * C));
    for (int64_t b = 0; b < B; ++b) {
        const int64_t L = clamp_len(lengths, b, T);
        int64_t Lo = conv_out(L, pt, pb, KT, st);
        if (Lo > To) Lo = To;
        #pragma omp parallel for schedule(static)
        for (int64_t c = 0; c < C; ++c)       /* scatter of every unmasked output, per channel */
            for (int64_t i = 0; i < Lo; ++i)
                for (int64_t j = 0; j < Fo; ++j) {
                    const double g = dy[((b * To + i) * Fo + j) * C + c];
                    for (int64_t p = 0; p < KT; ++p)
                        for (int64_t q = 0; q < KF; ++q) {
                            const int64_t t = st * i + p - pt, f = sf * j + q - pf;
                            if (t < 0 || t >= L || f < 0 || f >= F) continue;
                            dx[((b * T + t) * F + f) * C + c] += g * w[(p * KF + q) * C + c];
                        }
                }
    }
    return 0;
}

int oracle_dwconv2d_bwd_dw(const double *x, const double *dy, const int32_t *lengths, int64_t B, int64_t T,
                           int64_t F, int64_t C, int64_t KT, int64_t KF, int64_t st, int64_t sf, int64_t pt,
                           int64_t pb, int64_t pf, double *dw, double *dbias)
{
    if (!conv2d_args_ok(B, T, F, C, KT, KF, st, sf, pt, pb, pf)) return 1;
    const int64_t To = conv_out(T, pt, pb, KT, st), Fo = conv_out(F, pf, pf, KF, sf);
    #pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < C; ++c) {
        double gb = 0.0;
        for (int64_t pq = 0; pq < KT * KF; ++pq) dw[pq * C + c] = 0.0;
        for (int64_t b = 0; b < B; ++b) {
            const int64_t L = clamp_len(lengths, b, T);
            int64_t Lo = conv_out(L, pt, pb, KT, st);
            if (Lo > To) Lo = To;
            for (int64_t i = 0; i < Lo; ++i)
                for (int64_t j = 0; j < Fo; ++j) {
                    const double g = dy[((b * To + i) * Fo + j) * C + c];
                    gb += g;
                    for (int64_t p = 0; p < KT; ++p)
                        for (int64_t q = 0; q < KF; ++q)
                            dw[(p * KF + q) * C + c] += g * xpad2(x, b, st * i + p, sf * j + q, c, T, F, C, pt, pf, L);
                }
        }
        if (dbias) dbias[c] = gb;
    }
    return 0;
}
