// General depthwise conv2d with fused length masking (NeMo PR #16114, "Use Fused Kernels for
// Depthwise Striding Subsampler", section "What does this PR do ?", the second kernel: a depthwise
// conv with fused pre/post masking and causal padding, for the subsampler's later stages).
//
//   xpad[b,r,s,c] = x[b, r-pt, s-pf, c] if 0 <= r-pt < len_b and 0 <= s-pf < F, else 0
//   y[b,i,j,c]    = [i < Lo_b] (bias[c] + sum_{p,q} xpad[b, st i + p, sf j + q, c] w[p,q,c])
//   dx[b,t,f,c]   = [t < len_b] sum over the (i, j, p, q) with st i + p - pt = t, sf j + q - pf = f,
//                   i < Lo_b, of dy[b,i,j,c] w[p,q,c]            (the transpose, as a gather)
//   dW[p,q,c]     = sum_{b, i < Lo_b, j} dy[b,i,j,c] xpad[b, st i + p, sf j + q, c];  dbias = sum dy
//
// Channels-last, so a thread owns V consecutive channels (one 8- or 16-byte vector) of one output
// row and walks its columns; every access of a warp is 32 consecutive vectors.  The weight
// gradient keeps per-thread partial sums over a persistent share of the rows, writes one partial
// row per block and adds the rows in a fixed order (reproducible for given sizes on a given GPU model, no atomics).
#include "dw_internal.h"

namespace dwk {
namespace {

constexpr int kC2Threads = 128;
constexpr int kC2MaxRows = 592;   // weight-gradient partial rows (at most; 4 per SM)
constexpr int kC2Taps = 9;        // taps per weight-gradient pass

__device__ __forceinline__ int conv_len(int n, int p0, int p1, int k, int s) {
    const int m = n + p0 + p1 - k;
    return m < 0 ? 0 : m / s + 1;
}

template <typename T, int V>
__device__ __forceinline__ void ld_frame(const T *p, float2 (&f)[Pairs<V>::n]) {
    Vec<T, V> v;
    v.load(p);
    v.to_f2(f);
}

// KTC/KFC > 0: a compiled window (taps in registers); 0: runtime KT, KF.
template <typename T, int V, int KTC, int KFC>
__global__ void __launch_bounds__(kC2Threads)
dwconv2d_fwd_kernel(const T *__restrict__ x, const float *__restrict__ w, const float *__restrict__ bias,
                    T *__restrict__ y, const int32_t *__restrict__ lengths, int32_t *__restrict__ out_lengths, int B,
                    int Tn, int F, int C, int KTr, int KFr, int st, int sf, int pt, int pb, int pf, int To, int Fo,
                    int nCV) {
    constexpr int P = Pairs<V>::n;
    const int KT = KTC > 0 ? KTC : KTr, KF = KFC > 0 ? KFC : KFr;
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<int64_t>(B) * To * nCV) return;
    const int cv = static_cast<int>(idx % nCV);
    const int64_t rest = idx / nCV;
    const int i = static_cast<int>(rest % To), b = static_cast<int>(rest / To);
    const int c = cv * V;
    const int L = static_cast<int>(clamp_len(lengths, b, Tn));
    int Lo = conv_len(L, pt, pb, KT, st);
    if (Lo > To) Lo = To;
    if (out_lengths != nullptr && i == 0 && cv == 0) out_lengths[b] = Lo;
    T *yr = y + (static_cast<int64_t>(b) * To + i) * Fo * C + c;
    if (i >= Lo) {
        for (int j = 0; j < Fo; ++j) Vec<T, V>::store_zero(yr + static_cast<int64_t>(j) * C);
        return;
    }
    float2 bv[P];
    if (bias != nullptr) {
        load_param<V>(bias + c, bv);
    } else {
#pragma unroll
        for (int q = 0; q < P; ++q) bv[q] = make_float2(0.f, 0.f);
    }
    float2 wr[KTC > 0 ? KTC * KFC : 1][P];
    if constexpr (KTC > 0) {
#pragma unroll
        for (int t = 0; t < KTC * KFC; ++t) load_param<V>(w + static_cast<int64_t>(t) * C + c, wr[t]);
    }
    const T *xb = x + static_cast<int64_t>(b) * Tn * F * C + c;
    for (int j = 0; j < Fo; ++j) {
        float2 acc[P];
#pragma unroll
        for (int q = 0; q < P; ++q) acc[q] = bv[q];
#pragma unroll(KTC > 0 ? KTC : 1)
        for (int p = 0; p < KT; ++p) {
            const int r = st * i + p - pt;
            if (r < 0 || r >= L) continue;  // padding, or a frame at/after len_b
#pragma unroll(KFC > 0 ? KFC : 1)
            for (int qq = 0; qq < KF; ++qq) {
                const int f = sf * j + qq - pf;
                if (f < 0 || f >= F) continue;
                float2 xv[P], wv[P];
                ld_frame<T, V>(xb + (static_cast<int64_t>(r) * F + f) * C, xv);
                if constexpr (KTC > 0) {
#pragma unroll
                    for (int q = 0; q < P; ++q) wv[q] = wr[p * KFC + qq][q];
                } else {
                    load_param<V>(w + static_cast<int64_t>(p * KF + qq) * C + c, wv);
                }
#pragma unroll
                for (int q = 0; q < P; ++q) acc[q] = ffma2(xv[q], wv[q], acc[q]);
            }
        }
        Vec<T, V>::store(yr + static_cast<int64_t>(j) * C, acc);
    }
}

// Data gradient as a gather: input frame (t, f) collects every unmasked output whose window
// tap (p, q) lands on it.
template <typename T, int V, int KTC, int KFC>
__global__ void __launch_bounds__(kC2Threads)
dwconv2d_dx_kernel(const T *__restrict__ dy, const float *__restrict__ w, T *__restrict__ dx,
                   const int32_t *__restrict__ lengths, int B, int Tn, int F, int C, int KTr, int KFr, int st, int sf,
                   int pt, int pb, int pf, int To, int Fo, int nCV) {
    constexpr int P = Pairs<V>::n;
    const int KT = KTC > 0 ? KTC : KTr, KF = KFC > 0 ? KFC : KFr;
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<int64_t>(B) * Tn * nCV) return;
    const int cv = static_cast<int>(idx % nCV);
    const int64_t rest = idx / nCV;
    const int t = static_cast<int>(rest % Tn), b = static_cast<int>(rest / Tn);
    const int c = cv * V;
    const int L = static_cast<int>(clamp_len(lengths, b, Tn));
    int Lo = conv_len(L, pt, pb, KT, st);
    if (Lo > To) Lo = To;
    T *xr = dx + (static_cast<int64_t>(b) * Tn + t) * F * C + c;
    if (t >= L) {
        for (int f = 0; f < F; ++f) Vec<T, V>::store_zero(xr + static_cast<int64_t>(f) * C);
        return;
    }
    float2 wr[KTC > 0 ? KTC * KFC : 1][P];
    if constexpr (KTC > 0) {
#pragma unroll
        for (int q = 0; q < KTC * KFC; ++q) load_param<V>(w + static_cast<int64_t>(q) * C + c, wr[q]);
    }
    const T *gb = dy + static_cast<int64_t>(b) * To * Fo * C + c;
    for (int f = 0; f < F; ++f) {
        float2 acc[P];
#pragma unroll
        for (int q = 0; q < P; ++q) acc[q] = make_float2(0.f, 0.f);
#pragma unroll(KTC > 0 ? KTC : 1)
        for (int p = 0; p < KT; ++p) {
            const int u = t + pt - p;
            if (u < 0 || u % st != 0) continue;
            const int i = u / st;
            if (i >= Lo) continue;  // a masked (or absent) output row
#pragma unroll(KFC > 0 ? KFC : 1)
            for (int qq = 0; qq < KF; ++qq) {
                const int v = f + pf - qq;
                if (v < 0 || v % sf != 0) continue;
                const int j = v / sf;
                if (j >= Fo) continue;
                float2 gv[P], wv[P];
                ld_frame<T, V>(gb + (static_cast<int64_t>(i) * Fo + j) * C, gv);
                if constexpr (KTC > 0) {
#pragma unroll
                    for (int q = 0; q < P; ++q) wv[q] = wr[p * KFC + qq][q];
                } else {
                    load_param<V>(w + static_cast<int64_t>(p * KF + qq) * C + c, wv);
                }
#pragma unroll
                for (int q = 0; q < P; ++q) acc[q] = ffma2(gv[q], wv[q], acc[q]);
            }
        }
        Vec<T, V>::store(xr + static_cast<int64_t>(f) * C, acc);
    }
}

// Weight and bias gradient partials for taps [tap0, tap0 + kC2Taps): block g of channel group
// cgp walks output rows (b, i) g, g + G, ...; one partial row per block, [slot][C] with slots
// 0 .. KT*KF-1 the taps and KT*KF the bias.
template <typename T, bool VEC2>
__global__ void __launch_bounds__(kC2Threads)
dwconv2d_dw_kernel(const T *__restrict__ x, const T *__restrict__ dy, const int32_t *__restrict__ lengths,
                   float *__restrict__ partials, int B, int Tn, int F, int C, int KT, int KF, int st, int sf, int pt,
                   int pb, int pf, int To, int Fo, int nCG, int tap0, int with_bias) {
    const int cgp = blockIdx.x % nCG, g = blockIdx.x / nCG, G = gridDim.x / nCG;
    const int c = (cgp * kC2Threads + threadIdx.x) * 2;
    if (c >= C) return;
    const bool two = c + 1 < C;
    auto ld = [&](const T *p) -> float2 {
        if constexpr (VEC2) {  // C even and both activations aligned to a channel pair
            Vec<T, 2> v;
            v.load(p);
            float2 f[1];
            v.to_f2(f);
            return f[0];
        } else {
        Vec<T, 1> a;
        a.load(p);
        float2 fa[1];
        a.to_f2(fa);
        float yv = 0.f;
        if (two) {
            Vec<T, 1> bq;
            bq.load(p + 1);
            float2 fb[1];
            bq.to_f2(fb);
            yv = fb[0].x;
        }
        return make_float2(fa[0].x, yv);
        }
    };
    const int ntap = KT * KF;
    float2 acc[kC2Taps], accb = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < kC2Taps; ++k) acc[k] = make_float2(0.f, 0.f);
    const int64_t rows = static_cast<int64_t>(B) * To;
    for (int64_t row = g; row < rows; row += G) {
        const int b = static_cast<int>(row / To), i = static_cast<int>(row % To);
        const int L = static_cast<int>(clamp_len(lengths, b, Tn));
        int Lo = conv_len(L, pt, pb, KT, st);
        if (Lo > To) Lo = To;
        if (i >= Lo) continue;
        const T *gr = dy + (static_cast<int64_t>(b) * To + i) * Fo * C + c;
        const T *xb = x + static_cast<int64_t>(b) * Tn * F * C + c;
        for (int j = 0; j < Fo; ++j) {
            const float2 gv = ld(gr + static_cast<int64_t>(j) * C);
            if (with_bias) {
                accb.x += gv.x;
                accb.y += gv.y;
            }
#pragma unroll
            for (int k = 0; k < kC2Taps; ++k) {
                const int tap = tap0 + k;
                if (tap >= ntap) break;
                const int p = tap / KF, q = tap % KF;
                const int r = st * i + p - pt, f = sf * j + q - pf;
                if (r < 0 || r >= L || f < 0 || f >= F) continue;
                acc[k] = ffma2(gv, ld(xb + (static_cast<int64_t>(r) * F + f) * C), acc[k]);
            }
        }
    }
    float *row = partials + static_cast<int64_t>(g) * (ntap + 1) * C + c;
    auto put = [&](int slot, float2 v) {
        row[static_cast<int64_t>(slot) * C] = v.x;
        if (two) row[static_cast<int64_t>(slot) * C + 1] = v.y;
    };
#pragma unroll
    for (int k = 0; k < kC2Taps; ++k)
        if (tap0 + k < ntap) put(tap0 + k, acc[k]);
    if (with_bias) put(ntap, accb);
}

// dW / dbias = the partial rows summed in a fixed order (8 row groups, then a fixed tree).
__global__ void __launch_bounds__(256)
dwconv2d_dw_finalize_kernel(const float *__restrict__ partials, int G, int ntap, int C, float *__restrict__ dw,
                            float *__restrict__ dbias) {
    __shared__ float red[8][33];
    const int col = threadIdx.x % 32, rg = threadIdx.x / 32;
    const int64_t E = static_cast<int64_t>(ntap + 1) * C;
    const int64_t e = static_cast<int64_t>(blockIdx.x) * 32 + col;
    float s = 0.f;
    if (e < E)
        for (int r = rg; r < G; r += 8) s += __ldg(partials + static_cast<int64_t>(r) * E + e);
    red[rg][col] = s;
    __syncthreads();
    if (rg == 0 && e < E) {
        const float t = ((red[0][col] + red[1][col]) + (red[2][col] + red[3][col])) +
                        ((red[4][col] + red[5][col]) + (red[6][col] + red[7][col]));
        const int64_t slot = e / C, c = e % C;
        if (slot < ntap) dw[slot * C + c] = t;
        else if (dbias != nullptr) dbias[c] = t;
    }
}

__global__ void dwconv2d_out_lengths_kernel(const int32_t *__restrict__ lengths, int32_t *__restrict__ out_lengths,
                                            int B, int Tn, int KT, int st, int pt, int pb, int To) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= B) return;
    const int Lo = conv_len(static_cast<int>(clamp_len(lengths, b, Tn)), pt, pb, KT, st);
    out_lengths[b] = Lo < To ? Lo : To;
}

__global__ void dwconv2d_dw_zero_kernel(float *dw, float *dbias, int ntap, int C) {
    const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (e < static_cast<int64_t>(ntap) * C) dw[e] = 0.f;
    if (dbias != nullptr && e < C) dbias[e] = 0.f;
}

template <typename T, int V>
cudaError_t launch_fwd(const Conv2dArgs &a, cudaStream_t s) {
    const int nCV = static_cast<int>(a.C / V);
    const int64_t grid = (a.B * a.To * nCV + kC2Threads - 1) / kC2Threads;
    if (grid > kMaxGrid) return cudaErrorInvalidConfiguration;
#define DW_C2_ARGS                                                                                            \
    static_cast<const T *>(a.x), a.w, a.bias, static_cast<T *>(a.y), a.lengths, a.out_lengths,              \
        static_cast<int>(a.B), static_cast<int>(a.T), static_cast<int>(a.F), static_cast<int>(a.C), a.KT, a.KF, \
        a.st, a.sf, a.pt, a.pb, a.pf, static_cast<int>(a.To), static_cast<int>(a.Fo), nCV
    if (a.KT == 3 && a.KF == 3) dwconv2d_fwd_kernel<T, V, 3, 3><<<static_cast<unsigned>(grid), kC2Threads, 0, s>>>(DW_C2_ARGS);
    else dwconv2d_fwd_kernel<T, V, 0, 0><<<static_cast<unsigned>(grid), kC2Threads, 0, s>>>(DW_C2_ARGS);
#undef DW_C2_ARGS
    return cudaGetLastError();
}

template <typename T, int V>
cudaError_t launch_dx(const Conv2dArgs &a, cudaStream_t s) {
    const int nCV = static_cast<int>(a.C / V);
    const int64_t grid = (a.B * a.T * nCV + kC2Threads - 1) / kC2Threads;
    if (grid > kMaxGrid) return cudaErrorInvalidConfiguration;
#define DW_C2_ARGS                                                                                            \
    static_cast<const T *>(a.x), a.w, static_cast<T *>(a.y), a.lengths, static_cast<int>(a.B),              \
        static_cast<int>(a.T), static_cast<int>(a.F), static_cast<int>(a.C), a.KT, a.KF, a.st, a.sf, a.pt, a.pb, \
        a.pf, static_cast<int>(a.To), static_cast<int>(a.Fo), nCV
    if (a.KT == 3 && a.KF == 3) dwconv2d_dx_kernel<T, V, 3, 3><<<static_cast<unsigned>(grid), kC2Threads, 0, s>>>(DW_C2_ARGS);
    else dwconv2d_dx_kernel<T, V, 0, 0><<<static_cast<unsigned>(grid), kC2Threads, 0, s>>>(DW_C2_ARGS);
#undef DW_C2_ARGS
    return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch_vec(const Conv2dArgs &a, cudaStream_t s, bool dx) {
    switch (a.vec_width) {
        case 4: return dx ? launch_dx<T, 4>(a, s) : launch_fwd<T, 4>(a, s);
        case 2: return dx ? launch_dx<T, 2>(a, s) : launch_fwd<T, 2>(a, s);
        default: return dx ? launch_dx<T, 1>(a, s) : launch_fwd<T, 1>(a, s);
    }
}

}  // namespace

cudaError_t conv2d_fwd_launch(const Conv2dArgs &a, cudaStream_t s) {
    if (a.B == 0) return cudaSuccess;
    if (a.To == 0 || a.Fo == 0) {  // no output elements; the output lengths are still reported
        if (a.out_lengths == nullptr) return cudaSuccess;
        dwconv2d_out_lengths_kernel<<<static_cast<unsigned>((a.B + 127) / 128), 128, 0, s>>>(
            a.lengths, a.out_lengths, static_cast<int>(a.B), static_cast<int>(a.T), a.KT, a.st, a.pt, a.pb,
            static_cast<int>(a.To));
        return cudaGetLastError();
    }
    const cudaError_t e = conv2d_fwd_tma_launch(a, s);
    if (e != cudaErrorNotSupported) return e;
    return with_dtype(a.dtype, [&](auto tag) { return dispatch_vec<decltype(tag)>(a, s, false); });
}

cudaError_t conv2d_dx_launch(const Conv2dArgs &a, cudaStream_t s) {
    if (a.B == 0 || a.T == 0) return cudaSuccess;
    const cudaError_t e = conv2d_dx_tma_launch(a, s);
    if (e != cudaErrorNotSupported) return e;
    return with_dtype(a.dtype, [&](auto tag) { return dispatch_vec<decltype(tag)>(a, s, true); });
}

int conv2d_dw_partial_rows(int64_t B, int64_t To) {
    const int64_t rows = B * To;
    return static_cast<int>(rows < 1 ? 1 : (rows < kC2MaxRows ? rows : kC2MaxRows));
}

size_t conv2d_dw_workspace_bytes(int64_t B, int64_t To, int64_t C, int KT, int KF) {
    return static_cast<size_t>(conv2d_dw_partial_rows(B, To)) * (static_cast<size_t>(KT) * KF + 1) *
           static_cast<size_t>(C) * sizeof(float);
}

cudaError_t conv2d_dw_launch(const Conv2dArgs &a, float *dw, float *dbias, float *partials, cudaStream_t s) {
    const int ntap = a.KT * a.KF;
    if (a.B == 0 || a.To == 0 || a.Fo == 0) {
        dwconv2d_dw_zero_kernel<<<static_cast<unsigned>((static_cast<int64_t>(ntap) * a.C + 255) / 256), 256, 0, s>>>(
            dw, dbias, ntap, static_cast<int>(a.C));
        return cudaGetLastError();
    }
    const int64_t E = static_cast<int64_t>(ntap + 1) * a.C;
    {
        int Gt = 0;
        const cudaError_t e = conv2d_dw_tma_partials(a, partials, conv2d_dw_partial_rows(a.B, a.To), &Gt, s);
        if (e != cudaErrorNotSupported) {
            if (e != cudaSuccess) return e;
            // the same [rows][taps + 1][C] layout as the conv1d weight gradient
            return launch_finalize_rows(partials, dw, dbias, Gt, ntap, a.C, s);
        }
    }
    const int64_t nCG = (a.C + 2 * kC2Threads - 1) / (2 * kC2Threads);
    int G = conv2d_dw_partial_rows(a.B, a.To);
    const int64_t cap = (static_cast<int64_t>(sm_count()) * 8) / nCG;
    if (cap >= 1 && cap < G) G = static_cast<int>(cap);
    const int64_t grid = static_cast<int64_t>(G) * nCG;
    if (grid > kMaxGrid) return cudaErrorInvalidConfiguration;
    for (int tap0 = 0; tap0 < ntap; tap0 += kC2Taps) {
        const int wb = tap0 == 0 ? 1 : 0;
#define DW_C2_DW(TT, VV)                                                                                       \
    dwconv2d_dw_kernel<TT, VV><<<static_cast<unsigned>(grid), kC2Threads, 0, s>>>(                                 \
        static_cast<const TT *>(a.x), static_cast<const TT *>(a.y), a.lengths, partials, static_cast<int>(a.B),   \
        static_cast<int>(a.T), static_cast<int>(a.F), static_cast<int>(a.C), a.KT, a.KF, a.st, a.sf, a.pt, a.pb, \
        a.pf, static_cast<int>(a.To), static_cast<int>(a.Fo), static_cast<int>(nCG), tap0, wb)
        const bool v2 = a.vec_width >= 2;
        with_dtype(a.dtype, [&](auto tag) {
            using TT = decltype(tag);
            if (v2) DW_C2_DW(TT, true);
            else DW_C2_DW(TT, false);
            return 0;
        });
#undef DW_C2_DW
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    dwconv2d_dw_finalize_kernel<<<static_cast<unsigned>((E + 31) / 32), 256, 0, s>>>(partials, G, ntap,
                                                                                      static_cast<int>(a.C), dw, dbias);
    return cudaGetLastError();
}

}  // namespace dwk
