// Depthwise conv1d over time, forward and data gradient, channels-last [B][T][C].
//
//   y[b,t,c] = [t < len_b] * (bias[c] + sum_{k<K} xpad[b,t+k,c] * w[k,c])
//
// The SSM_CONV form of the depthwise conv over the input padded to T + K - 1 frames
// (parakeet.cpp PR #102, "faster GPU decode: one SSM_CONV for the depthwise conv",
// section "What changes"), with the pre/post masking and causal padding fused into the
// kernel as NeMo PR #16114 does ("Use Fused Kernels for Depthwise Striding Subsampler",
// section "What does this PR do ?", second kernel).
//
// The data gradient is the same correlation with the taps reversed (w[K-1-k]), the pads
// swapped (pad_left' = K-1-pad_left) and no bias; the masks are the same.  `flip` selects
// the reversed taps when the weights are loaded, so one engine serves both.
//
// Design (HBM-bound: ~2 B read + 2 B written per bf16 output, K FMAs):
//  - a thread owns V consecutive channels (a pair when C is even and the pointers allow it,
//    else one) and R consecutive frames; lanes run along C, so each warp load/store of bf16
//    pairs covers 128 contiguous bytes;
//  - it loads the R + K - 1 input frames it needs once, as raw words, into registers, and
//    accumulates in float32 pairs with packed FMA (fma.rn.f32x2): each input is unpacked once
//    and scattered into the K outputs it feeds;
//  - the K - 1 halo frames shared with the neighbouring frame run are re-read by the
//    neighbour warp and hit L1/L2, so DRAM sees each input frame about once;
//  - input frames at or beyond len_b are never loaded (predicated off), and a run that lies
//    wholly beyond len_b only stores zeros.
#include "dw_internal.h"

namespace dwk {

template <typename T, int V, int K, int R>
__global__ void __launch_bounds__(256)
conv1d_fwd_vec_kernel(const T *__restrict__ x, const float *__restrict__ w,
                      const float *__restrict__ bias, T *__restrict__ y,
                      const int32_t *__restrict__ lengths, int64_t Tn, int64_t C, int pad_left,
                      int flip, int TX, int nT, int nC) {
    constexpr int NP = Pairs<V>::n;
    const int tx = threadIdx.x % TX, ty = threadIdx.x / TX;
    const int TY = blockDim.x / TX;
    int64_t lin = blockIdx.x;
    const int ct = static_cast<int>(lin % nC);
    lin /= nC;
    const int tt = static_cast<int>(lin % nT);
    const int64_t b = lin / nT;
    const int64_t c0 = (static_cast<int64_t>(ct) * TX + tx) * V;
    if (c0 >= C) return;
    const int64_t t0 = (static_cast<int64_t>(tt) * TY + ty) * R;
    if (t0 >= Tn) return;
    const int64_t L = clamp_len(lengths, b, Tn);
    const T *xb = x + b * Tn * C + c0;
    T *yb = y + b * Tn * C + c0;

    if (t0 >= L) {  // the whole run is masked: zeros only, nothing read
#pragma unroll
        for (int r = 0; r < R; ++r)
            if (t0 + r < Tn) Vec<T, V>::store_zero(yb + (t0 + r) * C);
        return;
    }

    Vec<T, V> raw[R + K - 1];
#pragma unroll
    for (int i = 0; i < R + K - 1; ++i) {
        const int64_t j = t0 - pad_left + i;
        if (j >= 0 && j < L) raw[i].load(xb + j * C);
        else raw[i].zero();
    }

    float2 wv[K][NP];
#pragma unroll
    for (int k = 0; k < K; ++k) load_param<V>(w + static_cast<int64_t>(flip ? K - 1 - k : k) * C + c0, wv[k]);
    float2 acc[R][NP];
    {
        float2 bv[NP];
        if (bias) load_param<V>(bias + c0, bv);
        else {
#pragma unroll
            for (int p = 0; p < NP; ++p) bv[p] = make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int p = 0; p < NP; ++p) acc[r][p] = bv[p];
    }

    // input frame i feeds output r = i - k through tap k
#pragma unroll
    for (int i = 0; i < R + K - 1; ++i) {
        float2 xf[NP];
        raw[i].to_f2(xf);
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const int r = i - k;
            if (r >= 0 && r < R) {
#pragma unroll
                for (int p = 0; p < NP; ++p) acc[r][p] = ffma2(xf[p], wv[k][p], acc[r][p]);
            }
        }
        // output r = i - (K-1) has received its last term
        const int rd = i - (K - 1);
        if (rd >= 0) {
            const int64_t t = t0 + rd;
            if (t < Tn) {
                if (t < L) Vec<T, V>::store(yb + t * C, acc[rd]);
                else Vec<T, V>::store_zero(yb + t * C);
            }
        }
    }
}

// Any K, any vector width: taps in a runtime loop; each output re-reads its inputs
// (served from L1).  The general fallback for widths without a specialisation.
template <typename T, int V, int R>
__global__ void __launch_bounds__(256)
conv1d_fwd_vec_anyk_kernel(const T *__restrict__ x, const float *__restrict__ w,
                           const float *__restrict__ bias, T *__restrict__ y,
                           const int32_t *__restrict__ lengths, int64_t Tn, int64_t C, int K,
                           int pad_left, int flip, int TX, int nT, int nC) {
    constexpr int NP = Pairs<V>::n;
    const int tx = threadIdx.x % TX, ty = threadIdx.x / TX;
    const int TY = blockDim.x / TX;
    int64_t lin = blockIdx.x;
    const int ct = static_cast<int>(lin % nC);
    lin /= nC;
    const int tt = static_cast<int>(lin % nT);
    const int64_t b = lin / nT;
    const int64_t c0 = (static_cast<int64_t>(ct) * TX + tx) * V;
    if (c0 >= C) return;
    const int64_t t0 = (static_cast<int64_t>(tt) * TY + ty) * R;
    if (t0 >= Tn) return;
    const int64_t L = clamp_len(lengths, b, Tn);
    const T *xb = x + b * Tn * C + c0;
    T *yb = y + b * Tn * C + c0;
    if (t0 >= L) {
#pragma unroll
        for (int r = 0; r < R; ++r)
            if (t0 + r < Tn) Vec<T, V>::store_zero(yb + (t0 + r) * C);
        return;
    }
    float2 acc[R][NP];
    {
        float2 bv[NP];
        if (bias) load_param<V>(bias + c0, bv);
        else {
#pragma unroll
            for (int p = 0; p < NP; ++p) bv[p] = make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int p = 0; p < NP; ++p) acc[r][p] = bv[p];
    }
    for (int k = 0; k < K; ++k) {
        float2 wk[NP];
        load_param<V>(w + static_cast<int64_t>(flip ? K - 1 - k : k) * C + c0, wk);
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int64_t j = t0 + r + k - pad_left;
            if (j >= 0 && j < L) {
                Vec<T, V> v;
                v.load(xb + j * C);
                float2 xf[NP];
                v.to_f2(xf);
#pragma unroll
                for (int p = 0; p < NP; ++p) acc[r][p] = ffma2(xf[p], wk[p], acc[r][p]);
            }
        }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int64_t t = t0 + r;
        if (t < Tn) {
            if (t < L) Vec<T, V>::store(yb + t * C, acc[r]);
            else Vec<T, V>::store_zero(yb + t * C);
        }
    }
}

namespace {

constexpr int kThreads = 256;

int pow2_at_most(int64_t v, int cap) {
    int p = 1;
    while (p < cap && p < v) p <<= 1;
    return p;
}

template <typename T, int V, int K>
cudaError_t launch_vec_k(const Conv1dArgs &a, cudaStream_t s) {
    constexpr int R = (K <= 9) ? 16 : 8;
    const int64_t Cv = (a.C + V - 1) / V;
    const int TX = pow2_at_most(Cv, 32);
    const int TY = kThreads / TX;
    const int nC = static_cast<int>((Cv + TX - 1) / TX);
    const int nT = static_cast<int>((a.T + static_cast<int64_t>(TY) * R - 1) / (static_cast<int64_t>(TY) * R));
    const int64_t grid = a.B * nT * static_cast<int64_t>(nC);
    if (grid > kMaxGrid) return cudaErrorInvalidConfiguration;
    conv1d_fwd_vec_kernel<T, V, K, R><<<static_cast<unsigned>(grid), kThreads, 0, s>>>(
        static_cast<const T *>(a.x), a.w, a.bias, static_cast<T *>(a.y), a.lengths, a.T, a.C,
        a.pad_left, a.flip, TX, nT, nC);
    return cudaGetLastError();
}

template <typename T, int V>
cudaError_t launch_vec_anyk(const Conv1dArgs &a, cudaStream_t s) {
    constexpr int R = 8;
    const int64_t Cv = (a.C + V - 1) / V;
    const int TX = pow2_at_most(Cv, 32);
    const int TY = kThreads / TX;
    const int nC = static_cast<int>((Cv + TX - 1) / TX);
    const int nT = static_cast<int>((a.T + static_cast<int64_t>(TY) * R - 1) / (static_cast<int64_t>(TY) * R));
    const int64_t grid = a.B * nT * static_cast<int64_t>(nC);
    if (grid > kMaxGrid) return cudaErrorInvalidConfiguration;
    conv1d_fwd_vec_anyk_kernel<T, V, R><<<static_cast<unsigned>(grid), kThreads, 0, s>>>(
        static_cast<const T *>(a.x), a.w, a.bias, static_cast<T *>(a.y), a.lengths, a.T, a.C, a.K,
        a.pad_left, a.flip, TX, nT, nC);
    return cudaGetLastError();
}

template <typename T, int V>
cudaError_t dispatch_k(const Conv1dArgs &a, cudaStream_t s) {
    switch (a.K) {
        case 1: return launch_vec_k<T, V, 1>(a, s);
        case 2: return launch_vec_k<T, V, 2>(a, s);
        case 3: return launch_vec_k<T, V, 3>(a, s);
        case 4: return launch_vec_k<T, V, 4>(a, s);
        case 5: return launch_vec_k<T, V, 5>(a, s);
        case 7: return launch_vec_k<T, V, 7>(a, s);
        case 9: return launch_vec_k<T, V, 9>(a, s);
        case 15: return launch_vec_k<T, V, 15>(a, s);
        case 31: return launch_vec_k<T, V, 31>(a, s);
        default: return launch_vec_anyk<T, V>(a, s);
    }
}

template <typename T>
cudaError_t dispatch_dtype(const Conv1dArgs &a, cudaStream_t s) {
    if (a.vec_width >= 2) return dispatch_k<T, 2>(a, s);
    return dispatch_k<T, 1>(a, s);
}

}  // namespace

cudaError_t conv1d_fwd_launch(const Conv1dArgs &a, cudaStream_t s) {
    if (a.B == 0 || a.T == 0) return cudaSuccess;
    if (a.bf16) return dispatch_dtype<bf16>(a, s);
    return dispatch_dtype<float>(a, s);
}

}  // namespace dwk
