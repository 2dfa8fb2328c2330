// Streaming causal depthwise conv1d, one chunk, with a cache of each stream's K-1 most recent
// input frames (parakeet.cpp PR #102, "What changes": the streaming encoder keeps its own
// depthwise conv with a cache).
//
//   xcat_b      = [cache_b (K-1 frames) ; x_b frames 0 .. len_b-1]
//   y[b,t,c]    = [t < len_b] (bias[c] + sum_k xcat_b[t+k, c] w[k,c])
//   cache_b    <- xcat_b frames len_b .. len_b+K-2
//
// A chunk is small (one to a few dozen frames per stream), so this is a latency-bound op: one
// thread owns V channels of one stream for a segment of the chunk's frames, V chosen so that
// enough threads run.  With a compile-time K it slides a register window of K frames along time
// (every input frame is read once); other widths read the window from global memory.
#include "dw_internal.h"

namespace dwk {
namespace {

constexpr int kStreamThreads = 128;

template <typename T, int V>
__device__ __forceinline__ void load_frame(const T *p, float2 (&f)[Pairs<V>::n]) {
    Vec<T, V> v;
    v.load(p);
    v.to_f2(f);
}

// The cache is read and then rewritten by the same kernel, so it is read with plain (coherent)
// loads rather than through the read-only path.
template <typename T, int V>
__device__ __forceinline__ void load_cached(Vec<T, V> &v, const T *p) {
    v.r = *reinterpret_cast<const decltype(v.r) *>(p);
}
template <typename T, int V>
__device__ __forceinline__ void load_cached_frame(const T *p, float2 (&f)[Pairs<V>::n]) {
    Vec<T, V> v;
    load_cached<T, V>(v, p);
    v.to_f2(f);
}

// Thread layout: idx = ((b * nCV) + channel vector) * nSeg + segment; segment s covers frames
// [s S, s S + S).  S >= K - 1, so only segment 0 reads cached frames, and segment 0's thread
// alone rewrites the cache (after it has read every old cache frame): no other thread touches
// the cache, so the in-place update is race free.
struct StreamIdx {
    int b, c, t0, t1;
};
__device__ __forceinline__ bool stream_idx(int B, int Tn, int nCV, int V, int S, int nSeg, StreamIdx &r) {
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<int64_t>(B) * nCV * nSeg) return false;
    const int seg = static_cast<int>(idx % nSeg);
    const int64_t bc = idx / nSeg;
    r.b = static_cast<int>(bc / nCV);
    r.c = static_cast<int>(bc % nCV) * V;
    r.t0 = seg * S;
    r.t1 = r.t0 + S < Tn ? r.t0 + S : Tn;
    return true;
}

// Compile-time K: the window win[0..K-1] holds xcat frames t .. t+K-1 of this thread's channels.
template <typename T, int V, int K>
__global__ void __launch_bounds__(kStreamThreads)
conv1d_stream_kernel(const T *__restrict__ x, const float *__restrict__ w, const float *__restrict__ bias,
                     T *__restrict__ y, T *cache, const int32_t *__restrict__ lengths, int B, int Tn, int C,
                     int nCV, int S, int nSeg) {
    constexpr int H = K - 1;
    constexpr int P = Pairs<V>::n;
    launch_dependents();     // the next chunk's kernel may start its own set-up
    grid_dependency_wait();  // launched programmatically: the previous chunk's cache writes are visible after this
    StreamIdx r;
    if (!stream_idx(B, Tn, nCV, V, S, nSeg, r)) return;
    const int c = r.c;
    const int L = static_cast<int>(clamp_len(lengths, r.b, Tn));
    const T *xb = x + static_cast<int64_t>(r.b) * Tn * C + c;
    T *yb = y + static_cast<int64_t>(r.b) * Tn * C + c;
    T *cb = cache + static_cast<int64_t>(r.b) * H * C + c;
    const int tv = L < r.t1 ? L : r.t1;  // frames [t0, tv) of this segment are valid

    if (r.t0 < tv) {
        float2 wr[K][P], bv[P];
#pragma unroll
        for (int k = 0; k < K; ++k) load_param<V>(w + k * C + c, wr[k]);
        if (bias != nullptr) {
            load_param<V>(bias + c, bv);
        } else {
#pragma unroll
            for (int p = 0; p < P; ++p) bv[p] = make_float2(0.f, 0.f);
        }
        float2 win[K][P];
#pragma unroll
        for (int j = 0; j < H; ++j) {  // xcat frame t0 + j: cached, or chunk frame t0 + j - H (< L)
            const int f = r.t0 + j;
            if (f < H) load_cached_frame<T, V>(cb + f * C, win[j]);
            else load_frame<T, V>(xb + static_cast<int64_t>(f - H) * C, win[j]);
        }
        for (int t = r.t0; t < tv; ++t) {
            load_frame<T, V>(xb + static_cast<int64_t>(t) * C, win[H]);
            float2 acc[P];
#pragma unroll
            for (int p = 0; p < P; ++p) acc[p] = bv[p];
#pragma unroll
            for (int k = 0; k < K; ++k)
#pragma unroll
                for (int p = 0; p < P; ++p) acc[p] = ffma2(win[k][p], wr[k][p], acc[p]);
            Vec<T, V>::store(yb + static_cast<int64_t>(t) * C, acc);
#pragma unroll
            for (int j = 0; j < H; ++j)
#pragma unroll
                for (int p = 0; p < P; ++p) win[j][p] = win[j + 1][p];
        }
    }
    for (int t = tv > r.t0 ? tv : r.t0; t < r.t1; ++t) Vec<T, V>::store_zero(yb + static_cast<int64_t>(t) * C);
    // segment 0: new cache = xcat frames L .. L+H-1, gathered before any store
    if constexpr (H > 0) {
        if (r.t0 == 0) {
            Vec<T, V> nc[H];
#pragma unroll
            for (int i = 0; i < H; ++i) {
                if (L + i < H) load_cached<T, V>(nc[i], cb + (L + i) * C);
                else nc[i].load(xb + static_cast<int64_t>(L + i - H) * C);
            }
#pragma unroll
            for (int i = 0; i < H; ++i) {
                float2 f[P];
                nc[i].to_f2(f);
                Vec<T, V>::store(cb + i * C, f);
            }
        }
    }
}

// Any K: the window is read from global memory (cache frames, then the chunk's valid frames).
template <typename T, int V>
__global__ void __launch_bounds__(kStreamThreads)
conv1d_stream_anyk_kernel(const T *__restrict__ x, const float *__restrict__ w, const float *__restrict__ bias,
                          T *__restrict__ y, T *cache, const int32_t *__restrict__ lengths, int B, int Tn, int C,
                          int K, int nCV, int S, int nSeg) {
    constexpr int P = Pairs<V>::n;
    const int H = K - 1;
    launch_dependents();     // the next chunk's kernel may start its own set-up
    grid_dependency_wait();  // launched programmatically: the previous chunk's cache writes are visible after this
    StreamIdx r;
    if (!stream_idx(B, Tn, nCV, V, S, nSeg, r)) return;
    const int c = r.c;
    const int L = static_cast<int>(clamp_len(lengths, r.b, Tn));
    const T *xb = x + static_cast<int64_t>(r.b) * Tn * C + c;
    T *yb = y + static_cast<int64_t>(r.b) * Tn * C + c;
    T *cb = cache + static_cast<int64_t>(r.b) * H * C + c;
    float2 bv[P];
    if (bias != nullptr) {
        load_param<V>(bias + c, bv);
    } else {
#pragma unroll
        for (int p = 0; p < P; ++p) bv[p] = make_float2(0.f, 0.f);
    }
    for (int t = r.t0; t < r.t1; ++t) {
        if (t >= L) {
            Vec<T, V>::store_zero(yb + static_cast<int64_t>(t) * C);
            continue;
        }
        float2 acc[P];
#pragma unroll
        for (int p = 0; p < P; ++p) acc[p] = bv[p];
        for (int k = 0; k < K; ++k) {
            const int j = t + k;  // xcat frame; j - H <= t < L, so chunk frames here are valid
            float2 xv[P], wv[P];
            if (j < H) load_cached_frame<T, V>(cb + static_cast<int64_t>(j) * C, xv);
            else load_frame<T, V>(xb + static_cast<int64_t>(j - H) * C, xv);
            load_param<V>(w + static_cast<int64_t>(k) * C + c, wv);
#pragma unroll
            for (int p = 0; p < P; ++p) acc[p] = ffma2(xv[p], wv[p], acc[p]);
        }
        Vec<T, V>::store(yb + static_cast<int64_t>(t) * C, acc);
    }
    // segment 0: new cache in ascending order; frame i reads xcat frame L + i >= i, which no
    // earlier iteration has overwritten
    if (r.t0 == 0) {
        for (int i = 0; i < H; ++i) {
            float2 f[P];
            if (L + i < H) load_cached_frame<T, V>(cb + static_cast<int64_t>(L + i) * C, f);
            else load_frame<T, V>(xb + static_cast<int64_t>(L + i - H) * C, f);
            Vec<T, V>::store(cb + static_cast<int64_t>(i) * C, f);
        }
    }
}

template <typename T, int V>
cudaError_t launch_stream(const StreamArgs &a, cudaStream_t s) {
    const int nCV = static_cast<int>(a.C / V);
    // segments of at least K-1 frames (only segment 0 sees the cache), at least 8 frames each
    const int S = static_cast<int>(a.T <= 8 ? a.T : (a.K - 1 > 8 ? a.K - 1 : 8));
    const int nSeg = static_cast<int>((a.T + S - 1) / S);
    const int64_t threads = a.B * nCV * nSeg;
    const int64_t grid = (threads + kStreamThreads - 1) / kStreamThreads;
    if (grid > kMaxGrid) return cudaErrorInvalidConfiguration;
    const T *x = static_cast<const T *>(a.x);
    T *y = static_cast<T *>(a.y), *cache = static_cast<T *>(a.cache);
    const int B = static_cast<int>(a.B), Tn = static_cast<int>(a.T), C = static_cast<int>(a.C);
    const dim3 g3(static_cast<unsigned>(grid)), b3(kStreamThreads);
#define DW_STREAM_K(KK)                                                                                   \
    case KK:                                                                                              \
        return launch_programmatic(conv1d_stream_kernel<T, V, KK>, g3, b3, 0, s, x, a.w, a.bias, y, cache, \
                                   a.lengths, B, Tn, C, nCV, S, nSeg);
    switch (a.K) {
        DW_STREAM_K(1) DW_STREAM_K(2) DW_STREAM_K(3) DW_STREAM_K(4) DW_STREAM_K(5) DW_STREAM_K(7)
        DW_STREAM_K(9) DW_STREAM_K(15)
        default:
            return launch_programmatic(conv1d_stream_anyk_kernel<T, V>, g3, b3, 0, s, x, a.w, a.bias, y, cache,
                                       a.lengths, B, Tn, C, a.K, nCV, S, nSeg);
    }
#undef DW_STREAM_K
}

}  // namespace

cudaError_t conv1d_stream_launch(const StreamArgs &a, cudaStream_t s) {
    if (a.B == 0 || a.T == 0) return cudaSuccess;
    // A chunk is latency bound: take the widest channel vector that still gives about 64k
    // threads (every SM busy), never below 2 channels when the vector path is allowed.
    int v = a.vec_width;
    const int64_t segs = a.T <= 8 ? 1 : (a.T + 7) / 8;
    while (v > 2 && a.B * (a.C / v) * segs < (int64_t(1) << 16)) v /= 2;
    return with_dtype(a.dtype, [&](auto tag) {
        using T = decltype(tag);
        if constexpr (sizeof(T) == 2) {
            switch (v) {
                case 8: return launch_stream<T, 8>(a, s);
                case 4: return launch_stream<T, 4>(a, s);
                case 2: return launch_stream<T, 2>(a, s);
                default: return launch_stream<T, 1>(a, s);
            }
        } else {
            switch (v) {
                case 4: return launch_stream<T, 4>(a, s);
                case 2: return launch_stream<T, 2>(a, s);
                default: return launch_stream<T, 1>(a, s);
            }
        }
    });
}

}  // namespace dwk
