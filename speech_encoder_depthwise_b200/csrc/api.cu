// The C ABI (include/dwconv.h): argument validation on the host, then dispatch to the
// kernels.  Nothing here allocates, synchronizes or aborts.  Every argument check runs
// before the first CUDA call, so invalid calls return without touching the device.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "api_internal.h"

namespace dwk {
cudaError_t subsample_out_lengths_launch(const int32_t *lengths, int32_t *out_lengths, int64_t B, int64_t T,
                                         cudaStream_t s);
}

namespace {
thread_local int g_last_cuda_error = 0;
}  // namespace

namespace dwapi {
dw_status_t cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return DW_OK;
    g_last_cuda_error = static_cast<int>(e);
    return DW_ERR_CUDA;
}
}  // namespace dwapi

namespace {

using dwapi::cuda_status;

size_t dtype_size(dw_dtype_t t) { return t == DW_F32 ? 4 : 2; }

bool valid_dtype(dw_dtype_t t) { return t == DW_F32 || t == DW_BF16 || t == DW_F16; }

// n = a*b*c without overflow of int64 (all >= 0)
bool mul3(int64_t a, int64_t b, int64_t c, int64_t *n) {
    __int128 p = static_cast<__int128>(a) * b * c;
    if (p > static_cast<__int128>(INT64_MAX / 4)) return false;
    *n = static_cast<int64_t>(p);
    return true;
}

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
    return pa < pb + nb && pb < pa + na;
}

bool aligned(const void *p, size_t n) { return p == nullptr || reinterpret_cast<uintptr_t>(p) % n == 0; }

// Widest channel vector (4, 2 or 1 channels) that C and every pointer allow: activations
// aligned to the vector, float32 parameters to 8 bytes (they are read as float2).
int pick_vec_width(int64_t C, size_t esize, std::initializer_list<const void *> acts,
                   std::initializer_list<const void *> params) {
    for (const void *p : params)
        if (!aligned(p, 8)) return 1;
    for (int v : {4, 2}) {
        if (C % v != 0) continue;
        bool ok = true;
        for (const void *p : acts) ok = ok && aligned(p, v * esize);
        if (ok) return v;
    }
    return 1;
}

// Channel counts beyond this are rejected: frame offsets are kept in 32 bits inside a run.
constexpr int64_t kMaxChannels = 1 << 22;

dw_status_t check_conv1d_common(const void *in, const float *w, const void *out, int64_t B, int64_t T,
                                int64_t C, int K, int pad_left, dw_dtype_t dt, int64_t *n) {
    if (!valid_dtype(dt)) return DW_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || C < 1 || K < 1 || pad_left < 0 || pad_left > K - 1) return DW_ERR_INVALID_ARG;
    if (C > kMaxChannels || K > 4096) return DW_ERR_UNSUPPORTED;
    if (!mul3(B, T, C, n)) return DW_ERR_INVALID_ARG;
    if (*n == 0) return DW_OK;
    if (in == nullptr || w == nullptr || out == nullptr) return DW_ERR_INVALID_ARG;
    const size_t bytes = static_cast<size_t>(*n) * dtype_size(dt);
    if (overlaps(in, bytes, out, bytes)) return DW_ERR_INVALID_ARG;
    return DW_OK;
}

// Geometry of a depthwise conv2d: every size in range and the output sizes (To, Fo).  Bounds
// keep every frame index inside the kernels (stride i + tap - pad and the like) in 32 bits.
dw_status_t conv2d_geometry(int64_t B, int64_t T, int64_t F, int64_t C, int KT, int KF, int st, int sf, int pt,
                            int pb, int pf, int64_t *To, int64_t *Fo) {
    if (B < 0 || T < 0 || F < 1 || C < 1 || KT < 1 || KF < 1 || st < 1 || sf < 1 || pt < 0 || pb < 0 || pf < 0)
        return DW_ERR_INVALID_ARG;
    constexpr int64_t kLim = (int64_t(1) << 30);
    if (B >= kLim || T + pt + pb >= kLim || F + 2 * static_cast<int64_t>(pf) >= kLim || KT >= kLim ||
        KF >= kLim)
        return DW_ERR_INVALID_ARG;
    if (C > kMaxChannels) return DW_ERR_UNSUPPORTED;
    auto out = [](int64_t n, int64_t p0, int64_t p1, int64_t k, int64_t s) -> int64_t {
        const int64_t m = n + p0 + p1 - k;
        return m < 0 ? 0 : m / s + 1;
    };
    *To = out(T, pt, pb, KT, st);
    *Fo = out(F, pf, pf, KF, sf);
    int64_t n = 0;
    if (!mul3(B, T, F * C, &n) || !mul3(B, *To, *Fo * C, &n)) return DW_ERR_INVALID_ARG;
    return DW_OK;
}

dwk::Conv2dArgs conv2d_args(int64_t B, int64_t T, int64_t F, int64_t C, int64_t To, int64_t Fo, int KT, int KF,
                            int st, int sf, int pt, int pb, int pf, dw_dtype_t dt) {
    dwk::Conv2dArgs a;
    a.x = nullptr; a.w = nullptr; a.bias = nullptr; a.y = nullptr; a.lengths = nullptr; a.out_lengths = nullptr;
    a.B = B; a.T = T; a.F = F; a.C = C; a.To = To; a.Fo = Fo;
    a.KT = KT; a.KF = KF; a.st = st; a.sf = sf; a.pt = pt; a.pb = pb; a.pf = pf;
    a.dtype = static_cast<int>(dt);
    a.vec_width = 1;
    return a;
}

// Packed sequences: x/y [N][C], item b on rows offsets[b] .. offsets[b+1]-1.
dw_status_t packed_common(const void *in, const float *w, void *out, const int32_t *offsets, int64_t B, int64_t N,
                          int64_t C, int K, int pad_left, dw_dtype_t dt, dwk::Conv1dArgs *a) {
    int64_t n = 0;
    dw_status_t st = check_conv1d_common(in, w, out, 1, N, C, K, pad_left, dt, &n);
    if (st != DW_OK) return st;
    if (B < 0) return DW_ERR_INVALID_ARG;
    if (N >= (int64_t(1) << 30) || B >= (int64_t(1) << 30)) return DW_ERR_UNSUPPORTED;  // 32-bit row indices
    if (n > 0 && B > 0 && offsets == nullptr) return DW_ERR_INVALID_ARG;
    a->B = B; a->T = N; a->C = C; a->K = K;
    a->dtype = static_cast<int>(dt);
    a->lengths = nullptr;
    return DW_OK;
}

}  // namespace

namespace dwapi {
dw_status_t bwd_dw_prepare(const void *x, const void *dy, float *dw, float *dbias, const int32_t *lengths,
                           int64_t B, int64_t T, int64_t C, int K, int pad_left, dw_dtype_t io_dtype,
                           dwk::DwArgs *a, int64_t *n) {
    if (!valid_dtype(io_dtype)) return DW_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || C < 1 || K < 1 || pad_left < 0 || pad_left > K - 1) return DW_ERR_INVALID_ARG;
    if (C > kMaxChannels || K > 4096) return DW_ERR_UNSUPPORTED;
    if (!mul3(B, T, C, n)) return DW_ERR_INVALID_ARG;
    if (dw == nullptr) return DW_ERR_INVALID_ARG;
    if (static_cast<int64_t>(K + 1) * C > dwk::kMaxGrid * 256LL) return DW_ERR_INVALID_ARG;
    if (*n > 0 && (x == nullptr || dy == nullptr)) return DW_ERR_INVALID_ARG;
    a->x = x; a->dy = dy; a->dw = dw; a->dbias = dbias; a->lengths = lengths;
    a->B = B; a->T = T; a->C = C; a->K = K; a->pad_left = pad_left;
    a->dtype = static_cast<int>(io_dtype);
    a->partials = nullptr;
    a->G = 0;
    a->vec_width = *n > 0 ? pick_vec_width(C, dtype_size(io_dtype), {x, dy}, {}) : 1;
    return DW_OK;
}
}  // namespace dwapi

extern "C" {

const char *dw_status_string(dw_status_t s) {
    switch (s) {
        case DW_OK: return "DW_OK";
        case DW_ERR_INVALID_ARG: return "DW_ERR_INVALID_ARG: invalid argument";
        case DW_ERR_UNSUPPORTED: return "DW_ERR_UNSUPPORTED: request not supported by this build";
        case DW_ERR_WORKSPACE: return "DW_ERR_WORKSPACE: workspace missing or too small";
        case DW_ERR_CUDA: return "DW_ERR_CUDA: a CUDA call or kernel launch failed";
        case DW_ERR_TIMEOUT: return "DW_ERR_TIMEOUT: a device-side wait gave up";
    }
    return "unknown dw_status_t";
}

int dw_last_cuda_error(void) { return g_last_cuda_error; }

dw_status_t dw_selftest_wait_timeout(int *done, dw_stream_t stream) {
    if (done == nullptr) return DW_ERR_INVALID_ARG;
    return cuda_status(dwk::selftest_wait_timeout_launch(done, static_cast<cudaStream_t>(stream)));
}

dw_status_t dw_device_error(void) {
    if (cudaDeviceSynchronize() != cudaSuccess) return cuda_status(cudaGetLastError());
    const unsigned int e = dwk::conv1d_fwd_take_error() | dwk::conv1d_dw_take_error() | dwk::subsample_tc_take_error() |
                           dwk::conv2d_tma_take_error() | dwk::selftest_take_error();
    return e ? DW_ERR_TIMEOUT : DW_OK;
}

dw_status_t dwconv1d_fwd(const void *x, const float *w, const float *bias, void *y, const int32_t *lengths,
                         int64_t B, int64_t T, int64_t C, int K, int pad_left, dw_dtype_t io_dtype,
                         dw_stream_t stream) {
    int64_t n = 0;
    dw_status_t st = check_conv1d_common(x, w, y, B, T, C, K, pad_left, io_dtype, &n);
    if (st != DW_OK || n == 0) return st;
    dwk::Conv1dArgs a;
    a.x = x; a.w = w; a.bias = bias; a.y = y; a.lengths = lengths;
    a.B = B; a.T = T; a.C = C; a.K = K; a.pad_left = pad_left; a.flip = 0;
    a.dtype = static_cast<int>(io_dtype);
    a.vec_width = pick_vec_width(C, dtype_size(io_dtype), {x, y}, {w, bias});
    return cuda_status(dwk::conv1d_fwd_launch(a, static_cast<cudaStream_t>(stream)));
}

dw_status_t dwconv1d_bwd_dx(const void *dy, const float *w, void *dx, const int32_t *lengths, int64_t B,
                            int64_t T, int64_t C, int K, int pad_left, dw_dtype_t io_dtype, dw_stream_t stream) {
    int64_t n = 0;
    dw_status_t st = check_conv1d_common(dy, w, dx, B, T, C, K, pad_left, io_dtype, &n);
    if (st != DW_OK || n == 0) return st;
    dwk::Conv1dArgs a;
    a.x = dy; a.w = w; a.bias = nullptr; a.y = dx; a.lengths = lengths;
    a.B = B; a.T = T; a.C = C; a.K = K;
    a.pad_left = K - 1 - pad_left;  // correlation with reversed taps: the pads swap
    a.flip = 1;
    a.dtype = static_cast<int>(io_dtype);
    a.vec_width = pick_vec_width(C, dtype_size(io_dtype), {dy, dx}, {w});
    return cuda_status(dwk::conv1d_fwd_launch(a, static_cast<cudaStream_t>(stream)));
}

dw_status_t dwconv1d_bwd(const void *x, const void *dy, const float *w, void *dx, float *dw, float *dbias,
                         const int32_t *lengths, int64_t B, int64_t T, int64_t C, int K, int pad_left,
                         dw_dtype_t io_dtype, void *workspace, size_t workspace_bytes, dw_stream_t stream) {
    int64_t n = 0;
    dw_status_t st = check_conv1d_common(dy, w, dx, B, T, C, K, pad_left, io_dtype, &n);
    if (st != DW_OK) return st;
    if (n > 0) {
        if (x == nullptr) return DW_ERR_INVALID_ARG;
        const size_t bytes = static_cast<size_t>(n) * dtype_size(io_dtype);
        if (overlaps(dx, bytes, x, bytes)) return DW_ERR_INVALID_ARG;
    }
    // the weight-gradient entry validates the rest and serves the degenerate sizes
    if (n == 0)
        return dwconv1d_bwd_dw(x, dy, dw, dbias, lengths, B, T, C, K, pad_left, io_dtype, workspace,
                               workspace_bytes, stream);
    if (dw == nullptr) return DW_ERR_INVALID_ARG;
    const size_t need = dwk::conv1d_dw_workspace_bytes(B, T, C, K);
    if (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 16)) return DW_ERR_WORKSPACE;
    const size_t out_bytes = static_cast<size_t>(K) * C * sizeof(float);
    if (overlaps(workspace, need, dw, out_bytes) ||
        (dbias && overlaps(workspace, need, dbias, static_cast<size_t>(C) * sizeof(float))))
        return DW_ERR_INVALID_ARG;
    dwk::DwArgs a;
    a.x = x; a.dy = dy; a.dw = dw; a.dbias = dbias; a.lengths = lengths;
    a.B = B; a.T = T; a.C = C; a.K = K; a.pad_left = pad_left;
    a.dtype = static_cast<int>(io_dtype);
    a.partials = static_cast<float *>(workspace);
    a.G = dwk::conv1d_dw_partial_rows(B, T, C, K);
    a.vec_width = pick_vec_width(C, dtype_size(io_dtype), {x, dy, dx}, {w});
    a.w = w;
    a.dx = dx;
    const cudaError_t e = dwk::conv1d_bwd_fused_launch(a, static_cast<cudaStream_t>(stream));
    if (e != cudaErrorNotSupported) return cuda_status(e);
    // no fused instance for these sizes: the two gradients, one after the other
    st = dwconv1d_bwd_dx(dy, w, dx, lengths, B, T, C, K, pad_left, io_dtype, stream);
    if (st != DW_OK) return st;
    return dwconv1d_bwd_dw(x, dy, dw, dbias, lengths, B, T, C, K, pad_left, io_dtype, workspace, workspace_bytes,
                           stream);
}

dw_status_t dwconv1d_fwd_packed(const void *x, const float *w, const float *bias, void *y, const int32_t *offsets,
                                int64_t B, int64_t N, int64_t C, int K, int pad_left, dw_dtype_t io_dtype,
                                dw_stream_t stream) {
    dwk::Conv1dArgs a;
    dw_status_t st = packed_common(x, w, y, offsets, B, N, C, K, pad_left, io_dtype, &a);
    if (st != DW_OK || B == 0 || N == 0) return st;
    a.x = x; a.w = w; a.bias = bias; a.y = y; a.pad_left = pad_left; a.flip = 0;
    a.vec_width = pick_vec_width(C, dtype_size(io_dtype), {x, y}, {w, bias});
    return cuda_status(dwk::conv1d_fwd_packed_launch(a, offsets, static_cast<cudaStream_t>(stream)));
}

dw_status_t dwconv1d_bwd_dx_packed(const void *dy, const float *w, void *dx, const int32_t *offsets, int64_t B,
                                   int64_t N, int64_t C, int K, int pad_left, dw_dtype_t io_dtype,
                                   dw_stream_t stream) {
    dwk::Conv1dArgs a;
    dw_status_t st = packed_common(dy, w, dx, offsets, B, N, C, K, pad_left, io_dtype, &a);
    if (st != DW_OK || B == 0 || N == 0) return st;
    a.x = dy; a.w = w; a.bias = nullptr; a.y = dx;
    a.pad_left = K - 1 - pad_left;  // correlation with reversed taps: the pads swap
    a.flip = 1;
    a.vec_width = pick_vec_width(C, dtype_size(io_dtype), {dy, dx}, {w});
    return cuda_status(dwk::conv1d_fwd_packed_launch(a, offsets, static_cast<cudaStream_t>(stream)));
}

size_t dwconv1d_bwd_dw_packed_workspace_size(int64_t B, int64_t N, int64_t C, int K) {
    if (B < 0 || N < 0 || C < 1 || K < 1) return 0;
    int64_t n = 0;
    if (!mul3(1, N, C, &n)) return 0;
    return dwk::conv1d_dw_packed_workspace_bytes(N, C, K);
}

dw_status_t dwconv1d_bwd_dw_packed(const void *x, const void *dy, float *dw, float *dbias, const int32_t *offsets,
                                   int64_t B, int64_t N, int64_t C, int K, int pad_left, dw_dtype_t io_dtype,
                                   void *workspace, size_t workspace_bytes, dw_stream_t stream) {
    if (!valid_dtype(io_dtype)) return DW_ERR_INVALID_ARG;
    if (B < 0 || N < 0 || C < 1 || K < 1 || pad_left < 0 || pad_left > K - 1) return DW_ERR_INVALID_ARG;
    if (C > kMaxChannels || K > 4096) return DW_ERR_UNSUPPORTED;
    if (N >= (int64_t(1) << 30) || B >= (int64_t(1) << 30)) return DW_ERR_UNSUPPORTED;
    int64_t n = 0;
    if (!mul3(1, N, C, &n)) return DW_ERR_INVALID_ARG;
    if (dw == nullptr) return DW_ERR_INVALID_ARG;
    const size_t out_bytes = static_cast<size_t>(K) * C * sizeof(float), gb = static_cast<size_t>(C) * sizeof(float);
    if (dbias != nullptr && overlaps(dw, out_bytes, dbias, gb)) return DW_ERR_INVALID_ARG;
    dwk::DwArgs a;
    a.x = x; a.dy = dy; a.dw = dw; a.dbias = dbias; a.lengths = nullptr;
    a.B = B; a.T = N; a.C = C; a.K = K; a.pad_left = pad_left;
    a.dtype = static_cast<int>(io_dtype);
    a.partials = static_cast<float *>(workspace);
    a.G = 0;
    a.vec_width = 1;
    if (B > 0 && N > 0) {
        if (x == nullptr || dy == nullptr || offsets == nullptr) return DW_ERR_INVALID_ARG;
        const size_t need = dwk::conv1d_dw_packed_workspace_bytes(N, C, K);
        if (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 16)) return DW_ERR_WORKSPACE;
        if (overlaps(workspace, need, dw, out_bytes) || (dbias && overlaps(workspace, need, dbias, gb)))
            return DW_ERR_INVALID_ARG;
        a.vec_width = pick_vec_width(C, dtype_size(io_dtype), {x, dy}, {});
    } else {
        a.B = 0;  // no rows: the gradients are zeros
    }
    return cuda_status(dwk::conv1d_dw_packed_launch(a, offsets, static_cast<cudaStream_t>(stream)));
}

dw_status_t dwconv1d_stream_fwd(const void *x, const float *w, const float *bias, void *y, void *cache,
                                const int32_t *lengths, int64_t B, int64_t T, int64_t C, int K,
                                dw_dtype_t io_dtype, dw_stream_t stream) {
    int64_t n = 0;
    dw_status_t st = check_conv1d_common(x, w, y, B, T, C, K, K - 1, io_dtype, &n);
    if (st != DW_OK || n == 0) return st;
    const size_t es = dtype_size(io_dtype);
    const size_t cache_bytes = static_cast<size_t>(B) * static_cast<size_t>(K - 1) * static_cast<size_t>(C) * es;
    if (K > 1) {
        if (cache == nullptr) return DW_ERR_INVALID_ARG;
        const size_t bytes = static_cast<size_t>(n) * es;
        if (overlaps(cache, cache_bytes, x, bytes) || overlaps(cache, cache_bytes, y, bytes)) return DW_ERR_INVALID_ARG;
    }
    dwk::StreamArgs a;
    a.x = x; a.w = w; a.bias = bias; a.y = y; a.cache = cache; a.lengths = lengths;
    a.B = B; a.T = T; a.C = C; a.K = K;
    a.dtype = static_cast<int>(io_dtype);
    a.vec_width = pick_vec_width(C, es, {x, y, cache}, {w, bias});
    // bf16 rows of 8 channels move as one 16-byte word when everything lines up
    if (a.dtype != 0 && a.vec_width == 4 && C % 8 == 0 && aligned(x, 16) && aligned(y, 16) && aligned(cache, 16))
        a.vec_width = 8;
    return cuda_status(dwk::conv1d_stream_launch(a, static_cast<cudaStream_t>(stream)));
}

size_t dwconv1d_bwd_dw_workspace_size(int64_t B, int64_t T, int64_t C, int K) {
    if (B <= 0 || T <= 0 || C < 1 || K < 1) return 0;
    int64_t n = 0;
    if (!mul3(B, T, C, &n)) return 0;
    return dwk::conv1d_dw_workspace_bytes(B, T, C, K);
}


dw_status_t dwconv1d_bwd_dw(const void *x, const void *dy, float *dw, float *dbias, const int32_t *lengths,
                            int64_t B, int64_t T, int64_t C, int K, int pad_left, dw_dtype_t io_dtype,
                            void *workspace, size_t workspace_bytes, dw_stream_t stream) {
    dwk::DwArgs a;
    int64_t n = 0;
    const dw_status_t st = dwapi::bwd_dw_prepare(x, dy, dw, dbias, lengths, B, T, C, K, pad_left, io_dtype, &a, &n);
    if (st != DW_OK) return st;
    a.partials = static_cast<float *>(workspace);
    if (n > 0) {
        const size_t need = dwk::conv1d_dw_workspace_bytes(B, T, C, K);
        if (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 16)) return DW_ERR_WORKSPACE;
        const size_t out_bytes = static_cast<size_t>(K) * C * sizeof(float);
        if (overlaps(workspace, need, dw, out_bytes) ||
            (dbias && overlaps(workspace, need, dbias, static_cast<size_t>(C) * sizeof(float))))
            return DW_ERR_INVALID_ARG;
        a.G = dwk::conv1d_dw_partial_rows(B, T, C, K);
    }
    return cuda_status(dwk::conv1d_dw_launch(a, static_cast<cudaStream_t>(stream)));
}

size_t dw_subsample_bwd_workspace_size(int64_t B, int64_t T, int64_t F, int64_t C) {
    if (B < 0 || T < 0 || F < 1 || C < 1) return 0;
    int64_t n = 0;
    if (!mul3(B, T, F, &n) || !mul3(B, T, C, &n)) return 0;
    return dwk::subsample_bwd_workspace_bytes(B, T, F, C);
}

dw_status_t dw_subsample_bwd(const float *mel, const float *w0, const float *b0, const float *w1,
                             const void *dout, const int32_t *lengths, float *dw0, float *db0, float *dw1,
                             float *db1, int64_t B, int64_t T, int64_t F, int64_t C, int causal,
                             dw_dtype_t dout_dtype, void *workspace, size_t workspace_bytes, dw_stream_t stream) {
    if (!valid_dtype(dout_dtype)) return DW_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || F < 1 || C < 1 || (causal != 0 && causal != 1)) return DW_ERR_INVALID_ARG;
    if (C > kMaxChannels) return DW_ERR_UNSUPPORTED;
    int64_t n = 0;
    if (!mul3(B, T, F, &n)) return DW_ERR_INVALID_ARG;
    if (!dw0 || !db0 || !dw1 || !db1) return DW_ERR_INVALID_ARG;
    auto s2 = [](int64_t v) -> int64_t { return v >= 1 ? (v - 1) / 2 + 1 : 0; };
    const int64_t T4 = s2(s2(T)), F4 = s2(s2(F));
    int64_t nout = 0;
    if (!mul3(B, T4 * F4, C, &nout)) return DW_ERR_INVALID_ARG;
    dwk::SubsampleBwdArgs a;
    a.mel = mel; a.w0 = w0; a.b0 = b0; a.w1 = w1; a.dout = dout; a.lengths = lengths;
    a.dw0 = dw0; a.db0 = db0; a.dw1 = dw1; a.db1 = db1;
    a.partials = static_cast<float *>(workspace);
    a.B = B; a.T = T; a.F = F; a.C = C; a.causal = causal; a.dout_dtype = static_cast<int>(dout_dtype);
    if (nout > 0) {
        if (!mel || !w0 || !b0 || !w1 || !dout) return DW_ERR_INVALID_ARG;
        const size_t need = dwk::subsample_bwd_workspace_bytes(B, T, F, C);
        if (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 16)) return DW_ERR_WORKSPACE;
        const size_t g = static_cast<size_t>(9) * C * sizeof(float), gb = static_cast<size_t>(C) * sizeof(float);
        if (overlaps(workspace, need, dw0, g) || overlaps(workspace, need, dw1, g) ||
            overlaps(workspace, need, db0, gb) || overlaps(workspace, need, db1, gb))
            return DW_ERR_INVALID_ARG;
    }
    return cuda_status(dwk::subsample_bwd_launch(a, static_cast<cudaStream_t>(stream)));
}

dw_status_t dwconv2d_fwd(const void *x, const float *w, const float *bias, void *y, const int32_t *lengths,
                         int32_t *out_lengths, int64_t B, int64_t T, int64_t F, int64_t C, int KT, int KF,
                         int stride_t, int stride_f, int pad_t, int pad_b, int pad_f, dw_dtype_t io_dtype,
                         dw_stream_t stream) {
    if (!valid_dtype(io_dtype)) return DW_ERR_INVALID_ARG;
    int64_t To = 0, Fo = 0;
    dw_status_t st = conv2d_geometry(B, T, F, C, KT, KF, stride_t, stride_f, pad_t, pad_b, pad_f, &To, &Fo);
    if (st != DW_OK) return st;
    const int64_t nin = B * T * F * C, nout = B * To * Fo * C;
    if (nout == 0 && out_lengths == nullptr) return DW_OK;
    if (nout > 0) {
        if (x == nullptr || w == nullptr || y == nullptr) return DW_ERR_INVALID_ARG;
        const size_t es = dtype_size(io_dtype);
        if (overlaps(x, static_cast<size_t>(nin) * es, y, static_cast<size_t>(nout) * es)) return DW_ERR_INVALID_ARG;
    }
    if (B == 0) return DW_OK;
    dwk::Conv2dArgs a = conv2d_args(B, T, F, C, To, Fo, KT, KF, stride_t, stride_f, pad_t, pad_b, pad_f, io_dtype);
    a.x = x; a.w = w; a.bias = bias; a.y = y; a.lengths = lengths; a.out_lengths = out_lengths;
    a.vec_width = pick_vec_width(C, dtype_size(io_dtype), {x, y}, {w, bias});
    return cuda_status(dwk::conv2d_fwd_launch(a, static_cast<cudaStream_t>(stream)));
}

dw_status_t dwconv2d_bwd_dx(const void *dy, const float *w, void *dx, const int32_t *lengths, int64_t B,
                            int64_t T, int64_t F, int64_t C, int KT, int KF, int stride_t, int stride_f, int pad_t,
                            int pad_b, int pad_f, dw_dtype_t io_dtype, dw_stream_t stream) {
    if (!valid_dtype(io_dtype)) return DW_ERR_INVALID_ARG;
    int64_t To = 0, Fo = 0;
    dw_status_t st = conv2d_geometry(B, T, F, C, KT, KF, stride_t, stride_f, pad_t, pad_b, pad_f, &To, &Fo);
    if (st != DW_OK) return st;
    const int64_t nin = B * T * F * C, nout = B * To * Fo * C;
    if (nin == 0) return DW_OK;
    if (dx == nullptr || w == nullptr) return DW_ERR_INVALID_ARG;
    if (nout > 0) {
        if (dy == nullptr) return DW_ERR_INVALID_ARG;
        const size_t es = dtype_size(io_dtype);
        if (overlaps(dy, static_cast<size_t>(nout) * es, dx, static_cast<size_t>(nin) * es)) return DW_ERR_INVALID_ARG;
    }
    dwk::Conv2dArgs a = conv2d_args(B, T, F, C, To, Fo, KT, KF, stride_t, stride_f, pad_t, pad_b, pad_f, io_dtype);
    a.x = dy; a.w = w; a.y = dx; a.lengths = lengths;
    a.vec_width = pick_vec_width(C, dtype_size(io_dtype), {dy, dx}, {w});
    return cuda_status(dwk::conv2d_dx_launch(a, static_cast<cudaStream_t>(stream)));
}

size_t dwconv2d_bwd_dw_workspace_size(int64_t B, int64_t T, int64_t F, int64_t C, int KT, int KF, int stride_t,
                                      int stride_f, int pad_t, int pad_b, int pad_f) {
    int64_t To = 0, Fo = 0;
    if (conv2d_geometry(B, T, F, C, KT, KF, stride_t, stride_f, pad_t, pad_b, pad_f, &To, &Fo) != DW_OK) return 0;
    return dwk::conv2d_dw_workspace_bytes(B, To, C, KT, KF);
}

dw_status_t dwconv2d_bwd_dw(const void *x, const void *dy, float *dw, float *dbias, const int32_t *lengths,
                            int64_t B, int64_t T, int64_t F, int64_t C, int KT, int KF, int stride_t, int stride_f,
                            int pad_t, int pad_b, int pad_f, dw_dtype_t io_dtype, void *workspace,
                            size_t workspace_bytes, dw_stream_t stream) {
    if (!valid_dtype(io_dtype)) return DW_ERR_INVALID_ARG;
    int64_t To = 0, Fo = 0;
    dw_status_t st = conv2d_geometry(B, T, F, C, KT, KF, stride_t, stride_f, pad_t, pad_b, pad_f, &To, &Fo);
    if (st != DW_OK) return st;
    if (dw == nullptr) return DW_ERR_INVALID_ARG;
    const int64_t ntap = static_cast<int64_t>(KT) * KF;
    if ((ntap + 1) * C > dwk::kMaxGrid * 32LL) return DW_ERR_INVALID_ARG;
    const size_t out_bytes = static_cast<size_t>(ntap) * C * sizeof(float), gb = static_cast<size_t>(C) * sizeof(float);
    if (dbias != nullptr && overlaps(dw, out_bytes, dbias, gb)) return DW_ERR_INVALID_ARG;
    dwk::Conv2dArgs a = conv2d_args(B, T, F, C, To, Fo, KT, KF, stride_t, stride_f, pad_t, pad_b, pad_f, io_dtype);
    a.x = x; a.y = const_cast<void *>(dy); a.lengths = lengths;
    float *partials = nullptr;
    if (B * To * Fo > 0) {
        if (x == nullptr || dy == nullptr) return DW_ERR_INVALID_ARG;
        const size_t need = dwk::conv2d_dw_workspace_bytes(B, To, C, KT, KF);
        if (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 16)) return DW_ERR_WORKSPACE;
        if (overlaps(workspace, need, dw, out_bytes) || (dbias && overlaps(workspace, need, dbias, gb)))
            return DW_ERR_INVALID_ARG;
        partials = static_cast<float *>(workspace);
        const size_t es = dtype_size(io_dtype);
        a.vec_width = (C % 2 == 0 && aligned(x, 2 * es) && aligned(dy, 2 * es)) ? 2 : 1;
    }
    return cuda_status(dwk::conv2d_dw_launch(a, dw, dbias, partials, static_cast<cudaStream_t>(stream)));
}

namespace {

dw_status_t subsample_fwd(const float *mel, const float *w0, const float *b0, const float *w1, const float *b1,
                          void *out, const int32_t *lengths, int32_t *out_lengths, int64_t B, int64_t T, int64_t F,
                          int64_t C, int causal, dw_dtype_t out_dtype, bool tensor_cores, cudaStream_t s) {
    if (!valid_dtype(out_dtype)) return DW_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || F < 1 || C < 1 || (causal != 0 && causal != 1)) return DW_ERR_INVALID_ARG;
    int64_t n = 0;
    if (!mul3(B, T, F, &n)) return DW_ERR_INVALID_ARG;
    auto s2 = [](int64_t v) -> int64_t { return v >= 1 ? (v - 1) / 2 + 1 : 0; };
    const int64_t T4 = s2(s2(T)), F4 = s2(s2(F));
    int64_t nout = 0;
    if (!mul3(B, T4 * F4, C, &nout)) return DW_ERR_INVALID_ARG;
    if (out_lengths == nullptr && nout == 0) return DW_OK;
    if (nout > 0) {
        if (!mel || !w0 || !b0 || !w1 || !b1 || !out) return DW_ERR_INVALID_ARG;
        if (overlaps(mel, static_cast<size_t>(n) * 4, out, static_cast<size_t>(nout) * dtype_size(out_dtype)))
            return DW_ERR_INVALID_ARG;
    }
    if (nout > 0) {  // the fused kernel also writes out_lengths
        dwk::SubsampleArgs a;
        a.mel = mel; a.w0 = w0; a.b0 = b0; a.w1 = w1; a.b1 = b1; a.out = out;
        a.lengths = lengths; a.out_lengths = out_lengths;
        a.B = B; a.T = T; a.F = F; a.C = C; a.causal = causal; a.out_dtype = static_cast<int>(out_dtype);
        return cuda_status(dwk::subsample_launch(a, tensor_cores, s));
    }
    if (out_lengths != nullptr && B > 0)  // no frames: only the (zero) output lengths
        return cuda_status(dwk::subsample_out_lengths_launch(lengths, out_lengths, B, T, s));
    return DW_OK;
}

}  // namespace

dw_status_t dw_subsample_fwd(const float *mel, const float *w0, const float *b0, const float *w1,
                             const float *b1, void *out, const int32_t *lengths, int32_t *out_lengths,
                             int64_t B, int64_t T, int64_t F, int64_t C, int causal, dw_dtype_t out_dtype,
                             dw_stream_t stream) {
    return subsample_fwd(mel, w0, b0, w1, b1, out, lengths, out_lengths, B, T, F, C, causal, out_dtype, true,
                         static_cast<cudaStream_t>(stream));
}

dw_status_t dw_subsample_fwd_simt(const float *mel, const float *w0, const float *b0, const float *w1,
                                  const float *b1, void *out, const int32_t *lengths, int32_t *out_lengths,
                                  int64_t B, int64_t T, int64_t F, int64_t C, int causal, dw_dtype_t out_dtype,
                                  dw_stream_t stream) {
    return subsample_fwd(mel, w0, b0, w1, b1, out, lengths, out_lengths, B, T, F, C, causal, out_dtype, false,
                         static_cast<cudaStream_t>(stream));
}

}  // extern "C"
