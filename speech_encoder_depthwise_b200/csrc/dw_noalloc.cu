// dwconv1d_bwd_dw_noalloc: the weight/bias gradient with its scratch memory inside the
// library, for callers that cannot allocate device memory.
//
// Who needs it: code embedded in a host application that owns every byte of device memory
// through its own allocator and gives plug-ins no allocation handle, and streaming loops that
// must not call cudaMalloc after start-up because an allocation can block on the whole
// device.  Such callers cannot provide the workspace that dwconv1d_bwd_dw takes.
//
// The scratch is a fixed-size array in device memory that belongs to the library: every GPU
// that loads the library holds it until the process exits.  All calls share it and it keeps
// the contents of the last call; the kernels overwrite every partial sum they later read, so
// nothing has to be cleared between calls.  Calls that overlap on the GPU (other streams,
// other host threads) race on the array and must be serialised by the caller.
#include <mutex>

#include "dw_internal.h"
#include "dwconv.h"

namespace {

constexpr size_t kScratchBytes = size_t(2) << 20;  // 2 MiB

static __device__ __align__(256) unsigned char g_dw_scratch[kScratchBytes];

// Device address of g_dw_scratch on the current device.  In host code the array's name is
// only a host-side stand-in, so the address is looked up with cudaGetSymbolAddress, once per
// device, with that device current.
cudaError_t scratch_address(void **out) {
    static std::mutex mu;
    static void *addr[64];
    static bool have[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!have[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_dw_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = p;
        have[dev] = true;
    }
    *out = addr[dev];
    return cudaSuccess;
}

bool aligned_to(const void *p, size_t n) { return p == nullptr || reinterpret_cast<uintptr_t>(p) % n == 0; }

}  // namespace

extern "C" dw_status_t dwconv1d_bwd_dw_noalloc(const void *x, const void *dy, float *dw, float *dbias,
                                               const int32_t *lengths, int64_t B, int64_t T, int64_t C, int K,
                                               int pad_left, dw_dtype_t io_dtype, dw_stream_t stream) {
    if (io_dtype != DW_F32 && io_dtype != DW_BF16 && io_dtype != DW_F16) return DW_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || C < 1 || K < 1 || pad_left < 0 || pad_left > K - 1) return DW_ERR_INVALID_ARG;
    if (C > (int64_t(1) << 22) || K > 4096) return DW_ERR_UNSUPPORTED;
    if (dw == nullptr) return DW_ERR_INVALID_ARG;
    const __int128 n = static_cast<__int128>(B) * T * C;
    if (n > static_cast<__int128>(INT64_MAX / 4)) return DW_ERR_INVALID_ARG;
    // one partial row [K+1][C] float32 must fit the scratch; larger sizes are rejected
    const size_t row_bytes = static_cast<size_t>(K + 1) * static_cast<size_t>(C) * sizeof(float);
    if (row_bytes > kScratchBytes) return DW_ERR_UNSUPPORTED;

    dwk::DwArgs a;
    a.x = x; a.dy = dy; a.dw = dw; a.dbias = dbias; a.lengths = lengths;
    a.B = B; a.T = T; a.C = C; a.K = K; a.pad_left = pad_left;
    a.dtype = static_cast<int>(io_dtype);
    a.partials = nullptr;
    a.G = 0;
    a.vec_width = 1;
    if (n > 0) {
        if (x == nullptr || dy == nullptr) return DW_ERR_INVALID_ARG;
        void *scratch = nullptr;
        const cudaError_t e = scratch_address(&scratch);
        if (e != cudaSuccess) return DW_ERR_CUDA;
        const int rows_fit = static_cast<int>(kScratchBytes / row_bytes);
        const int rows = dwk::conv1d_dw_partial_rows(B, T, C, K);
        a.partials = static_cast<float *>(scratch);
        a.G = rows < rows_fit ? rows : rows_fit;
        const size_t es = io_dtype == DW_F32 ? 4 : 2;
        for (int v : {4, 2}) {
            if (C % v == 0 && aligned_to(x, v * es) && aligned_to(dy, v * es)) {
                a.vec_width = v;
                break;
            }
        }
    }
    return dwk::conv1d_dw_launch(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? DW_OK : DW_ERR_CUDA;
}
