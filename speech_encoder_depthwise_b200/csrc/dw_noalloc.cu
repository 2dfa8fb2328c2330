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
//
// The argument checks are those of dwconv1d_bwd_dw (shared code), plus the scratch's limit.
#include <mutex>

#include "api_internal.h"

namespace {

constexpr size_t kScratchBytes = size_t(2) << 20;  // 2 MiB

static __device__ __align__(256) unsigned char g_dw_scratch[kScratchBytes];

// The driver's context queries, looked up once through the runtime (the library does not link
// the driver library); null where the driver does not provide them.
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

template <typename Fn>
Fn driver_entry(const char *name) {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &f, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<Fn>(f);
}

// Unique id of the calling thread's current context (ids are never reused within a process).
bool current_context_id(unsigned long long *id) {
    static const CtxGetCurrentFn get_current = driver_entry<CtxGetCurrentFn>("cuCtxGetCurrent");
    static const CtxGetIdFn get_id = driver_entry<CtxGetIdFn>("cuCtxGetId");
    CUcontext ctx = nullptr;
    if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr)
        return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_dw_scratch on the current device.  In host code the array's name is
// only a host-side stand-in, so the address is looked up with cudaGetSymbolAddress on the
// first call on each device, with that device current, and again whenever the device's
// context has changed since (after cudaDeviceReset the old address is no longer valid).
cudaError_t scratch_address(void **out) {
    static std::mutex mu;
    static void *addr[64];
    static unsigned long long ctx_of[64];
    static bool have[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    unsigned long long id = 0;
    bool known = current_context_id(&id);
    std::lock_guard<std::mutex> lock(mu);
    if (!(have[dev] && known && ctx_of[dev] == id)) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_dw_scratch);
        if (e != cudaSuccess) return e;
        if (!known) known = current_context_id(&id);  // the lookup may have created the context
        addr[dev] = p;
        ctx_of[dev] = id;
        have[dev] = known;  // without a context id the address is looked up again next time
    }
    *out = addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" dw_status_t dwconv1d_bwd_dw_noalloc(const void *x, const void *dy, float *dw, float *dbias,
                                               const int32_t *lengths, int64_t B, int64_t T, int64_t C, int K,
                                               int pad_left, dw_dtype_t io_dtype, dw_stream_t stream) {
    dwk::DwArgs a;
    int64_t n = 0;
    const dw_status_t st = dwapi::bwd_dw_prepare(x, dy, dw, dbias, lengths, B, T, C, K, pad_left, io_dtype, &a, &n);
    if (st != DW_OK) return st;
    // one partial row [K+1][C] float32 must fit the scratch; larger sizes are rejected
    const size_t row_bytes = static_cast<size_t>(K + 1) * static_cast<size_t>(C) * sizeof(float);
    if (row_bytes > kScratchBytes) return DW_ERR_UNSUPPORTED;
    if (n > 0) {
        void *scratch = nullptr;
        const cudaError_t e = scratch_address(&scratch);
        if (e != cudaSuccess) return dwapi::cuda_status(e);
        const int rows_fit = static_cast<int>(kScratchBytes / row_bytes);
        const int rows = dwk::conv1d_dw_partial_rows(B, T, C, K);
        a.partials = static_cast<float *>(scratch);
        a.G = rows < rows_fit ? rows : rows_fit;  // fewer partial rows than the workspace path: same sums, other order
    }
    return dwapi::cuda_status(dwk::conv1d_dw_launch(a, static_cast<cudaStream_t>(stream)));
}
