// Host-side helpers shared by the launchers: device properties, per-kernel attributes and
// tensor-map encoding for the bulk tensor copies.  No allocation, no synchronization.
#include <mutex>

#include "dw_internal.h"

namespace dwk {

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) return 148;
    return n;
}

// The limit only ever grows, and never below the 48 KiB default: a kernel launched with
// different amounts of shared memory keeps working for every size requested so far.
cudaError_t ensure_smem_attr(const void *kern, int bytes) {
    static std::mutex mu;
    static struct Entry { const void *k; int dev; int bytes; } done[256];
    static int n_done = 0;
    constexpr int kDefault = 48 * 1024;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const int want = bytes > kDefault ? bytes : kDefault;
    std::lock_guard<std::mutex> lock(mu);
    Entry *hit = nullptr;
    for (int i = 0; i < n_done; ++i)
        if (done[i].k == kern && done[i].dev == dev) hit = &done[i];
    if (hit != nullptr && hit->bytes >= want) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, want);
    if (e != cudaSuccess) return e;
    if (hit != nullptr) hit->bytes = want;
    else if (n_done < 256) done[n_done++] = {kern, dev, want};
    return cudaSuccess;
}

TensorMapEncodeTiledFn tensor_map_encoder() {
    static TensorMapEncodeTiledFn fn = []() -> TensorMapEncodeTiledFn {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<TensorMapEncodeTiledFn>(p);
    }();
    return fn;
}

cudaError_t make_act_map(CUtensorMap *map, const void *base, int dtype, int64_t B, int64_t T, int64_t C,
                         int box_c, int box_t) {
    TensorMapEncodeTiledFn enc = tensor_map_encoder();
    if (enc == nullptr) return cudaErrorNotSupported;
    const int64_t es = dtype_bytes(dtype);
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(C * es), static_cast<cuuint64_t>(T * C * es)};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_c), static_cast<cuuint32_t>(box_t), 1u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    const CUresult r = enc(map, tma_dtype(dtype), 3,
                           const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace dwk
