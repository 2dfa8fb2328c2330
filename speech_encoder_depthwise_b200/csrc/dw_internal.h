// Internal launch interface between the C ABI layer (api.cu) and the kernels.
// Arguments arrive here already validated; launchers only pick a kernel and launch it.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <type_traits>

#include "dw_common.cuh"

namespace dwk {

constexpr int64_t kMaxGrid = 0x7fffffffLL;

struct Conv1dArgs {
    const void *x;        // input [B][T][C] (dy for the data gradient)
    const float *w;       // [K][C]
    const float *bias;    // [C] or null
    void *y;              // output [B][T][C]
    const int32_t *lengths;
    int64_t B, T, C;
    int K;
    int pad_left;         // left pad of THIS correlation (already swapped for the data gradient)
    int flip;             // 1: use w[K-1-k] as tap k
    int dtype;            // I/O element type: 0 float32, 1 bf16, 2 fp16
    int vec_width;        // 2: even-channel vector path allowed; 1: scalar path
};

struct DwArgs {
    const void *x, *dy;
    float *dw, *dbias;
    const int32_t *lengths;
    int64_t B, T, C;
    int K, pad_left, dtype, vec_width;  // dtype: 0 float32, 1 bf16, 2 fp16
    float *partials;      // workspace: [G][K+1][C] float32
    int G;                // partial rows (blocks per channel tile)
    const float *w = nullptr;  // [K][C]: taps of the data gradient (fused backward only)
    void *dx = nullptr;        // [B][T][C]: data gradient (fused backward only)
};

struct StreamArgs {
    const void *x;        // chunk [B][T][C]
    const float *w;       // [K][C]
    const float *bias;    // [C] or null
    void *y;              // [B][T][C]
    void *cache;          // [B][K-1][C], read and rewritten
    const int32_t *lengths;
    int64_t B, T, C;
    int K, dtype, vec_width;  // dtype: 0 float32, 1 bf16, 2 fp16; vec_width: 8 (16-bit types only), 4, 2 or 1
};

struct SubsampleArgs {
    const float *mel, *w0, *b0, *w1, *b1;
    void *out;
    const int32_t *lengths;
    int32_t *out_lengths;
    int64_t B, T, F, C;
    int causal, out_dtype;  // out_dtype: 0 float32, 1 bf16, 2 fp16
};

// General depthwise conv2d, channels-last [B][T][F][C], taps [KT][KF][C].  The data gradient
// takes dy as x and writes dx through y; the weight gradient takes x and dy (as y).
struct Conv2dArgs {
    const void *x;
    const float *w;           // [KT][KF][C] (forward and data gradient)
    const float *bias;        // [C] or null (forward)
    void *y;
    const int32_t *lengths;
    int32_t *out_lengths;     // [B] or null (forward)
    int64_t B, T, F, C, To, Fo;
    int KT, KF, st, sf, pt, pb, pf;
    int dtype, vec_width;     // dtype: 0 float32, 1 bf16, 2 fp16; vec_width: 4, 2 or 1 channels per thread
};

// Raise a kernel's dynamic shared memory limit to `bytes`, once per (kernel, device).
cudaError_t ensure_smem_attr(const void *kern, int bytes);

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime (no link
// against the driver library); null if unavailable.
typedef CUresult (*TensorMapEncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                           const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                           const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                           CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
TensorMapEncodeTiledFn tensor_map_encoder();

// dtype code of an element type (0 float32, 1 bf16, 2 fp16) and the matching tensor-map type.
template <typename T> constexpr int dtype_code() { return sizeof(T) == 4 ? 0 : (std::is_same<T, bf16>::value ? 1 : 2); }
inline CUtensorMapDataType tma_dtype(int dtype) {
    return dtype == 1 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                      : (dtype == 2 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32);
}
inline int dtype_bytes(int dtype) { return dtype == 0 ? 4 : 2; }

// Tensor map over a channels-last [B][T][C] activation (dims innermost first: C, T, B) with
// a box of box_c channels x box_t frames x 1 item; out-of-range elements read as zero.
cudaError_t make_act_map(CUtensorMap *map, const void *base, int dtype, int64_t B, int64_t T, int64_t C,
                         int box_c, int box_t);

int sm_count();

// Launch with programmatic stream serialization: the kernel may start while the previous one in
// the stream drains, and must call grid_dependency_wait before touching memory that one writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_programmatic(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Args &&>(args)...);
}

cudaError_t conv1d_fwd_launch(const Conv1dArgs &a, cudaStream_t s);
// Packed sequences: a.B items, a.T = N rows of x/y [N][C], item b on rows offsets[b] .. offsets[b+1]-1.
cudaError_t conv1d_fwd_packed_launch(const Conv1dArgs &a, const int32_t *offsets, cudaStream_t s);
// Reads and clears the device error word of the conv1d forward kernels (synchronous).
unsigned int conv1d_fwd_take_error();

// dW/dbias: the number of partial rows G and the workspace bytes follow from the sizes alone.
int conv1d_dw_partial_rows(int64_t B, int64_t T, int64_t C, int K);
size_t conv1d_dw_workspace_bytes(int64_t B, int64_t T, int64_t C, int K);
cudaError_t conv1d_dw_launch(const DwArgs &a, cudaStream_t s);
// Packed batches (a.T = N rows, a.B items on rows offsets[b] .. offsets[b+1]-1): partial rows
// [rows][K+1][C] in a.partials, then the fixed-order finalize.
int conv1d_dw_packed_rows(int64_t N);
size_t conv1d_dw_packed_workspace_bytes(int64_t N, int64_t C, int K);
cudaError_t conv1d_dw_packed_launch(const DwArgs &a, const int32_t *offsets, cudaStream_t s);
// dx and dW/dbias in one pass over dy; cudaErrorNotSupported when no fused instance fits.
cudaError_t conv1d_bwd_fused_launch(const DwArgs &a, cudaStream_t s);
// dW / dbias = partial rows [Gp][K+1][C] (slots 0..K-1 the taps, slot K the bias) summed in a
// fixed order; launched programmatically after the kernel that wrote them.
cudaError_t launch_finalize_rows(const float *partials, float *dw, float *dbias, int Gp, int K, int64_t C,
                                 cudaStream_t s);
unsigned int conv1d_dw_take_error();

cudaError_t conv1d_stream_launch(const StreamArgs &a, cudaStream_t s);

// tensor_cores: the tcgen05 kernel where eligible; false keeps every size on the FP32 SIMT kernel.
cudaError_t subsample_launch(const SubsampleArgs &a, bool tensor_cores, cudaStream_t s);

cudaError_t conv2d_fwd_launch(const Conv2dArgs &a, cudaStream_t s);
cudaError_t conv2d_dx_launch(const Conv2dArgs &a, cudaStream_t s);
int conv2d_dw_partial_rows(int64_t B, int64_t To);
size_t conv2d_dw_workspace_bytes(int64_t B, int64_t To, int64_t C, int KT, int KF);
cudaError_t conv2d_dw_launch(const Conv2dArgs &a, float *dw, float *dbias, float *partials, cudaStream_t s);
// TMA-staged kernels for the 3x3 window (16-byte aligned rows); cudaErrorNotSupported otherwise.
cudaError_t conv2d_fwd_tma_launch(const Conv2dArgs &a, cudaStream_t s);
cudaError_t conv2d_dx_tma_launch(const Conv2dArgs &a, cudaStream_t s);
// Writes partial rows [G][10][C] (G <= max_rows) for the fixed-order finalize.
cudaError_t conv2d_dw_tma_partials(const Conv2dArgs &a, float *partials, int max_rows, int *G, cudaStream_t s);
unsigned int conv2d_tma_take_error();

// A one-block kernel whose bounded mbarrier wait must run out (nothing completes the barrier);
// writes 2 to *done when it gave up, 1 if the wait (impossibly) succeeded.
cudaError_t selftest_wait_timeout_launch(int *done, cudaStream_t s);
unsigned int selftest_take_error();

struct SubsampleBwdArgs {
    const float *mel, *w0, *b0, *w1;
    const void *dout;             // [B][T4][F4][C] bf16, fp16 or float32
    const int32_t *lengths;
    float *dw0, *db0, *dw1, *db1;  // [3][3][C], [C], [3][3][C], [C]
    float *partials;              // workspace: [rows][20][C]
    int64_t B, T, F, C;
    int causal, dout_dtype;  // 0 float32, 1 bf16, 2 fp16
};
int subsample_bwd_partial_rows(int64_t B, int64_t T, int64_t F);
size_t subsample_bwd_workspace_bytes(int64_t B, int64_t T, int64_t F, int64_t C);
cudaError_t subsample_bwd_launch(const SubsampleBwdArgs &a, cudaStream_t s);
// Tensor-core subsampler backward for 16-bit dout with C a multiple of 8 (16-byte aligned dout
// rows): writes partial rows [rows][20][C] (rows <= max_rows) for the fixed-order finalize;
// cudaErrorNotSupported where the SIMT kernel must serve.
cudaError_t subsample_bwd_tc_launch(const SubsampleBwdArgs &a, int max_rows, int *rows, cudaStream_t s);
// Tensor-core subsampler: usable when the output rows are 16-byte aligned (C * element size a
// multiple of 16, aligned base); the SIMT kernel serves every other case.
bool subsample_tc_eligible(const SubsampleArgs &a);
cudaError_t subsample_tc_launch(const SubsampleArgs &a, cudaStream_t s);
unsigned int subsample_tc_take_error();

}  // namespace dwk
