/*
 * dwconv.h - C ABI of a B200 (sm_100a) library for the depthwise-convolution hot path of a
 * conformer speech encoder: the time-axis depthwise conv1d (forward, data gradient, weight
 * and bias gradients) and the fused depthwise-striding subsampler front.
 *
 * Conventions shared by every entry point
 *  - Memory: every tensor pointer is a DEVICE pointer owned by the caller.  The library
 *    allocates nothing, never synchronizes, and enqueues its kernels on `stream`
 *    (a cudaStream_t; NULL means the legacy default stream).  Results are ready when the
 *    stream reaches them.
 *  - Stream order: the kernels are launched with programmatic stream serialization, so one
 *    may start while the previous kernel in the stream drains.  Until that kernel has
 *    completed it only initialises its own shared memory and warms L2 with prefetches, then
 *    it waits for it (griddepcontrol.wait) before its first read: inputs written by earlier
 *    work in the stream, lengths included, are always seen.  Each kernel also lets the next
 *    one start early.  A caller's kernel launched normally after a call waits for the call to
 *    complete as usual; one launched with programmatic serialization must itself wait
 *    (cudaGridDependencySynchronize) before it reads the call's outputs.
 *  - Layout: activations are channels-last and C-contiguous: x[B][T][C] (C fastest).
 *    Weights and biases are float32: w[K][C], bias[C], w0/w1[3][3][C] (C fastest).  A
 *    PyTorch depthwise weight [C][1][K] is the transpose of w.
 *  - Lengths: `lengths` is a device int32 array [B] or NULL.  NULL means every item has
 *    T valid frames.  Values outside [0, T] are clamped into it by the kernels.
 *  - Masking: frame t of item b is valid when t < lengths[b].  Invalid input frames count
 *    as zero; invalid output frames are written as +0.0.
 *  - Errors: every call returns a dw_status_t and never aborts or traps.  Argument errors
 *    are found on the host before any CUDA call.  A failed launch returns DW_ERR_CUDA.
 *    C above 4,194,304 channels or K above 4096 returns DW_ERR_UNSUPPORTED.
 *    B == 0 or T == 0 is a valid no-op.  Misaligned pointers, or a C that is not a
 *    multiple of the vector width, take a narrower (slower) path and stay correct.
 *  - Arithmetic: bf16, fp16 or float32 I/O, float32 accumulation, 16-bit stores rounded to
 *    nearest even.  The subsampler's conv0 runs on the tensor cores (float32-accurate split),
 *    and so do its backward's conv0 recompute and dw0/db0 reduction; everything else runs on the
 *    FP32 pipes.
 */
#ifndef DWCONV_B200_H
#define DWCONV_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum dw_status {
    DW_OK = 0,
    DW_ERR_INVALID_ARG = 1,  /* null pointer, bad size, bad padding, aliasing */
    DW_ERR_UNSUPPORTED = 2,  /* a valid request this build cannot serve (e.g. no sm_100 device) */
    DW_ERR_WORKSPACE = 3,    /* workspace missing or smaller than the *_workspace_size result */
    DW_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed */
    DW_ERR_TIMEOUT = 5       /* a bounded wait inside a kernel gave up (see dw_device_error) */
} dw_status_t;

/*
 * Element type of the activations (x, y, dy, dx, the stream cache).  Weights, biases and
 * gradients of weights are always float32, and so is the arithmetic.  DW_F16 (IEEE binary16;
 * "GPU inference for speech", section "Precision": inference usually runs in FP16 or BF16) is
 * accepted wherever an io_dtype, out_dtype or dout_dtype is taken.
 */
typedef enum dw_dtype {
    DW_F32 = 0,   /* IEEE float32 */
    DW_BF16 = 1,  /* bfloat16 (upper half of a float32) */
    DW_F16 = 2    /* IEEE float16 */
} dw_dtype_t;

typedef void *dw_stream_t; /* a cudaStream_t */

/*
 * dwconv1d_fwd - depthwise conv1d forward with fused pre/post masking and padding.
 *
 *   y[b,t,c] = [t < len_b] * (bias[c] + sum_{k<K} xpad[b,t+k,c] * w[k,c])
 *   xpad[b,j,c] = x[b, j - pad_left, c] if 0 <= j - pad_left < len_b, else 0
 *
 * The sum over k of x[t+k,c] * w[k,c] over the input padded to T + K - 1 frames is the
 * SSM_CONV form of the depthwise conv (parakeet.cpp PR #102, "faster GPU decode: one
 * SSM_CONV for the depthwise conv", section "What changes"); masking before and after the
 * conv and the causal padding are fused as in NeMo PR #16114 ("Use Fused Kernels for
 * Depthwise Striding Subsampler", section "What does this PR do ?", second kernel).
 *
 *  x        [B][T][C] io_dtype, device, read only
 *  w        [K][C] float32, device
 *  bias     [C] float32, device, or NULL (no bias)
 *  y        [B][T][C] io_dtype, device, written in full; must not overlap x
 *  lengths  [B] int32, device, or NULL
 *  B, T, C  sizes, B >= 0, T >= 0, C >= 1
 *  K        kernel width, K >= 1 (any width)
 *  pad_left 0 <= pad_left <= K-1; pad_right = K-1-pad_left.  Symmetric ('same') padding:
 *           pad_left = (K-1)/2; causal padding: pad_left = K-1.
 */
dw_status_t dwconv1d_fwd(const void *x, const float *w, const float *bias, void *y,
                         const int32_t *lengths, int64_t B, int64_t T, int64_t C, int K,
                         int pad_left, dw_dtype_t io_dtype, dw_stream_t stream);

/*
 * dwconv1d_bwd_dx - data gradient of dwconv1d_fwd (backward of NeMo PR #16114's
 * depthwise kernel, section "What does this PR do ?").
 *
 *   dz[b,t,c] = [t < len_b] dy[b,t,c]
 *   dx[b,s,c] = [s < len_b] * sum_{k<K} dz[b, s + pad_left - k, c] * w[k,c]   (dz = 0 outside [0,T))
 *
 * i.e. the forward correlation with the taps reversed and the pads swapped, no bias.
 *
 *  dy       [B][T][C] io_dtype, device          dx [B][T][C] io_dtype, device, written in full,
 *  w        [K][C] float32, device                 must not overlap dy
 *  other arguments as in dwconv1d_fwd (pad_left is the FORWARD pass's left pad).
 */
dw_status_t dwconv1d_bwd_dx(const void *dy, const float *w, void *dx, const int32_t *lengths,
                            int64_t B, int64_t T, int64_t C, int K, int pad_left,
                            dw_dtype_t io_dtype, dw_stream_t stream);

/*
 * dwconv1d_fwd_packed - dwconv1d_fwd over a packed batch: the B sequences lie back to back in
 * x [N][C], sequence b on rows offsets[b] .. offsets[b+1]-1, with no padding rows ("GPU
 * inference for speech", section "Where the time goes": padding short clips to long ones is
 * wasted compute, fixed by length bucketing and packed sequences).  Each sequence is convolved
 * on its own, with its own padding:
 *
 *   y[n,c] = bias[c] + sum_{k<K} xs[t + k - pad_left, c] * w[k,c]     for row n = offsets[b] + t
 *   xs[j,c] = x[offsets[b] + j, c] if 0 <= j < offsets[b+1] - offsets[b], else 0
 *
 * which equals dwconv1d_fwd on the padded batch with lengths[b] = offsets[b+1] - offsets[b], row
 * for row.  Work and traffic follow N, not B * max length.
 *
 *  x, y     [N][C] io_dtype, device; y must not overlap x.  Rows no sequence covers are left
 *           unchanged.
 *  offsets  [B+1] int32, device: 0 = offsets[0] <= offsets[1] <= ... <= offsets[B] <= N.  The
 *           kernels clamp every offset into [0, N] (memory safety only; other values give
 *           unspecified rows).
 *  w, bias, K, pad_left, io_dtype: as dwconv1d_fwd.  B >= 0, N >= 0 (either 0: no-op);
 *  N or B of 2^30 or more returns DW_ERR_UNSUPPORTED.
 */
dw_status_t dwconv1d_fwd_packed(const void *x, const float *w, const float *bias, void *y,
                                const int32_t *offsets, int64_t B, int64_t N, int64_t C, int K,
                                int pad_left, dw_dtype_t io_dtype, dw_stream_t stream);

/*
 * dwconv1d_bwd_dx_packed - data gradient of dwconv1d_fwd_packed (dwconv1d_bwd_dx sequence by
 * sequence): dx[n,c] = sum_{k<K} dys[t + pad_left - k, c] * w[k,c] for row n = offsets[b] + t,
 * dys = dy of sequence b, zero outside it.  Arguments as dwconv1d_fwd_packed (pad_left is the
 * forward pass's).
 */
dw_status_t dwconv1d_bwd_dx_packed(const void *dy, const float *w, void *dx,
                                   const int32_t *offsets, int64_t B, int64_t N, int64_t C, int K,
                                   int pad_left, dw_dtype_t io_dtype, dw_stream_t stream);

/*
 * dwconv1d_bwd_dw_packed_workspace_size - bytes of device workspace dwconv1d_bwd_dw_packed needs
 * (depends on N, C and K only); 0 for invalid sizes.
 */
size_t dwconv1d_bwd_dw_packed_workspace_size(int64_t B, int64_t N, int64_t C, int K);

/*
 * dwconv1d_bwd_dw_packed - weight and bias gradients of dwconv1d_fwd_packed:
 *   dW[k,c] = sum over sequences b and their frames t of dy[offsets[b]+t, c] xs_b[t + k - pad_left, c]
 *   dbias[c] = sum over the rows of every sequence of dy[n, c]
 * with xs_b = x of sequence b, zero outside it.  float32 partial sums per block go to `workspace`
 * and a second kernel adds them in a fixed order (bitwise reproducible for given sizes on a
 * given GPU model: the grid follows the SM count).  No atomics.  Rows no sequence covers are
 * ignored.
 *
 *  x, dy      [N][C] io_dtype, device;  offsets as dwconv1d_fwd_packed
 *  dw         [K][C] float32, device, overwritten;  dbias [C] float32, or NULL
 *  workspace  at least dwconv1d_bwd_dw_packed_workspace_size(B, N, C, K) bytes, 16-byte aligned,
 *             contents on entry ignored.  With B == 0 or N == 0 the gradients are zeros.
 */
dw_status_t dwconv1d_bwd_dw_packed(const void *x, const void *dy, float *dw, float *dbias,
                                   const int32_t *offsets, int64_t B, int64_t N, int64_t C, int K,
                                   int pad_left, dw_dtype_t io_dtype, void *workspace,
                                   size_t workspace_bytes, dw_stream_t stream);

/*
 * dwconv1d_stream_fwd - one chunk of a streaming causal depthwise conv1d with a cache of each
 * stream's K-1 most recent input frames (parakeet.cpp PR #102, section "What changes": the
 * streaming encoder keeps its own depthwise conv with a cache).
 *
 *   xcat_b      = [cache_b (K-1 frames) ; x_b frames 0 .. len_b-1]
 *   y[b,t,c]    = [t < len_b] (bias[c] + sum_{k<K} xcat_b[t+k,c] w[k,c])
 *   cache_b    <- xcat_b frames len_b .. len_b+K-2   (rewritten in place)
 *
 * Feeding a stream chunk by chunk from a zero cache gives exactly the frames of dwconv1d_fwd
 * with causal padding (pad_left = K-1) over the whole stream.
 *
 *  x        [B][T][C] io_dtype, device: this chunk; frames t >= len_b are not part of the
 *           stream (they are neither used nor cached)
 *  w, bias  as dwconv1d_fwd
 *  y        [B][T][C] io_dtype, device, written in full (zeros at t >= len_b); must not
 *           overlap x or cache
 *  cache    [B][K-1][C] io_dtype, device, read and rewritten; may be NULL when K == 1;
 *           must not overlap x or y.  A new stream starts from a zeroed cache.
 *  lengths  [B] int32, device, or NULL (all T frames valid): valid frames of this chunk
 *  B >= 0, T >= 0 (T == 0 leaves the cache unchanged), C >= 1, K >= 1
 */
dw_status_t dwconv1d_stream_fwd(const void *x, const float *w, const float *bias, void *y,
                                void *cache, const int32_t *lengths, int64_t B, int64_t T,
                                int64_t C, int K, dw_dtype_t io_dtype, dw_stream_t stream);

/*
 * dwconv1d_bwd_dw_workspace_size - bytes of device workspace dwconv1d_bwd_dw needs for
 * these sizes (independent of pointers, dtype and device).  Returns 0 when B*T == 0.
 */
size_t dwconv1d_bwd_dw_workspace_size(int64_t B, int64_t T, int64_t C, int K);

/*
 * dwconv1d_bwd_dw - weight and bias gradients of dwconv1d_fwd (NeMo PR #16114, section
 * "What does this PR do ?", backward; deterministic like its "honor deterministic path").
 *
 *   dW[k,c]   = sum_{b,t} dz[b,t,c] * xpad[b,t+k,c]
 *   dbias[c]  = sum_{b,t} dz[b,t,c],           dz[b,t,c] = [t < len_b] dy[b,t,c]
 *
 * float32 accumulation in a fixed order: per-block partial sums go to `workspace`, then a
 * second kernel adds them in a fixed order.  Results are bitwise reproducible for given
 * sizes on a given GPU model (the grid, and so the order of the sums, follows the SM count).
 * No atomics.
 *
 *  x, dy     [B][T][C] io_dtype, device
 *  dw        [K][C] float32, device, overwritten
 *  dbias     [C] float32, device, overwritten, or NULL
 *  workspace device buffer of at least dwconv1d_bwd_dw_workspace_size(B,T,C,K) bytes,
 *            16-byte aligned; contents on entry are ignored
 *  With B*T == 0 the gradients are written as zeros (workspace may be NULL).
 */
dw_status_t dwconv1d_bwd_dw(const void *x, const void *dy, float *dw, float *dbias,
                            const int32_t *lengths, int64_t B, int64_t T, int64_t C, int K,
                            int pad_left, dw_dtype_t io_dtype, void *workspace,
                            size_t workspace_bytes, dw_stream_t stream);

/*
 * dwconv1d_bwd - the data gradient and the weight/bias gradients of dwconv1d_fwd in one pass
 * that reads dy once (NeMo PR #16114, section "What does this PR do ?", the depthwise kernel's
 * backward).  Results equal dwconv1d_bwd_dx followed by dwconv1d_bwd_dw: dx up to float32
 * summation order, dW/dbias bitwise reproducible for given sizes on a given GPU model, like
 * dwconv1d_bwd_dw.
 *
 *  x, dy, dx  [B][T][C] io_dtype, device; dx is written in full and must not overlap x or dy
 *  w          [K][C] float32 (the forward taps)
 *  dw, dbias, workspace, workspace_bytes: as dwconv1d_bwd_dw
 *  other arguments as dwconv1d_fwd (pad_left is the forward pass's).
 * Sizes without a fused instance run the two gradients one after the other (same results).
 */
dw_status_t dwconv1d_bwd(const void *x, const void *dy, const float *w, void *dx, float *dw,
                         float *dbias, const int32_t *lengths, int64_t B, int64_t T, int64_t C,
                         int K, int pad_left, dw_dtype_t io_dtype, void *workspace,
                         size_t workspace_bytes, dw_stream_t stream);

/*
 * dwconv1d_bwd_dw_noalloc - dwconv1d_bwd_dw without a caller-provided workspace: it allocates
 * nothing and uses a scratch array that the library keeps in device memory.  The papers have
 * no counterpart to this entry point; it exists for callers that cannot allocate device
 * memory: code embedded in a host that owns all device memory through its own allocator and
 * hands plug-ins no allocation handle, and streaming loops that must not call cudaMalloc after
 * start-up because an allocation can block on the whole device.
 *
 *  Scratch: 2 MiB (2,097,152 bytes) of device memory per GPU that loads the library, held
 *  until the process exits.  One partial row of (K+1)*C float32 must fit in it: larger
 *  (K+1)*C returns DW_ERR_UNSUPPORTED without touching the device.  Within that limit the
 *  results equal dwconv1d_bwd_dw's up to float32 summation order (the same order whenever
 *  the scratch holds as many partial rows as dwconv1d_bwd_dw_workspace_size would provide).
 *  The first call on a device looks up the scratch's device address (cudaGetSymbolAddress),
 *  and so does the first call after the device's context has changed (cudaDeviceReset), so
 *  that first call should come before any stream capture.  All calls share the scratch and
 *  it keeps the last call's contents; calls that overlap on the GPU race on it, so the caller
 *  must serialise them.  Every partial sum read is written by the same call first.  Argument
 *  checks, results and errors are those of dwconv1d_bwd_dw (a failed launch returns
 *  DW_ERR_CUDA and sets dw_last_cuda_error), plus the scratch limit above.
 */
dw_status_t dwconv1d_bwd_dw_noalloc(const void *x, const void *dy, float *dw, float *dbias,
                                    const int32_t *lengths, int64_t B, int64_t T, int64_t C, int K,
                                    int pad_left, dw_dtype_t io_dtype, dw_stream_t stream);

/*
 * dw_subsample_fwd - fused front of the depthwise-striding subsampler (NeMo PR #16114, "Use
 * Fused Kernels for Depthwise Striding Subsampler", section "What does this PR do ?", first
 * kernel: mel [B,T,F,1] -> conv0 [B,T/2,F/2,C] -> ReLU -> masking -> conv_dw1 [B,T/4,F/4,C]).
 * The conv0 output never goes to device memory.
 *
 *   melpad = mel with frames t >= len_b zeroed, padded Pt|Pb in time and 1|1 in frequency
 *   h[b,i,j,c]   = [i < ceil(len_b/2)] * ReLU(b0[c] + sum_{p,q<3} melpad[2i+p, 2j+q] * w0[p,q,c])
 *   out[b,i,j,c] = [i < ceil(len_b/4)] * (b1[c] + sum_{p,q<3} hpad[b, 2i+p, 2j+q, c] * w1[p,q,c])
 *   hpad = h padded Pt|Pb in time and 1|1 in frequency; Pt|Pb = 1|1, or 2|0 when causal.
 *
 *  mel          [B][T][F] float32, device
 *  w0, w1       [3][3][C] float32, device;  b0, b1 [C] float32, device
 *  out          [B][T4][F4][C] out_dtype, device, written in full, where
 *               T2 = ceil(T/2), T4 = ceil(T2/2), F2 = ceil(F/2), F4 = ceil(F2/2)
 *  lengths      [B] int32, device, or NULL
 *  out_lengths  [B] int32, device, or NULL; receives ceil(ceil(len_b/2)/2)
 *  B >= 0, T >= 0, F >= 1, C >= 1; causal 0 or 1; out_dtype DW_BF16, DW_F16 or DW_F32
 */
dw_status_t dw_subsample_fwd(const float *mel, const float *w0, const float *b0,
                             const float *w1, const float *b1, void *out,
                             const int32_t *lengths, int32_t *out_lengths, int64_t B,
                             int64_t T, int64_t F, int64_t C, int causal,
                             dw_dtype_t out_dtype, dw_stream_t stream);

/*
 * dw_subsample_fwd_simt - the same operation, arguments and results as dw_subsample_fwd, computed
 * entirely on the FP32 FMA pipes: conv0, ReLU, the masks and conv_dw1 as packed float32 FMAs, no
 * tensor cores, for every size and alignment.  The NeMo PR's kernel runs conv0 as a TF32 dot
 * (NeMo PR #16114, "What does this PR do ?"); dw_subsample_fwd runs it on the tcgen05 tensor
 * cores with float32-accurate operand splits whenever the output rows are 16-byte aligned.  This
 * entry point is the all-FP32 design of the depthwise path: the kernel whose throughput is
 * stated against the FP32 peak.  Results agree with dw_subsample_fwd within float32 rounding.
 */
dw_status_t dw_subsample_fwd_simt(const float *mel, const float *w0, const float *b0,
                                  const float *w1, const float *b1, void *out,
                                  const int32_t *lengths, int32_t *out_lengths, int64_t B,
                                  int64_t T, int64_t F, int64_t C, int causal,
                                  dw_dtype_t out_dtype, dw_stream_t stream);

/*
 * dw_subsample_bwd_workspace_size - bytes of device workspace dw_subsample_bwd needs for these
 * sizes (independent of pointers, dtype and device).
 */
size_t dw_subsample_bwd_workspace_size(int64_t B, int64_t T, int64_t F, int64_t C);

/*
 * dw_subsample_bwd - backward of dw_subsample_fwd (NeMo PR #16114, "Use Fused Kernels for
 * Depthwise Striding Subsampler", section "What does this PR do ?": the fused kernels come with
 * backward passes): the gradients of sum(out * dout) with respect to the weights and biases.
 *
 *   doutm[i,j,c] = [i < ceil(len_b/4)] dout[i,j,c];  z = b0 + conv0(melpad) (recomputed)
 *   db1 = sum doutm;   dw1[p,q,c] = sum doutm[i,j,c] hpad[2i+p, 2j+q, c]
 *   dh  = conv_dw1 transposed applied to doutm (taps w1);  dz = [r < ceil(len_b/2)] [z > 0] dh
 *   db0 = sum dz;      dw0[p,q,c] = sum dz[r,s,c] melpad[2r+p, 2s+q]
 * The mel input takes no gradient.  float32 accumulation (z and the dw0/db0 sums on the tensor
 * cores with float32-accurate operand splits when dout rows are 16-byte aligned and 16-bit);
 * the per-block partial sums go to `workspace` and a second kernel adds them in a fixed order
 * (reproducible for given sizes on a given GPU model).  No atomics.
 *
 *  mel, w0, b0, w1, lengths, B, T, F, C, causal: as dw_subsample_fwd (b1 is not needed)
 *  dout         [B][T4][F4][C] dout_dtype (DW_BF16, DW_F16 or DW_F32), device
 *  dw0, dw1     [3][3][C] float32, device, overwritten;  db0, db1 [C] float32, overwritten
 *  workspace    device buffer of at least dw_subsample_bwd_workspace_size(B,T,F,C) bytes,
 *               16-byte aligned; contents on entry are ignored
 *  With no output frames the gradients are written as zeros (workspace may be NULL).
 */
dw_status_t dw_subsample_bwd(const float *mel, const float *w0, const float *b0,
                             const float *w1, const void *dout, const int32_t *lengths,
                             float *dw0, float *db0, float *dw1, float *db1, int64_t B,
                             int64_t T, int64_t F, int64_t C, int causal, dw_dtype_t dout_dtype,
                             void *workspace, size_t workspace_bytes, dw_stream_t stream);

/*
 * dwconv2d_fwd - general depthwise conv2d over channels-last [B][T][F][C] with fused length
 * masking and causal padding (NeMo PR #16114, "Use Fused Kernels for Depthwise Striding
 * Subsampler", section "What does this PR do ?", second kernel: a depthwise conv with fused
 * masking and causal padding, used by the subsampler's later depthwise stages).
 *
 *   xpad[b,r,s,c] = x[b, r-pad_t, s-pad_f, c] if 0 <= r-pad_t < len_b and 0 <= s-pad_f < F, else 0
 *   To = (T + pad_t + pad_b - KT) / stride_t + 1,  Fo = (F + 2 pad_f - KF) / stride_f + 1
 *        (0 when the window does not fit)
 *   Lo_b = min(To, (len_b + pad_t + pad_b - KT) / stride_t + 1)   (0 when it does not fit)
 *   y[b,i,j,c] = [i < Lo_b] (bias[c] + sum_{p<KT, q<KF} xpad[b, stride_t i + p, stride_f j + q, c] w[p,q,c])
 *
 * Frames t >= len_b count as padding (the pre-mask); output rows i >= Lo_b are written as +0.0
 * (the post-mask).  Causal time padding is pad_t = KT-1, pad_b = 0; symmetric is pad_t = pad_b.
 * float32 accumulation, one rounding to io_dtype.
 *
 *  x            [B][T][F][C] io_dtype, device
 *  w            [KT][KF][C] float32, device;  bias [C] float32, device, or NULL
 *  y            [B][To][Fo][C] io_dtype, device, written in full; must not overlap x
 *  lengths      [B] int32, device, or NULL (all T frames valid); values are clamped to [0, T]
 *  out_lengths  [B] int32, device, or NULL; receives Lo_b
 *  B >= 0, T >= 0, F >= 1, C >= 1, KT, KF >= 1, strides >= 1, pads >= 0; each of T, F, C, To,
 *  Fo below 2^31.  Invalid arguments return DW_ERR_INVALID_ARG before any device work.
 */
dw_status_t dwconv2d_fwd(const void *x, const float *w, const float *bias, void *y,
                         const int32_t *lengths, int32_t *out_lengths, int64_t B, int64_t T,
                         int64_t F, int64_t C, int KT, int KF, int stride_t, int stride_f,
                         int pad_t, int pad_b, int pad_f, dw_dtype_t io_dtype, dw_stream_t stream);

/*
 * dwconv2d_bwd_dx - data gradient of dwconv2d_fwd: the transpose of the masked map,
 *   dx[b,t,f,c] = [t < len_b] sum over (i, j, p, q) with stride_t i + p - pad_t = t,
 *                 stride_f j + q - pad_f = f and i < Lo_b of dy[b,i,j,c] w[p,q,c]
 * computed as a gather (each dx element is written once, no atomics).
 *
 *  dy  [B][To][Fo][C] io_dtype, device;  dx [B][T][F][C] io_dtype, device, written in full
 *      (+0.0 at t >= len_b); must not overlap dy
 *  other arguments as dwconv2d_fwd.
 */
dw_status_t dwconv2d_bwd_dx(const void *dy, const float *w, void *dx, const int32_t *lengths,
                            int64_t B, int64_t T, int64_t F, int64_t C, int KT, int KF,
                            int stride_t, int stride_f, int pad_t, int pad_b, int pad_f,
                            dw_dtype_t io_dtype, dw_stream_t stream);

/*
 * dwconv2d_bwd_dw_workspace_size - bytes of device workspace dwconv2d_bwd_dw needs for these
 * sizes (independent of pointers, dtype and device); 0 for invalid sizes.
 */
size_t dwconv2d_bwd_dw_workspace_size(int64_t B, int64_t T, int64_t F, int64_t C, int KT, int KF,
                                      int stride_t, int stride_f, int pad_t, int pad_b, int pad_f);

/*
 * dwconv2d_bwd_dw - weight and bias gradients of dwconv2d_fwd:
 *   dW[p,q,c] = sum_{b, i < Lo_b, j} dy[b,i,j,c] xpad[b, stride_t i + p, stride_f j + q, c]
 *   dbias[c]  = sum_{b, i < Lo_b, j} dy[b,i,j,c]
 * float32 accumulation; per-block partial sums go to `workspace` and a second kernel adds them
 * in a fixed order: bitwise reproducible for given sizes on a given GPU model.  No atomics.
 *
 *  x, dy        as dwconv2d_fwd / dwconv2d_bwd_dx
 *  dw           [KT][KF][C] float32, device, overwritten;  dbias [C] float32, or NULL
 *  workspace    device buffer of at least dwconv2d_bwd_dw_workspace_size(...) bytes, 16-byte
 *               aligned; contents on entry are ignored
 *  With no output elements the gradients are written as zeros (workspace may be NULL).
 */
dw_status_t dwconv2d_bwd_dw(const void *x, const void *dy, float *dw, float *dbias,
                            const int32_t *lengths, int64_t B, int64_t T, int64_t F, int64_t C,
                            int KT, int KF, int stride_t, int stride_f, int pad_t, int pad_b,
                            int pad_f, dw_dtype_t io_dtype, void *workspace,
                            size_t workspace_bytes, dw_stream_t stream);

/* dw_status_string - a static, human-readable name for a status code. */
const char *dw_status_string(dw_status_t status);

/* dw_last_cuda_error - the cudaError_t behind the most recent DW_ERR_CUDA on this thread. */
int dw_last_cuda_error(void);

/*
 * dw_device_error - reads and clears the device-side error words of the library's kernels.
 * Pipelined kernels wait on shared-memory barriers for their own bulk copies; every such
 * wait is bounded, and a wait that gives up records an error here instead of hanging.
 * SYNCHRONOUS: waits for all work on the current device.  Returns DW_OK when no kernel
 * recorded an error since the previous call, DW_ERR_TIMEOUT when one did, DW_ERR_CUDA when
 * the query itself failed.
 */
dw_status_t dw_device_error(void);

/*
 * dw_selftest_wait_timeout - checks the bounded waits: launches one block that runs the kernels'
 * bounded mbarrier wait (with a limit 256 times shorter than theirs) on an mbarrier nothing will
 * complete.  The wait gives up after its poll limit,
 * records the error that dw_device_error() then reports as DW_ERR_TIMEOUT, writes 2 to *done
 * (a device int32) and returns; no fault is raised and the context stays usable.
 */
dw_status_t dw_selftest_wait_timeout(int *done, dw_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DWCONV_B200_H */
