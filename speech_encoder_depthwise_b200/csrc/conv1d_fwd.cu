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
#include <type_traits>

#include "dw_internal.h"

namespace dwk {

template <typename T, int V, int K, int R>
__global__ void __launch_bounds__(256, 2)
conv1d_fwd_vec_kernel(const T *__restrict__ x, const float *__restrict__ w,
                      const float *__restrict__ bias, T *__restrict__ y,
                      const int32_t *__restrict__ lengths, int64_t Tn, int C, int pad_left,
                      int flip, int TX, int nT, int nC, int64_t units) {
    constexpr int NP = Pairs<V>::n;
    const int tx = threadIdx.x % TX, ty = threadIdx.x / TX;
    const int TY = blockDim.x / TX;
    // The grid is a multiple of nC and units run channel-tile fastest, so a block keeps one
    // channel tile (and its weights in registers) for every unit it is dealt.
    const int ct = static_cast<int>(blockIdx.x % nC);
    const int c0 = (ct * TX + tx) * V;
    if (c0 >= C) return;
    const uint32_t rs = static_cast<uint32_t>(C) * sizeof(T);  // bytes between frames

    float2 wv[K][NP], bv[NP];
#pragma unroll
    for (int k = 0; k < K; ++k) load_param<V>(w + static_cast<int64_t>(flip ? K - 1 - k : k) * C + c0, wv[k]);
    if (bias) load_param<V>(bias + c0, bv);
    else {
#pragma unroll
        for (int p = 0; p < NP; ++p) bv[p] = make_float2(0.f, 0.f);
    }

    for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
        const int64_t bt = u / nC;
        const int64_t b = bt / nT;
        const int64_t t0 = ((bt % nT) * TY + ty) * R;
        if (t0 >= Tn) continue;
        const int64_t L = clamp_len(lengths, b, Tn);
        const char *xi = reinterpret_cast<const char *>(x + b * Tn * C + c0);  // frame 0 of item b
        char *yt = reinterpret_cast<char *>(y + (b * Tn + t0) * C + c0);      // frame t0 of item b
        if (t0 >= L) {  // the whole run is masked: zeros only, nothing read
#pragma unroll
            for (int r = 0; r < R; ++r)
                if (t0 + r < Tn) Vec<T, V>::store_zero(reinterpret_cast<T *>(yt + static_cast<uint32_t>(r) * rs));
            continue;
        }
        const int64_t j0 = t0 - pad_left;
        Vec<T, V> raw[R + K - 1];
        if (j0 >= 0 && j0 + R + K - 1 <= L) {  // every input frame of the run is valid
            const char *xj = xi + j0 * rs;
#pragma unroll
            for (int i = 0; i < R + K - 1; ++i)
                raw[i].load(reinterpret_cast<const T *>(xj + static_cast<uint32_t>(i) * rs));
        } else {
#pragma unroll
            for (int i = 0; i < R + K - 1; ++i) {
                const int64_t j = j0 + i;
                if (j >= 0 && j < L) raw[i].load(reinterpret_cast<const T *>(xi + j * rs));
                else raw[i].zero();
            }
        }
        const bool full = t0 + R <= L;  // every output of the run is valid
        float2 acc[R][NP];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int p = 0; p < NP; ++p) acc[r][p] = bv[p];
        // input frame i feeds output r = i - k through tap k; output r is complete after i = r + K - 1
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
            const int rd = i - (K - 1);
            if (rd >= 0) {
                T *dst = reinterpret_cast<T *>(yt + static_cast<uint32_t>(rd) * rs);
                if (full || t0 + rd < L) Vec<T, V>::store(dst, acc[rd]);
                else if (t0 + rd < Tn) Vec<T, V>::store_zero(dst);
            }
        }
    }
}

// ---------------------------------------------------------------------------------------
// Pipelined variant for the common case (16-byte frame rows, specialised K): a persistent
// block per SM, one producer warp and kTmaConsumers consumer warps.  For each tile the
// producer issues ONE tensor copy (cp.async.bulk.tensor: CT channels x (TT + K - 1) frames,
// starting K-1 halo frames early) into a kTmaStages-deep shared-memory ring; completion is
// counted in bytes on the stage's "full" mbarrier.  Frames before 0 or past T arrive as zeros
// (the padding).  Each block keeps one channel tile, so its weights stay in registers, and its
// first ring-full of copies goes out before any length is known.  Consumers read their R + K - 1 rows from shared memory with the same
// register window as above, mask frames in [len_b, T), store straight to global memory and
// release the stage on its "empty" mbarrier.  HBM never waits on compute: up to kTmaStages
// tiles are in flight per SM while the consumers work on one.  Wholly masked tiles are not
// read at all.
// ---------------------------------------------------------------------------------------
// Tuned on B200 (sweeps over consumer warps, frames per thread, ring depth, blocks per SM and
// tile width): 3 blocks of 4 consumer warps per SM, 3 stages, 12 frames per thread (K = 15: 8
// with 4 channels a thread, 16 with 2), tiles 128 channels wide (256-byte bf16 rows; narrower
// rows cost DRAM efficiency).
#ifndef DW_FWD_CONSUMERS
#define DW_FWD_CONSUMERS 4
#endif
#ifndef DW_FWD_R
#define DW_FWD_R 12
#endif
#ifndef DW_FWD_R_WIDE
#define DW_FWD_R_WIDE 16
#endif
#ifndef DW_FWD_STAGES
#define DW_FWD_STAGES 3
#endif
#ifndef DW_FWD_BLOCKS
#define DW_FWD_BLOCKS 3
#endif

constexpr int kTmaConsumers = DW_FWD_CONSUMERS;  // consumer warps per block
constexpr int kTmaR = DW_FWD_R;                  // frames per consumer thread, K <= 9
constexpr int kTmaRWide = DW_FWD_R_WIDE;         // frames per consumer thread, K > 9
#ifndef DW_FWD_R_WIDE4
#define DW_FWD_R_WIDE4 8
#endif
constexpr int kTmaRWide4 = DW_FWD_R_WIDE4;       // frames per consumer thread, K = 15 with 4 channels
constexpr int kTmaStages = DW_FWD_STAGES;        // shared-memory ring depth
constexpr int kTmaBlocks = DW_FWD_BLOCKS;        // resident blocks per SM

constexpr int kTmaThreads = 32 * (1 + kTmaConsumers);

template <typename T, int V, int K>
struct TmaShape {
    static constexpr int R = (K > 9) ? (V >= 4 ? kTmaRWide4 : kTmaRWide) : kTmaR;
    static constexpr int WPR = (V >= 4) ? 1 : 2;      // consumer warps side by side: 128-channel tiles
    static constexpr int CT = 32 * V * WPR;           // channels per tile
    static constexpr int TT = (kTmaConsumers / WPR) * R;  // output frames per tile
    static constexpr int ROWS = TT + K - 1;           // input rows per tile
    static constexpr int ROWB = CT * static_cast<int>(sizeof(T));
    static constexpr int STAGE_BYTES = ROWS * ROWB;
    static constexpr int SMEM = 128 + kTmaStages * STAGE_BYTES;
};

// PACKED: the items are sequences of a packed batch, x and y [N][C] with item b on rows
// offsets[b] .. offsets[b+1]-1 (`lengths` then points to offsets[B+1], Tn = N).  Each item has
// exactly its own frames (no padding rows), so only its frame-runs are dealt, in order, through a
// prefix table of runs per item that warp 0 builds in shared memory; input rows of the
// neighbouring items inside a tile are masked like frames past a length.
template <typename T, int V, int K, bool PACKED = false>
__global__ void __launch_bounds__(kTmaThreads, kTmaBlocks)
conv1d_fwd_tma_kernel(const __grid_constant__ CUtensorMap xmap, const float *__restrict__ w,
                      const float *__restrict__ bias, T *__restrict__ y, const int32_t *__restrict__ lengths,
                      int B, int Tn, int C, int pad_left, int flip, int nT, int nC, int ntiles) {
    using S = TmaShape<T, V, K>;
    constexpr int NP = Pairs<V>::n;
    constexpr int R = S::R;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem_raw);
    uint64_t *empty = full + kTmaStages;
    unsigned char *stages = smem_raw + 128;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    // Each block keeps one channel tile (the grid is a multiple of nC), so its weights stay in
    // registers, and walks that tile's (item, frame-run) positions q0, q0 + qstride, ...
    const int my_ct = static_cast<int>(blockIdx.x % nC);
    const int q0 = static_cast<int>(blockIdx.x / nC), qstride = static_cast<int>(gridDim.x / nC);
    int nq = ntiles / nC;  // positions per channel tile
    // packed items: runs before item b (pv[b]), its first row and its length
    int *pv = reinterpret_cast<int *>(stages + static_cast<size_t>(kTmaStages) * S::STAGE_BYTES);
    int *pst = pv + (B + 1), *plen = pst + B;
    launch_dependents();  // the next kernel in the stream may start its own set-up
    if (threadIdx.x == 0) {
        for (int i = 0; i < kTmaStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kTmaConsumers);
        }
        fence_barrier_init();
    }
    if constexpr (!PACKED) {
        // While the previous kernel drains, warm L2 with this block's first ring-full of tiles (the
        // same boxes the producer copies after the wait), its taps and bias, and the lengths.
        if (threadIdx.x == 0) {
            prefetch_tmap(&xmap);
            for (int i = 0, q = q0; i < kTmaStages && q < nq; ++i, q += qstride)
                tma_prefetch_3d(&xmap, my_ct * S::CT, (q % nT) * S::TT - pad_left, q / nT);
        } else if (warp == 1) {  // taps and bias over the tile's channels: (K + 1) rows of CT floats
            constexpr int kLines = S::CT * 4 / 128;
            for (int i = lane; i < (K + 1) * kLines; i += 32) {
                const int row = i / kLines, c = my_ct * S::CT + (i % kLines) * 32;
                if (c < C && (row < K || bias != nullptr)) prefetch_l2(row < K ? w + static_cast<int64_t>(row) * C + c : bias + c);
            }
        } else if (warp == 2 && lengths != nullptr) {
            for (int i = lane * 32; i < B; i += 32 * 32) prefetch_l2(lengths + i);
        }
    }
    grid_dependency_wait();  // launched programmatically: the previous kernel's writes are visible after this
    if constexpr (PACKED) {
        if (warp == 0) {  // offsets are clamped into [0, N] and made non-decreasing
            int run = 0;
            if (lane == 0) pv[0] = 0;
            for (int base = 0; base < B; base += 32) {
                const int bb = base + lane;
                int nv = 0;
                if (bb < B) {
                    int s0 = __ldg(lengths + bb), e = __ldg(lengths + bb + 1);
                    s0 = s0 < 0 ? 0 : (s0 > Tn ? Tn : s0);
                    e = e < s0 ? s0 : (e > Tn ? Tn : e);
                    pst[bb] = s0;
                    plen[bb] = e - s0;
                    nv = (e - s0 + S::TT - 1) / S::TT;
                }
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int t = __shfl_up_sync(0xffffffffu, nv, o);
                    if (lane >= o) nv += t;
                }
                if (bb < B) pv[bb + 1] = run + nv;
                run += __shfl_sync(0xffffffffu, nv, 31);
            }
        }
    }
    __syncthreads();
    if constexpr (PACKED) nq = pv[B];
    // position q of the channel tile -> item b, first frame t0 (within the item), the item's
    // length L, its first row r0 in x/y and its frame count TN (T, or L when packed)
    auto unit_at = [&](int q, int &b, int &t0, int &L, int64_t &r0, int &TN) {
        if constexpr (PACKED) {
            b = TileOrder::find(pv, B, q);
            t0 = (q - pv[b]) * S::TT;
            L = plen[b];
            r0 = pst[b];
            TN = L;
        } else {
            b = q / nT;
            t0 = (q % nT) * S::TT;
            L = static_cast<int>(clamp_len(lengths, b, Tn));
            r0 = static_cast<int64_t>(b) * Tn;
            TN = Tn;
        }
    };
    if (warp == 0) {  // producer warp: one elected lane, one tensor copy per tile
        if (lane == 0) prefetch_tmap(&xmap);
        int it = 0;
        for (int q = q0; q < nq; q += qstride, ++it) {
            const int s = it % kTmaStages;
            const uint32_t ph = (it / kTmaStages) & 1;
            int b, t0, L, TN;
            int64_t r0 = 0;
            if (PACKED || (it >= kTmaStages && lane == 0)) {
                unit_at(q, b, t0, L, r0, TN);
            } else {
                // the first ring-full of tiles is issued without waiting for the item's length (a
                // wholly masked one is read needlessly); later tiles skip the read when t0 >= len
                b = q / nT;
                t0 = (q % nT) * S::TT;
                L = Tn;
            }
            if (!__all_sync(0xffffffffu, mbar_wait(&empty[s], ph ^ 1))) return;
            if (lane == 0) {
                if (t0 < L) {  // rows before frame 0 or past T arrive as zeros; rows in [L, T) are masked by the consumers
                    mbar_arrive_expect_tx(&full[s], S::STAGE_BYTES);
                    // padded: item b of the [B][T][C] map; packed: rows of the [1][N][C] map
                    tma_load_3d(stages + static_cast<size_t>(s) * S::STAGE_BYTES, &xmap, my_ct * S::CT,
                                static_cast<int>(PACKED ? r0 : 0) + t0 - pad_left, PACKED ? 0 : b, &full[s]);
                } else {
                    mbar_arrive(&full[s]);  // a wholly masked tile: nothing to read
                }
            }
            __syncwarp();
        }
        return;
    }

    // consumer warps: warp g+1 computes frames [t0 + g R, t0 + g R + R) of each tile
    const int g = (warp - 1) / S::WPR;                  // row group
    const int wc = ((warp - 1) % S::WPR) * 32 * V;      // first channel of this warp within the tile
    const int cv = my_ct * S::CT + wc + lane * V;
    const bool active = cv < C;
    float2 wv[K][NP], bv[NP];
    if (active) {  // the block's channel tile never changes: weights stay in registers
#pragma unroll
        for (int k = 0; k < K; ++k) load_param<V>(w + static_cast<int64_t>(flip ? K - 1 - k : k) * C + cv, wv[k]);
        if (bias) load_param<V>(bias + cv, bv);
        else {
#pragma unroll
            for (int p = 0; p < NP; ++p) bv[p] = make_float2(0.f, 0.f);
        }
    }
    int it = 0;
    for (int q = q0; q < nq; q += qstride, ++it) {
        const int s = it % kTmaStages;
        const uint32_t ph = (it / kTmaStages) & 1;
        int b, t0, L, TN;
        int64_t r0;
        unit_at(q, b, t0, L, r0, TN);  // before the wait below
        const int tg = t0 + g * R;
        float2 acc[R][NP];
        if (active && tg < L) {
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int p = 0; p < NP; ++p) acc[r][p] = bv[p];
        }
        if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph))) return;
        if (active && tg < TN) {
            T *yp = y + (r0 + tg) * C + cv;
            if (tg >= L) {
#pragma unroll
                for (int r = 0; r < R; ++r)
                    if (tg + r < TN) Vec<T, V>::store_zero(yp + static_cast<int64_t>(r) * C);
            } else {
                const unsigned char *sp = stages + static_cast<size_t>(s) * S::STAGE_BYTES +
                                          (g * R) * S::ROWB + (wc + lane * V) * static_cast<int>(sizeof(T));
                const int jb = tg - pad_left;  // frame of this thread's first row
                // CHECK = false: every row and every output of the run is inside [0, len_b)
                auto run = [&](auto check) {
                    constexpr bool CHECK = decltype(check)::value;
                    T *dst = yp;
#pragma unroll
                    for (int i = 0; i < R + K - 1; ++i) {
                        Vec<T, V> v;
                        v.r = *reinterpret_cast<const decltype(v.r) *>(sp + i * S::ROWB);
                        if constexpr (CHECK) {
                            if (jb + i < 0 || jb + i >= L) v.zero();
                        }
                        float2 xf[NP];
                        v.to_f2(xf);
#pragma unroll
                        for (int k = 0; k < K; ++k) {
                            const int r = i - k;
                            if (r >= 0 && r < R) {
#pragma unroll
                                for (int p = 0; p < NP; ++p) acc[r][p] = ffma2(xf[p], wv[k][p], acc[r][p]);
                            }
                        }
                        const int rd = i - (K - 1);
                        if (rd >= 0) {
                            if constexpr (CHECK) {
                                if (tg + rd < L) Vec<T, V>::store(dst, acc[rd]);
                                else if (tg + rd < TN) Vec<T, V>::store_zero(dst);
                            } else {
                                Vec<T, V>::store(dst, acc[rd]);
                            }
                            dst += C;
                        }
                    }
                };
                if (jb >= 0 && jb + R + K - 1 <= L) run(std::false_type{});  // implies tg + R <= L
                else run(std::true_type{});
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
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

// Blocks resident per SM for a kernel at 256 threads, and the SM count of the current device.
template <typename Kern>
int resident_blocks(Kern kern) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kThreads, 0) != cudaSuccess || n < 1) n = 1;
    return n;
}

template <typename T, int V, int K>
cudaError_t launch_vec_k(const Conv1dArgs &a, cudaStream_t s) {
    constexpr int R = (K <= 9) ? 16 : 8;
    const int64_t Cv = (a.C + V - 1) / V;
    const int TX = pow2_at_most(Cv, 32);
    const int TY = kThreads / TX;
    const int nC = static_cast<int>((Cv + TX - 1) / TX);
    const int nT = static_cast<int>((a.T + static_cast<int64_t>(TY) * R - 1) / (static_cast<int64_t>(TY) * R));
    const int64_t units = a.B * nT * static_cast<int64_t>(nC);
    auto kern = conv1d_fwd_vec_kernel<T, V, K, R>;
    static const int occ = resident_blocks(kern);
    int64_t grid = static_cast<int64_t>(sm_count()) * occ;
    grid = (grid / nC) * nC;
    if (grid < nC) grid = nC;
    if (grid > units) grid = units;          // units is a multiple of nC
    if (grid > kMaxGrid) return cudaErrorInvalidConfiguration;
    kern<<<static_cast<unsigned>(grid), kThreads, 0, s>>>(
        static_cast<const T *>(a.x), a.w, a.bias, static_cast<T *>(a.y), a.lengths, a.T, static_cast<int>(a.C),
        a.pad_left, a.flip, TX, nT, nC, units);
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

// Packed sequences, any K, any C, any alignment: thread = (row n, V channels).  The row's item
// comes from a binary search over offsets; its inputs outside the item count as zero.  Rows
// that no item covers are left unchanged.
template <typename T, int V>
__global__ void __launch_bounds__(256)
conv1d_fwd_packed_kernel(const T *__restrict__ x, const float *__restrict__ w, const float *__restrict__ bias,
                         T *__restrict__ y, const int32_t *__restrict__ offsets, int B, int N, int C, int K,
                         int pad_left, int flip, int nCV) {
    constexpr int NP = Pairs<V>::n;
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<int64_t>(N) * nCV) return;
    const int n = static_cast<int>(idx / nCV), c = static_cast<int>(idx % nCV) * V;
    auto off = [&](int b) {
        const int o = __ldg(offsets + b);
        return o < 0 ? 0 : (o > N ? N : o);
    };
    int lo = 0, hi = B;  // the last item b with off(b) <= n
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (off(mid) <= n) lo = mid;
        else hi = mid;
    }
    const int s0 = off(lo), e = off(lo + 1);
    if (n < s0 || n >= e) return;
    const int t = n - s0, L = e - s0;
    float2 acc[NP];
    if (bias != nullptr) {
        load_param<V>(bias + c, acc);
    } else {
#pragma unroll
        for (int p = 0; p < NP; ++p) acc[p] = make_float2(0.f, 0.f);
    }
    for (int k = 0; k < K; ++k) {
        const int j = t - pad_left + k;
        if (j < 0 || j >= L) continue;
        Vec<T, V> v;
        v.load(x + (static_cast<int64_t>(s0) + j) * C + c);
        float2 xf[NP], wf[NP];
        v.to_f2(xf);
        load_param<V>(w + static_cast<int64_t>(flip ? K - 1 - k : k) * C + c, wf);
#pragma unroll
        for (int p = 0; p < NP; ++p) acc[p] = ffma2(xf[p], wf[p], acc[p]);
    }
    Vec<T, V>::store(y + static_cast<int64_t>(n) * C + c, acc);
}

template <typename T, int V, int K>
cudaError_t launch_tma(const Conv1dArgs &a, cudaStream_t s) {
    using S = TmaShape<T, V, K>;
    auto kern = conv1d_fwd_tma_kernel<T, V, K>;
    const cudaError_t attr = ensure_smem_attr(reinterpret_cast<const void *>(kern), S::SMEM);
    if (attr != cudaSuccess) return attr;
    const int nC = static_cast<int>((a.C + S::CT - 1) / S::CT);
    const int nT = static_cast<int>((a.T + S::TT - 1) / S::TT);
    const int64_t ntiles = a.B * static_cast<int64_t>(nT) * nC;
    if (ntiles > kMaxGrid) return cudaErrorInvalidConfiguration;
    CUtensorMap xmap;
    const cudaError_t me = make_act_map(&xmap, a.x, dtype_code<T>(), a.B, a.T, a.C, S::CT, S::ROWS);
    if (me != cudaSuccess) return me;
    int64_t grid = static_cast<int64_t>(sm_count()) * kTmaBlocks;
    if (grid > ntiles) grid = ntiles;
    grid = grid / nC * nC;  // whole channel tiles per block walk
    if (grid < nC) grid = nC;
    // programmatic dependent launch: the blocks come up while the previous kernel drains and
    // wait for it (grid_dependency_wait) before touching memory
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kTmaThreads);
    cfg.dynamicSmemBytes = S::SMEM;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, xmap, a.w, a.bias, static_cast<T *>(a.y), a.lengths, static_cast<int>(a.B),
                              static_cast<int>(a.T), static_cast<int>(a.C), a.pad_left, a.flip, nT, nC,
                              static_cast<int>(ntiles));
}

// Packed sequences: x and y [N][C], item b on rows offsets[b] .. offsets[b+1]-1.  The tensor
// map views x as one item of N frames; at most kOrderMaxItems items per launch (the run table
// lives in shared memory), so larger batches go in slices of consecutive items.
template <typename T, int V, int K>
cudaError_t launch_tma_packed(const Conv1dArgs &a, const int32_t *offsets, cudaStream_t s) {
    using S = TmaShape<T, V, K>;
    auto kern = conv1d_fwd_tma_kernel<T, V, K, true>;
    const int smem = S::SMEM + static_cast<int>((3 * kOrderMaxItems + 1) * sizeof(int));
    const cudaError_t attr = ensure_smem_attr(reinterpret_cast<const void *>(kern), smem);
    if (attr != cudaSuccess) return attr;
    const int nC = static_cast<int>((a.C + S::CT - 1) / S::CT);
    CUtensorMap xmap;
    const cudaError_t me = make_act_map(&xmap, a.x, dtype_code<T>(), 1, a.T, a.C, S::CT, S::ROWS);
    if (me != cudaSuccess) return me;
    // every block deals runs of its channel tile; the grid is a multiple of nC
    int64_t grid = static_cast<int64_t>(sm_count()) * kTmaBlocks;
    const int64_t runs_max = (a.T + S::TT - 1) / S::TT + a.B;  // at most one partial run per item
    if (grid > runs_max * nC) grid = runs_max * nC;
    grid = grid / nC * nC;
    if (grid < nC) grid = nC;
    for (int64_t b0 = 0; b0 < a.B; b0 += kOrderMaxItems) {
        const int nb = static_cast<int>(a.B - b0 < kOrderMaxItems ? a.B - b0 : kOrderMaxItems);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(grid));
        cfg.blockDim = dim3(kTmaThreads);
        cfg.dynamicSmemBytes = static_cast<size_t>(smem);
        cfg.stream = s;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        at[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, xmap, a.w, a.bias, static_cast<T *>(a.y), offsets + b0,
                                                 nb, static_cast<int>(a.T), static_cast<int>(a.C), a.pad_left, a.flip,
                                                 0, nC, 0);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// The pipelined kernel copies whole frame rows in 16-byte units: C * sizeof(T) a multiple of
// 16 and x 16-byte aligned.  Frame and item indices are 32-bit there.
template <typename T>
bool tma_ok(const Conv1dArgs &a) {
    return (a.C * static_cast<int64_t>(sizeof(T))) % 16 == 0 && reinterpret_cast<uintptr_t>(a.x) % 16 == 0 &&
           a.T < (1LL << 30) && a.B < (1LL << 30);
}

template <typename T, int V>
cudaError_t dispatch_k(const Conv1dArgs &a, cudaStream_t s) {
    if constexpr (V >= 2) {
        if (tma_ok<T>(a)) {
            switch (a.K) {
                case 1: return launch_tma<T, V, 1>(a, s);
                case 2: return launch_tma<T, V, 2>(a, s);
                case 3: return launch_tma<T, V, 3>(a, s);
                case 4: return launch_tma<T, V, 4>(a, s);
                case 5: return launch_tma<T, V, 5>(a, s);
                case 7: return launch_tma<T, V, 7>(a, s);
                case 9: return launch_tma<T, V, 9>(a, s);
                default: break;
            }
            if constexpr (V == 2 || V == 4) {
                if (a.K == 15) return launch_tma<T, V, 15>(a, s);
            }
        }
    }
    switch (a.K) {
        case 1: return launch_vec_k<T, V, 1>(a, s);
        case 2: return launch_vec_k<T, V, 2>(a, s);
        case 3: return launch_vec_k<T, V, 3>(a, s);
        case 4: return launch_vec_k<T, V, 4>(a, s);
        case 5: return launch_vec_k<T, V, 5>(a, s);
        case 7: return launch_vec_k<T, V, 7>(a, s);
        case 9: return launch_vec_k<T, V, 9>(a, s);
        default: break;
    }
    if constexpr (V <= 2) {
        if (a.K == 15) return launch_vec_k<T, V, 15>(a, s);
    }
    return launch_vec_anyk<T, (V > 2 ? 2 : V)>(a, s);
}

template <typename T>
cudaError_t dispatch_dtype(const Conv1dArgs &a, cudaStream_t s) {
    // 4 bf16 channels (8 bytes) per thread up to K = 9, and for K = 15 on the pipelined kernel with
    // 8 frames per thread (26.0 against 27.9 us for pairs at 32x750x1024); pairs for other wide
    // kernels and for float32 (8 bytes), which keeps the register window under 128 registers.
    if constexpr (sizeof(T) == 2) {
#ifdef DW_FWD_V8
        if (a.vec_width >= 8 && a.K <= 9) return dispatch_k<T, 8>(a, s);
#endif
        if (a.vec_width >= 4 && (a.K <= 9 || (a.K == 15 && tma_ok<T>(a)))) return dispatch_k<T, 4>(a, s);
    }
    if (a.vec_width >= 2) return dispatch_k<T, 2>(a, s);
    return dispatch_k<T, 1>(a, s);
}

template <typename T>
cudaError_t dispatch_packed(const Conv1dArgs &a, const int32_t *offsets, cudaStream_t s) {
    if (tma_ok<T>(a) && a.vec_width >= 2) {
        if constexpr (sizeof(T) == 2) {
            if (a.vec_width >= 4) {
                switch (a.K) {
                    case 1: return launch_tma_packed<T, 4, 1>(a, offsets, s);
                    case 2: return launch_tma_packed<T, 4, 2>(a, offsets, s);
                    case 3: return launch_tma_packed<T, 4, 3>(a, offsets, s);
                    case 4: return launch_tma_packed<T, 4, 4>(a, offsets, s);
                    case 5: return launch_tma_packed<T, 4, 5>(a, offsets, s);
                    case 7: return launch_tma_packed<T, 4, 7>(a, offsets, s);
                    case 9: return launch_tma_packed<T, 4, 9>(a, offsets, s);
                    default: break;
                }
            }
        }
        switch (a.K) {
            case 1: return launch_tma_packed<T, 2, 1>(a, offsets, s);
            case 2: return launch_tma_packed<T, 2, 2>(a, offsets, s);
            case 3: return launch_tma_packed<T, 2, 3>(a, offsets, s);
            case 4: return launch_tma_packed<T, 2, 4>(a, offsets, s);
            case 5: return launch_tma_packed<T, 2, 5>(a, offsets, s);
            case 7: return launch_tma_packed<T, 2, 7>(a, offsets, s);
            case 9: return launch_tma_packed<T, 2, 9>(a, offsets, s);
            case 15: return launch_tma_packed<T, 2, 15>(a, offsets, s);
            default: break;
        }
    }
    const int V = a.vec_width >= 2 ? 2 : 1;
    const int nCV = static_cast<int>(a.C / V);
    const int64_t grid = (a.T * nCV + 255) / 256;
    if (grid > kMaxGrid) return cudaErrorInvalidConfiguration;
#define DW_PK(VV)                                                                                              \
    conv1d_fwd_packed_kernel<T, VV><<<static_cast<unsigned>(grid), 256, 0, s>>>(                               \
        static_cast<const T *>(a.x), a.w, a.bias, static_cast<T *>(a.y), offsets, static_cast<int>(a.B),       \
        static_cast<int>(a.T), static_cast<int>(a.C), a.K, a.pad_left, a.flip, nCV)
    if (V == 2) DW_PK(2);
    else DW_PK(1);
#undef DW_PK
    return cudaGetLastError();
}

}  // namespace

cudaError_t conv1d_fwd_packed_launch(const Conv1dArgs &a, const int32_t *offsets, cudaStream_t s) {
    if (a.B == 0 || a.T == 0) return cudaSuccess;
    return with_dtype(a.dtype, [&](auto tag) { return dispatch_packed<decltype(tag)>(a, offsets, s); });
}

unsigned int conv1d_fwd_take_error() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, dw_device_error_flag, sizeof(v)) != cudaSuccess) return 0;
    if (v) cudaMemcpyToSymbol(dw_device_error_flag, &zero, sizeof(zero));
    return v;
}

cudaError_t conv1d_fwd_launch(const Conv1dArgs &a, cudaStream_t s) {
    if (a.B == 0 || a.T == 0) return cudaSuccess;
    return with_dtype(a.dtype, [&](auto tag) { return dispatch_dtype<decltype(tag)>(a, s); });
}

}  // namespace dwk
