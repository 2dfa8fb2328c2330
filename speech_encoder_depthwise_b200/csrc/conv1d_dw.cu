// Weight and bias gradients of the depthwise conv1d, channels-last [B][T][C].
//
//   dW[k,c]  = sum_{b,t} dz[b,t,c] * xpad[b,t+k,c]
//   dbias[c] = sum_{b,t} dz[b,t,c],          dz[b,t,c] = [t < len_b] dy[b,t,c]
//
// The backward of the depthwise kernel with fused masking and padding (NeMo PR #16114,
// "Use Fused Kernels for Depthwise Striding Subsampler", section "What does this PR do ?"),
// kept deterministic as that PR's "honor deterministic path" commit asks: float32 sums in a
// fixed order, no atomics.
//
// Two launches:
//  1. partial kernel, grid (G, channel tiles), thread-block clusters of 8 along G.  A thread
//     owns V channels and walks R frames of each (item, frame-run) unit it is dealt (static
//     round robin over units, so the order of every sum is fixed).  It keeps K+1 float32
//     accumulator pairs in registers, reading each dy frame once and each x frame once per
//     run (halo frames re-read from L1/L2).  The block then sums its rows in shared memory,
//     and the 8 blocks of a cluster sum each other's results through distributed shared
//     memory, so only G/8 partial rows [K+1][C] reach the workspace.
//  2. finalize kernel: dW[k][c] and dbias[c] = the partial rows added in row order.
// Widths without a specialisation run in passes of 8 taps over the same data.
#include <cooperative_groups.h>
#include <type_traits>

#include "dw_internal.h"

namespace cg = cooperative_groups;

namespace dwk {

constexpr int kDwThreads = 256;
constexpr int kDwCluster = 8;
constexpr int kDwTapBlock = 8;   // taps per pass for widths without a specialisation
constexpr int kDwMaxRows = 256;  // partial rows at most (blocks, or clusters, per channel tile)
constexpr int kDwMaxRows16 = 16; // partial rows of the register-tiled kernel

template <typename T, int V, int KB, int R>
__global__ void __cluster_dims__(kDwCluster, 1, 1) __launch_bounds__(kDwThreads, 2)
conv1d_dw_partial_kernel(const T *__restrict__ x, const T *__restrict__ dy,
                         const int32_t *__restrict__ lengths, float *__restrict__ partials,
                         int64_t B, int64_t Tn, int C, int K, int k_off, int pad_left, int TX,
                         int nTC, int with_bias) {
    extern __shared__ float smem[];  // [TY][KB+1][CT]
    constexpr int NP = Pairs<V>::n;
    const int tx = threadIdx.x % TX, ty = threadIdx.x / TX;
    const int TY = blockDim.x / TX;
    const int CT = TX * V;
    const int g = blockIdx.x, G = gridDim.x;
    const int ct = blockIdx.y;
    const int c0 = (ct * TX + tx) * V;
    const bool active = c0 < C;
    const uint32_t rs = static_cast<uint32_t>(C) * sizeof(T);

    float2 acc[KB][NP], accb[NP];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        accb[p] = make_float2(0.f, 0.f);
#pragma unroll
        for (int k = 0; k < KB; ++k) acc[k][p] = make_float2(0.f, 0.f);
    }

    if (active) {
        const int64_t units = B * nTC;
        const int64_t TU = static_cast<int64_t>(TY) * R;
        for (int64_t u = g; u < units; u += G) {
            const int64_t b = u / nTC;
            const int64_t t0 = (u % nTC) * TU + static_cast<int64_t>(ty) * R;
            const int64_t L = clamp_len(lengths, b, Tn);
            if (t0 >= L) continue;
            const char *xi = reinterpret_cast<const char *>(x + b * Tn * C + c0);
            const char *di = reinterpret_cast<const char *>(dy + b * Tn * C + c0);
            const int64_t j0 = t0 + k_off - pad_left;  // x frame paired with dz[t0] through tap k_off
            Vec<T, V> rdy[R], rx[R + KB - 1];
            if (t0 + R <= L && j0 >= 0 && j0 + R + KB - 1 <= L) {  // every frame of the run is valid
                const char *dp = di + t0 * rs;
                const char *xp = xi + j0 * rs;
#pragma unroll
                for (int r = 0; r < R; ++r) rdy[r].load(reinterpret_cast<const T *>(dp + static_cast<uint32_t>(r) * rs));
#pragma unroll
                for (int i = 0; i < R + KB - 1; ++i)
                    rx[i].load(reinterpret_cast<const T *>(xp + static_cast<uint32_t>(i) * rs));
            } else {
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    if (t0 + r < L) rdy[r].load(reinterpret_cast<const T *>(di + (t0 + r) * rs));
                    else rdy[r].zero();
                }
#pragma unroll
                for (int i = 0; i < R + KB - 1; ++i) {
                    const int64_t j = j0 + i;
                    if (j >= 0 && j < L) rx[i].load(reinterpret_cast<const T *>(xi + j * rs));
                    else rx[i].zero();
                }
            }
            float2 dz[R][NP];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                rdy[r].to_f2(dz[r]);
#pragma unroll
                for (int p = 0; p < NP; ++p) {
                    accb[p].x += dz[r][p].x;
                    accb[p].y += dz[r][p].y;
                }
            }
            // x frame i meets dz[r] through tap k = i - r
#pragma unroll
            for (int i = 0; i < R + KB - 1; ++i) {
                float2 xf[NP];
                rx[i].to_f2(xf);
#pragma unroll
                for (int k = 0; k < KB; ++k) {
                    const int r = i - k;
                    if (r >= 0 && r < R) {
#pragma unroll
                        for (int p = 0; p < NP; ++p) acc[k][p] = ffma2(dz[r][p], xf[p], acc[k][p]);
                    }
                }
            }
        }
    }

    // block: rows -> shared memory -> sum over rows in row order (into row 0)
    const int E = (KB + 1) * CT;
    float *mine = smem + static_cast<size_t>(ty) * E;
#pragma unroll
    for (int k = 0; k <= KB; ++k) {
#pragma unroll
        for (int p = 0; p < NP; ++p) {
            const float2 v = (k < KB) ? acc[k][p] : accb[p];
            if (2 * p < V) mine[k * CT + tx * V + 2 * p] = v.x;
            if (2 * p + 1 < V) mine[k * CT + tx * V + 2 * p + 1] = v.y;
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        float s = smem[e];
        for (int r = 1; r < TY; ++r) s += smem[static_cast<size_t>(r) * E + e];
        smem[e] = s;
    }

    // cluster: block rank q sums entries [q*chunk, (q+1)*chunk) over the ranks in rank order
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    const int nrank = static_cast<int>(cluster.num_blocks());
    const int rank = static_cast<int>(cluster.block_rank());
    const int chunk = (E + nrank - 1) / nrank;
    const int64_t prow = g / nrank;
    for (int e = rank * chunk + threadIdx.x; e < min(E, (rank + 1) * chunk); e += blockDim.x) {
        float s = 0.f;
        for (int q = 0; q < nrank; ++q) s += cluster.map_shared_rank(smem, q)[e];
        const int kk = e / CT;
        const int64_t c = static_cast<int64_t>(ct) * CT + (e % CT);
        if (c >= C) continue;
        if (kk == KB) {
            if (with_bias) partials[(prow * (K + 1) + K) * C + c] = s;
        } else if (k_off + kk < K) {
            partials[(prow * (K + 1) + k_off + kk) * C + c] = s;
        }
    }
    cluster.sync();  // keep this block's shared memory alive until every rank has read it
}

// ---------------------------------------------------------------------------------------
// Pipelined variant (16-byte frame rows, specialised K): grid (G, channel tiles), 2 blocks per
// SM, clusters of 1-8 blocks along G chosen at launch.  Warp 0 streams each unit into a
// kDwStages-deep shared-memory ring with two tensor copies (x: the TT frames plus the halo,
// dy: the TT frames), counted in bytes on the stage's "full" mbarrier; 8 consumer warps
// accumulate dW/dbias for their R frames in registers across all units the block is dealt,
// then release the stage on its "empty" mbarrier.  At the end every warp (the producer adds
// zeros) joins the block and cluster reductions of the register-tiled kernel above.
// ---------------------------------------------------------------------------------------
#ifndef DW_DW_CONSUMERS
#define DW_DW_CONSUMERS 8
#endif
#ifndef DW_DW_R
#define DW_DW_R 8
#endif
#ifndef DW_DW_STAGES
#define DW_DW_STAGES 3
#endif
#ifndef DW_DW_BLOCKS
#define DW_DW_BLOCKS 2
#endif
#ifndef DW_DW_ORDERED
#define DW_DW_ORDERED 1
#endif
constexpr int kDwConsumers = DW_DW_CONSUMERS;  // consumer warps per block
constexpr int kDwR = DW_DW_R;                  // frames per consumer thread per unit
constexpr int kDwStages = DW_DW_STAGES;        // shared-memory ring depth
constexpr int kDwBlocks = DW_DW_BLOCKS;        // resident blocks per SM

// FUSED: the same pass also computes the data gradient, so the dy tile carries K-1 halo rows
// (the dx correlation reads dy frames s + pad_left - k).  Its threads hold two sets of
// accumulators, so it runs one block per SM (more registers per thread).
template <typename T, int V, int KB, bool FUSED = false>
struct DwTmaShape {
    static constexpr int CONS = kDwConsumers;  // consumer warps
    static constexpr int R = kDwR;             // frames per consumer thread per unit
    static constexpr int THREADS = 32 * (1 + CONS);
    static constexpr int CT = 32 * V;
    static constexpr int TT = CONS * R;
    static constexpr int XROWS = TT + KB - 1;
    static constexpr int DROWS = FUSED ? TT + KB - 1 : TT;
    static constexpr int ROWB = CT * static_cast<int>(sizeof(T));
    static constexpr int STAGE_BYTES = (XROWS + DROWS) * ROWB;
    static constexpr int RED_BYTES = CONS * (KB + 1) * CT * 4;
    static constexpr int BODY = (kDwStages * STAGE_BYTES > RED_BYTES) ? kDwStages * STAGE_BYTES : RED_BYTES;
    static constexpr int SMEM = 128 + BODY;  // plus the tile-order tables, sized at launch
};

// Used for the one-pass data + weight gradient (FUSED) and for batches of more than
// kOrderMaxItems items; the span-balanced kernel below takes every other pipelined case.
template <typename T, int V, int KB, bool FUSED = false>
__global__ void __launch_bounds__(DwTmaShape<T, V, KB, FUSED>::THREADS, FUSED ? 1 : kDwBlocks)
conv1d_dw_tma_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap dmap,
                     const int32_t *__restrict__ lengths, float *__restrict__ partials, int B, int Tn, int C, int K,
                     int k_off, int pad_left, int nT, int with_bias, int ordered, const float *__restrict__ wgt,
                     T *__restrict__ dx) {
    using S = DwTmaShape<T, V, KB, FUSED>;
    const int padR = K - 1 - pad_left;  // the data gradient's left pad
    constexpr int NP = Pairs<V>::n;
    constexpr int R = S::R;
    launch_dependents();  // the finalize may be scheduled now; it waits for this grid to finish
    extern __shared__ __align__(128) unsigned char smem_raw[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem_raw);
    uint64_t *empty = full + kDwStages;
    unsigned char *stages = smem_raw + 128;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int g = blockIdx.x, G = gridDim.x, ct = blockIdx.y;
    const int c0 = ct * S::CT;
    // the frame-runs to walk: only the valid ones (first frame < len_b), in balanced order, or
    // every (item, run) pair when B is too large for the order's shared-memory tables
    int *ord_mem = reinterpret_cast<int *>(stages + S::BODY);
    TileOrder order{ord_mem, ord_mem + (B + 1), ord_mem + 2 * (B + 1), B, nT, 1, 0};
    grid_dependency_wait();  // launched programmatically: the previous kernel's writes are visible after this
    if (ordered) order.build(ord_mem, ord_mem + (B + 1), ord_mem + 2 * (B + 1), lengths, Tn, S::TT);
    if (threadIdx.x == 0) {
        for (int i = 0; i < kDwStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], S::CONS);
        }
        fence_barrier_init();
    }
    __syncthreads();
    if (ordered) order.V = order.pv[B];
    // the fused pass also walks the wholly masked units: their dx frames are written as zeros
    const int units = (ordered && !FUSED) ? order.V : B * nT;
    auto unit_at = [&](int u, int &b, int &t0, int &L) {
        if (ordered) {
            int tt, ctd;
            order.map(u, b, tt, ctd, L);
            t0 = tt * S::TT;
        } else {
            b = u / nT;
            t0 = (u % nT) * S::TT;
            L = static_cast<int>(clamp_len(lengths, b, Tn));
        }
    };
    float2 acc[KB][NP], accb[NP];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        accb[p] = make_float2(0.f, 0.f);
#pragma unroll
        for (int k = 0; k < KB; ++k) acc[k][p] = make_float2(0.f, 0.f);
    }
    bool ok = true;

    if (warp == 0) {  // producer warp: one elected lane, two tensor copies (x with halo, dy) per unit
        if (lane == 0) {
            prefetch_tmap(&xmap);
            prefetch_tmap(&dmap);
        }
        int it = 0;
        for (int u = g; u < units && ok; u += G, ++it) {
            const int s = it % kDwStages;
            const uint32_t ph = (it / kDwStages) & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(&empty[s], ph ^ 1));
            if (!ok) break;
            if (lane == 0) {
                int b, t0, L;
                if (ordered || it >= kDwStages) {
                    unit_at(u, b, t0, L);
                } else {  // the first ring-full is issued before any length is read
                    b = u / nT;
                    t0 = (u % nT) * S::TT;
                    L = Tn;
                }
                if (t0 < L) {  // frames before 0 or past T arrive as zeros; [L, T) is masked by the consumers
                    unsigned char *st = stages + static_cast<size_t>(s) * S::STAGE_BYTES;
                    mbar_arrive_expect_tx(&full[s], S::STAGE_BYTES);
                    tma_load_3d(st, &xmap, c0, t0 + k_off - pad_left, b, &full[s]);
                    tma_load_3d(st + S::XROWS * S::ROWB, &dmap, c0, FUSED ? t0 - padR : t0, b, &full[s]);
                } else {
                    mbar_arrive(&full[s]);  // a wholly masked unit: nothing to read
                }
            }
            __syncwarp();
        }
    } else {  // consumer warp cw computes frames [t0 + cw R, t0 + cw R + R) of every unit
        const int cw = warp - 1;
        const bool active = c0 + lane * V < C;
        float2 wv[FUSED ? KB : 1][NP];  // the data gradient's taps, this thread's channels
        if constexpr (FUSED) {
            if (active) {
#pragma unroll
                for (int k = 0; k < KB; ++k) load_param<V>(wgt + static_cast<int64_t>(k) * C + c0 + lane * V, wv[k]);
            }
        }
        int it = 0;
        for (int u = g; u < units && ok; u += G, ++it) {
            const int s = it % kDwStages;
            const uint32_t ph = (it / kDwStages) & 1;
            int b, t0, L;
            unit_at(u, b, t0, L);
            ok = __all_sync(0xffffffffu, mbar_wait(&full[s], ph));
            if (!ok) break;
            const int tg = t0 + cw * R;
            if constexpr (FUSED) {
                // data gradient: dx[s] = [s < len_b] sum_k dz[s + pad_left - k] w[k] for this thread's
                // R frames; tile row i holds dy frame tg - padR + i
                if (active && tg < Tn) {
                    T *dxp = dx + (static_cast<int64_t>(b) * Tn + tg) * C + c0 + lane * V;
                    const int nr = Tn - tg < R ? Tn - tg : R;
                    if (tg < L) {
                        const unsigned char *zp = stages + static_cast<size_t>(s) * S::STAGE_BYTES +
                                                  lane * V * sizeof(T) + (S::XROWS + cw * R) * S::ROWB;
                        const int f0 = tg - padR;
                        auto dxrun = [&](auto check) {
                            constexpr bool CHECK = decltype(check)::value;
                            float2 da[R][NP];
#pragma unroll
                            for (int r = 0; r < R; ++r)
#pragma unroll
                                for (int p = 0; p < NP; ++p) da[r][p] = make_float2(0.f, 0.f);
#pragma unroll
                            for (int i = 0; i < R + KB - 1; ++i) {
                                Vec<T, V> v;
                                v.r = *reinterpret_cast<const decltype(v.r) *>(zp + i * S::ROWB);
                                if constexpr (CHECK) {
                                    if (f0 + i < 0 || f0 + i >= L) v.zero();
                                }
                                float2 z[NP];
                                v.to_f2(z);
#pragma unroll
                                for (int k = 0; k < KB; ++k) {
                                    const int r = i - (KB - 1) + k;
                                    if (r >= 0 && r < R) {
#pragma unroll
                                        for (int p = 0; p < NP; ++p) da[r][p] = ffma2(z[p], wv[k][p], da[r][p]);
                                    }
                                }
                            }
#pragma unroll
                            for (int r = 0; r < R; ++r) {
                                if (r < nr) {
                                    if (CHECK && tg + r >= L) Vec<T, V>::store_zero(dxp + static_cast<int64_t>(r) * C);
                                    else Vec<T, V>::store(dxp + static_cast<int64_t>(r) * C, da[r]);
                                }
                            }
                        };
                        if (f0 >= 0 && f0 + R + KB - 1 <= L && nr == R) dxrun(std::false_type{});
                        else dxrun(std::true_type{});
                    } else {
                        for (int r = 0; r < nr; ++r) Vec<T, V>::store_zero(dxp + static_cast<int64_t>(r) * C);
                    }
                }
            }
            if (active && tg < L) {
                const unsigned char *st = stages + static_cast<size_t>(s) * S::STAGE_BYTES + lane * V * sizeof(T);
                const unsigned char *dp = st + (S::XROWS + (FUSED ? padR : 0) + cw * R) * S::ROWB;
                const unsigned char *xp = st + (cw * R) * S::ROWB;
                const int jb = tg + k_off - pad_left;  // frame of this thread's first x row
                // CHECK = false: every dy and x row of the run is inside [0, len_b)
                auto run = [&](auto check) {
                    constexpr bool CHECK = decltype(check)::value;
                    float2 dz[R][NP];
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        Vec<T, V> v;
                        v.r = *reinterpret_cast<const decltype(v.r) *>(dp + r * S::ROWB);
                        if constexpr (CHECK) {
                            if (tg + r >= L) v.zero();
                        }
                        v.to_f2(dz[r]);
#pragma unroll
                        for (int p = 0; p < NP; ++p) {
                            accb[p].x += dz[r][p].x;
                            accb[p].y += dz[r][p].y;
                        }
                    }
#pragma unroll
                    for (int i = 0; i < R + KB - 1; ++i) {
                        Vec<T, V> v;
                        v.r = *reinterpret_cast<const decltype(v.r) *>(xp + i * S::ROWB);
                        if constexpr (CHECK) {
                            if (jb + i < 0 || jb + i >= L) v.zero();
                        }
                        float2 xf[NP];
                        v.to_f2(xf);
#pragma unroll
                        for (int k = 0; k < KB; ++k) {
                            const int r = i - k;
                            if (r >= 0 && r < R) {
#pragma unroll
                                for (int p = 0; p < NP; ++p) acc[k][p] = ffma2(dz[r][p], xf[p], acc[k][p]);
                            }
                        }
                    }
                };
                if (tg + R <= L && jb >= 0 && jb + R + KB - 1 <= L) run(std::false_type{});
                else run(std::true_type{});
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
    }
    // every warp has left the pipeline; the stage memory now holds the block reduction
    __syncthreads();
    const int E = (KB + 1) * S::CT;
    float *red = reinterpret_cast<float *>(stages);
    if (warp > 0) {
        float *mine = red + static_cast<size_t>(warp - 1) * E;
#pragma unroll
        for (int k = 0; k <= KB; ++k) {
#pragma unroll
            for (int p = 0; p < NP; ++p) {
                const float2 v = (k < KB) ? acc[k][p] : accb[p];
                if (2 * p < V) mine[k * S::CT + lane * V + 2 * p] = v.x;
                if (2 * p + 1 < V) mine[k * S::CT + lane * V + 2 * p + 1] = v.y;
            }
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        float sum = red[e];
        for (int r = 1; r < S::CONS; ++r) sum += red[static_cast<size_t>(r) * E + e];
        red[e] = sum;
    }
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    const int nrank = static_cast<int>(cluster.num_blocks());
    const int rank = static_cast<int>(cluster.block_rank());
    const int chunk = (E + nrank - 1) / nrank;
    const int64_t prow = g / nrank;
    for (int e = rank * chunk + threadIdx.x; e < min(E, (rank + 1) * chunk); e += blockDim.x) {
        float sum = 0.f;
        for (int q = 0; q < nrank; ++q) sum += cluster.map_shared_rank(red, q)[e];
        const int kk = e / S::CT;
        const int64_t c = static_cast<int64_t>(c0) + (e % S::CT);
        if (c >= C) continue;
        if (kk == KB) {
            if (with_bias) partials[(prow * (K + 1) + K) * C + c] = sum;
        } else if (k_off + kk < K) {
            partials[(prow * (K + 1) + k_off + kk) * C + c] = sum;
        }
    }
    cluster.sync();
}

// ---------------------------------------------------------------------------------------
// Span-balanced variant (the default for 16-byte rows, specialised K and up to kOrderMaxItems
// items): grid (G, channel tiles), kDwBlocks blocks per SM, no clusters.  The valid frames of
// all items (t < len_b; in a packed batch every row of every sequence), item after item, form
// one sequence of V frames per channel tile: block j of the tile's G blocks takes the contiguous
// span [V j / G, V (j+1) / G) of it, cut into tiles of at most TT frames that never cross an
// item, so every block reads the same number of frames to within one.  The producer copies a
// tile of n frames as ceil((n + K - 1) / SB) tensor boxes of x (halo included) and ceil(n / SB)
// boxes of dy, SB rows each, so a short tile reads little beyond its own rows.  The consumers
// accumulate dW/dbias for their R frames of every tile in registers, as in the kernel above.  At
// the end the block adds its warps' sums in a fixed order through shared memory and writes one
// partial row; the finalize kernel adds the G rows in a fixed order (no atomics, reproducible
// for given sizes on a given GPU model).  The lengths are prefetched into L2 before the
// dependency wait: a prefetch only warms the cache, so writes of the previous kernel are seen.
// ---------------------------------------------------------------------------------------
constexpr int kDwSB = 8;  // rows per tensor box

// FUSED: the same pass also computes the data gradient dx[s] = [s < len_b] sum_k dz[s + pad_left
// - k] w[k] of every valid frame, so the dy tile carries the K - 1 halo rows too; each block also
// writes the zeros of its share of the masked frames' dx (an equal share of the sequence of
// masked frames, len_b <= t < T), while its first tiles load.  Two sets of accumulators per
// thread: one block per SM.
template <typename T, int V, int KB, bool FUSED = false>
struct DwSpanShape {
    static constexpr int CONS = kDwConsumers;
    static constexpr int R = kDwR;
    static constexpr int THREADS = 32 * (1 + CONS);
    static constexpr int CT = 32 * V;
    static constexpr int TT = CONS * R;
    static constexpr int ROWB = CT * static_cast<int>(sizeof(T));
    static constexpr int XROWS = (TT + KB - 1 + kDwSB - 1) / kDwSB * kDwSB;
    static constexpr int DROWS = ((FUSED ? TT + KB - 1 : TT) + kDwSB - 1) / kDwSB * kDwSB;
    static constexpr int BOX_BYTES = kDwSB * ROWB;
    static constexpr int STAGE_BYTES = (XROWS + DROWS) * ROWB;
    static constexpr int STAGES = FUSED ? 5 : kDwStages;  // one block per SM when fused: a deeper ring
    static constexpr int RED_BYTES = CONS * (KB + 1) * CT * 4;
    static constexpr int BODY = (STAGES * STAGE_BYTES > RED_BYTES) ? STAGES * STAGE_BYTES : RED_BYTES;
    static constexpr int SMEM = 128 + BODY;  // plus the item tables, sized at launch
};

// PACKED: x and dy [N][C], `lengths` = offsets[B+1] (clamped into [0, N], non-decreasing), Tn = N.
template <typename T, int V, int KB, bool PACKED, bool FUSED = false>
__global__ void __launch_bounds__(DwSpanShape<T, V, KB, FUSED>::THREADS, FUSED ? 1 : kDwBlocks)
conv1d_dw_span_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap dmap,
                      const int32_t *__restrict__ lengths, float *__restrict__ partials, int B, int Tn, int C,
                      int K, int k_off, int pad_left, int with_bias, const float *__restrict__ wgt,
                      T *__restrict__ dx) {
    static_assert(!(PACKED && FUSED), "the one-pass backward takes padded batches");
    using S = DwSpanShape<T, V, KB, FUSED>;
    const int padR = K - 1 - pad_left;  // the data gradient's left pad
    constexpr int NP = Pairs<V>::n;
    constexpr int R = S::R;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem_raw);
    uint64_t *empty = full + S::STAGES;
    unsigned char *stages = smem_raw + 128;
    // per item: valid frames before it (pv), its valid frames (plen), its first row (pst) and
    // (FUSED) its masked frames before it (pm)
    int *pv = reinterpret_cast<int *>(stages + S::BODY);
    int *plen = pv + (B + 1), *pst = plen + B, *pm = pst + B;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int jj = static_cast<int>(blockIdx.x), G = static_cast<int>(gridDim.x), ct = static_cast<int>(blockIdx.y);
    const int c0 = ct * S::CT;
    launch_dependents();  // the finalize may be scheduled now; it waits for this grid to finish
    if (threadIdx.x == 0) {
        for (int i = 0; i < S::STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], S::CONS);
        }
        fence_barrier_init();
    }
    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&xmap);
            prefetch_tmap(&dmap);
        }
        if (lengths != nullptr)  // one 128-byte line per 32 entries
            for (int i = lane * 32; i < (PACKED ? B + 1 : B); i += 32 * 32) prefetch_l2(lengths + i);
    }
    grid_dependency_wait();  // launched programmatically: the previous kernel's writes are visible after this
    for (int bb = static_cast<int>(threadIdx.x); bb < B; bb += static_cast<int>(blockDim.x)) {
        int s0 = 0, L;
        if constexpr (PACKED) {
            s0 = __ldg(lengths + bb);
            int e = __ldg(lengths + bb + 1);
            s0 = s0 < 0 ? 0 : (s0 > Tn ? Tn : s0);
            e = e < s0 ? s0 : (e > Tn ? Tn : e);
            L = e - s0;
        } else {
            L = static_cast<int>(clamp_len(lengths, bb, Tn));
        }
        plen[bb] = L;
        pst[bb] = s0;
    }
    __syncthreads();
    if (warp == 0) {  // prefix sums of the valid (and, FUSED, of the masked) frames
        int run = 0, run_m = 0;
        if (lane == 0) {
            pv[0] = 0;
            if (FUSED) pm[0] = 0;
        }
        for (int base = 0; base < B; base += 32) {
            const int bb = base + lane;
            int v = bb < B ? plen[bb] : 0, m = bb < B ? Tn - plen[bb] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, v, o), tm = __shfl_up_sync(0xffffffffu, m, o);
                if (lane >= o) {
                    v += t;
                    m += tm;
                }
            }
            if (bb < B) {
                pv[bb + 1] = run + v;
                if (FUSED) pm[bb + 1] = run_m + m;
            }
            run += __shfl_sync(0xffffffffu, v, 31);
            run_m += __shfl_sync(0xffffffffu, m, 31);
        }
    }
    __syncthreads();
    const int v_begin = static_cast<int>(static_cast<int64_t>(pv[B]) * jj / G);
    const int v_end = static_cast<int>(static_cast<int64_t>(pv[B]) * (jj + 1) / G);
    // the tile that starts at position p of the valid sequence: item b (advanced in place; items
    // without valid frames are skipped), its first frame t0 and its frame count n
    auto tile_at = [&](int p, int &b, int &t0, int &n) {
        while (pv[b + 1] <= p) ++b;
        t0 = p - pv[b];
        const int left = plen[b] - t0, span = v_end - p;
        n = left < span ? left : span;
        if (n > S::TT) n = S::TT;
    };
    float2 acc[KB][NP], accb[NP];
#pragma unroll
    for (int q = 0; q < NP; ++q) {
        accb[q] = make_float2(0.f, 0.f);
#pragma unroll
        for (int k = 0; k < KB; ++k) acc[k][q] = make_float2(0.f, 0.f);
    }

    if (warp == 0) {  // producer warp: one elected lane issues the tile's tensor boxes
        int b = v_begin < v_end ? TileOrder::find(pv, B, v_begin) : 0;
        int it = 0;
        for (int p = v_begin; p < v_end; ++it) {
            int t0, n;
            tile_at(p, b, t0, n);
            const int s = it % S::STAGES;
            const uint32_t ph = (it / S::STAGES) & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&empty[s], ph ^ 1))) break;
            if (lane == 0) {
                const int nbx = (n + KB - 1 + kDwSB - 1) / kDwSB;
                const int nby = ((FUSED ? n + KB - 1 : n) + kDwSB - 1) / kDwSB;
                unsigned char *st = stages + static_cast<size_t>(s) * S::STAGE_BYTES;
                mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>((nbx + nby) * S::BOX_BYTES));
                // padded: frames of item b of the [B][T][C] maps; packed: rows of the [1][N][C] maps.
                // FUSED: the dy rows start K-1-pad_left frames early (the data gradient's halo).
                const int r0 = PACKED ? pst[b] : 0, bi = PACKED ? 0 : b;
                const int d0 = r0 + t0 - (FUSED ? padR : 0);
                for (int i = 0; i < nbx; ++i)
                    tma_load_3d(st + i * S::BOX_BYTES, &xmap, c0, r0 + t0 + k_off - pad_left + i * kDwSB, bi, &full[s]);
                for (int i = 0; i < nby; ++i)
                    tma_load_3d(st + S::XROWS * S::ROWB + i * S::BOX_BYTES, &dmap, c0, d0 + i * kDwSB, bi, &full[s]);
            }
            __syncwarp();
            p += n;
        }
    } else {  // consumer warp cw: frames [t0 + cw R, t0 + cw R + R) of every tile
        const int cw = warp - 1;
        const bool active = c0 + lane * V < C;
        float2 wv[FUSED ? KB : 1][NP];  // the data gradient's taps, this thread's channels
        if constexpr (FUSED) {
            if (active) {
#pragma unroll
                for (int k = 0; k < KB; ++k) load_param<V>(wgt + static_cast<int64_t>(k) * C + c0 + lane * V, wv[k]);
            }
            // this block's share of the masked frames: dx zeros, issued while the first tiles load
            const int m_begin = static_cast<int>(static_cast<int64_t>(pm[B]) * jj / G);
            const int m_end = static_cast<int>(static_cast<int64_t>(pm[B]) * (jj + 1) / G);
            if (active && m_begin + cw < m_end) {
                int mb = TileOrder::find(pm, B, m_begin + cw);
                for (int m = m_begin + cw; m < m_end; m += S::CONS) {
                    while (pm[mb + 1] <= m) ++mb;
                    const int t = plen[mb] + (m - pm[mb]);
                    Vec<T, V>::store_zero(dx + (static_cast<int64_t>(mb) * Tn + t) * C + c0 + lane * V);
                }
            }
        }
        int b = v_begin < v_end ? TileOrder::find(pv, B, v_begin) : 0;
        int it = 0;
        for (int p = v_begin; p < v_end; ++it) {
            int t0, n;
            tile_at(p, b, t0, n);
            const int s = it % S::STAGES;
            const uint32_t ph = (it / S::STAGES) & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph))) break;
            const int tg = t0 + cw * R;   // this warp's first frame
            const int nr = n - cw * R;    // its frame count (R at most; none when <= 0)
            if constexpr (FUSED) {
                // data gradient of this warp's frames: dy tile row i holds frame tg - padR + i - cw R
                if (active && nr > 0) {
                    const int L = plen[b];
                    T *dxp = dx + (static_cast<int64_t>(b) * Tn + tg) * C + c0 + lane * V;
                    const unsigned char *zp = stages + static_cast<size_t>(s) * S::STAGE_BYTES + lane * V * sizeof(T) +
                                              (S::XROWS + cw * R) * S::ROWB;
                    const int f0 = tg - padR;  // frame of this warp's first dy row
                    auto dxrun = [&](auto check) {
                        constexpr bool CHECK = decltype(check)::value;
                        float2 da[R][NP];
#pragma unroll
                        for (int r = 0; r < R; ++r)
#pragma unroll
                            for (int q = 0; q < NP; ++q) da[r][q] = make_float2(0.f, 0.f);
#pragma unroll
                        for (int i = 0; i < R + KB - 1; ++i) {
                            Vec<T, V> v;
                            v.r = *reinterpret_cast<const decltype(v.r) *>(zp + i * S::ROWB);
                            if constexpr (CHECK) {  // frames outside [0, len_b), and rows past this warp's reach
                                if (f0 + i < 0 || f0 + i >= L || i >= nr + KB - 1) v.zero();
                            }
                            float2 z[NP];
                            v.to_f2(z);
#pragma unroll
                            for (int k = 0; k < KB; ++k) {
                                const int r = i - (KB - 1) + k;
                                if (r >= 0 && r < R) {
#pragma unroll
                                    for (int q = 0; q < NP; ++q) da[r][q] = ffma2(z[q], wv[k][q], da[r][q]);
                                }
                            }
                        }
#pragma unroll
                        for (int r = 0; r < R; ++r)
                            if (!CHECK || r < nr) Vec<T, V>::store(dxp + static_cast<int64_t>(r) * C, da[r]);
                    };
                    if (nr >= R && f0 >= 0 && f0 + R + KB - 1 <= L) dxrun(std::false_type{});
                    else dxrun(std::true_type{});
                }
            }
            if (active && nr > 0) {
                const int L = plen[b];
                const unsigned char *st = stages + static_cast<size_t>(s) * S::STAGE_BYTES + lane * V * sizeof(T);
                const unsigned char *dp = st + (S::XROWS + (FUSED ? padR : 0) + cw * R) * S::ROWB;
                const unsigned char *xp = st + (cw * R) * S::ROWB;
                const int jb = tg + k_off - pad_left;  // frame of this warp's first x row
                // CHECK = false: all R frames are this warp's and every x row is inside [0, len_b).
                // With CHECK, rows past this warp's frames (not loaded, or of the next warp) are
                // zeroed as well, so that nothing stale meets a zero dz.
                auto run = [&](auto check) {
                    constexpr bool CHECK = decltype(check)::value;
                    float2 dz[R][NP];
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        Vec<T, V> v;
                        v.r = *reinterpret_cast<const decltype(v.r) *>(dp + r * S::ROWB);
                        if constexpr (CHECK) {
                            if (r >= nr) v.zero();
                        }
                        v.to_f2(dz[r]);
#pragma unroll
                        for (int q = 0; q < NP; ++q) {
                            accb[q].x += dz[r][q].x;
                            accb[q].y += dz[r][q].y;
                        }
                    }
#pragma unroll
                    for (int i = 0; i < R + KB - 1; ++i) {
                        Vec<T, V> v;
                        v.r = *reinterpret_cast<const decltype(v.r) *>(xp + i * S::ROWB);
                        if constexpr (CHECK) {
                            if (jb + i < 0 || jb + i >= L || i >= nr + KB - 1) v.zero();
                        }
                        float2 xf[NP];
                        v.to_f2(xf);
#pragma unroll
                        for (int k = 0; k < KB; ++k) {
                            const int r = i - k;
                            if (r >= 0 && r < R) {
#pragma unroll
                                for (int q = 0; q < NP; ++q) acc[k][q] = ffma2(dz[r][q], xf[q], acc[k][q]);
                            }
                        }
                    }
                };
                if (nr >= R && jb >= 0 && jb + R + KB - 1 <= L) run(std::false_type{});
                else run(std::true_type{});
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            p += n;
        }
    }
    // every warp has left the pipeline; the stage memory now holds the block's sums, as channel
    // pairs (V is even here: 2 or 4 channels a thread)
    static_assert(V % 2 == 0, "pairs of channels");
    __syncthreads();
    const int E2 = (KB + 1) * S::CT / 2;
    float2 *red = reinterpret_cast<float2 *>(stages);
    if (warp > 0) {
        float2 *mine = red + static_cast<size_t>(warp - 1) * E2;
#pragma unroll
        for (int k = 0; k <= KB; ++k) {
#pragma unroll
            for (int q = 0; q < NP; ++q) mine[(k * S::CT + lane * V) / 2 + q] = (k < KB) ? acc[k][q] : accb[q];
        }
    }
    __syncthreads();
    for (int e = static_cast<int>(threadIdx.x); e < E2; e += static_cast<int>(blockDim.x)) {
        float2 sum = red[e];
#pragma unroll
        for (int r = 1; r < S::CONS; ++r) {
            const float2 t = red[static_cast<size_t>(r) * E2 + e];
            sum.x += t.x;
            sum.y += t.y;
        }
        const int kk = (2 * e) / S::CT;
        const int64_t c = static_cast<int64_t>(c0) + (2 * e) % S::CT;  // even; C is even on this path
        if (c >= C) continue;
        float *row = nullptr;
        if (kk == KB) {
            if (with_bias) row = partials + (static_cast<int64_t>(jj) * (K + 1) + K) * C;
        } else if (k_off + kk < K) {
            row = partials + (static_cast<int64_t>(jj) * (K + 1) + k_off + kk) * C;
        }
        if (row != nullptr) *reinterpret_cast<float2 *>(row + c) = sum;
    }
}

// dW[k][c] / dbias[c] = sum over the partial rows.  A block covers 32 consecutive (k, c) entries
// with 8 row groups: group r adds rows r, r+8, r+16, ... in order, then the 8 group sums are
// added in a fixed tree.  The order depends only on the row count, so results are reproducible.
__global__ void __launch_bounds__(256)
conv1d_dw_finalize_kernel(const float *__restrict__ partials, float *__restrict__ dw,
                          float *__restrict__ dbias, int Gp, int K, int64_t C) {
    __shared__ float red[8][33];
    launch_dependents();     // the next kernel may start its own set-up
    grid_dependency_wait();  // launched programmatically after the partial kernel
    const int col = threadIdx.x % 32, rg = threadIdx.x / 32;
    const int64_t E = static_cast<int64_t>(K + 1) * C;
    const int64_t e = static_cast<int64_t>(blockIdx.x) * 32 + col;
    float s = 0.f;
    if (e < E) {
#pragma unroll 4
        for (int g = rg; g < Gp; g += 8) s += __ldg(partials + static_cast<int64_t>(g) * E + e);
    }
    red[rg][col] = s;
    __syncthreads();
    if (rg == 0 && e < E) {
        const float t = ((red[0][col] + red[1][col]) + (red[2][col] + red[3][col])) +
                        ((red[4][col] + red[5][col]) + (red[6][col] + red[7][col]));
        const int64_t k = e / C, c = e % C;
        if (k < K) dw[k * C + c] = t;
        else if (dbias) dbias[c] = t;
    }
}

// The same sum for (K+1)*C a multiple of 4, with every load of a thread in flight at once: a
// block covers 64 consecutive entries (16 lanes x float4) with 16 row groups; group r loads rows
// r, r+16, r+32, ... (at most 16 per thread; G <= 256) and adds them in order, then the 16 group
// sums are added in a fixed tree.  Reproducible for a given row count.
constexpr int kFinGroups = 16;
__global__ void __launch_bounds__(256)
conv1d_dw_finalize4_kernel(const float *__restrict__ partials, float *__restrict__ dw,
                           float *__restrict__ dbias, int Gp, int K, int64_t C) {
    __shared__ float4 red[kFinGroups][16];
    launch_dependents();     // the next kernel may start its own set-up
    grid_dependency_wait();  // launched programmatically after the partial kernel
    const int lane = threadIdx.x % 16, rg = threadIdx.x / 16;
    const int64_t E4 = static_cast<int64_t>(K + 1) * C / 4;
    const int64_t e4 = static_cast<int64_t>(blockIdx.x) * 16 + lane;
    const float4 *p4 = reinterpret_cast<const float4 *>(partials);
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    if (e4 < E4) {
        float4 v[kDwMaxRows / kFinGroups];
#pragma unroll
        for (int i = 0; i < kDwMaxRows / kFinGroups; ++i) {
            const int g = rg + i * kFinGroups;
            v[i] = g < Gp ? __ldg(p4 + static_cast<int64_t>(g) * E4 + e4) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int i = 0; i < kDwMaxRows / kFinGroups; ++i) {
            s.x += v[i].x;
            s.y += v[i].y;
            s.z += v[i].z;
            s.w += v[i].w;
        }
    }
    red[rg][lane] = s;
    __syncthreads();
    if (rg == 0 && e4 < E4) {
        float4 t[kFinGroups];
#pragma unroll
        for (int r = 0; r < kFinGroups; ++r) t[r] = red[r][lane];
#pragma unroll
        for (int w = 1; w < kFinGroups; w <<= 1) {
#pragma unroll
            for (int r = 0; r + w < kFinGroups; r += 2 * w) {
                t[r].x += t[r + w].x;
                t[r].y += t[r + w].y;
                t[r].z += t[r + w].z;
                t[r].w += t[r + w].w;
            }
        }
        const float o[4] = {t[0].x, t[0].y, t[0].z, t[0].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int64_t e = 4 * e4 + q, k = e / C, c = e % C;
            if (k < K) dw[k * C + c] = o[q];
            else if (dbias) dbias[c] = o[q];
        }
    }
}

// dW / dbias from Gp partial rows [Gp][K+1][C] (programmatic dependent launch).
cudaError_t launch_finalize_rows(const float *partials, float *dw, float *dbias, int Gp, int K, int64_t C,
                                 cudaStream_t s) {
    const int64_t n = static_cast<int64_t>(K + 1) * C;
    const bool vec = n % 4 == 0 && reinterpret_cast<uintptr_t>(partials) % 16 == 0 && Gp <= kDwMaxRows;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(vec ? (n / 4 + 15) / 16 : (n + 31) / 32));
    cfg.blockDim = dim3(256);
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (vec) return cudaLaunchKernelEx(&cfg, conv1d_dw_finalize4_kernel, partials, dw, dbias, Gp, K, C);
    return cudaLaunchKernelEx(&cfg, conv1d_dw_finalize_kernel, partials, dw, dbias, Gp, K, C);
}

__global__ void conv1d_dw_zero_kernel(float *__restrict__ dw, float *__restrict__ dbias, int K, int64_t C) {
    const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (e < static_cast<int64_t>(K) * C) dw[e] = 0.f;
    if (dbias && e < C) dbias[e] = 0.f;
}

// Upper bound on the partial rows (one per block, or per cluster of blocks, of a channel tile):
// one per 64 frames, at most kDwMaxRows, and no more than keep the workspace within 64 MiB when
// the rows are wide.  The workspace is sized for it, so it depends on the sizes alone.
int conv1d_dw_partial_rows(int64_t B, int64_t T, int64_t C, int K) {
    const int64_t frames = B * T;
    if (frames <= 0) return 0;
    int64_t gp = (frames + 63) / 64;
    if (gp > kDwMaxRows) gp = kDwMaxRows;
    const int64_t row_bytes = static_cast<int64_t>(K + 1) * C * static_cast<int64_t>(sizeof(float));
    const int64_t cap = (int64_t(64) << 20) / (row_bytes > 0 ? row_bytes : 1);
    if (gp > cap) gp = cap;
    if (gp < 1) gp = 1;
    return static_cast<int>(gp);
}

size_t conv1d_dw_workspace_bytes(int64_t B, int64_t T, int64_t C, int K) {
    const int gp = conv1d_dw_partial_rows(B, T, C, K);
    return static_cast<size_t>(gp) * static_cast<size_t>(K + 1) * static_cast<size_t>(C) * sizeof(float);
}

namespace {

int pow2_at_most(int64_t v, int cap) {
    int p = 1;
    while (p < cap && p < v) p <<= 1;
    return p;
}

// Partial rows actually used: enough clusters to fill every SM once (two blocks per SM), at most
// the workspace's row count.  Fixed for given sizes on a given GPU, so results are reproducible.
int used_rows(int max_rows, int nCT, int blocks_per_sm) {
    const int64_t slots = static_cast<int64_t>(sm_count()) * blocks_per_sm;
    int64_t gp = slots / (static_cast<int64_t>(kDwCluster) * nCT);
    if (gp < 1) gp = 1;
    if (gp > max_rows) gp = max_rows;
    return static_cast<int>(gp);
}

template <typename T, int V, int KB>
cudaError_t launch_pass(const DwArgs &a, int gp, int k_off, int with_bias, cudaStream_t s) {
    constexpr int R = (V >= 4 || KB > 9) ? 8 : 16;
    const int64_t Cv = (a.C + V - 1) / V;
    const int TX = pow2_at_most(Cv, 32);
    const int TY = kDwThreads / TX;
    const int nCT = static_cast<int>((Cv + TX - 1) / TX);
    const int nTC = static_cast<int>((a.T + static_cast<int64_t>(TY) * R - 1) / (static_cast<int64_t>(TY) * R));
    if (nCT > 65535) return cudaErrorInvalidConfiguration;
    const size_t smem = static_cast<size_t>(TY) * (KB + 1) * TX * V * sizeof(float);
    conv1d_dw_partial_kernel<T, V, KB, R><<<dim3(gp * kDwCluster, nCT), kDwThreads, smem, s>>>(
        static_cast<const T *>(a.x), static_cast<const T *>(a.dy), a.lengths, a.partials, a.B, a.T,
        static_cast<int>(a.C), a.K, k_off, a.pad_left, TX, nTC, with_bias);
    return cudaGetLastError();
}

// Grid rows G and cluster size for the pipelined kernel: as many blocks per channel tile as
// fit on the device at once, in clusters as large as that allows (fewer partial rows).
template <typename T, int V, int KB, bool FUSED = false>
cudaError_t launch_tma_pass(const DwArgs &a, int k_off, int with_bias, int *gp_out, cudaStream_t s) {
    using S = DwTmaShape<T, V, KB, FUSED>;
    auto kern = conv1d_dw_tma_kernel<T, V, KB, FUSED>;
    const int ordered = (DW_DW_ORDERED && a.B <= kOrderMaxItems) ? 1 : 0;
    const int smem = S::SMEM + (ordered ? static_cast<int>((3 * (a.B + 1) * sizeof(int) + 15) / 16 * 16) : 0);
    const cudaError_t attr = ensure_smem_attr(reinterpret_cast<const void *>(kern),
                                              S::SMEM + static_cast<int>(3 * (kOrderMaxItems + 1) * sizeof(int)) + 16);
    if (attr != cudaSuccess) return attr;
    const int nCT = static_cast<int>((a.C + S::CT - 1) / S::CT);
    const int nT = static_cast<int>((a.T + S::TT - 1) / S::TT);
    const int64_t units = a.B * nT;
    if (nCT > 65535 || units >= (1LL << 31)) return cudaErrorInvalidConfiguration;
    int best_g = 0, best_c = 1;
    for (int c : {8, 4, 2, 1}) {
        cudaLaunchConfig_t q = {};
        q.gridDim = dim3(c, nCT);
        q.blockDim = dim3(S::THREADS);
        q.dynamicSmemBytes = smem;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = c;
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        q.attrs = at;
        q.numAttrs = 1;
        int nclu = 0;
        if (cudaOccupancyMaxActiveClusters(&nclu, kern, &q) != cudaSuccess || nclu < 1) {
            (void)cudaGetLastError();
            continue;
        }
        int64_t gg = (static_cast<int64_t>(nclu) * c / nCT) / c * c;  // blocks per channel tile
        const int64_t ucap = (units + c - 1) / c * c;                  // no more blocks than units
        if (gg > ucap) gg = ucap;
        if (gg / c > a.G) gg = static_cast<int64_t>(a.G) * c;          // workspace rows
        // a smaller cluster must fill clearly more of the GPU to be worth its extra partial rows
        if (gg > best_g + best_g / 32) {
            best_g = static_cast<int>(gg);
            best_c = c;
        }
    }
    if (best_g < 1) {  // more channel tiles than resident blocks: one block per tile, in waves
        best_g = 1;
        best_c = 1;
    }
    *gp_out = best_g / best_c;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(best_g, nCT);
    cfg.blockDim = dim3(S::THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = best_c;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cudaLaunchAttribute at2[2] = {at[0], {}};
    at2[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at2[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at2;
    cfg.numAttrs = 2;
    CUtensorMap xmap, dmap;
    cudaError_t me = make_act_map(&xmap, a.x, dtype_code<T>(), a.B, a.T, a.C, S::CT, S::XROWS);
    if (me == cudaSuccess) me = make_act_map(&dmap, a.dy, dtype_code<T>(), a.B, a.T, a.C, S::CT, S::DROWS);
    if (me != cudaSuccess) return me;
    return cudaLaunchKernelEx(&cfg, kern, xmap, dmap, a.lengths, a.partials, static_cast<int>(a.B),
                              static_cast<int>(a.T), static_cast<int>(a.C), a.K, k_off, a.pad_left, nT, with_bias,
                              ordered, a.w, static_cast<T *>(a.dx));
}

// The span-balanced kernel for a padded batch (offsets == null) or a packed one: grid (G, channel
// tiles), G = the blocks per channel tile that fit on the device at once, at most a.G (the
// workspace's partial rows) and no more than the frames fill tiles of TT.
template <typename T, int V, int KB, bool FUSED = false>
cudaError_t launch_span_pass(const DwArgs &a, const int32_t *offsets, int *gp_out, cudaStream_t s) {
    using S = DwSpanShape<T, V, KB, FUSED>;
    const bool packed = offsets != nullptr;
    auto kern = FUSED ? conv1d_dw_span_kernel<T, V, KB, false, FUSED>
                      : (packed ? conv1d_dw_span_kernel<T, V, KB, true> : conv1d_dw_span_kernel<T, V, KB, false>);
    const int smem = S::SMEM + static_cast<int>((4 * a.B + 2) * sizeof(int));
    const cudaError_t attr = ensure_smem_attr(reinterpret_cast<const void *>(kern),
                                              S::SMEM + static_cast<int>((4 * kOrderMaxItems + 2) * sizeof(int)));
    if (attr != cudaSuccess) return attr;
    const int64_t nCT = (a.C + S::CT - 1) / S::CT;
    if (nCT > 65535) return cudaErrorInvalidConfiguration;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, S::THREADS, smem) != cudaSuccess || per_sm < 1) {
        (void)cudaGetLastError();
        per_sm = 1;
    }
    const int64_t frames = packed ? a.T : a.B * a.T;  // an upper bound on the valid frames
    int64_t G = static_cast<int64_t>(sm_count()) * per_sm / nCT;
    const int64_t gmax = (frames + S::TT - 1) / S::TT;
    if (G > gmax) G = gmax;
    if (G > a.G) G = a.G;
    if (G < 1) G = 1;  // more channel tiles than resident blocks: one block per tile, in waves
    *gp_out = static_cast<int>(G);
    CUtensorMap xmap, dmap;
    const int64_t mB = packed ? 1 : a.B;
    cudaError_t me = make_act_map(&xmap, a.x, dtype_code<T>(), mB, a.T, a.C, S::CT, kDwSB);
    if (me == cudaSuccess) me = make_act_map(&dmap, a.dy, dtype_code<T>(), mB, a.T, a.C, S::CT, kDwSB);
    if (me != cudaSuccess) return me;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(G), static_cast<unsigned>(nCT));
    cfg.blockDim = dim3(S::THREADS);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, xmap, dmap, packed ? offsets : a.lengths, a.partials, static_cast<int>(a.B),
                              static_cast<int>(a.T), static_cast<int>(a.C), a.K, 0, a.pad_left, 1, a.w,
                              static_cast<T *>(a.dx));
}

template <typename T>
bool dw_tma_ok(const DwArgs &a) {
    return (a.C * static_cast<int64_t>(sizeof(T))) % 16 == 0 && reinterpret_cast<uintptr_t>(a.x) % 16 == 0 &&
           reinterpret_cast<uintptr_t>(a.dy) % 16 == 0 && a.T < (1LL << 30) && a.B < (1LL << 30) &&
           a.B * a.T < (1LL << 31);
}

template <typename T, int V>
int channel_tiles(int64_t C) {
    const int64_t Cv = (C + V - 1) / V;
    const int TX = pow2_at_most(Cv, 32);
    return static_cast<int>((Cv + TX - 1) / TX);
}

template <typename T, int V>
cudaError_t launch_partials(const DwArgs &a, int *gp_out, cudaStream_t s) {
    if constexpr (V >= 2) {
        if (dw_tma_ok<T>(a) && a.B <= kOrderMaxItems) {
            switch (a.K) {
                case 1: return launch_span_pass<T, V, 1>(a, nullptr, gp_out, s);
                case 2: return launch_span_pass<T, V, 2>(a, nullptr, gp_out, s);
                case 3: return launch_span_pass<T, V, 3>(a, nullptr, gp_out, s);
                case 4: return launch_span_pass<T, V, 4>(a, nullptr, gp_out, s);
                case 5: return launch_span_pass<T, V, 5>(a, nullptr, gp_out, s);
                case 7: return launch_span_pass<T, V, 7>(a, nullptr, gp_out, s);
                case 9: return launch_span_pass<T, V, 9>(a, nullptr, gp_out, s);
                default: break;
            }
            if constexpr (V == 2) {
                if (a.K == 15) return launch_span_pass<T, V, 15>(a, nullptr, gp_out, s);
            }
        }
        if (dw_tma_ok<T>(a)) {
            switch (a.K) {
                case 1: return launch_tma_pass<T, V, 1>(a, 0, 1, gp_out, s);
                case 2: return launch_tma_pass<T, V, 2>(a, 0, 1, gp_out, s);
                case 3: return launch_tma_pass<T, V, 3>(a, 0, 1, gp_out, s);
                case 4: return launch_tma_pass<T, V, 4>(a, 0, 1, gp_out, s);
                case 5: return launch_tma_pass<T, V, 5>(a, 0, 1, gp_out, s);
                case 7: return launch_tma_pass<T, V, 7>(a, 0, 1, gp_out, s);
                case 9: return launch_tma_pass<T, V, 9>(a, 0, 1, gp_out, s);
                default: break;
            }
            if constexpr (V == 2) {
                if (a.K == 15) return launch_tma_pass<T, V, 15>(a, 0, 1, gp_out, s);
            }
        }
    }
    const int gp = used_rows(a.G < kDwMaxRows16 ? a.G : kDwMaxRows16, channel_tiles<T, V>(a.C), 2);
    *gp_out = gp;
    switch (a.K) {
        case 1: return launch_pass<T, V, 1>(a, gp, 0, 1, s);
        case 2: return launch_pass<T, V, 2>(a, gp, 0, 1, s);
        case 3: return launch_pass<T, V, 3>(a, gp, 0, 1, s);
        case 4: return launch_pass<T, V, 4>(a, gp, 0, 1, s);
        case 5: return launch_pass<T, V, 5>(a, gp, 0, 1, s);
        case 7: return launch_pass<T, V, 7>(a, gp, 0, 1, s);
        case 9: return launch_pass<T, V, 9>(a, gp, 0, 1, s);
        default: break;
    }
    if constexpr (V <= 2) {
        if (a.K == 15) return launch_pass<T, V, 15>(a, gp, 0, 1, s);
    }
    for (int k_off = 0; k_off < a.K; k_off += kDwTapBlock) {
        cudaError_t e = launch_pass<T, (V > 2 ? 2 : V), kDwTapBlock>(a, gp, k_off, k_off == 0, s);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

template <typename T>
cudaError_t launch_dtype(const DwArgs &a, int *gp, cudaStream_t s) {
    if constexpr (sizeof(T) == 2) {
        if (a.vec_width >= 4 && a.K <= 9) return launch_partials<T, 4>(a, gp, s);
    }
    if (a.vec_width >= 2) return launch_partials<T, 2>(a, gp, s);
    return launch_partials<T, 1>(a, gp, s);
}

// The fused data + weight gradient pass; cudaErrorNotSupported when the pipelined kernel has no
// instance for these sizes (the caller then runs the two gradients separately).
template <typename T>
cudaError_t launch_fused_partials(const DwArgs &a, int *gp, cudaStream_t s) {
    if (!dw_tma_ok<T>(a) || a.vec_width < 2) return cudaErrorNotSupported;
    if (a.B <= kOrderMaxItems) {  // the span-balanced kernel in its one-pass form
        if constexpr (sizeof(T) == 2) {
            if (a.vec_width >= 4) {
                switch (a.K) {
                    case 1: return launch_span_pass<T, 4, 1, true>(a, nullptr, gp, s);
                    case 2: return launch_span_pass<T, 4, 2, true>(a, nullptr, gp, s);
                    case 3: return launch_span_pass<T, 4, 3, true>(a, nullptr, gp, s);
                    case 4: return launch_span_pass<T, 4, 4, true>(a, nullptr, gp, s);
                    case 5: return launch_span_pass<T, 4, 5, true>(a, nullptr, gp, s);
                    case 7: return launch_span_pass<T, 4, 7, true>(a, nullptr, gp, s);
                    case 9: return launch_span_pass<T, 4, 9, true>(a, nullptr, gp, s);
                    default: break;
                }
            }
        }
        switch (a.K) {
            case 1: return launch_span_pass<T, 2, 1, true>(a, nullptr, gp, s);
            case 2: return launch_span_pass<T, 2, 2, true>(a, nullptr, gp, s);
            case 3: return launch_span_pass<T, 2, 3, true>(a, nullptr, gp, s);
            case 4: return launch_span_pass<T, 2, 4, true>(a, nullptr, gp, s);
            case 5: return launch_span_pass<T, 2, 5, true>(a, nullptr, gp, s);
            case 7: return launch_span_pass<T, 2, 7, true>(a, nullptr, gp, s);
            case 9: return launch_span_pass<T, 2, 9, true>(a, nullptr, gp, s);
            case 15: return launch_span_pass<T, 2, 15, true>(a, nullptr, gp, s);
            default: return cudaErrorNotSupported;
        }
    }
    if constexpr (sizeof(T) == 2) {
        if (a.vec_width >= 4) {
            switch (a.K) {
                case 1: return launch_tma_pass<T, 4, 1, true>(a, 0, 1, gp, s);
                case 2: return launch_tma_pass<T, 4, 2, true>(a, 0, 1, gp, s);
                case 3: return launch_tma_pass<T, 4, 3, true>(a, 0, 1, gp, s);
                case 4: return launch_tma_pass<T, 4, 4, true>(a, 0, 1, gp, s);
                case 5: return launch_tma_pass<T, 4, 5, true>(a, 0, 1, gp, s);
                case 7: return launch_tma_pass<T, 4, 7, true>(a, 0, 1, gp, s);
                case 9: return launch_tma_pass<T, 4, 9, true>(a, 0, 1, gp, s);
                default: break;
            }
        }
    }
    switch (a.K) {
        case 1: return launch_tma_pass<T, 2, 1, true>(a, 0, 1, gp, s);
        case 2: return launch_tma_pass<T, 2, 2, true>(a, 0, 1, gp, s);
        case 3: return launch_tma_pass<T, 2, 3, true>(a, 0, 1, gp, s);
        case 4: return launch_tma_pass<T, 2, 4, true>(a, 0, 1, gp, s);
        case 5: return launch_tma_pass<T, 2, 5, true>(a, 0, 1, gp, s);
        case 7: return launch_tma_pass<T, 2, 7, true>(a, 0, 1, gp, s);
        case 9: return launch_tma_pass<T, 2, 9, true>(a, 0, 1, gp, s);
        case 15: return launch_tma_pass<T, 2, 15, true>(a, 0, 1, gp, s);
        default: return cudaErrorNotSupported;
    }
}

cudaError_t launch_finalize(const DwArgs &a, int gp, cudaStream_t s) {
    return launch_finalize_rows(a.partials, a.dw, a.dbias, gp, a.K, a.C, s);
}

}  // namespace

cudaError_t conv1d_bwd_fused_launch(const DwArgs &a, cudaStream_t s) {
    if (a.B == 0 || a.T == 0) return cudaErrorNotSupported;  // nothing to fuse
    int gp = 0;
    const cudaError_t e = with_dtype(a.dtype, [&](auto tag) { return launch_fused_partials<decltype(tag)>(a, &gp, s); });
    if (e != cudaSuccess) return e;
    return launch_finalize(a, gp, s);
}

unsigned int conv1d_dw_take_error() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, dw_device_error_flag, sizeof(v)) != cudaSuccess) return 0;
    if (v) cudaMemcpyToSymbol(dw_device_error_flag, &zero, sizeof(zero));
    return v;
}

// ---------------------------------------------------------------------------------------
// Packed batches: x and dy [N][C], item b on rows offsets[b] .. offsets[b+1]-1, each item with its
// own padding.  Grid (G, channel tiles of 32 V channels); block g walks rows N g / G .. N (g+1) / G,
// its 8 warps each a contiguous share, tracking the item of the current row as it goes (offsets
// clamped into [0, N]).  A thread keeps a window of the kDwPackedTaps x frames t - pad + k_off + k
// of the current row t (zero outside the item) and slides it one frame per row, so each row costs
// one dy and one x load: dbias += dz, dW[k_off + k] += dz win[k].  Widths beyond kDwPackedTaps run
// in passes.  The warps' sums are added in a fixed order in shared memory and each block writes
// partial row g; the finalize kernel adds the rows in order (reproducible, no atomics).
constexpr int kDwPackedTaps = 16;

template <typename T, int V>
__global__ void __launch_bounds__(256)
conv1d_dw_packed_kernel(const T *__restrict__ x, const T *__restrict__ dy, const int32_t *__restrict__ offsets,
                        float *__restrict__ partials, int B, int N, int C, int K, int k_off, int kb, int pad_left,
                        int with_bias, int G) {
    constexpr int NP = Pairs<V>::n;
    constexpr int KT = kDwPackedTaps;
    extern __shared__ float red[];  // [8][KT + 1][32 V]
    const int lane = threadIdx.x % 32, wp = threadIdx.x / 32;
    const int CT = 32 * V;
    const int cl = lane * V, c = blockIdx.y * CT + cl;
    const bool act = c < C;
    auto off = [&](int b) {
        const int o = __ldg(offsets + b);
        return o < 0 ? 0 : (o > N ? N : o);
    };
    const int64_t g = blockIdx.x;
    const int rb = static_cast<int>(static_cast<int64_t>(N) * g / G), re = static_cast<int>(static_cast<int64_t>(N) * (g + 1) / G);
    const int n0 = rb + static_cast<int>(static_cast<int64_t>(re - rb) * wp / 8);
    const int n1 = rb + static_cast<int>(static_cast<int64_t>(re - rb) * (wp + 1) / 8);
    float2 acc[KT][NP], accb[NP];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        accb[p] = make_float2(0.f, 0.f);
#pragma unroll
        for (int k = 0; k < KT; ++k) acc[k][p] = make_float2(0.f, 0.f);
    }
    if (act && n0 < n1) {
        int lo = 0, hi = B;  // the last item whose first row is <= n0
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (off(mid) <= n0) lo = mid;
            else hi = mid;
        }
        int b = lo, s0 = off(b), e = off(b + 1);
        if (e < s0) e = s0;
        auto load_x = [&](int j, int L, float2 (&f)[NP]) {  // frame j of the current item, zero outside
            if (j >= 0 && j < L) {
                Vec<T, V> v;
                v.load(x + (static_cast<int64_t>(s0) + j) * C + c);
                v.to_f2(f);
            } else {
#pragma unroll
                for (int p = 0; p < NP; ++p) f[p] = make_float2(0.f, 0.f);
            }
        };
        // window: slot (k + r) % KT holds frame j0 + k of row r of the current group of KT rows,
        // so every slot index is a compile-time constant; the frame that enters for row r + 1
        // (j0 + KT) takes the slot row r's frame j0 leaves
        float2 win[KT][NP];
        bool fresh = true;  // the window must be (re)filled for the current row
        for (int base = n0; base < n1; base += KT) {
#pragma unroll
            for (int r = 0; r < KT; ++r) {
                const int n = base + r;
                if (n < n1) {
                    while (n >= e && b + 1 < B) {  // the next item
                        ++b;
                        s0 = off(b);
                        e = off(b + 1);
                        if (e < s0) e = s0;
                        fresh = true;
                    }
                    if (n < s0 || n >= e) {  // a row no item covers
                        fresh = true;
                    } else {
                        const int t = n - s0, L = e - s0, j0 = t - pad_left + k_off;
                        if (fresh) {
#pragma unroll
                            for (int k = 0; k < KT; ++k) load_x(j0 + k, L, win[(k + r) % KT]);
                            fresh = false;
                        }
                        Vec<T, V> v;
                        v.load(dy + static_cast<int64_t>(n) * C + c);
                        float2 dz[NP];
                        v.to_f2(dz);
#pragma unroll
                        for (int p = 0; p < NP; ++p) {
                            accb[p].x += dz[p].x;
                            accb[p].y += dz[p].y;
                        }
#pragma unroll
                        for (int k = 0; k < KT; ++k) {
                            if (k < kb) {
#pragma unroll
                                for (int p = 0; p < NP; ++p)
                                    acc[k][p] = ffma2(dz[p], win[(k + r) % KT][p], acc[k][p]);
                            }
                        }
                        load_x(j0 + KT, L, win[r % KT]);  // frame j0 + KT for the next row
                    }
                }
            }
        }
    }
    // fixed-order sum over the 8 warps: red[warp][slot][channel of the tile]
#pragma unroll
    for (int kk = 0; kk <= KT; ++kk) {
        float2 v[NP];
#pragma unroll
        for (int p = 0; p < NP; ++p) v[p] = kk < KT ? acc[kk][p] : accb[p];
        float *d = red + (wp * (KT + 1) + kk) * CT + cl;
        if constexpr (V == 1) {
            d[0] = v[0].x;
        } else {
#pragma unroll
            for (int p = 0; p < NP; ++p) {
                d[2 * p] = v[p].x;
                d[2 * p + 1] = v[p].y;
            }
        }
    }
    __syncthreads();
    const int E = (KT + 1) * CT;
    for (int i = threadIdx.x; i < E; i += blockDim.x) {
        const int kk = i / CT, ch = blockIdx.y * CT + i % CT;
        if (ch >= C) continue;
        float t = 0.f;
        {
            float r[8];
#pragma unroll
            for (int w = 0; w < 8; ++w) r[w] = red[w * E + i];
            t = ((r[0] + r[1]) + (r[2] + r[3])) + ((r[4] + r[5]) + (r[6] + r[7]));
        }
        if (kk == KT) {
            if (with_bias) partials[(g * (K + 1) + K) * C + ch] = t;
        } else if (kk < kb) {
            partials[(g * (K + 1) + k_off + kk) * C + ch] = t;
        }
    }
}

constexpr int kDwPackedRows = 256;  // partial rows of the packed weight gradient (at most)

int conv1d_dw_packed_rows(int64_t N) {
    const int64_t g = (N + 127) / 128;
    return static_cast<int>(g < 1 ? 1 : (g > kDwPackedRows ? kDwPackedRows : g));
}

size_t conv1d_dw_packed_workspace_bytes(int64_t N, int64_t C, int K) {
    return static_cast<size_t>(conv1d_dw_packed_rows(N)) * static_cast<size_t>(K + 1) * static_cast<size_t>(C) *
           sizeof(float);
}

cudaError_t conv1d_dw_packed_launch(const DwArgs &a, const int32_t *offsets, cudaStream_t s) {
    const int64_t n = static_cast<int64_t>(a.K + 1) * a.C;
    if (a.B == 0 || a.T == 0) {
        conv1d_dw_zero_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(a.dw, a.dbias, a.K, a.C);
        return cudaGetLastError();
    }
    if (a.B <= kOrderMaxItems) {  // the pipelined kernel in its packed mode
        int gp = 0;
        const cudaError_t et = with_dtype(a.dtype, [&](auto tag) -> cudaError_t {
            using T = decltype(tag);
            if (!dw_tma_ok<T>(a) || a.vec_width < 2) return cudaErrorNotSupported;
            DwArgs b = a;
            b.G = conv1d_dw_packed_rows(a.T);
            if constexpr (sizeof(T) == 2) {
                if (a.vec_width >= 4) {
                    switch (a.K) {
                        case 1: return launch_span_pass<T, 4, 1>(b, offsets, &gp, s);
                        case 2: return launch_span_pass<T, 4, 2>(b, offsets, &gp, s);
                        case 3: return launch_span_pass<T, 4, 3>(b, offsets, &gp, s);
                        case 4: return launch_span_pass<T, 4, 4>(b, offsets, &gp, s);
                        case 5: return launch_span_pass<T, 4, 5>(b, offsets, &gp, s);
                        case 7: return launch_span_pass<T, 4, 7>(b, offsets, &gp, s);
                        case 9: return launch_span_pass<T, 4, 9>(b, offsets, &gp, s);
                        default: return cudaErrorNotSupported;
                    }
                }
            }
            switch (a.K) {
                case 1: return launch_span_pass<T, 2, 1>(b, offsets, &gp, s);
                case 2: return launch_span_pass<T, 2, 2>(b, offsets, &gp, s);
                case 3: return launch_span_pass<T, 2, 3>(b, offsets, &gp, s);
                case 4: return launch_span_pass<T, 2, 4>(b, offsets, &gp, s);
                case 5: return launch_span_pass<T, 2, 5>(b, offsets, &gp, s);
                case 7: return launch_span_pass<T, 2, 7>(b, offsets, &gp, s);
                case 9: return launch_span_pass<T, 2, 9>(b, offsets, &gp, s);
                case 15: return launch_span_pass<T, 2, 15>(b, offsets, &gp, s);
                default: return cudaErrorNotSupported;
            }
        });
        if (et != cudaErrorNotSupported) {
            if (et != cudaSuccess) return et;
            return launch_finalize_rows(a.partials, a.dw, a.dbias, gp, a.K, a.C, s);
        }
    }
    const int G = conv1d_dw_packed_rows(a.T);
    const int V = a.vec_width >= 2 ? 2 : 1;
    const int64_t nCT = (a.C + 32 * V - 1) / (32 * V);
    if (nCT > 65535) return cudaErrorInvalidConfiguration;
    const size_t red_bytes = static_cast<size_t>(8) * (kDwPackedTaps + 1) * 32 * V * sizeof(float);
    for (int k_off = 0; k_off < a.K; k_off += kDwPackedTaps) {
        const int kb = a.K - k_off < kDwPackedTaps ? a.K - k_off : kDwPackedTaps;
        const cudaError_t e = with_dtype(a.dtype, [&](auto tag) {
            using T = decltype(tag);
            const dim3 grid(static_cast<unsigned>(G), static_cast<unsigned>(nCT));
            if (V == 2)
                conv1d_dw_packed_kernel<T, 2><<<grid, 256, red_bytes, s>>>(
                    static_cast<const T *>(a.x), static_cast<const T *>(a.dy), offsets, a.partials, static_cast<int>(a.B),
                    static_cast<int>(a.T), static_cast<int>(a.C), a.K, k_off, kb, a.pad_left, k_off == 0 ? 1 : 0, G);
            else
                conv1d_dw_packed_kernel<T, 1><<<grid, 256, red_bytes, s>>>(
                    static_cast<const T *>(a.x), static_cast<const T *>(a.dy), offsets, a.partials, static_cast<int>(a.B),
                    static_cast<int>(a.T), static_cast<int>(a.C), a.K, k_off, kb, a.pad_left, k_off == 0 ? 1 : 0, G);
            return cudaGetLastError();
        });
        if (e != cudaSuccess) return e;
    }
    return launch_finalize_rows(a.partials, a.dw, a.dbias, G, a.K, a.C, s);
}

cudaError_t conv1d_dw_launch(const DwArgs &a, cudaStream_t s) {
    const int64_t n = static_cast<int64_t>(a.K + 1) * a.C;
    if (a.B == 0 || a.T == 0) {
        conv1d_dw_zero_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(a.dw, a.dbias, a.K, a.C);
        return cudaGetLastError();
    }
    int gp = 0;
    cudaError_t e = with_dtype(a.dtype, [&](auto tag) { return launch_dtype<decltype(tag)>(a, &gp, s); });
    if (e != cudaSuccess) return e;
    return launch_finalize(a, gp, s);
}

}  // namespace dwk
