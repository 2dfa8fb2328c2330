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

#include "dw_internal.h"

namespace cg = cooperative_groups;

namespace dwk {

constexpr int kDwThreads = 256;
constexpr int kDwCluster = 8;
constexpr int kDwTapBlock = 8;   // taps per pass for widths without a specialisation

template <typename T, int V, int KB, int R>
__global__ void __cluster_dims__(kDwCluster, 1, 1) __launch_bounds__(kDwThreads)
conv1d_dw_partial_kernel(const T *__restrict__ x, const T *__restrict__ dy,
                         const int32_t *__restrict__ lengths, float *__restrict__ partials,
                         int64_t B, int64_t Tn, int64_t C, int K, int k_off, int pad_left, int TX,
                         int nTC, int with_bias) {
    extern __shared__ float smem[];  // [TY][KB+1][CT]
    constexpr int NP = Pairs<V>::n;
    const int tx = threadIdx.x % TX, ty = threadIdx.x / TX;
    const int TY = blockDim.x / TX;
    const int CT = TX * V;
    const int g = blockIdx.x, G = gridDim.x;
    const int ct = blockIdx.y;
    const int64_t c0 = (static_cast<int64_t>(ct) * TX + tx) * V;
    const bool active = c0 < C;

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
            const T *xb = x + b * Tn * C + c0;
            const T *db = dy + b * Tn * C + c0;
            Vec<T, V> rdy[R], rx[R + KB - 1];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                if (t0 + r < L) rdy[r].load(db + (t0 + r) * C);
                else rdy[r].zero();
            }
#pragma unroll
            for (int i = 0; i < R + KB - 1; ++i) {
                const int64_t j = t0 + k_off - pad_left + i;
                if (j >= 0 && j < L) rx[i].load(xb + j * C);
                else rx[i].zero();
            }
            float2 xf[R + KB - 1][NP];
#pragma unroll
            for (int i = 0; i < R + KB - 1; ++i) rx[i].to_f2(xf[i]);
#pragma unroll
            for (int r = 0; r < R; ++r) {
                float2 dz[NP];
                rdy[r].to_f2(dz);
#pragma unroll
                for (int p = 0; p < NP; ++p) {
                    accb[p].x += dz[p].x;
                    accb[p].y += dz[p].y;
                }
#pragma unroll
                for (int k = 0; k < KB; ++k)
#pragma unroll
                    for (int p = 0; p < NP; ++p) acc[k][p] = ffma2(dz[p], xf[r + k][p], acc[k][p]);
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

__global__ void __launch_bounds__(256)
conv1d_dw_finalize_kernel(const float *__restrict__ partials, float *__restrict__ dw,
                          float *__restrict__ dbias, int Gp, int K, int64_t C) {
    const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (e >= static_cast<int64_t>(K + 1) * C) return;
    const int64_t k = e / C, c = e % C;
    float s = 0.f;
    for (int g = 0; g < Gp; ++g) s += partials[(static_cast<int64_t>(g) * (K + 1) + k) * C + c];
    if (k < K) dw[k * C + c] = s;
    else if (dbias) dbias[c] = s;
}

__global__ void conv1d_dw_zero_kernel(float *__restrict__ dw, float *__restrict__ dbias, int K, int64_t C) {
    const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (e < static_cast<int64_t>(K) * C) dw[e] = 0.f;
    if (dbias && e < C) dbias[e] = 0.f;
}

int conv1d_dw_partial_rows(int64_t B, int64_t T, int64_t /*C*/, int /*K*/) {
    const int64_t frames = B * T;
    if (frames <= 0) return 0;
    int64_t gp = (frames + 2047) / 2048;
    if (gp < 1) gp = 1;
    if (gp > 16) gp = 16;
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

template <typename T, int V, int KB>
cudaError_t launch_pass(const DwArgs &a, int k_off, int with_bias, cudaStream_t s) {
    constexpr int R = (KB <= 9) ? 16 : 8;
    const int64_t Cv = (a.C + V - 1) / V;
    const int TX = pow2_at_most(Cv, 32);
    const int TY = kDwThreads / TX;
    const int nCT = static_cast<int>((Cv + TX - 1) / TX);
    const int nTC = static_cast<int>((a.T + static_cast<int64_t>(TY) * R - 1) / (static_cast<int64_t>(TY) * R));
    const int G = a.G * kDwCluster;
    if (nCT > 65535) return cudaErrorInvalidConfiguration;
    const size_t smem = static_cast<size_t>(TY) * (KB + 1) * TX * V * sizeof(float);
    conv1d_dw_partial_kernel<T, V, KB, R><<<dim3(G, nCT), kDwThreads, smem, s>>>(
        static_cast<const T *>(a.x), static_cast<const T *>(a.dy), a.lengths, a.partials, a.B, a.T,
        a.C, a.K, k_off, a.pad_left, TX, nTC, with_bias);
    return cudaGetLastError();
}

template <typename T, int V>
cudaError_t launch_partials(const DwArgs &a, cudaStream_t s) {
    switch (a.K) {
        case 1: return launch_pass<T, V, 1>(a, 0, 1, s);
        case 2: return launch_pass<T, V, 2>(a, 0, 1, s);
        case 3: return launch_pass<T, V, 3>(a, 0, 1, s);
        case 4: return launch_pass<T, V, 4>(a, 0, 1, s);
        case 5: return launch_pass<T, V, 5>(a, 0, 1, s);
        case 7: return launch_pass<T, V, 7>(a, 0, 1, s);
        case 9: return launch_pass<T, V, 9>(a, 0, 1, s);
        case 15: return launch_pass<T, V, 15>(a, 0, 1, s);
        default:
            for (int k_off = 0; k_off < a.K; k_off += kDwTapBlock) {
                cudaError_t e = launch_pass<T, V, kDwTapBlock>(a, k_off, k_off == 0, s);
                if (e != cudaSuccess) return e;
            }
            return cudaSuccess;
    }
}

template <typename T>
cudaError_t launch_dtype(const DwArgs &a, cudaStream_t s) {
    if (a.vec_width >= 2) return launch_partials<T, 2>(a, s);
    return launch_partials<T, 1>(a, s);
}

}  // namespace

cudaError_t conv1d_dw_launch(const DwArgs &a, cudaStream_t s) {
    const int64_t n = static_cast<int64_t>(a.K + 1) * a.C;
    if (a.B == 0 || a.T == 0) {
        conv1d_dw_zero_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(a.dw, a.dbias, a.K, a.C);
        return cudaGetLastError();
    }
    cudaError_t e = a.bf16 ? launch_dtype<bf16>(a, s) : launch_dtype<float>(a, s);
    if (e != cudaSuccess) return e;
    conv1d_dw_finalize_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(a.partials, a.dw, a.dbias,
                                                                                   a.G, a.K, a.C);
    return cudaGetLastError();
}

}  // namespace dwk
