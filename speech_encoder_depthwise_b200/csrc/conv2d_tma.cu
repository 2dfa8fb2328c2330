// Depthwise conv2d with a 3x3 window (any strides and pads): shared-memory tiled kernels fed by
// TMA tensor copies (NeMo PR #16114, "Use Fused Kernels for Depthwise Striding Subsampler",
// section "What does this PR do ?", the depthwise conv with fused masking and causal padding).
// The same map as the general kernels in conv2d.cu:
//
//   xpad[b,r,s,c] = x[b, r-pt, s-pf, c] if 0 <= r-pt < len_b and 0 <= s-pf < F, else 0
//   y[b,i,j,c]    = [i < Lo_b] (bias[c] + sum_{p,q<3} xpad[b, st i + p, sf j + q, c] w[p,q,c])
//
// Each CTA is persistent and walks tiles (item, block of rows, block of columns, channel slab).
// One thread issues a single 4-D TMA copy per tile (box = channel slab x columns x rows x 1) into
// one of two shared-memory stages while the block computes on the other, so every input
// element crosses HBM once (plus a small row halo).  Padding outside the tensor arrives as TMA
// zero fill; frames at or after len_b are real data and are skipped at compute time.  Tiles
// whose rows are all masked only store zeros and issue no copy.
#include "dw_internal.h"

namespace dwk {
namespace {

constexpr int kC2V = 4;             // channels per thread (8 bytes bf16, 16 bytes float32)
constexpr int kC2StageMax = 49152;  // bytes of one stage

__device__ __forceinline__ void tma_load_4d(void *dst, const void *tmap, int c, int f, int t, int b, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, "
        "%5}], [%6];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c), "r"(f), "r"(t), "r"(b), "r"(smem_addr(bar))
        : "memory");
}

// L2 prefetch of one tensor box (no destination, nothing to wait for): safe before the dependency
// wait, since it only fills the cache.
__device__ __forceinline__ void tma_prefetch_4d(const void *tmap, int c, int f, int t, int b) {
    asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                     reinterpret_cast<uint64_t>(tmap)),
                 "r"(c), "r"(f), "r"(t), "r"(b)
                 : "memory");
}

// Before the dependency wait: the taps (9 rows over the slab's CS channels) and the lengths into L2.
__device__ __forceinline__ void c2_prefetch_params(const float *w, const int32_t *lengths, int C, int c0, int CS, int B,
                                                   int tid, int nthreads) {
    const int lines = (CS * 4 + 127) / 128;
    for (int i = tid; i < 9 * lines; i += nthreads) {
        const int c = c0 + (i % lines) * 32;
        if (w != nullptr && c < C) prefetch_l2(w + static_cast<int64_t>(i / lines) * C + c);
    }
    if (lengths != nullptr)
        for (int i = tid * 32; i < B; i += nthreads * 32) prefetch_l2(lengths + i);
}

__device__ __forceinline__ int out_len(const int32_t *lengths, int b, int Tn, int pt, int pb, int st, int To) {
    const int L = static_cast<int>(clamp_len(lengths, b, Tn));
    const int m = L + pt + pb - 3;
    const int Lo = m < 0 ? 0 : m / st + 1;
    return Lo < To ? Lo : To;
}

// Geometry and tiling, passed by value.
struct C2Geo {
    int B, T, F, C, To, Fo, st, sf, pt, pb, pf;
    int TI, TJ, CS;      // tile: rows, columns (of the map's output), channels
    int BR, BF;          // box rows, box columns of the staged tensor
    int nI, nJ, nCS;     // tiles per axis
    int stage_bytes;     // bytes of one stage (all staged boxes, each 128-byte aligned)
    int tx_bytes;        // bytes the copies of one stage deliver
};

template <typename T>
__device__ __forceinline__ void lds_vec(const T *p, float2 (&f)[2]) {
    if constexpr (sizeof(T) == 2) {
        const uint2 r = *reinterpret_cast<const uint2 *>(p);
        f[0] = Half16<T>::unpack(r.x);
        f[1] = Half16<T>::unpack(r.y);
    } else {
        const float4 r = *reinterpret_cast<const float4 *>(p);
        f[0] = make_float2(r.x, r.y);
        f[1] = make_float2(r.z, r.w);
    }
}

// Decode tile index -> (b, row block, column block, channel slab), channel slab fastest.
__device__ __forceinline__ void decode(const C2Geo &g, int tile, int &b, int &it, int &jt, int &cs) {
    cs = tile % g.nCS;
    int r = tile / g.nCS;
    jt = r % g.nJ;
    r /= g.nJ;
    it = r % g.nI;
    b = r / g.nI;
}

// Shared memory: two mbarriers in the first 128 bytes, then [2 stages][stage_bytes], then (the
// data gradient only) the per-tile row table.
constexpr int kC2Head = 128;
struct C2Smem {
    unsigned char *stage[2];
    uint64_t *full;
};
__device__ __forceinline__ C2Smem c2_smem(unsigned char *raw, int stage_bytes) {
    C2Smem s;
    s.full = reinterpret_cast<uint64_t *>(raw);
    s.stage[0] = raw + kC2Head;
    s.stage[1] = raw + kC2Head + stage_bytes;
    return s;
}

// ------------------------------------------------------------------------------ forward
// Tile = TI output rows x TJ output columns x CS channels of one item; the box covers input rows
// st*i0 - pt .. + BR and columns sf*j0 - pf .. + BF.  Thread = (column j, channel vector cv) and
// walks the TI rows; blockDim = TJ * CS/4 rounded up to a warp.
template <typename T, int ST>
__global__ void __launch_bounds__(512)
c2_fwd_tma_kernel(const __grid_constant__ CUtensorMap xmap, const float *__restrict__ w,
                  const float *__restrict__ bias, T *__restrict__ y, const int32_t *__restrict__ lengths,
                  int32_t *__restrict__ out_lengths, C2Geo g) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    const C2Smem sm = c2_smem(smem_raw, g.stage_bytes);
    const int tid = threadIdx.x;
    const int CSV = g.CS / kC2V;
    const int cv = tid % CSV, jl = tid / CSV;
    const bool active = jl < g.TJ;
    const int ntiles = g.B * g.nI * g.nJ * g.nCS;
    launch_dependents();  // the next kernel in the stream may start its own set-up
    if (tid == 0) {
        prefetch_tmap(&xmap);
        mbar_init(&sm.full[0], 1);
        mbar_init(&sm.full[1], 1);
        fence_barrier_init();
        if (static_cast<int>(blockIdx.x) < ntiles) {  // the first tile's box, before its length is known
            int b, it, jt, cs;
            decode(g, blockIdx.x, b, it, jt, cs);
            tma_prefetch_4d(&xmap, cs * g.CS, jt * g.TJ * g.sf - g.pf, it * g.TI * g.st - g.pt, b);
        }
    } else {
        c2_prefetch_params(w, lengths, g.C, (static_cast<int>(blockIdx.x) % g.nCS) * g.CS, g.CS, g.B, tid - 1,
                           static_cast<int>(blockDim.x) - 1);
    }
    grid_dependency_wait();  // launched programmatically: the previous kernel's writes are visible after this
    if (blockIdx.x == 0 && out_lengths != nullptr)
        for (int b = tid; b < g.B; b += blockDim.x) out_lengths[b] = out_len(lengths, b, g.T, g.pt, g.pb, g.st, g.To);
    __syncthreads();

    auto valid = [&](int tile) {
        int b, it, jt, cs;
        decode(g, tile, b, it, jt, cs);
        return it * g.TI < out_len(lengths, b, g.T, g.pt, g.pb, g.st, g.To);
    };
    int cursor = blockIdx.x, issued = 0;  // producer state (thread 0)
    auto issue_next = [&]() {
        while (cursor < ntiles && !valid(cursor)) cursor += gridDim.x;
        if (cursor >= ntiles) return;
        int b, it, jt, cs;
        decode(g, cursor, b, it, jt, cs);
        const int s = issued & 1;
        mbar_arrive_expect_tx(&sm.full[s], static_cast<uint32_t>(g.tx_bytes));
        tma_load_4d(sm.stage[s], &xmap, cs * g.CS, jt * g.TJ * g.sf - g.pf, it * g.TI * g.st - g.pt, b, &sm.full[s]);
        ++issued;
        cursor += gridDim.x;
    };
    if (tid == 0) issue_next();

    // the grid is a multiple of nCS, so the block's channel slab, and its taps, never change
    float2 wr[9][2], bv[2];
    {
        const int c = (static_cast<int>(blockIdx.x) % g.nCS) * g.CS + cv * kC2V;
        if (active && c < g.C) {
#pragma unroll
            for (int k = 0; k < 9; ++k) load_param<kC2V>(w + static_cast<int64_t>(k) * g.C + c, wr[k]);
            if (bias != nullptr) {
                load_param<kC2V>(bias + c, bv);
            } else {
                bv[0] = bv[1] = make_float2(0.f, 0.f);
            }
        }
    }
    int n = 0;  // valid tiles consumed
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        int b, it, jt, cs;
        decode(g, tile, b, it, jt, cs);
        const int L = static_cast<int>(clamp_len(lengths, b, g.T));
        const int Lo = out_len(lengths, b, g.T, g.pt, g.pb, g.st, g.To);
        const int i0 = it * g.TI, j = jt * g.TJ + jl, c = cs * g.CS + cv * kC2V;
        const bool col_ok = active && j < g.Fo && c < g.C;
        T *yb = y + ((static_cast<int64_t>(b) * g.To) * g.Fo + j) * g.C + c;
        const int64_t row_stride = static_cast<int64_t>(g.Fo) * g.C;
        if (i0 >= Lo) {  // every row masked: zeros, no copy
            if (col_ok)
                for (int i = i0; i < i0 + g.TI && i < g.To; ++i) Vec<T, kC2V>::store_zero(yb + i * row_stride);
            continue;
        }
        if (tid == 0) issue_next();  // the next valid tile into the other stage
        const int s = n & 1;
        const bool ok = mbar_wait(&sm.full[s], (n >> 1) & 1);
        if (__syncthreads_or(!ok)) {  // a copy never arrived (error word set): drain and leave
            if (tid == 0 && issued > n + 1) mbar_wait(&sm.full[s ^ 1], ((n + 1) >> 1) & 1);
            return;
        }
        if (col_ok) {
            // this thread's column of the box; 32-bit element offsets inside the stage
            const T *tb = reinterpret_cast<const T *>(sm.stage[s]) + (jl * g.sf * g.CS + cv * kC2V);
            const int RS = g.BF * g.CS;  // box row stride
            auto put = [&](int i, const float2 (&acc)[2]) {
                if (i >= g.To) return;
                if (i < Lo) Vec<T, kC2V>::store(yb + i * row_stride, acc);
                else Vec<T, kC2V>::store_zero(yb + i * row_stride);
            };
            if constexpr (ST > 0) {
                // two output rows per step: input rows i*ST + pp - pt, pp < ST + 3, feed row i
                // through tap pp and row i+1 through tap pp - ST (two independent chains)
                for (int il = 0; il < g.TI; il += 2) {
                    const int i = i0 + il;
                    if (i >= g.To || i >= Lo) {
                        put(i, bv);
                        put(i + 1, bv);
                        continue;
                    }
                    float2 a0[2] = {bv[0], bv[1]}, a1[2] = {bv[0], bv[1]};
#pragma unroll
                    for (int pp = 0; pp < ST + 3; ++pp) {
                        if (i * ST + pp - g.pt >= L) break;  // this and later frames are padding
                        const T *row = tb + (il * ST + pp) * RS;
#pragma unroll
                        for (int q = 0; q < 3; ++q) {
                            float2 xv[2];
                            lds_vec<T>(row + q * g.CS, xv);
                            if (pp < 3) {
                                a0[0] = ffma2(xv[0], wr[pp * 3 + q][0], a0[0]);
                                a0[1] = ffma2(xv[1], wr[pp * 3 + q][1], a0[1]);
                            }
                            if (pp >= ST && pp - ST < 3) {
                                a1[0] = ffma2(xv[0], wr[(pp - ST) * 3 + q][0], a1[0]);
                                a1[1] = ffma2(xv[1], wr[(pp - ST) * 3 + q][1], a1[1]);
                            }
                        }
                    }
                    put(i, a0);
                    put(i + 1, a1);
                }
            } else {
                for (int il = 0; il < g.TI; ++il) {
                    const int i = i0 + il;
                    if (i >= g.To || i >= Lo) {
                        put(i, bv);
                        continue;
                    }
                    float2 acc[2] = {bv[0], bv[1]};
#pragma unroll
                    for (int p = 0; p < 3; ++p) {
                        if (i * g.st + p - g.pt >= L) break;  // frames at/after len_b are padding
                        const T *row = tb + (il * g.st + p) * RS;
#pragma unroll
                        for (int q = 0; q < 3; ++q) {
                            float2 xv[2];
                            lds_vec<T>(row + q * g.CS, xv);
                            acc[0] = ffma2(xv[0], wr[p * 3 + q][0], acc[0]);
                            acc[1] = ffma2(xv[1], wr[p * 3 + q][1], acc[1]);
                        }
                    }
                    put(i, acc);
                }
            }
        }
        __syncthreads();  // stage s is free for the copy issued at the next valid tile
        ++n;
    }
}


// ------------------------------------------------------------------------------ data gradient
// dx[b,t,f,c] = [t < len_b] sum over taps (p, q) with (t + pt - p) = st i, (f + pf - q) = sf j,
// 0 <= i < Lo_b, 0 <= j < Fo of dy[b,i,j,c] w[p,q,c]  (the transpose of the forward map, as a gather).
// Tile = TI rows x TJ columns of dx x CS channels; the box covers dy rows floor((t0+pt-2)/st) ..
// + BR and columns floor((f0+pf-2)/sf) .. + BF.  Per tile, a table gives for each (dx row, p)
// the box row of its dy term or -1; each thread's column gives the same for q.
template <typename T>
__global__ void __launch_bounds__(512)
c2_dx_tma_kernel(const __grid_constant__ CUtensorMap gmap, const float *__restrict__ w, T *__restrict__ dx,
                 const int32_t *__restrict__ lengths, C2Geo g) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    const C2Smem sm = c2_smem(smem_raw, g.stage_bytes);
    int *rowtab = reinterpret_cast<int *>(sm.stage[1] + g.stage_bytes);  // [TI][3]
    const int tid = threadIdx.x;
    const int CSV = g.CS / kC2V;
    const int cv = tid % CSV, jl = tid / CSV;
    const bool active = jl < g.TJ;
    const int ntiles = g.B * g.nI * g.nJ * g.nCS;
    auto floordiv = [](int a, int d) { return a >= 0 ? a / d : -((-a + d - 1) / d); };
    launch_dependents();  // the next kernel in the stream may start its own set-up
    if (tid == 0) {
        prefetch_tmap(&gmap);
        mbar_init(&sm.full[0], 1);
        mbar_init(&sm.full[1], 1);
        fence_barrier_init();
        if (static_cast<int>(blockIdx.x) < ntiles) {  // the first tile's box, before its length is known
            int b, it, jt, cs;
            decode(g, blockIdx.x, b, it, jt, cs);
            tma_prefetch_4d(&gmap, cs * g.CS, floordiv(jt * g.TJ + g.pf - 2, g.sf), floordiv(it * g.TI + g.pt - 2, g.st), b);
        }
    } else {
        c2_prefetch_params(w, lengths, g.C, (static_cast<int>(blockIdx.x) % g.nCS) * g.CS, g.CS, g.B, tid - 1,
                           static_cast<int>(blockDim.x) - 1);
    }
    grid_dependency_wait();  // launched programmatically: the previous kernel's writes are visible after this
    __syncthreads();
    auto valid = [&](int tile) {
        int b, it, jt, cs;
        decode(g, tile, b, it, jt, cs);
        return it * g.TI < static_cast<int>(clamp_len(lengths, b, g.T));
    };
    int cursor = blockIdx.x, issued = 0;
    auto issue_next = [&]() {
        while (cursor < ntiles && !valid(cursor)) cursor += gridDim.x;
        if (cursor >= ntiles) return;
        int b, it, jt, cs;
        decode(g, cursor, b, it, jt, cs);
        const int s = issued & 1;
        mbar_arrive_expect_tx(&sm.full[s], static_cast<uint32_t>(g.tx_bytes));
        tma_load_4d(sm.stage[s], &gmap, cs * g.CS, floordiv(jt * g.TJ + g.pf - 2, g.sf),
                    floordiv(it * g.TI + g.pt - 2, g.st), b, &sm.full[s]);
        ++issued;
        cursor += gridDim.x;
    };
    if (tid == 0) issue_next();

    // the grid is a multiple of nCS, so the block's channel slab, and its taps, never change
    float2 wr[9][2];
    {
        const int c = (static_cast<int>(blockIdx.x) % g.nCS) * g.CS + cv * kC2V;
        if (active && c < g.C) {
#pragma unroll
            for (int k = 0; k < 9; ++k) load_param<kC2V>(w + static_cast<int64_t>(k) * g.C + c, wr[k]);
        }
    }
    int n = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        int b, it, jt, cs;
        decode(g, tile, b, it, jt, cs);
        const int L = static_cast<int>(clamp_len(lengths, b, g.T));
        const int t0 = it * g.TI, f = jt * g.TJ + jl, c = cs * g.CS + cv * kC2V;
        const bool col_ok = active && f < g.F && c < g.C;
        T *xb = dx + ((static_cast<int64_t>(b) * g.T) * g.F + f) * g.C + c;
        const int64_t row_stride = static_cast<int64_t>(g.F) * g.C;
        if (t0 >= L) {
            if (col_ok)
                for (int t = t0; t < t0 + g.TI && t < g.T; ++t) Vec<T, kC2V>::store_zero(xb + t * row_stride);
            continue;
        }
        if (tid == 0) issue_next();
        const int Lo = out_len(lengths, b, g.T, g.pt, g.pb, g.st, g.To);
        const int ia = floordiv(t0 + g.pt - 2, g.st);
        for (int e = tid; e < g.TI * 3; e += blockDim.x) {  // (row, p) -> box row or -1
            const int u = t0 + e / 3 + g.pt - e % 3;
            int rb = -1;
            if (u >= 0 && u % g.st == 0 && u / g.st < Lo) rb = u / g.st - ia;
            rowtab[e] = rb;
        }
        int cb[3];
        {
            const int ja = floordiv(jt * g.TJ + g.pf - 2, g.sf);
#pragma unroll
            for (int q = 0; q < 3; ++q) {
                const int v = f + g.pf - q;
                cb[q] = (v >= 0 && v % g.sf == 0 && v / g.sf < g.Fo) ? v / g.sf - ja : -1;
            }
        }
        const int s = n & 1;
        const bool ok = mbar_wait(&sm.full[s], (n >> 1) & 1);
        if (__syncthreads_or(!ok)) {
            if (tid == 0 && issued > n + 1) mbar_wait(&sm.full[s ^ 1], ((n + 1) >> 1) & 1);
            return;
        }
        if (col_ok) {
            const T *tileb = reinterpret_cast<const T *>(sm.stage[s]) + cv * kC2V;
            for (int tl = 0; tl < g.TI; ++tl) {
                const int t = t0 + tl;
                if (t >= g.T) break;
                if (t >= L) {
                    Vec<T, kC2V>::store_zero(xb + t * row_stride);
                    continue;
                }
                float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
                for (int p = 0; p < 3; ++p) {
                    const int rb = rowtab[tl * 3 + p];
                    if (rb < 0) continue;
#pragma unroll
                    for (int q = 0; q < 3; ++q) {
                        if (cb[q] < 0) continue;
                        float2 gv[2];
                        lds_vec<T>(tileb + (static_cast<int64_t>(rb) * g.BF + cb[q]) * g.CS, gv);
                        acc[0] = ffma2(gv[0], wr[p * 3 + q][0], acc[0]);
                        acc[1] = ffma2(gv[1], wr[p * 3 + q][1], acc[1]);
                    }
                }
                Vec<T, kC2V>::store(xb + t * row_stride, acc);
            }
        }
        __syncthreads();
        ++n;
    }
}

// Stride 2 in both axes: dx row pairs (t, t+1) and column pairs (f, f+1) with t, f even draw
// on a 2x2 block of dy: rows ilo = floor((t + pt - 1)/2) and ilo+1, columns likewise.  Which
// taps link them depends only on the parity of pt (rows) and of pf (columns), the same for the
// whole launch (RODD, CODD).  For one axis, with "lo"/"hi" the first/second dy row of the pair:
//   pad even: out0 = hi*tap0 + lo*tap2,  out1 = hi*tap1
//   pad odd:  out0 = lo*tap1,            out1 = hi*tap0 + lo*tap2
// Thread = (column pair m, channel vector cv) walking the row pairs of the tile, keeping the
// "hi" dy row of one step as the "lo" row of the next: two shared-memory loads per 4 outputs.
__host__ __device__ constexpr int ph_n(bool odd, int r) { return (odd ? r == 1 : r == 0) ? 2 : 1; }
__host__ __device__ constexpr int ph_sel(bool odd, int r, int e) {
    return ph_n(odd, r) == 2 ? (e == 0 ? 1 : 0) : (odd ? 0 : 1);
}
__host__ __device__ constexpr int ph_tap(bool odd, int r, int e) { return ph_n(odd, r) == 2 ? (e == 0 ? 0 : 2) : 1; }

template <typename T, bool RODD, bool CODD>
__global__ void __launch_bounds__(512)
c2_dx2_tma_kernel(const __grid_constant__ CUtensorMap gmap, const float *__restrict__ w, T *__restrict__ dx,
                  const int32_t *__restrict__ lengths, C2Geo g) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    const C2Smem sm = c2_smem(smem_raw, g.stage_bytes);
    const int tid = threadIdx.x;
    const int CSV = g.CS / kC2V;
    const int cv = tid % CSV, m = tid / CSV;
    const bool active = m < g.TJ / 2;
    const int ntiles = g.B * g.nI * g.nJ * g.nCS;
    auto floordiv = [](int a, int d) { return a >= 0 ? a / d : -((-a + d - 1) / d); };
    launch_dependents();  // the next kernel in the stream may start its own set-up
    if (tid == 0) {
        prefetch_tmap(&gmap);
        mbar_init(&sm.full[0], 1);
        mbar_init(&sm.full[1], 1);
        fence_barrier_init();
        if (static_cast<int>(blockIdx.x) < ntiles) {  // the first tile's box, before its length is known
            int b, it, jt, cs;
            decode(g, blockIdx.x, b, it, jt, cs);
            tma_prefetch_4d(&gmap, cs * g.CS, floordiv(jt * g.TJ + g.pf - 1, 2), floordiv(it * g.TI + g.pt - 1, 2), b);
        }
    } else {
        c2_prefetch_params(w, lengths, g.C, (static_cast<int>(blockIdx.x) % g.nCS) * g.CS, g.CS, g.B, tid - 1,
                           static_cast<int>(blockDim.x) - 1);
    }
    grid_dependency_wait();  // launched programmatically: the previous kernel's writes are visible after this
    __syncthreads();
    auto valid = [&](int tile) {
        int b, it, jt, cs;
        decode(g, tile, b, it, jt, cs);
        return it * g.TI < static_cast<int>(clamp_len(lengths, b, g.T));
    };
    int cursor = blockIdx.x, issued = 0;
    auto issue_next = [&]() {
        while (cursor < ntiles && !valid(cursor)) cursor += gridDim.x;
        if (cursor >= ntiles) return;
        int b, it, jt, cs;
        decode(g, cursor, b, it, jt, cs);
        const int s = issued & 1;
        mbar_arrive_expect_tx(&sm.full[s], static_cast<uint32_t>(g.tx_bytes));
        tma_load_4d(sm.stage[s], &gmap, cs * g.CS, floordiv(jt * g.TJ + g.pf - 1, 2),
                    floordiv(it * g.TI + g.pt - 1, 2), b, &sm.full[s]);
        ++issued;
        cursor += gridDim.x;
    };
    if (tid == 0) issue_next();

    // the grid is a multiple of nCS, so the block's channel slab, and its taps, never change
    float2 wr[9][2];
    {
        const int c = (static_cast<int>(blockIdx.x) % g.nCS) * g.CS + cv * kC2V;
        if (active && c < g.C) {
#pragma unroll
            for (int k = 0; k < 9; ++k) load_param<kC2V>(w + static_cast<int64_t>(k) * g.C + c, wr[k]);
        }
    }
    int n = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        int b, it, jt, cs;
        decode(g, tile, b, it, jt, cs);
        const int L = static_cast<int>(clamp_len(lengths, b, g.T));
        const int t0 = it * g.TI, f = jt * g.TJ + 2 * m, c = cs * g.CS + cv * kC2V;
        const bool col_ok = active && f < g.F && c < g.C;
        const bool col1_ok = f + 1 < g.F;
        T *xb = dx + ((static_cast<int64_t>(b) * g.T) * g.F + f) * g.C + c;
        const int64_t row_stride = static_cast<int64_t>(g.F) * g.C;
        auto put = [&](int t, int e, const float2 (&v)[2]) {  // dx[t, f + e]
            if (t >= g.T || (e == 1 && !col1_ok)) return;
            if (t < L) Vec<T, kC2V>::store(xb + t * row_stride + e * g.C, v);
            else Vec<T, kC2V>::store_zero(xb + t * row_stride + e * g.C);
        };
        if (t0 >= L) {
            if (col_ok) {
                const float2 z[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                for (int t = t0; t < t0 + g.TI; ++t) {
                    put(t, 0, z);
                    put(t, 1, z);
                }
            }
            continue;
        }
        if (tid == 0) issue_next();
        const int Lo = out_len(lengths, b, g.T, g.pt, g.pb, 2, g.To);
        const int ia = floordiv(t0 + g.pt - 1, 2);
        const int s = n & 1;
        const bool ok = mbar_wait(&sm.full[s], (n >> 1) & 1);
        if (__syncthreads_or(!ok)) {
            if (tid == 0 && issued > n + 1) mbar_wait(&sm.full[s ^ 1], ((n + 1) >> 1) & 1);
            return;
        }
        if (col_ok) {
            const T *tb = reinterpret_cast<const T *>(sm.stage[s]) + (m * g.CS + cv * kC2V);
            const int RS = g.BF * g.CS;
            float2 d[2][2][2];  // [lo/hi row][lo/hi column][pair]
            auto load_row = [&](int k, float2 (&r)[2][2]) {  // box row k = dy row ia + k
                const int i = ia + k;
                if (i >= 0 && i < Lo) {
                    lds_vec<T>(tb + k * RS, r[0]);
                    lds_vec<T>(tb + k * RS + g.CS, r[1]);
                } else {
                    r[0][0] = r[0][1] = r[1][0] = r[1][1] = make_float2(0.f, 0.f);
                }
            };
            load_row(0, d[0]);
            for (int k = 0; 2 * k < g.TI; ++k) {
                const int t = t0 + 2 * k;
                if (t >= g.T) break;
                load_row(k + 1, d[1]);
                float2 out[2][2][2];
#pragma unroll
                for (int r = 0; r < 2; ++r)
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
                        for (int e = 0; e < ph_n(RODD, r); ++e)
#pragma unroll
                            for (int h = 0; h < ph_n(CODD, cc); ++h) {
                                const int rs = ph_sel(RODD, r, e), cs2 = ph_sel(CODD, cc, h);
                                const int tap = ph_tap(RODD, r, e) * 3 + ph_tap(CODD, cc, h);
                                acc[0] = ffma2(d[rs][cs2][0], wr[tap][0], acc[0]);
                                acc[1] = ffma2(d[rs][cs2][1], wr[tap][1], acc[1]);
                            }
                        out[r][cc][0] = acc[0];
                        out[r][cc][1] = acc[1];
                    }
                put(t, 0, out[0][0]);
                put(t, 1, out[0][1]);
                put(t + 1, 0, out[1][0]);
                put(t + 1, 1, out[1][1]);
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    d[0][cc][0] = d[1][cc][0];
                    d[0][cc][1] = d[1][cc][1];
                }
            }
        }
        __syncthreads();
        ++n;
    }
}

// ------------------------------------------------------------------------------ weight gradient
// dW[p,q,c] = sum_{b, i < Lo_b, j} dy[b,i,j,c] xpad[b, st i + p, sf j + q, c];  dbias = sum dy.
// CTA (slab cs, index gi) walks tiles gi, gi + G, ... of its channel slab; per tile it stages the
// x box of the forward tile and the dy box (TI rows x TJ columns).  Thread = (channel vector cv,
// tile column pg) keeps 9 + 1 accumulator vectors over the rows of its column (two rows per step,
// sharing their common input row); at the end the columns are added in a fixed order through
// shared memory and the CTA writes partial row gi: partials[gi][slot][c], slots 0..8 the taps
// and 9 the bias.
template <typename T, int ST>
__global__ void __launch_bounds__(512)
c2_dw_tma_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap gmap,
                 const int32_t *__restrict__ lengths, float *__restrict__ partials, C2Geo g, int G, int xbytes) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    const C2Smem sm = c2_smem(smem_raw, g.stage_bytes);
    const int tid = threadIdx.x;
    const int CSV = g.CS / kC2V;
    const int cv = tid % CSV, pg = tid / CSV, NPG = blockDim.x / CSV;
    const int cs = blockIdx.x % g.nCS, gi = blockIdx.x / g.nCS;
    const int c = cs * g.CS + cv * kC2V;
    const int ntiles = g.B * g.nI * g.nJ;  // tiles of one slab
    auto dec = [&](int tile, int &b, int &it, int &jt) {
        jt = tile % g.nJ;
        const int r = tile / g.nJ;
        it = r % g.nI;
        b = r / g.nI;
    };
    launch_dependents();  // the finalize may be scheduled now; it waits for this grid to finish
    if (tid == 0) {
        prefetch_tmap(&xmap);
        prefetch_tmap(&gmap);
        mbar_init(&sm.full[0], 1);
        mbar_init(&sm.full[1], 1);
        fence_barrier_init();
        if (gi < ntiles) {  // the first tile's boxes, before its length is known
            int b, it, jt;
            dec(gi, b, it, jt);
            tma_prefetch_4d(&xmap, cs * g.CS, jt * g.TJ * g.sf - g.pf, it * g.TI * g.st - g.pt, b);
            tma_prefetch_4d(&gmap, cs * g.CS, jt * g.TJ, it * g.TI, b);
        }
    } else if (lengths != nullptr) {
        for (int i = (tid - 1) * 32; i < g.B; i += (static_cast<int>(blockDim.x) - 1) * 32) prefetch_l2(lengths + i);
    }
    grid_dependency_wait();  // launched programmatically: the previous kernel's writes are visible after this
    __syncthreads();
    auto valid = [&](int tile) {
        int b, it, jt;
        dec(tile, b, it, jt);
        return it * g.TI < out_len(lengths, b, g.T, g.pt, g.pb, g.st, g.To);
    };
    int cursor = gi, issued = 0;
    auto issue_next = [&]() {
        while (cursor < ntiles && !valid(cursor)) cursor += G;
        if (cursor >= ntiles) return;
        int b, it, jt;
        dec(cursor, b, it, jt);
        const int s = issued & 1;
        mbar_arrive_expect_tx(&sm.full[s], static_cast<uint32_t>(g.tx_bytes));
        tma_load_4d(sm.stage[s], &xmap, cs * g.CS, jt * g.TJ * g.sf - g.pf, it * g.TI * g.st - g.pt, b, &sm.full[s]);
        tma_load_4d(sm.stage[s] + xbytes, &gmap, cs * g.CS, jt * g.TJ, it * g.TI, b, &sm.full[s]);
        ++issued;
        cursor += G;
    };
    if (tid == 0) issue_next();

    float2 acc[10][2];
#pragma unroll
    for (int k = 0; k < 10; ++k) acc[k][0] = acc[k][1] = make_float2(0.f, 0.f);
    int n = 0;
    for (int tile = gi; tile < ntiles; tile += G) {
        int b, it, jt;
        dec(tile, b, it, jt);
        const int Lo = out_len(lengths, b, g.T, g.pt, g.pb, g.st, g.To);
        const int i0 = it * g.TI, j0 = jt * g.TJ;
        if (i0 >= Lo) continue;  // no unmasked output row: nothing to add
        if (tid == 0) issue_next();
        const int L = static_cast<int>(clamp_len(lengths, b, g.T));
        const int s = n & 1;
        const bool ok = mbar_wait(&sm.full[s], (n >> 1) & 1);
        if (__syncthreads_or(!ok)) {
            if (tid == 0 && issued > n + 1) mbar_wait(&sm.full[s ^ 1], ((n + 1) >> 1) & 1);
            return;
        }
        const int jl = pg;  // this thread's column of the tile
        if (c < g.C && jl < g.TJ && j0 + jl < g.Fo) {
            const T *xs = reinterpret_cast<const T *>(sm.stage[s]) + (jl * g.sf * g.CS + cv * kC2V);
            const T *gs = reinterpret_cast<const T *>(sm.stage[s] + xbytes) + (jl * g.CS + cv * kC2V);
            const int RS = g.BF * g.CS, GS = g.TJ * g.CS;  // box row strides (x, dy)
            auto add_bias = [&](const float2 (&gv)[2]) {
                acc[9][0].x += gv[0].x;
                acc[9][0].y += gv[0].y;
                acc[9][1].x += gv[1].x;
                acc[9][1].y += gv[1].y;
            };
            if constexpr (ST > 0) {
                // two output rows per step; input row i*ST + pp - pt meets row i through tap pp
                // and row i+1 through tap pp - ST
                for (int il = 0; il < g.TI; il += 2) {
                    const int i = i0 + il;
                    if (i >= Lo) break;  // later rows are masked too
                    float2 g0[2], g1[2];
                    lds_vec<T>(gs + il * GS, g0);
                    if (i + 1 < Lo) {
                        lds_vec<T>(gs + (il + 1) * GS, g1);
                    } else {
                        g1[0] = g1[1] = make_float2(0.f, 0.f);
                    }
                    add_bias(g0);
                    add_bias(g1);
#pragma unroll
                    for (int pp = 0; pp < ST + 3; ++pp) {
                        const int r = i * ST + pp - g.pt;
                        if (r >= L) break;     // this and later frames are padding
                        if (r < 0) continue;   // zero fill
                        const T *xr = xs + (il * ST + pp) * RS;
#pragma unroll
                        for (int q = 0; q < 3; ++q) {
                            float2 xv[2];
                            lds_vec<T>(xr + q * g.CS, xv);
                            if (pp < 3) {
                                acc[pp * 3 + q][0] = ffma2(g0[0], xv[0], acc[pp * 3 + q][0]);
                                acc[pp * 3 + q][1] = ffma2(g0[1], xv[1], acc[pp * 3 + q][1]);
                            }
                            if (pp >= ST && pp - ST < 3) {
                                acc[(pp - ST) * 3 + q][0] = ffma2(g1[0], xv[0], acc[(pp - ST) * 3 + q][0]);
                                acc[(pp - ST) * 3 + q][1] = ffma2(g1[1], xv[1], acc[(pp - ST) * 3 + q][1]);
                            }
                        }
                    }
                }
            } else {
                for (int il = 0; il < g.TI; ++il) {
                    const int i = i0 + il;
                    if (i >= Lo) break;
                    float2 gv[2];
                    lds_vec<T>(gs + il * GS, gv);
                    add_bias(gv);
#pragma unroll
                    for (int p = 0; p < 3; ++p) {
                        const int r = i * g.st + p - g.pt;
                        if (r >= L) break;
                        if (r < 0) continue;
                        const T *xr = xs + (il * g.st + p) * RS;
#pragma unroll
                        for (int q = 0; q < 3; ++q) {
                            float2 xv[2];
                            lds_vec<T>(xr + q * g.CS, xv);
                            acc[p * 3 + q][0] = ffma2(gv[0], xv[0], acc[p * 3 + q][0]);
                            acc[p * 3 + q][1] = ffma2(gv[1], xv[1], acc[p * 3 + q][1]);
                        }
                    }
                }
            }
        }
        __syncthreads();
        ++n;
    }
    // fixed-order sum over the position groups (the stages are free: the last copy was consumed)
    float *red = reinterpret_cast<float *>(sm.stage[0]);  // [NPG][10][CS]
#pragma unroll
    for (int k = 0; k < 10; ++k) {
        float *d = red + (static_cast<int64_t>(pg) * 10 + k) * g.CS + cv * kC2V;
        d[0] = acc[k][0].x;
        d[1] = acc[k][0].y;
        d[2] = acc[k][1].x;
        d[3] = acc[k][1].y;
    }
    __syncthreads();
    for (int e = tid; e < 10 * g.CS; e += blockDim.x) {
        const int k = e / g.CS, ch = e % g.CS;
        if (cs * g.CS + ch >= g.C) continue;
        float sum = 0.f;
        for (int q = 0; q < NPG; ++q) sum += red[(static_cast<int64_t>(q) * 10 + k) * g.CS + ch];
        partials[(static_cast<int64_t>(gi) * 10 + k) * g.C + cs * g.CS + ch] = sum;
    }
}

// ------------------------------------------------------------------------------ host side
cudaError_t make_map_4d(CUtensorMap *map, const void *base, int dtype, int64_t B, int64_t T, int64_t F, int64_t C,
                        int box_c, int box_f, int box_t) {
    TensorMapEncodeTiledFn enc = tensor_map_encoder();
    if (enc == nullptr) return cudaErrorNotSupported;
    const cuuint64_t es = static_cast<cuuint64_t>(dtype_bytes(dtype));
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(F), static_cast<cuuint64_t>(T),
                                static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(C) * es, static_cast<cuuint64_t>(F * C) * es,
                                   static_cast<cuuint64_t>(T * F * C) * es};
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(box_c), static_cast<cuuint32_t>(box_f),
                               static_cast<cuuint32_t>(box_t), 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = enc(map, tma_dtype(dtype), 4,
                           const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorNotSupported;
}

bool aligned16(const void *p) { return reinterpret_cast<uintptr_t>(p) % 16 == 0; }
bool aligned8(const void *p) { return p == nullptr || reinterpret_cast<uintptr_t>(p) % 8 == 0; }

// 3x3 window; channels-last rows 16-byte aligned; every count of the tensor map in range.
bool c2_eligible(const Conv2dArgs &a, const void *act0, const void *act1) {
    const int es = dtype_bytes(a.dtype);
    if (a.KT != 3 || a.KF != 3) return false;
    if ((a.C * es) % 16 != 0 || !aligned16(act0) || !aligned16(act1)) return false;
    if (!aligned8(a.w) || !aligned8(a.bias)) return false;
    if (a.B * a.T >= (int64_t(1) << 31) || a.B * a.To >= (int64_t(1) << 31)) return false;
    return true;
}

// Smallest power-of-two channel slab >= C, between 32 and cs_max (C is a multiple of 4 here).
int pick_cs(int64_t C, int cs_max) {
    int cs = 32;
    while (cs < cs_max && cs < C) cs *= 2;
    return cs;
}

int blocks_per_sm(const void *kern, int threads, size_t smem) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, smem) != cudaSuccess || n < 1) n = 1;
    return n;
}

template <typename T>
cudaError_t fwd_tma(const Conv2dArgs &a, cudaStream_t s) {
    const int es = sizeof(T);
    C2Geo g{};
    g.B = static_cast<int>(a.B); g.T = static_cast<int>(a.T); g.F = static_cast<int>(a.F); g.C = static_cast<int>(a.C);
    g.To = static_cast<int>(a.To); g.Fo = static_cast<int>(a.Fo);
    g.st = a.st; g.sf = a.sf; g.pt = a.pt; g.pb = a.pb; g.pf = a.pf;
    g.CS = pick_cs(a.C, 64);
    g.TJ = static_cast<int>((a.Fo + (a.Fo + 15) / 16 - 1) / ((a.Fo + 15) / 16));  // <= 16, even split
    g.BF = a.sf * (g.TJ - 1) + 3;
    if (g.BF > 256) return cudaErrorNotSupported;
    const int pix = g.BF * g.CS * es;
    g.TI = 0;
    for (int ti : {4, 2, 1}) {
        const int br = a.st * (ti - 1) + 3;
        if (br <= 256 && br * pix <= kC2StageMax / 2) {
            g.TI = ti;
            break;
        }
    }
    if (g.TI == 0) return cudaErrorNotSupported;
    g.BR = a.st * (g.TI - 1) + 3;
    g.nI = static_cast<int>((a.To + g.TI - 1) / g.TI);
    g.nJ = static_cast<int>((a.Fo + g.TJ - 1) / g.TJ);
    g.nCS = static_cast<int>((a.C + g.CS - 1) / g.CS);
    g.stage_bytes = g.tx_bytes = g.BR * pix;
    CUtensorMap map;
    cudaError_t e = make_map_4d(&map, a.x, dtype_code<T>(), a.B, a.T, a.F, a.C, g.CS, g.BF, g.BR);
    if (e != cudaSuccess) return e;
    const int threads = ((g.TJ * (g.CS / kC2V) + 31) / 32) * 32;
    const size_t smem = kC2Head + 2 * static_cast<size_t>(g.stage_bytes);
    // the row-pair path needs an even row count per tile and a compiled stride
    auto kern = (g.TI % 2 == 0 && a.st == 2) ? c2_fwd_tma_kernel<T, 2>
                : (g.TI % 2 == 0 && a.st == 1) ? c2_fwd_tma_kernel<T, 1> : c2_fwd_tma_kernel<T, 0>;
    if ((e = ensure_smem_attr(reinterpret_cast<const void *>(kern), static_cast<int>(smem))) != cudaSuccess) return e;
    const int64_t ntiles = static_cast<int64_t>(g.B) * g.nI * g.nJ * g.nCS;
    if (ntiles >= (int64_t(1) << 30)) return cudaErrorNotSupported;  // tile indices stay far from int overflow
    const int64_t cap = static_cast<int64_t>(sm_count()) * blocks_per_sm(reinterpret_cast<const void *>(kern), threads, smem);
    int64_t gridl = ntiles < cap ? ntiles : cap;
    gridl = gridl / g.nCS * g.nCS;  // whole channel slabs per block (its taps stay in registers)
    if (gridl < g.nCS) gridl = g.nCS;
    const int grid = static_cast<int>(gridl);
    return launch_programmatic(kern, dim3(grid), dim3(threads), smem, s, map, a.w, a.bias, static_cast<T *>(a.y),
                               a.lengths, a.out_lengths, g);
}

// Stride 2 x 2: the 2x2-block kernel.  Tiles of TI (even) dx rows x TJ (even) columns; the box
// holds dy rows ia .. ia + TI/2 and columns ja .. ja + TJ/2.
template <typename T>
cudaError_t dx2_tma(const Conv2dArgs &a, cudaStream_t s) {
    const int es = sizeof(T);
    C2Geo g{};
    g.B = static_cast<int>(a.B); g.T = static_cast<int>(a.T); g.F = static_cast<int>(a.F); g.C = static_cast<int>(a.C);
    g.To = static_cast<int>(a.To); g.Fo = static_cast<int>(a.Fo);
    g.st = 2; g.sf = 2; g.pt = a.pt; g.pb = a.pb; g.pf = a.pf;
    g.CS = pick_cs(a.C, 64);
    const int csv = g.CS / kC2V;
    {  // column pairs per tile: at most 512 threads, the F columns split evenly over the tiles
        const int64_t maxp = 512 / csv, pairs = (a.F + 1) / 2, nj = (pairs + maxp - 1) / maxp;
        g.TJ = static_cast<int>(2 * ((pairs + nj - 1) / nj));
    }
    g.BF = g.TJ / 2 + 1;
    const int pix = g.BF * g.CS * es;
    g.TI = 0;
    for (int ti : {16, 8, 4, 2}) {
        if ((ti / 2 + 1) * pix <= kC2StageMax / 2) {
            g.TI = ti;
            break;
        }
    }
    if (g.TI == 0 || g.BF > 256) return cudaErrorNotSupported;
    g.BR = g.TI / 2 + 1;
    g.nI = static_cast<int>((a.T + g.TI - 1) / g.TI);
    g.nJ = static_cast<int>((a.F + g.TJ - 1) / g.TJ);
    g.nCS = static_cast<int>((a.C + g.CS - 1) / g.CS);
    g.stage_bytes = g.tx_bytes = g.BR * pix;
    CUtensorMap map;
    cudaError_t e = make_map_4d(&map, a.x, dtype_code<T>(), a.B, a.To, a.Fo, a.C, g.CS, g.BF, g.BR);
    if (e != cudaSuccess) return e;
    const int threads = ((g.TJ / 2 * csv + 31) / 32) * 32;
    const size_t smem = kC2Head + 2 * static_cast<size_t>(g.stage_bytes);
    const bool ro = (a.pt & 1) != 0, co = (a.pf & 1) != 0;
    auto kern = ro ? (co ? c2_dx2_tma_kernel<T, true, true> : c2_dx2_tma_kernel<T, true, false>)
                   : (co ? c2_dx2_tma_kernel<T, false, true> : c2_dx2_tma_kernel<T, false, false>);
    if ((e = ensure_smem_attr(reinterpret_cast<const void *>(kern), static_cast<int>(smem))) != cudaSuccess) return e;
    const int64_t ntiles = static_cast<int64_t>(g.B) * g.nI * g.nJ * g.nCS;
    if (ntiles >= (int64_t(1) << 30)) return cudaErrorNotSupported;
    const int64_t cap = static_cast<int64_t>(sm_count()) * blocks_per_sm(reinterpret_cast<const void *>(kern), threads, smem);
    int64_t gridl = ntiles < cap ? ntiles : cap;
    gridl = gridl / g.nCS * g.nCS;  // whole channel slabs per block (its taps stay in registers)
    if (gridl < g.nCS) gridl = g.nCS;
    const int grid = static_cast<int>(gridl);
    return launch_programmatic(kern, dim3(grid), dim3(threads), smem, s, map, a.w, static_cast<T *>(a.y), a.lengths, g);
}

template <typename T>
cudaError_t dx_tma(const Conv2dArgs &a, cudaStream_t s) {
    if (a.st == 2 && a.sf == 2) return dx2_tma<T>(a, s);
    const int es = sizeof(T);
    C2Geo g{};
    g.B = static_cast<int>(a.B); g.T = static_cast<int>(a.T); g.F = static_cast<int>(a.F); g.C = static_cast<int>(a.C);
    g.To = static_cast<int>(a.To); g.Fo = static_cast<int>(a.Fo);
    g.st = a.st; g.sf = a.sf; g.pt = a.pt; g.pb = a.pb; g.pf = a.pf;
    g.CS = pick_cs(a.C, 128);
    const int csv = g.CS / kC2V;
    {  // columns per tile: at most 512 threads, the F columns split evenly over the tiles
        const int64_t maxj = 512 / csv, nj = (a.F + maxj - 1) / maxj;
        g.TJ = static_cast<int>((a.F + nj - 1) / nj);
    }
    g.BF = (g.TJ + a.sf) / a.sf + 1;
    const int pix = g.BF * g.CS * es;
    g.TI = 0;
    for (int ti : {32, 16, 8, 4, 2, 1}) {
        const int br = (ti + a.st) / a.st + 1;
        if (br <= 256 && br * pix <= kC2StageMax) {
            g.TI = ti;
            break;
        }
    }
    if (g.TI == 0 || g.BF > 256) return cudaErrorNotSupported;
    g.BR = (g.TI + a.st) / a.st + 1;
    g.nI = static_cast<int>((a.T + g.TI - 1) / g.TI);
    g.nJ = static_cast<int>((a.F + g.TJ - 1) / g.TJ);
    g.nCS = static_cast<int>((a.C + g.CS - 1) / g.CS);
    g.stage_bytes = g.tx_bytes = g.BR * pix;
    CUtensorMap map;
    cudaError_t e = make_map_4d(&map, a.x, dtype_code<T>(), a.B, a.To, a.Fo, a.C, g.CS, g.BF, g.BR);
    if (e != cudaSuccess) return e;
    const int threads = ((g.TJ * csv + 31) / 32) * 32;
    const size_t smem = kC2Head + 2 * static_cast<size_t>(g.stage_bytes) + static_cast<size_t>(g.TI) * 3 * sizeof(int);
    auto kern = c2_dx_tma_kernel<T>;
    if ((e = ensure_smem_attr(reinterpret_cast<const void *>(kern), static_cast<int>(smem))) != cudaSuccess) return e;
    const int64_t ntiles = static_cast<int64_t>(g.B) * g.nI * g.nJ * g.nCS;
    if (ntiles >= (int64_t(1) << 30)) return cudaErrorNotSupported;  // tile indices stay far from int overflow
    const int64_t cap = static_cast<int64_t>(sm_count()) * blocks_per_sm(reinterpret_cast<const void *>(kern), threads, smem);
    int64_t gridl = ntiles < cap ? ntiles : cap;
    gridl = gridl / g.nCS * g.nCS;  // whole channel slabs per block (its taps stay in registers)
    if (gridl < g.nCS) gridl = g.nCS;
    const int grid = static_cast<int>(gridl);
    return launch_programmatic(kern, dim3(grid), dim3(threads), smem, s, map, a.w, static_cast<T *>(a.y), a.lengths, g);
}

template <typename T>
cudaError_t dw_tma(const Conv2dArgs &a, float *partials, int max_rows, int *G_out, cudaStream_t s) {
    const int es = sizeof(T);
    C2Geo g{};
    g.B = static_cast<int>(a.B); g.T = static_cast<int>(a.T); g.F = static_cast<int>(a.F); g.C = static_cast<int>(a.C);
    g.To = static_cast<int>(a.To); g.Fo = static_cast<int>(a.Fo);
    g.st = a.st; g.sf = a.sf; g.pt = a.pt; g.pb = a.pb; g.pf = a.pf;
    g.CS = pick_cs(a.C, 64);
    g.TJ = static_cast<int>((a.Fo + (a.Fo + 15) / 16 - 1) / ((a.Fo + 15) / 16));  // <= 16, even split
    g.BF = a.sf * (g.TJ - 1) + 3;
    if (g.BF > 256) return cudaErrorNotSupported;
    const int pix = g.BF * g.CS * es;
    g.TI = 0;
    for (int ti : {4, 2, 1}) {
        const int br = a.st * (ti - 1) + 3;
        const int xb = ((br * pix + 127) / 128) * 128;
        if (br <= 256 && xb + ti * g.TJ * g.CS * es <= kC2StageMax) {
            g.TI = ti;
            break;
        }
    }
    if (g.TI == 0) return cudaErrorNotSupported;
    g.BR = a.st * (g.TI - 1) + 3;
    g.nI = static_cast<int>((a.To + g.TI - 1) / g.TI);
    g.nJ = static_cast<int>((a.Fo + g.TJ - 1) / g.TJ);
    g.nCS = static_cast<int>((a.C + g.CS - 1) / g.CS);
    const int xbytes = ((g.BR * pix + 127) / 128) * 128;
    g.stage_bytes = xbytes + g.TI * g.TJ * g.CS * es;
    g.tx_bytes = g.BR * pix + g.TI * g.TJ * g.CS * es;
    CUtensorMap xm, gm;
    cudaError_t e = make_map_4d(&xm, a.x, dtype_code<T>(), a.B, a.T, a.F, a.C, g.CS, g.BF, g.BR);
    if (e != cudaSuccess) return e;
    if ((e = make_map_4d(&gm, a.y, dtype_code<T>(), a.B, a.To, a.Fo, a.C, g.CS, g.TJ, g.TI)) != cudaSuccess) return e;
    const int threads = ((g.TJ * (g.CS / kC2V) + 31) / 32) * 32;
    // the final reduction [groups][10][CS] float32 reuses the stages
    const size_t red = static_cast<size_t>(threads / (g.CS / kC2V)) * 10 * g.CS * sizeof(float);
    const size_t stages = 2 * static_cast<size_t>(g.stage_bytes);
    const size_t smem = kC2Head + (red > stages ? red : stages);
    auto kern = (g.TI % 2 == 0 && a.st == 2) ? c2_dw_tma_kernel<T, 2>
                : (g.TI % 2 == 0 && a.st == 1) ? c2_dw_tma_kernel<T, 1> : c2_dw_tma_kernel<T, 0>;
    if ((e = ensure_smem_attr(reinterpret_cast<const void *>(kern), static_cast<int>(smem))) != cudaSuccess) return e;
    const int64_t ntiles = static_cast<int64_t>(g.B) * g.nI * g.nJ;
    if (ntiles * g.nCS >= (int64_t(1) << 30)) return cudaErrorNotSupported;
    int64_t G = static_cast<int64_t>(sm_count()) * blocks_per_sm(reinterpret_cast<const void *>(kern), threads, smem) /
                g.nCS;
    if (G > ntiles) G = ntiles;
    if (G > max_rows) G = max_rows;
    if (G < 1) G = 1;
    *G_out = static_cast<int>(G);
    return launch_programmatic(kern, dim3(static_cast<unsigned>(G * g.nCS)), dim3(threads), smem, s, xm, gm, a.lengths,
                               partials, g, static_cast<int>(G), xbytes);
}

}  // namespace

cudaError_t conv2d_fwd_tma_launch(const Conv2dArgs &a, cudaStream_t s) {
    if (a.B == 0 || a.To == 0 || a.Fo == 0 || !c2_eligible(a, a.x, a.y)) return cudaErrorNotSupported;
    return with_dtype(a.dtype, [&](auto tag) { return fwd_tma<decltype(tag)>(a, s); });
}

cudaError_t conv2d_dx_tma_launch(const Conv2dArgs &a, cudaStream_t s) {
    if (a.B == 0 || a.T == 0 || a.To == 0 || a.Fo == 0 || !c2_eligible(a, a.x, a.y)) return cudaErrorNotSupported;
    return with_dtype(a.dtype, [&](auto tag) { return dx_tma<decltype(tag)>(a, s); });
}

cudaError_t conv2d_dw_tma_partials(const Conv2dArgs &a, float *partials, int max_rows, int *G, cudaStream_t s) {
    if (a.B == 0 || a.To == 0 || a.Fo == 0 || !c2_eligible(a, a.x, a.y)) return cudaErrorNotSupported;
    return with_dtype(a.dtype, [&](auto tag) { return dw_tma<decltype(tag)>(a, partials, max_rows, G, s); });
}

unsigned int conv2d_tma_take_error() {
    unsigned int h = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&h, dw_device_error_flag, sizeof(h)) != cudaSuccess) return 0;
    if (h) cudaMemcpyToSymbol(dw_device_error_flag, &zero, sizeof(zero));
    return h;
}

}  // namespace dwk
