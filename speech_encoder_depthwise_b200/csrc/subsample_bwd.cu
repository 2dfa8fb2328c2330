// Backward of the fused depthwise-striding subsampler front (NeMo PR #16114, "Use Fused Kernels
// for Depthwise Striding Subsampler", section "What does this PR do ?": the fused kernels come
// with their backward passes): the gradients of sum(out * dout) with respect to w0, b0, w1, b1.
//
// Every term is local to one h pixel (r, s) of one channel:
//   z      = b0 + sum_{p,q} melpad[2r+p, 2s+q] w0[p,q]          (recomputed, never stored)
//   h      = ReLU(z)                                             (rows r >= ceil(len/2) are 0)
//   for each tap (p, q) that maps an output pixel (i, j) onto (r, s), i.e. 2i+p-Pt = r and
//   2j+q-1 = s (one or two taps per axis), with doutm = [i < ceil(len/4)] dout[i, j]:
//       dh  += doutm w1[p,q]        dw1[p,q] += h doutm
//   dz     = [z > 0] dh
//   dw0[p,q] += dz melpad[2r+p, 2s+q]      db0 += dz
// and db1 += doutm[r/2, s/2] at even (r, s) (each output pixel exactly once).  Rows at or past
// ceil(len/2) contribute nothing: their h and dz are zero and the outputs they feed are masked.
//
// A persistent grid walks spatial tiles (item, 8 h rows, up to 20 h columns); a thread owns a
// channel pair and keeps all twenty gradient pairs in registers for its whole share of the
// tiles.  Per tile the mel window is staged once in shared memory as {m, m} pairs, and every
// thread stages its own window of dout values (requested together, so their latency overlaps).  Block b of a
// channel group writes one partial row; a finalize kernel adds the rows in a fixed order, so the
// results are reproducible for given sizes on a given GPU model.
#include "dw_internal.h"

namespace dwk {
namespace {

constexpr int kSbThreads = 128;                      // one thread per channel pair
constexpr int kSbRT = 8;                             // h rows per spatial tile
constexpr int kSbST = 20;                            // h columns per spatial tile
constexpr int kSbMR = 2 * kSbRT + 1;                 // staged mel rows
constexpr int kSbMC = 2 * kSbST + 1;                 // staged mel columns
constexpr int kSbSlots = 20;                         // dw0[9], db0, dw1[9], db1
constexpr int kSbMaxRows = 592;                      // partial rows per channel group (at most)
constexpr int kSbNRW = kSbRT / 2 + 2;                // output rows a tile's h rows read
constexpr int kSbNCW = kSbST / 2 + 3;                // output columns a tile's h columns read

// A thread's staged dout value: a 16-bit pair as one word (the values are exact in it), or a
// float pair.
template <typename TD> struct DWord {
    using type = float2;
    static __device__ __forceinline__ float2 get(float2 v) { return v; }
    static __device__ __forceinline__ void put(float2 v, float2 &w) { w = v; }
};
template <typename TD> struct DWord16 {
    using type = uint32_t;
    static __device__ __forceinline__ float2 get(uint32_t u) { return Half16<TD>::unpack(u); }
    static __device__ __forceinline__ void put(float2 v, uint32_t &w) { w = Half16<TD>::pack(v.x, v.y); }
};
template <> struct DWord<bf16> : DWord16<bf16> {};
template <> struct DWord<f16> : DWord16<f16> {};

template <typename TD, bool VEC>
__device__ __forceinline__ float2 load_dout(const TD *p, bool two) {
    if constexpr (VEC) {
        if constexpr (sizeof(TD) == 2) {
            return Half16<TD>::unpack(__ldg(reinterpret_cast<const unsigned int *>(p)));
        } else {
            return __ldg(reinterpret_cast<const float2 *>(p));
        }
    } else {
        auto f = [](const TD *q) -> float {
            if constexpr (sizeof(TD) == 2) return static_cast<float>(*q);
            else return __ldg(q);
        };
        return make_float2(f(p), two ? f(p + 1) : 0.f);
    }
}

__device__ __forceinline__ float2 relu_mask(float2 z, float2 v) {  // [z > 0] v, per channel
    return make_float2(z.x > 0.f ? v.x : 0.f, z.y > 0.f ? v.y : 0.f);
}

// One h row r of a tile, walking output columns k: output pixel column k feeds h columns 2k-1
// (tap q = 0), 2k (q = 1) and 2k+1 (q = 2), so each dout value is loaded once and the next
// column's values are loaded one step ahead.  EVEN: r + Pt even, so output rows iA = (r+Pt)/2
// (tap p = 0) and iB = iA - 1 (p = 2) feed the row; otherwise only iA = (r+Pt-1)/2 (p = 1).
template <typename TD, bool EVEN, typename W = typename DWord<TD>::type>
__device__ __forceinline__ void row_pass(int r, int R0, int S0, int send, int Pt, const W *win, int iLo, int kLo,
                                         const float2 (*sm)[kSbMC], const float2 (&W0)[9], const float2 (&W1)[9],
                                         float2 bias0, float2 (&gw0)[9], float2 (&gw1)[9], float2 &gb0,
                                         float2 &gb1) {
    constexpr int pA = EVEN ? 0 : 1;
    const int iA = EVEN ? (r + Pt) >> 1 : (r + Pt - 1) >> 1, iB = iA - 1;
    // this thread's staged window: [output row - iLo][output column - kLo], kSbThreads apart
    const W *rowA = win + (iA - iLo) * kSbNCW * kSbThreads, *rowB = win + (iB - iLo) * kSbNCW * kSbThreads;
    const float2 zero = make_float2(0.f, 0.f);
    auto load = [&](int k, float2 &a, float2 &bb) {
        a = DWord<TD>::get(rowA[(k - kLo) * kSbThreads]);
        bb = EVEN ? DWord<TD>::get(rowB[(k - kLo) * kSbThreads]) : zero;
    };
    // one h pixel (r, s) given its dh taps: recompute z, then every gradient term it owns
    auto pixel = [&](int s, float2 dh, const float2 (&d)[4], const int (&tap)[4], int nt, float2 db1v, bool own_b1) {
        const float2 *m0 = &sm[2 * (r - R0)][2 * (s - S0)];
        float2 mv[9];
#pragma unroll
        for (int p = 0; p < 3; ++p)
#pragma unroll
            for (int q = 0; q < 3; ++q) mv[3 * p + q] = m0[p * kSbMC + q];
        // three independent chains (one per tap row), then two adds: a short dependency chain
        float2 zr[3] = {bias0, make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int q = 0; q < 3; ++q)
#pragma unroll
            for (int p = 0; p < 3; ++p) zr[p] = ffma2(mv[3 * p + q], W0[3 * p + q], zr[p]);
        const float2 z = make_float2(zr[0].x + (zr[1].x + zr[2].x), zr[0].y + (zr[1].y + zr[2].y));
        const float2 h = make_float2(fmaxf(z.x, 0.f), fmaxf(z.y, 0.f));
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (u < nt) gw1[tap[u]] = ffma2(h, d[u], gw1[tap[u]]);
        if (own_b1) {
            gb1.x += db1v.x;
            gb1.y += db1v.y;
        }
        const float2 dz = relu_mask(z, dh);
        gb0.x += dz.x;
        gb0.y += dz.y;
#pragma unroll
        for (int t = 0; t < 9; ++t) gw0[t] = ffma2(dz, mv[t], gw0[t]);
    };
    const int k0 = S0 >> 1, k1 = send >> 1;  // h columns [S0, send) lie in output columns k0 .. k1;
                                             // the window holds columns k0 - 1 .. k1 + 1
    float2 pa, pb, ca, cb, na, nb;          // output column k-1, k and k+1 of rows iA, iB
    load(k0 - 1, pa, pb);
    load(k0, ca, cb);
    for (int k = k0; k <= k1; ++k) {
        load(k + 1, na, nb);
        const int so = 2 * k - 1, se = 2 * k;
        if (so >= S0 && so < send) {  // odd column: q = 0 from column k, q = 2 from column k-1
            float2 dh = ffma2(ca, W1[3 * pA + 0], ffma2(pa, W1[3 * pA + 2], zero));
            if (EVEN) dh = ffma2(cb, W1[6], ffma2(pb, W1[8], dh));
            const float2 d[4] = {ca, pa, cb, pb};
            const int tap[4] = {3 * pA + 0, 3 * pA + 2, 6, 8};
            pixel(so, dh, d, tap, EVEN ? 4 : 2, zero, false);
        }
        if (se >= S0 && se < send) {  // even column: q = 1 from column k
            float2 dh = ffma2(ca, W1[3 * pA + 1], zero);
            if (EVEN) dh = ffma2(cb, W1[7], dh);
            const float2 d[4] = {ca, cb, zero, zero};
            const int tap[4] = {3 * pA + 1, 7, 0, 0};
            // output pixel (r/2, k) is counted for db1 here, at h pixel (2i, 2k): its row is iA
            // when r + Pt is odd, iB when it is even
            pixel(se, dh, d, tap, EVEN ? 2 : 1, EVEN ? cb : ca, (r & 1) == 0);
        }
        pa = ca; pb = cb; ca = na; cb = nb;
    }
}

#ifndef DW_SB_MINB
#define DW_SB_MINB 4
#endif
template <typename TD, bool VEC>
__global__ void __launch_bounds__(kSbThreads, DW_SB_MINB)
dw_subsample_bwd_kernel(const float *__restrict__ mel, const float *__restrict__ w0, const float *__restrict__ b0,
                        const float *__restrict__ w1, const TD *__restrict__ dout,
                        const int32_t *__restrict__ lengths, float *__restrict__ partials, int B, int Tn, int F,
                        int C, int T2, int F2, int T4, int F4, int Pt, int nRT, int nST, int nCG) {
    using W = typename DWord<TD>::type;
    __shared__ __align__(16) float2 sm[kSbMR][kSbMC];
    extern __shared__ __align__(16) unsigned char dyn_smem[];
    W *win = reinterpret_cast<W *>(dyn_smem) + threadIdx.x;  // this thread's dout window
    const int cg = blockIdx.x % nCG, g = blockIdx.x / nCG, G = gridDim.x / nCG;
    const int c = (cg * kSbThreads + threadIdx.x) * 2;  // this thread's first channel
    const bool act = c < C, two = c + 1 < C;
    auto ld = [&](const float *p) { return make_float2(act ? __ldg(p) : 0.f, two ? __ldg(p + 1) : 0.f); };

    float2 W0[9], W1[9], bias0;
#pragma unroll
    for (int t = 0; t < 9; ++t) {
        W0[t] = ld(w0 + t * C + c);
        W1[t] = ld(w1 + t * C + c);
    }
    bias0 = ld(b0 + c);
    float2 gw0[9], gw1[9], gb0 = make_float2(0.f, 0.f), gb1 = make_float2(0.f, 0.f);
#pragma unroll
    for (int t = 0; t < 9; ++t) gw0[t] = gw1[t] = make_float2(0.f, 0.f);

    const int tiles = B * nRT * nST;
    for (int tile = g; tile < tiles; tile += G) {
        const int b = tile / (nRT * nST), rem = tile % (nRT * nST);
        const int R0 = (rem / nST) * kSbRT, S0 = (rem % nST) * kSbST;
        const int L = static_cast<int>(clamp_len(lengths, b, Tn));
        const int L2 = (L + 1) / 2, L4 = (L2 + 1) / 2;
        const int rend = min(R0 + kSbRT, L2), send = min(S0 + kSbST, F2);
        if (R0 >= rend) continue;  // every h row of the tile is masked: nothing to add
        // mel window: rows 2 R0 - Pt + [0, 2RT], columns 2 S0 - 1 + [0, 2ST]; zeros outside the
        // item and at frames t >= len
        __syncthreads();  // the previous tile's readers are done
        const float *mb = mel + static_cast<int64_t>(b) * Tn * F;
        for (int e = threadIdx.x; e < kSbMR * kSbMC; e += kSbThreads) {
            const int rr = e / kSbMC, cc = e % kSbMC;
            const int t = 2 * R0 - Pt + rr, f = 2 * S0 - 1 + cc;
            const float v = (t >= 0 && t < L && f >= 0 && f < F) ? __ldg(mb + static_cast<int64_t>(t) * F + f) : 0.f;
            sm[rr][cc] = make_float2(v, v);
        }
        __syncthreads();
        if (!act) continue;
        // this thread's dout values for the tile, all requested at once: output rows
        // iLo .. iLo + kSbNRW - 1 and columns kLo .. kLo + kSbNCW - 1, zero where masked or outside
        const TD *db = dout + static_cast<int64_t>(b) * T4 * F4 * C + c;
        const int i4 = L4 < T4 ? L4 : T4;  // output rows below this are unmasked
        const int iLo = (R0 + Pt - 2) >> 1, kLo = (S0 >> 1) - 1;
#pragma unroll 2
        for (int rr = 0; rr < kSbNRW; ++rr) {
            const int i = iLo + rr;
#pragma unroll
            for (int cc = 0; cc < kSbNCW; ++cc) {
                const int k = kLo + cc;
                float2 v = make_float2(0.f, 0.f);
                if (i >= 0 && i < i4 && k >= 0 && k < F4) v = load_dout<TD, VEC>(db + (static_cast<int64_t>(i) * F4 + k) * C, two);
                DWord<TD>::put(v, win[(rr * kSbNCW + cc) * kSbThreads]);
            }
        }
        for (int r = R0; r < rend; ++r) {
            // h row r receives taps p with r + Pt - p even: rows iA (p = 0 or 1) and, for p = 0,
            // also iB = iA - 1 with p = 2
            if (((r + Pt) & 1) == 0) row_pass<TD, true>(r, R0, S0, send, Pt, win, iLo, kLo, sm, W0, W1, bias0, gw0, gw1,
                                                        gb0, gb1);
            else row_pass<TD, false>(r, R0, S0, send, Pt, win, iLo, kLo, sm, W0, W1, bias0, gw0, gw1, gb0, gb1);
        }
    }
    if (!act) return;
    // partial row g: [slot][C], slots dw0 0..8, db0 9, dw1 10..18, db1 19
    float *row = partials + static_cast<int64_t>(g) * kSbSlots * C + c;
    auto put = [&](int slot, float2 v) {
        row[static_cast<int64_t>(slot) * C] = v.x;
        if (two) row[static_cast<int64_t>(slot) * C + 1] = v.y;
    };
#pragma unroll
    for (int t = 0; t < 9; ++t) {
        put(t, gw0[t]);
        put(10 + t, gw1[t]);
    }
    put(9, gb0);
    put(19, gb1);
}

// Sum of the partial rows in a fixed order: 8 row groups per column, then a fixed tree.
__global__ void __launch_bounds__(256)
dw_subsample_bwd_finalize_kernel(const float *__restrict__ partials, int G, int C, float *__restrict__ dw0,
                                 float *__restrict__ db0, float *__restrict__ dw1, float *__restrict__ db1) {
    __shared__ float red[8][33];
    const int col = threadIdx.x % 32, rg = threadIdx.x / 32;
    const int64_t E = static_cast<int64_t>(kSbSlots) * C;
    const int64_t e = static_cast<int64_t>(blockIdx.x) * 32 + col;
    float s = 0.f;
    if (e < E) {
        for (int r = rg; r < G; r += 8) s += __ldg(partials + static_cast<int64_t>(r) * E + e);
    }
    red[rg][col] = s;
    __syncthreads();
    if (rg == 0 && e < E) {
        const float t = ((red[0][col] + red[1][col]) + (red[2][col] + red[3][col])) +
                        ((red[4][col] + red[5][col]) + (red[6][col] + red[7][col]));
        const int slot = static_cast<int>(e / C), c = static_cast<int>(e % C);
        if (slot < 9) dw0[slot * C + c] = t;
        else if (slot == 9) db0[c] = t;
        else if (slot < 19) dw1[(slot - 10) * C + c] = t;
        else db1[c] = t;
    }
}

// The same sum for 16-byte aligned partials and at most kSbMaxRows4 rows: a block covers 64
// consecutive entries (16 lanes x float4) with 16 row groups; group r loads rows r, r+16, ... (all
// of its loads issued before the first add) and adds them in order, then the 16 group sums are
// added in a fixed tree.  Launched programmatically after the partial kernel.
constexpr int kSbFinGroups = 16, kSbMaxRows4 = 256;
__global__ void __launch_bounds__(256)
dw_subsample_bwd_finalize4_kernel(const float *__restrict__ partials, int G, int C, float *__restrict__ dw0,
                                  float *__restrict__ db0, float *__restrict__ dw1, float *__restrict__ db1) {
    __shared__ float4 red[kSbFinGroups][16];
    launch_dependents();     // the next kernel may start its own set-up
    grid_dependency_wait();  // the partial rows are complete and visible after this
    const int lane = threadIdx.x % 16, rg = threadIdx.x / 16;
    const int64_t E4 = static_cast<int64_t>(kSbSlots) * C / 4;
    const int64_t e4 = static_cast<int64_t>(blockIdx.x) * 16 + lane;
    const float4 *p4 = reinterpret_cast<const float4 *>(partials);
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    if (e4 < E4) {
        float4 v[kSbMaxRows4 / kSbFinGroups];
#pragma unroll
        for (int i = 0; i < kSbMaxRows4 / kSbFinGroups; ++i) {
            const int r = rg + i * kSbFinGroups;
            v[i] = r < G ? __ldg(p4 + static_cast<int64_t>(r) * E4 + e4) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int i = 0; i < kSbMaxRows4 / kSbFinGroups; ++i) {
            s.x += v[i].x;
            s.y += v[i].y;
            s.z += v[i].z;
            s.w += v[i].w;
        }
    }
    red[rg][lane] = s;
    __syncthreads();
    if (rg == 0 && e4 < E4) {
        float4 t[kSbFinGroups];
#pragma unroll
        for (int r = 0; r < kSbFinGroups; ++r) t[r] = red[r][lane];
#pragma unroll
        for (int w = 1; w < kSbFinGroups; w <<= 1) {
#pragma unroll
            for (int r = 0; r + w < kSbFinGroups; r += 2 * w) {
                t[r].x += t[r + w].x;
                t[r].y += t[r + w].y;
                t[r].z += t[r + w].z;
                t[r].w += t[r + w].w;
            }
        }
        const float o[4] = {t[0].x, t[0].y, t[0].z, t[0].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int64_t e = 4 * e4 + q;
            const int slot = static_cast<int>(e / C), c = static_cast<int>(e % C);
            if (slot < 9) dw0[slot * C + c] = o[q];
            else if (slot == 9) db0[c] = o[q];
            else if (slot < 19) dw1[(slot - 10) * C + c] = o[q];
            else db1[c] = o[q];
        }
    }
}

__global__ void dw_subsample_bwd_zero_kernel(float *dw0, float *db0, float *dw1, float *db1, int C) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e < 9 * C) {
        dw0[e] = 0.f;
        dw1[e] = 0.f;
    }
    if (e < C) {
        db0[e] = 0.f;
        db1[e] = 0.f;
    }
}

int64_t s2(int64_t n) { return n >= 1 ? (n - 1) / 2 + 1 : 0; }

}  // namespace

int subsample_bwd_partial_rows(int64_t B, int64_t T, int64_t F) {
    const int64_t T2 = s2(T), F2 = s2(F);
    const int64_t tiles = B * ((T2 + kSbRT - 1) / kSbRT) * ((F2 + kSbST - 1) / kSbST);
    return static_cast<int>(tiles < kSbMaxRows ? (tiles > 0 ? tiles : 1) : kSbMaxRows);
}

size_t subsample_bwd_workspace_bytes(int64_t B, int64_t T, int64_t F, int64_t C) {
    return static_cast<size_t>(subsample_bwd_partial_rows(B, T, F)) * kSbSlots * static_cast<size_t>(C) *
           sizeof(float);
}

cudaError_t subsample_bwd_launch(const SubsampleBwdArgs &a, cudaStream_t s) {
    const int Pt = a.causal ? 2 : 1;
    const int64_t T2 = s2(a.T), F2 = s2(a.F), T4 = s2(T2), F4 = s2(F2);
    if (a.B == 0 || T4 == 0) {
        dw_subsample_bwd_zero_kernel<<<static_cast<unsigned>((9 * a.C + 255) / 256), 256, 0, s>>>(
            a.dw0, a.db0, a.dw1, a.db1, static_cast<int>(a.C));
        return cudaGetLastError();
    }
    const int64_t E = static_cast<int64_t>(kSbSlots) * a.C;
    {
        int rows = 0;
        const cudaError_t et = subsample_bwd_tc_launch(a, subsample_bwd_partial_rows(a.B, a.T, a.F), &rows, s);
        if (et == cudaSuccess) {
            if (rows <= kSbMaxRows4 && reinterpret_cast<uintptr_t>(a.partials) % 16 == 0)
                return launch_programmatic(dw_subsample_bwd_finalize4_kernel, dim3(static_cast<unsigned>((E / 4 + 15) / 16)),
                                           dim3(256), 0, s, static_cast<const float *>(a.partials), rows,
                                           static_cast<int>(a.C), a.dw0, a.db0, a.dw1, a.db1);
            dw_subsample_bwd_finalize_kernel<<<static_cast<unsigned>((E + 31) / 32), 256, 0, s>>>(
                a.partials, rows, static_cast<int>(a.C), a.dw0, a.db0, a.dw1, a.db1);
            return cudaGetLastError();
        }
        if (et != cudaErrorNotSupported) return et;
    }
    const int nRT = static_cast<int>((T2 + kSbRT - 1) / kSbRT), nST = static_cast<int>((F2 + kSbST - 1) / kSbST);
    const int64_t nCG = (a.C + 2 * kSbThreads - 1) / (2 * kSbThreads);
    int G = subsample_bwd_partial_rows(a.B, a.T, a.F);
    // one wave of resident blocks over the device, never more than the workspace holds
    const bool half = a.dout_dtype != 0;
    const size_t dsmem = kSbNRW * kSbNCW * kSbThreads * (half ? sizeof(uint32_t) : sizeof(float2));
    int per_sm = 0;
    // the 16-bit instances share one occupancy (same registers and shared memory)
    const void *kern = half ? reinterpret_cast<const void *>(dw_subsample_bwd_kernel<bf16, true>)
                            : reinterpret_cast<const void *>(dw_subsample_bwd_kernel<float, true>);
    {
        const cudaError_t ea = ensure_smem_attr(kern, static_cast<int>(dsmem));
        if (ea != cudaSuccess) return ea;
    }
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kSbThreads, dsmem) != cudaSuccess || per_sm < 1) {
        (void)cudaGetLastError();
        per_sm = 2;
    }
    const int64_t per_group = (static_cast<int64_t>(sm_count()) * per_sm) / nCG;
    if (per_group >= 1 && per_group < G) G = static_cast<int>(per_group);
    const int64_t grid = static_cast<int64_t>(G) * nCG;
    if (grid > kMaxGrid || T4 * F4 * a.C >= (1LL << 31) || a.T * a.F >= (1LL << 31)) return cudaErrorInvalidConfiguration;
    const size_t es = half ? 2 : 4;
    cudaError_t e = cudaSuccess;
    const bool vec = (a.C % 2) == 0 && (reinterpret_cast<uintptr_t>(a.dout) % (2 * es)) == 0;
#define DW_SB_LAUNCH(TD, VV)                                                                                 \
    do {                                                                                                     \
    e = ensure_smem_attr(reinterpret_cast<const void *>(dw_subsample_bwd_kernel<TD, VV>),                    \
                         static_cast<int>(kSbNRW * kSbNCW * kSbThreads * sizeof(typename DWord<TD>::type)));   \
    if (e != cudaSuccess) return e;                                                                          \
    dw_subsample_bwd_kernel<TD, VV><<<static_cast<unsigned>(grid), kSbThreads,                              \
                                      kSbNRW * kSbNCW * kSbThreads * sizeof(typename DWord<TD>::type), s>>>(  \
        a.mel, a.w0, a.b0, a.w1, static_cast<const TD *>(a.dout), a.lengths, a.partials, static_cast<int>(a.B), \
        static_cast<int>(a.T), static_cast<int>(a.F), static_cast<int>(a.C), static_cast<int>(T2),          \
        static_cast<int>(F2), static_cast<int>(T4), static_cast<int>(F4), Pt, nRT, nST, static_cast<int>(nCG)); \
    } while (0)
    if (a.dout_dtype == 1) {
        if (vec) DW_SB_LAUNCH(bf16, true);
        else DW_SB_LAUNCH(bf16, false);
    } else if (a.dout_dtype == 2) {
        if (vec) DW_SB_LAUNCH(f16, true);
        else DW_SB_LAUNCH(f16, false);
    } else {
        if (vec) DW_SB_LAUNCH(float, true);
        else DW_SB_LAUNCH(float, false);
    }
#undef DW_SB_LAUNCH
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    dw_subsample_bwd_finalize_kernel<<<static_cast<unsigned>((E + 31) / 32), 256, 0, s>>>(
        a.partials, G, static_cast<int>(a.C), a.dw0, a.db0, a.dw1, a.db1);
    return cudaGetLastError();
}

}  // namespace dwk
