// Fused front of the depthwise-striding subsampler (NeMo PR #16114, "Use Fused Kernels for
// Depthwise Striding Subsampler", section "What does this PR do ?", first kernel):
//
//   mel [B,T,F] --conv0 3x3/s2, 1->C, +b0, ReLU, rows >= ceil(len/2) zeroed--> h [B,T2,F2,C]
//               --conv_dw1 depthwise 3x3/s2, +b1, rows >= ceil(len/4) zeroed--> out [B,T4,F4,C]
//
// h never leaves the SM.  Padding is zeros: 1|1 in time (2|0 when causal) and 1|1 in
// frequency, for both convolutions; mel frames at or beyond len_b count as zero.
//
// The path is FP32-FMA bound (9 FMAs per h element, 9 per output element, ~5 h elements
// per output), so the design is about keeping the FMA pipe fed:
//  - a block owns (item b, RI output rows, J output columns, up to 4 x 64 channels); each
//    thread owns one channel pair and computes with packed FMA (fma.rn.f32x2);
//  - the mel rows and columns the block needs are staged once in shared memory, each value
//    stored twice ({m, m}) so that a 16-byte shared load yields two ready FMA operands
//    broadcast to the whole warp;
//  - the thread walks its output rows top to bottom and its J columns left to right.  For
//    output row i it computes the two new h rows it needs (2i-Pt+1, 2i-Pt+2) column by column
//    and keeps the last one (2J+1 columns) in registers as the first h row of output row
//    i+1, so conv0 runs once per h element except for one h row per RI output rows and one
//    h column per column block;
//  - h rows that are masked or padding are skipped (zero), output rows at or beyond
//    ceil(len/4) only store zeros.
#include "dw_internal.h"

namespace dwk {

#ifndef DW_SUB_J
#define DW_SUB_J 4
#endif
#ifndef DW_SUB_RI
#define DW_SUB_RI 16
#endif
#ifndef DW_SUB_MINB
#define DW_SUB_MINB 5
#endif
constexpr int kSubJ = DW_SUB_J;          // output columns per thread
constexpr int kSubRI = DW_SUB_RI;        // output rows per block
constexpr int kSubWarpsMax = 4;          // channel tiles (64 channels each) per block
constexpr int kSubMinBlocks = DW_SUB_MINB;  // resident blocks per SM the register budget aims at

template <typename TO, bool VEC_STORE>
__device__ __forceinline__ void store_pair(TO *p, float2 v, bool has_y);

template <>
__device__ __forceinline__ void store_pair<bf16, true>(bf16 *p, float2 v, bool) {
    *reinterpret_cast<uint32_t *>(p) = pack_bf16x2(v.x, v.y);
}
template <>
__device__ __forceinline__ void store_pair<bf16, false>(bf16 *p, float2 v, bool has_y) {
    p[0] = __float2bfloat16_rn(v.x);
    if (has_y) p[1] = __float2bfloat16_rn(v.y);
}
template <>
__device__ __forceinline__ void store_pair<float, true>(float *p, float2 v, bool) {
    *reinterpret_cast<float2 *>(p) = v;
}
template <>
__device__ __forceinline__ void store_pair<float, false>(float *p, float2 v, bool has_y) {
    p[0] = v.x;
    if (has_y) p[1] = v.y;
}

__device__ __forceinline__ float2 relu2(float2 a) { return make_float2(fmaxf(a.x, 0.f), fmaxf(a.y, 0.f)); }

template <typename TO, bool VEC_STORE, int J, int RI>
__global__ void __launch_bounds__(kSubWarpsMax * 32, kSubMinBlocks)
dw_subsample_kernel(const float *__restrict__ mel, const float *__restrict__ w0,
                    const float *__restrict__ b0, const float *__restrict__ w1,
                    const float *__restrict__ b1, TO *__restrict__ out,
                    const int32_t *__restrict__ lengths, int32_t *__restrict__ out_lengths,
                    int B, int Tn, int F, int C, int T2, int F2, int T4, int F4, int Pt, int nCG,
                    int nJB, int nRC) {
    constexpr int NMR = 4 * RI + 3;   // mel rows a block reads
    constexpr int W = 4 * J + 8;      // staged mel columns: [4 j0 - 4, 4 j0 + 4 J + 4)
    __shared__ __align__(16) float2 sm[NMR][W];

    const int warps = blockDim.x / 32;
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
    int lin = blockIdx.x;
    const int cg = lin % nCG;
    lin /= nCG;
    const int jb = lin % nJB;
    lin /= nJB;
    const int rc = lin % nRC;
    const int b = lin / nRC;

    if (blockIdx.x == 0 && out_lengths != nullptr) {
        for (int q = threadIdx.x; q < B; q += blockDim.x) {
            const int Lq = static_cast<int>(clamp_len(lengths, q, Tn));
            out_lengths[q] = ((Lq + 1) / 2 + 1) / 2;
        }
    }
    const int L = static_cast<int>(clamp_len(lengths, b, Tn));
    const int L2 = (L + 1) / 2, L4 = (L2 + 1) / 2;
    const int hrows = L2 < T2 ? L2 : T2;   // h rows that are neither padding nor masked
    const int i0 = rc * RI;
    const int j0 = jb * J;
    const int mrow0 = 4 * i0 - 3 * Pt;     // first mel row staged
    const int mcol0 = 4 * j0 - 4;          // first mel column staged
    const int c = (cg * warps + warp) * 64 + 2 * lane;
    const bool has_x = c < C, has_y = c + 1 < C;
    const bool any_valid = i0 < L4;        // some output row of this block is unmasked

    if (any_valid) {
        const float *melb = mel + static_cast<int64_t>(b) * Tn * F;
        for (int e = threadIdx.x; e < NMR * W; e += blockDim.x) {
            const int rr = e / W, cc = e % W;
            const int mr = mrow0 + rr, mc = mcol0 + cc;
            float v = 0.f;
            if (mr >= 0 && mr < L && mc >= 0 && mc < F) v = __ldg(melb + mr * F + mc);  // frames >= len read as 0
            sm[rr][cc] = make_float2(v, v);
        }
    }
    __syncthreads();
    if (!has_x) return;

    TO *ob = out + static_cast<int64_t>(b) * T4 * F4 * C + c;
    const int jn = (F4 - j0) < J ? (F4 - j0) : J;  // columns of this block
    const int iend = (i0 + RI) < T4 ? (i0 + RI) : T4;
    if (!any_valid) {  // every row of this block is masked: zeros only
        for (int i = i0; i < iend; ++i)
            for (int jj = 0; jj < jn; ++jj)
                store_pair<TO, VEC_STORE>(ob + (i * F4 + j0 + jj) * C, make_float2(0.f, 0.f), has_y);
        return;
    }

    float2 w0r[9], w1r[9], b0r, b1r;
#pragma unroll
    for (int t = 0; t < 9; ++t) {
        w0r[t] = make_float2(__ldg(w0 + t * C + c), has_y ? __ldg(w0 + t * C + c + 1) : 0.f);
        w1r[t] = make_float2(__ldg(w1 + t * C + c), has_y ? __ldg(w1 + t * C + c + 1) : 0.f);
    }
    b0r = make_float2(__ldg(b0 + c), has_y ? __ldg(b0 + c + 1) : 0.f);
    b1r = make_float2(__ldg(b1 + c), has_y ? __ldg(b1 + c + 1) : 0.f);

    // carry[n] = h(first h row of the current output row, column 2 j0 - 1 + n)
    float2 carry[2 * J + 1];
    {
        const int r = 2 * i0 - Pt;               // staged row 0 is its first mel row
        const bool rv = r >= 0 && r < hrows;
#pragma unroll
        for (int n = 0; n < 2 * J + 1; ++n) {
            const int hc = 2 * j0 - 1 + n;
            float2 a = b0r;
#pragma unroll
            for (int p = 0; p < 3; ++p)
#pragma unroll
                for (int q = 0; q < 3; ++q) a = ffma2(sm[p][2 * n + 1 + q], w0r[p * 3 + q], a);
            carry[n] = (rv && hc >= 0 && hc < F2) ? relu2(a) : make_float2(0.f, 0.f);
        }
    }

    for (int i = i0; i < iend; ++i) {
        TO *orow = ob + (i * F4 + j0) * C;
        if (i >= L4) {  // this and every later row of the item are masked
            for (int jj = 0; jj < jn; ++jj) store_pair<TO, VEC_STORE>(orow + jj * C, make_float2(0.f, 0.f), has_y);
            continue;
        }
        const int r1 = 2 * i - Pt + 1, r2 = r1 + 1;   // the two new h rows
        const bool v1 = r1 >= 0 && r1 < hrows, v2 = r2 >= 0 && r2 < hrows;
        const int rr = 2 * r1 - Pt - mrow0;            // staged row of mel row 2 r1 - Pt
        // h column 2 j0 - 1 of rows r1, r2 (staged mel columns 1..3); column 3 then carries over
        float2 prev1 = b0r, prev2 = b0r, m0[5];
#pragma unroll
        for (int p = 0; p < 5; ++p) {
            const float2 m1 = sm[rr + p][1];
            const float4 m23 = *reinterpret_cast<const float4 *>(&sm[rr + p][2]);
            const float2 m[3] = {m1, make_float2(m23.x, m23.y), make_float2(m23.z, m23.w)};
            m0[p] = m[2];
            if (p <= 2) {
#pragma unroll
                for (int q = 0; q < 3; ++q) prev1 = ffma2(m[q], w0r[p * 3 + q], prev1);
            }
            if (p >= 2) {
#pragma unroll
                for (int q = 0; q < 3; ++q) prev2 = ffma2(m[q], w0r[(p - 2) * 3 + q], prev2);
            }
        }
        prev1 = (v1 && j0 > 0) ? relu2(prev1) : make_float2(0.f, 0.f);
        prev2 = (v2 && j0 > 0) ? relu2(prev2) : make_float2(0.f, 0.f);
#pragma unroll
        for (int jj = 0; jj < J; ++jj) {
            const int j = j0 + jj;
            const bool cv1 = 2 * j < F2, cv2 = 2 * j + 1 < F2;
            // mel columns 4j-1 .. 4j+3 are staged columns 3+4jj .. 7+4jj (column 3+4jj carries
            // over from the previous column).  Window row p feeds h row r1 through tap row p
            // (p <= 2) and h row r2 through tap row p-2 (p >= 2); each row is used as it arrives.
            float2 a1 = b0r, a2 = b0r, c1 = b0r, c2 = b0r;
#pragma unroll
            for (int p = 0; p < 5; ++p) {
                const float4 lo = *reinterpret_cast<const float4 *>(&sm[rr + p][4 + 4 * jj]);
                const float4 hi = *reinterpret_cast<const float4 *>(&sm[rr + p][6 + 4 * jj]);
                const float2 m[5] = {m0[p], make_float2(lo.x, lo.y), make_float2(lo.z, lo.w),
                                     make_float2(hi.x, hi.y), make_float2(hi.z, hi.w)};
                m0[p] = m[4];
                if (p <= 2) {
#pragma unroll
                    for (int q = 0; q < 3; ++q) {
                        a1 = ffma2(m[q], w0r[p * 3 + q], a1);
                        a2 = ffma2(m[q + 2], w0r[p * 3 + q], a2);
                    }
                }
                if (p >= 2) {
#pragma unroll
                    for (int q = 0; q < 3; ++q) {
                        c1 = ffma2(m[q], w0r[(p - 2) * 3 + q], c1);
                        c2 = ffma2(m[q + 2], w0r[(p - 2) * 3 + q], c2);
                    }
                }
            }
            a1 = (v1 && cv1) ? relu2(a1) : make_float2(0.f, 0.f);
            a2 = (v1 && cv2) ? relu2(a2) : make_float2(0.f, 0.f);
            c1 = (v2 && cv1) ? relu2(c1) : make_float2(0.f, 0.f);
            c2 = (v2 && cv2) ? relu2(c2) : make_float2(0.f, 0.f);

            // conv_dw1 as three independent row sums, added at the end
            float2 o0 = b1r, o1 = make_float2(0.f, 0.f), o2 = make_float2(0.f, 0.f);
            o0 = ffma2(carry[2 * jj], w1r[0], o0);
            o1 = ffma2(prev1, w1r[3], o1);
            o2 = ffma2(prev2, w1r[6], o2);
            o0 = ffma2(carry[2 * jj + 1], w1r[1], o0);
            o1 = ffma2(a1, w1r[4], o1);
            o2 = ffma2(c1, w1r[7], o2);
            o0 = ffma2(carry[2 * jj + 2], w1r[2], o0);
            o1 = ffma2(a2, w1r[5], o1);
            o2 = ffma2(c2, w1r[8], o2);
            const float2 o = make_float2(o0.x + o1.x + o2.x, o0.y + o1.y + o2.y);
            if (jj < jn) store_pair<TO, VEC_STORE>(orow + jj * C, o, has_y);

            carry[2 * jj] = prev2;
            carry[2 * jj + 1] = c1;
            prev1 = a2;
            prev2 = c2;
        }
        carry[2 * J] = prev2;
    }
}

cudaError_t subsample_launch(const SubsampleArgs &a, cudaStream_t s) {
    const int Pt = a.causal ? 2 : 1;
    auto s2 = [](int64_t n) -> int64_t { return n >= 1 ? (n - 1) / 2 + 1 : 0; };
    const int64_t T2 = s2(a.T), F2 = s2(a.F), T4 = s2(T2), F4 = s2(F2);
    if (a.B == 0 || T4 == 0) return cudaSuccess;
    const int64_t nCT = (a.C + 63) / 64;
    const int warps = static_cast<int>(nCT < kSubWarpsMax ? nCT : kSubWarpsMax);
    const int64_t nCG = (nCT + warps - 1) / warps;
    const int64_t nJB = (F4 + kSubJ - 1) / kSubJ;
    const int64_t nRC = (T4 + kSubRI - 1) / kSubRI;
    const int64_t grid = a.B * nRC * nJB * nCG;
    // indices inside the kernel are 32-bit: an item's output and mel planes must fit
    if (grid > kMaxGrid || T4 * F4 * a.C >= (1LL << 31) || a.T * a.F >= (1LL << 31) || 9 * a.C >= (1LL << 31))
        return cudaErrorInvalidConfiguration;
    const bool even = (a.C % 2) == 0;
    const bool aligned = (reinterpret_cast<uintptr_t>(a.out) % (a.bf16_out ? 4 : 8)) == 0;
    const bool vec = even && aligned;
#define DW_SUB_LAUNCH(TO, VS)                                                                           \
    dw_subsample_kernel<TO, VS, kSubJ, kSubRI><<<static_cast<unsigned>(grid), warps * 32, 0, s>>>(          \
        a.mel, a.w0, a.b0, a.w1, a.b1, static_cast<TO *>(a.out), a.lengths, a.out_lengths,                   \
        static_cast<int>(a.B), static_cast<int>(a.T), static_cast<int>(a.F), static_cast<int>(a.C),           \
        static_cast<int>(T2), static_cast<int>(F2), static_cast<int>(T4), static_cast<int>(F4), Pt,          \
        static_cast<int>(nCG), static_cast<int>(nJB), static_cast<int>(nRC))
    if (a.bf16_out) {
        if (vec) DW_SUB_LAUNCH(bf16, true);
        else DW_SUB_LAUNCH(bf16, false);
    } else {
        if (vec) DW_SUB_LAUNCH(float, true);
        else DW_SUB_LAUNCH(float, false);
    }
#undef DW_SUB_LAUNCH
    return cudaGetLastError();
}

__global__ void dw_out_lengths_kernel(const int32_t *__restrict__ lengths, int32_t *__restrict__ out_lengths,
                                      int64_t B, int64_t Tn) {
    const int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (b >= B) return;
    const int64_t L = clamp_len(lengths, b, Tn);
    out_lengths[b] = static_cast<int32_t>(((L + 1) / 2 + 1) / 2);
}

cudaError_t subsample_out_lengths_launch(const int32_t *lengths, int32_t *out_lengths, int64_t B, int64_t T,
                                         cudaStream_t s) {
    if (B == 0) return cudaSuccess;
    dw_out_lengths_kernel<<<static_cast<unsigned>((B + 255) / 256), 256, 0, s>>>(lengths, out_lengths, B, T);
    return cudaGetLastError();
}

}  // namespace dwk
