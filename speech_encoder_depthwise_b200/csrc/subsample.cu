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
#include <type_traits>

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
#ifndef DW_SUB_NPR
#define DW_SUB_NPR 1
#endif
constexpr int kSubJ = DW_SUB_J;          // output columns per thread
constexpr int kSubRI = DW_SUB_RI;        // output rows per block
constexpr int kSubWarpsMax = 4;          // channel tiles (64 channels each) per block
constexpr int kSubMinBlocks = DW_SUB_MINB;  // resident blocks per SM the register budget aims at
constexpr int kSubNPR = DW_SUB_NPR;         // channel pairs per thread
#ifndef DW_SUB_SCALAR
#define DW_SUB_SCALAR 0
#endif
// 1: mel staged as plain floats and conv0 as scalar FMAs with the mel value as a direct operand
// (one 16-byte shared load gives four mel columns); 0: mel staged as {m, m} pairs and conv0 as
// packed FMAs (one 16-byte load gives two columns).
constexpr bool kSubScalar = DW_SUB_SCALAR != 0;

// acc += m * w for a channel pair: packed FMA with a {m, m} pair, or two scalar FMAs.
__device__ __forceinline__ float2 mel_fma(float2 m, float2 w, float2 acc) { return ffma2(m, w, acc); }
__device__ __forceinline__ float2 mel_fma(float m, float2 w, float2 acc) {
    return make_float2(fmaf(m, w.x, acc.x), fmaf(m, w.y, acc.y));
}
__device__ __forceinline__ void stage_mel(float2 &dst, float v) { dst = make_float2(v, v); }
__device__ __forceinline__ void stage_mel(float &dst, float v) { dst = v; }

// Staged mel columns c .. c+3 of one row (c a multiple of 4): one 16-byte shared load of plain
// floats, or two of {m, m} pairs.
__device__ __forceinline__ void load4(const float *row, int c, float (&m)[4]) {
    const float4 v = *reinterpret_cast<const float4 *>(row + c);
    m[0] = v.x; m[1] = v.y; m[2] = v.z; m[3] = v.w;
}
__device__ __forceinline__ void load4(const float2 *row, int c, float2 (&m)[4]) {
    const float4 a = *reinterpret_cast<const float4 *>(row + c), b = *reinterpret_cast<const float4 *>(row + c + 2);
    m[0] = make_float2(a.x, a.y); m[1] = make_float2(a.z, a.w);
    m[2] = make_float2(b.x, b.y); m[3] = make_float2(b.z, b.w);
}

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
__device__ __forceinline__ void store_pair<f16, true>(f16 *p, float2 v, bool) {
    *reinterpret_cast<uint32_t *>(p) = pack_f16x2(v.x, v.y);
}
template <>
__device__ __forceinline__ void store_pair<f16, false>(f16 *p, float2 v, bool has_y) {
    p[0] = __float2half_rn(v.x);
    if (has_y) p[1] = __float2half_rn(v.y);
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

// Stores NPR channel pairs (2*NPR consecutive channels) of one output pixel.
template <typename TO, bool VEC_STORE, int NPR>
__device__ __forceinline__ void store_pairs(TO *p, const float2 (&v)[NPR], int nvalid) {
    if constexpr (VEC_STORE) {
        if constexpr (NPR == 1) {
            store_pair<TO, true>(p, v[0], true);
        } else if constexpr (sizeof(TO) == 2) {
            *reinterpret_cast<uint2 *>(p) =
                make_uint2(Half16<TO>::pack(v[0].x, v[0].y), Half16<TO>::pack(v[1].x, v[1].y));
        } else {
            *reinterpret_cast<float4 *>(p) = make_float4(v[0].x, v[0].y, v[1].x, v[1].y);
        }
    } else {
#pragma unroll
        for (int q = 0; q < NPR; ++q) {
            if (2 * q < nvalid) store_pair<TO, false>(p + 2 * q, v[q], 2 * q + 1 < nvalid);
        }
    }
}

template <typename TO, bool VEC_STORE, int J, int RI, int NPR>
__global__ void __launch_bounds__(kSubWarpsMax * 32, kSubMinBlocks)
dw_subsample_kernel(const float *__restrict__ mel, const float *__restrict__ w0,
                    const float *__restrict__ b0, const float *__restrict__ w1,
                    const float *__restrict__ b1, TO *__restrict__ out,
                    const int32_t *__restrict__ lengths, int32_t *__restrict__ out_lengths,
                    int B, int Tn, int F, int C, int T2, int F2, int T4, int F4, int Pt, int nCG,
                    int nJB, int nRC) {
    constexpr int NMR = 4 * RI + 3;   // mel rows a block reads
    constexpr int W = 4 * J + 8;      // staged mel columns: [4 j0 - 4, 4 j0 + 4 J + 4)
    constexpr int CW = 64 * NPR;      // channels per warp
    using MelT = typename std::conditional<kSubScalar, float, float2>::type;
    __shared__ __align__(16) MelT sm[NMR][W];

    const int warps = blockDim.x / 32;
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
    int lin = blockIdx.x;
    const int cg = lin % nCG;
    lin /= nCG;
    const int jb = lin % nJB;
    lin /= nJB;
    const int rc = lin % nRC;
    const int b = lin / nRC;
    launch_dependents();     // the next kernel in the stream may start its own set-up
    grid_dependency_wait();  // launched programmatically: the previous kernel's writes are visible after this

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
    const int c = (cg * warps + warp) * CW + 2 * NPR * lane;  // first channel of this thread
    const int nvalid = C - c;                                  // channels of this thread inside C
    const bool any_valid = i0 < L4;        // some output row of this block is unmasked

    if (any_valid) {
        const float *melb = mel + static_cast<int64_t>(b) * Tn * F;
        for (int e = threadIdx.x; e < NMR * W; e += blockDim.x) {
            const int rr = e / W, cc = e % W;
            const int mr = mrow0 + rr, mc = mcol0 + cc;
            float v = 0.f;
            if (mr >= 0 && mr < L && mc >= 0 && mc < F) v = __ldg(melb + mr * F + mc);  // frames >= len read as 0
            stage_mel(sm[rr][cc], v);
        }
    }
    __syncthreads();
    if (nvalid <= 0) return;

    TO *ob = out + static_cast<int64_t>(b) * T4 * F4 * C + c;
    const int jn = (F4 - j0) < J ? (F4 - j0) : J;  // columns of this block
    const int iend = (i0 + RI) < T4 ? (i0 + RI) : T4;
    float2 zero2[NPR];
#pragma unroll
    for (int q = 0; q < NPR; ++q) zero2[q] = make_float2(0.f, 0.f);
    if (!any_valid) {  // every row of this block is masked: zeros only
        for (int i = i0; i < iend; ++i)
            for (int jj = 0; jj < jn; ++jj) store_pairs<TO, VEC_STORE, NPR>(ob + (i * F4 + j0 + jj) * C, zero2, nvalid);
        return;
    }

    float2 w0r[9][NPR], w1r[9][NPR], b0r[NPR], b1r[NPR];
    {
        auto ld = [&](const float *p, int k) { return k < nvalid ? __ldg(p + k) : 0.f; };
#pragma unroll
        for (int q = 0; q < NPR; ++q) {
#pragma unroll
            for (int t = 0; t < 9; ++t) {
                w0r[t][q] = make_float2(ld(w0 + t * C + c, 2 * q), ld(w0 + t * C + c, 2 * q + 1));
                w1r[t][q] = make_float2(ld(w1 + t * C + c, 2 * q), ld(w1 + t * C + c, 2 * q + 1));
            }
            b0r[q] = make_float2(ld(b0 + c, 2 * q), ld(b0 + c, 2 * q + 1));
            b1r[q] = make_float2(ld(b1 + c, 2 * q), ld(b1 + c, 2 * q + 1));
        }
    }

    // carry[n] = h(first h row of the current output row, column 2 j0 - 1 + n)
    float2 carry[2 * J + 1][NPR];
    {
        const int r = 2 * i0 - Pt;               // staged row 0 is its first mel row
        const bool rv = r >= 0 && r < hrows;
#pragma unroll
        for (int n = 0; n < 2 * J + 1; ++n) {
            const int hc = 2 * j0 - 1 + n;
            const bool ok = rv && hc >= 0 && hc < F2;
#pragma unroll
            for (int q = 0; q < NPR; ++q) {
                float2 a = b0r[q];
#pragma unroll
                for (int p = 0; p < 3; ++p)
#pragma unroll
                    for (int qq = 0; qq < 3; ++qq) a = mel_fma(sm[p][2 * n + 1 + qq], w0r[p * 3 + qq][q], a);
                carry[n][q] = ok ? relu2(a) : make_float2(0.f, 0.f);
            }
        }
    }
    // every h column of this block is inside [0, F2) except possibly column 2 j0 - 1 (j0 == 0)
    const bool cols_all = 2 * (j0 + J) <= F2;

    for (int i = i0; i < iend; ++i) {
        TO *orow = ob + (i * F4 + j0) * C;
        if (i >= L4) {  // this and every later row of the item are masked
            for (int jj = 0; jj < jn; ++jj) store_pairs<TO, VEC_STORE, NPR>(orow + jj * C, zero2, nvalid);
            continue;
        }
        const int r1 = 2 * i - Pt + 1, r2 = r1 + 1;   // the two new h rows
        const bool v1 = r1 >= 0 && r1 < hrows, v2 = r2 >= 0 && r2 < hrows;
        const int rr = 2 * r1 - Pt - mrow0;            // staged row of mel row 2 r1 - Pt
        // h column 2 j0 - 1 of rows r1, r2 (staged mel columns 1..3); column 3 then carries over
        float2 prev1[NPR], prev2[NPR];
        MelT m0[5];
#pragma unroll
        for (int q = 0; q < NPR; ++q) prev1[q] = prev2[q] = b0r[q];
#pragma unroll
        for (int p = 0; p < 5; ++p) {
            MelT m4[4];
            load4(sm[rr + p], 0, m4);   // staged columns 0..3; columns 1..3 are mel 4 j0 - 3 .. 4 j0 - 1
            const MelT m[3] = {m4[1], m4[2], m4[3]};
            m0[p] = m[2];
#pragma unroll
            for (int q = 0; q < NPR; ++q) {
                if (p <= 2) {
#pragma unroll
                    for (int qq = 0; qq < 3; ++qq) prev1[q] = mel_fma(m[qq], w0r[p * 3 + qq][q], prev1[q]);
                }
                if (p >= 2) {
#pragma unroll
                    for (int qq = 0; qq < 3; ++qq) prev2[q] = mel_fma(m[qq], w0r[(p - 2) * 3 + qq][q], prev2[q]);
                }
            }
        }
#pragma unroll
        for (int q = 0; q < NPR; ++q) {
            prev1[q] = (v1 && j0 > 0) ? relu2(prev1[q]) : make_float2(0.f, 0.f);
            prev2[q] = (v2 && j0 > 0) ? relu2(prev2[q]) : make_float2(0.f, 0.f);
        }

        // one output row; CHECK adds the per-column and per-row validity selects
        auto row = [&](auto check) {
            constexpr bool CHECK = decltype(check)::value;
#pragma unroll
            for (int jj = 0; jj < J; ++jj) {
                const int j = j0 + jj;
                const bool cv1 = 2 * j < F2, cv2 = 2 * j + 1 < F2;
                // mel columns 4j-1 .. 4j+3 are staged columns 3+4jj .. 7+4jj (column 3+4jj carries
                // over from the previous column).  Window row p feeds h row r1 through tap row p
                // (p <= 2) and h row r2 through tap row p-2 (p >= 2); each row is used as it arrives.
                float2 a1[NPR], a2[NPR], c1[NPR], c2[NPR];
#pragma unroll
                for (int q = 0; q < NPR; ++q) a1[q] = a2[q] = c1[q] = c2[q] = b0r[q];
#pragma unroll
                for (int p = 0; p < 5; ++p) {
                    MelT m4[4];
                    load4(sm[rr + p], 4 + 4 * jj, m4);
                    const MelT m[5] = {m0[p], m4[0], m4[1], m4[2], m4[3]};
                    m0[p] = m[4];
#pragma unroll
                    for (int q = 0; q < NPR; ++q) {
                        if (p <= 2) {
#pragma unroll
                            for (int qq = 0; qq < 3; ++qq) {
                                a1[q] = mel_fma(m[qq], w0r[p * 3 + qq][q], a1[q]);
                                a2[q] = mel_fma(m[qq + 2], w0r[p * 3 + qq][q], a2[q]);
                            }
                        }
                        if (p >= 2) {
#pragma unroll
                            for (int qq = 0; qq < 3; ++qq) {
                                c1[q] = mel_fma(m[qq], w0r[(p - 2) * 3 + qq][q], c1[q]);
                                c2[q] = mel_fma(m[qq + 2], w0r[(p - 2) * 3 + qq][q], c2[q]);
                            }
                        }
                    }
                }
                float2 o[NPR];
#pragma unroll
                for (int q = 0; q < NPR; ++q) {
                    if constexpr (CHECK) {
                        a1[q] = (v1 && cv1) ? relu2(a1[q]) : make_float2(0.f, 0.f);
                        a2[q] = (v1 && cv2) ? relu2(a2[q]) : make_float2(0.f, 0.f);
                        c1[q] = (v2 && cv1) ? relu2(c1[q]) : make_float2(0.f, 0.f);
                        c2[q] = (v2 && cv2) ? relu2(c2[q]) : make_float2(0.f, 0.f);
                    } else {
                        a1[q] = relu2(a1[q]);
                        a2[q] = relu2(a2[q]);
                        c1[q] = relu2(c1[q]);
                        c2[q] = relu2(c2[q]);
                    }
                    // conv_dw1 as two independent sums, added at the end
                    float2 oa = b1r[q], ob2 = make_float2(0.f, 0.f);
                    oa = ffma2(carry[2 * jj][q], w1r[0][q], oa);
                    ob2 = ffma2(prev1[q], w1r[3][q], ob2);
                    oa = ffma2(carry[2 * jj + 1][q], w1r[1][q], oa);
                    ob2 = ffma2(a1[q], w1r[4][q], ob2);
                    oa = ffma2(carry[2 * jj + 2][q], w1r[2][q], oa);
                    ob2 = ffma2(a2[q], w1r[5][q], ob2);
                    oa = ffma2(prev2[q], w1r[6][q], oa);
                    ob2 = ffma2(c1[q], w1r[7][q], ob2);
                    oa = ffma2(c2[q], w1r[8][q], oa);
                    o[q] = make_float2(oa.x + ob2.x, oa.y + ob2.y);
                    carry[2 * jj][q] = prev2[q];
                    carry[2 * jj + 1][q] = c1[q];
                    prev1[q] = a2[q];
                    prev2[q] = c2[q];
                }
                if (jj < jn) store_pairs<TO, VEC_STORE, NPR>(orow + jj * C, o, nvalid);
            }
        };
        if (v1 && v2 && cols_all) row(std::false_type{});
        else row(std::true_type{});
#pragma unroll
        for (int q = 0; q < NPR; ++q) carry[2 * J][q] = prev2[q];
    }
}

cudaError_t subsample_launch(const SubsampleArgs &a, bool tensor_cores, cudaStream_t s) {
    const int Pt = a.causal ? 2 : 1;
    auto s2 = [](int64_t n) -> int64_t { return n >= 1 ? (n - 1) / 2 + 1 : 0; };
    const int64_t T2 = s2(a.T), F2 = s2(a.F), T4 = s2(T2), F4 = s2(F2);
    if (a.B == 0 || T4 == 0) return cudaSuccess;
    if (tensor_cores && subsample_tc_eligible(a)) {
        const cudaError_t e = subsample_tc_launch(a, s);
        if (e != cudaErrorNotSupported) return e;
    }
    const int64_t nCT = (a.C + 64 * kSubNPR - 1) / (64 * kSubNPR);
    const int warps = static_cast<int>(nCT < kSubWarpsMax ? nCT : kSubWarpsMax);
    const int64_t nCG = (nCT + warps - 1) / warps;
    const int64_t nJB = (F4 + kSubJ - 1) / kSubJ;
    const int64_t nRC = (T4 + kSubRI - 1) / kSubRI;
    const int64_t grid = a.B * nRC * nJB * nCG;
    // indices inside the kernel are 32-bit: an item's output and mel planes must fit
    if (grid > kMaxGrid || T4 * F4 * a.C >= (1LL << 31) || a.T * a.F >= (1LL << 31) || 9 * a.C >= (1LL << 31))
        return cudaErrorInvalidConfiguration;
    // vector stores of 2*kSubNPR channels need C a multiple of that and an aligned output
    const int vch = 2 * kSubNPR;
    const bool vec = (a.C % vch) == 0 &&
                     (reinterpret_cast<uintptr_t>(a.out) % (static_cast<uintptr_t>(vch) * dtype_bytes(a.out_dtype))) == 0;
#define DW_SUB_LAUNCH(TO, VS)                                                                           \
    return launch_programmatic(dw_subsample_kernel<TO, VS, kSubJ, kSubRI, kSubNPR>, dim3(static_cast<unsigned>(grid)), \
        dim3(warps * 32), 0, s, a.mel, a.w0, a.b0, a.w1, a.b1, static_cast<TO *>(a.out), a.lengths, a.out_lengths, \
        static_cast<int>(a.B), static_cast<int>(a.T), static_cast<int>(a.F), static_cast<int>(a.C),           \
        static_cast<int>(T2), static_cast<int>(F2), static_cast<int>(T4), static_cast<int>(F4), Pt,          \
        static_cast<int>(nCG), static_cast<int>(nJB), static_cast<int>(nRC))
    if (a.out_dtype == 1) {
        if (vec) DW_SUB_LAUNCH(bf16, true);
        DW_SUB_LAUNCH(bf16, false);
    } else if (a.out_dtype == 2) {
        if (vec) DW_SUB_LAUNCH(f16, true);
        DW_SUB_LAUNCH(f16, false);
    }
    if (vec) DW_SUB_LAUNCH(float, true);
    DW_SUB_LAUNCH(float, false);
#undef DW_SUB_LAUNCH
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
