// Shared device helpers: channel-vector loads/stores of bf16, fp16 or float32, 16-bit <->
// float32 conversion, packed float32x2 FMA.  sm_100a only.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dwk {

typedef __nv_bfloat16 bf16;
typedef __half f16;

__device__ __forceinline__ float bf16_lo(uint32_t p) { return __uint_as_float(p << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t p) { return __uint_as_float(p & 0xffff0000u); }

// Two floats to a bf16 pair, round to nearest even; `lo` lands in the low 16 bits.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

#ifdef DW_SCALAR_FMA
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    return make_float2(fmaf(a.x, b.x, c.x), fmaf(a.y, b.y, c.y));
}
#else
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
#endif

// Raw storage for V consecutive channels of element type T, loaded with one instruction.
// Words are 32-bit; a 16-bit pair (bf16 or fp16) sits in one word (low half = lower channel).
template <typename T, int V> struct Vec;

// The two 16-bit element types: unpacking a pair word to float32 and packing two float32 values
// (round to nearest even) into one.
__device__ __forceinline__ float2 f16_pair(uint32_t p) {
    __half2 h;
    *reinterpret_cast<uint32_t *>(&h) = p;
    return __half22float2(h);
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}
template <typename T> struct Half16;
template <> struct Half16<bf16> {
    static __device__ __forceinline__ float2 unpack(uint32_t p) { return make_float2(bf16_lo(p), bf16_hi(p)); }
    static __device__ __forceinline__ uint32_t pack(float lo, float hi) { return pack_bf16x2(lo, hi); }
    static __device__ __forceinline__ float one(unsigned short r) { return __uint_as_float(static_cast<uint32_t>(r) << 16); }
    static __device__ __forceinline__ bf16 cvt(float v) { return __float2bfloat16_rn(v); }
};
template <> struct Half16<f16> {
    static __device__ __forceinline__ float2 unpack(uint32_t p) { return f16_pair(p); }
    static __device__ __forceinline__ uint32_t pack(float lo, float hi) { return pack_f16x2(lo, hi); }
    static __device__ __forceinline__ float one(unsigned short r) { return __half2float(__ushort_as_half(r)); }
    static __device__ __forceinline__ f16 cvt(float v) { return __float2half_rn(v); }
};

template <typename T> struct Vec16x8 {
    using H = Half16<T>;
    uint4 r;
    __device__ __forceinline__ void load(const T *p) { r = __ldg(reinterpret_cast<const uint4 *>(p)); }
    __device__ __forceinline__ void zero() { r = make_uint4(0, 0, 0, 0); }
    __device__ __forceinline__ void to_f2(float2 (&f)[4]) const {
        f[0] = H::unpack(r.x); f[1] = H::unpack(r.y); f[2] = H::unpack(r.z); f[3] = H::unpack(r.w);
    }
    static __device__ __forceinline__ void store(T *p, const float2 (&f)[4]) {
        uint4 o = make_uint4(H::pack(f[0].x, f[0].y), H::pack(f[1].x, f[1].y), H::pack(f[2].x, f[2].y),
                             H::pack(f[3].x, f[3].y));
        *reinterpret_cast<uint4 *>(p) = o;
    }
    static __device__ __forceinline__ void store_zero(T *p) { *reinterpret_cast<uint4 *>(p) = make_uint4(0, 0, 0, 0); }
};

template <typename T> struct Vec16x4 {
    using H = Half16<T>;
    uint2 r;
    __device__ __forceinline__ void load(const T *p) { r = __ldg(reinterpret_cast<const uint2 *>(p)); }
    __device__ __forceinline__ void zero() { r = make_uint2(0, 0); }
    __device__ __forceinline__ void to_f2(float2 (&f)[2]) const { f[0] = H::unpack(r.x); f[1] = H::unpack(r.y); }
    static __device__ __forceinline__ void store(T *p, const float2 (&f)[2]) {
        *reinterpret_cast<uint2 *>(p) = make_uint2(H::pack(f[0].x, f[0].y), H::pack(f[1].x, f[1].y));
    }
    static __device__ __forceinline__ void store_zero(T *p) { *reinterpret_cast<uint2 *>(p) = make_uint2(0, 0); }
};

template <typename T> struct Vec16x2 {
    using H = Half16<T>;
    uint32_t r;
    __device__ __forceinline__ void load(const T *p) { r = __ldg(reinterpret_cast<const unsigned int *>(p)); }
    __device__ __forceinline__ void zero() { r = 0; }
    __device__ __forceinline__ void to_f2(float2 (&f)[1]) const { f[0] = H::unpack(r); }
    static __device__ __forceinline__ void store(T *p, const float2 (&f)[1]) {
        *reinterpret_cast<uint32_t *>(p) = H::pack(f[0].x, f[0].y);
    }
    static __device__ __forceinline__ void store_zero(T *p) { *reinterpret_cast<uint32_t *>(p) = 0u; }
};

// One channel (any C, any alignment): the value travels as a float2 with .y = 0, so the
// same pairwise arithmetic serves every width.  The slow, general fallback.
template <typename T> struct Vec16x1 {
    using H = Half16<T>;
    unsigned short r;
    __device__ __forceinline__ void load(const T *p) { r = __ldg(reinterpret_cast<const unsigned short *>(p)); }
    __device__ __forceinline__ void zero() { r = 0; }
    __device__ __forceinline__ void to_f2(float2 (&f)[1]) const { f[0] = make_float2(H::one(r), 0.f); }
    static __device__ __forceinline__ void store(T *p, const float2 (&f)[1]) { *p = H::cvt(f[0].x); }
    static __device__ __forceinline__ void store_zero(T *p) { *reinterpret_cast<unsigned short *>(p) = 0; }
};

template <> struct Vec<bf16, 8> : Vec16x8<bf16> {};
template <> struct Vec<bf16, 4> : Vec16x4<bf16> {};
template <> struct Vec<bf16, 2> : Vec16x2<bf16> {};
template <> struct Vec<bf16, 1> : Vec16x1<bf16> {};
template <> struct Vec<f16, 8> : Vec16x8<f16> {};
template <> struct Vec<f16, 4> : Vec16x4<f16> {};
template <> struct Vec<f16, 2> : Vec16x2<f16> {};
template <> struct Vec<f16, 1> : Vec16x1<f16> {};

template <> struct Vec<float, 4> {
    float4 r;
    __device__ __forceinline__ void load(const float *p) { r = __ldg(reinterpret_cast<const float4 *>(p)); }
    __device__ __forceinline__ void zero() { r = make_float4(0.f, 0.f, 0.f, 0.f); }
    __device__ __forceinline__ void to_f2(float2 (&f)[2]) const {
        f[0] = make_float2(r.x, r.y); f[1] = make_float2(r.z, r.w);
    }
    static __device__ __forceinline__ void store(float *p, const float2 (&f)[2]) {
        *reinterpret_cast<float4 *>(p) = make_float4(f[0].x, f[0].y, f[1].x, f[1].y);
    }
    static __device__ __forceinline__ void store_zero(float *p) {
        *reinterpret_cast<float4 *>(p) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
};

template <> struct Vec<float, 2> {
    float2 r;
    __device__ __forceinline__ void load(const float *p) { r = __ldg(reinterpret_cast<const float2 *>(p)); }
    __device__ __forceinline__ void zero() { r = make_float2(0.f, 0.f); }
    __device__ __forceinline__ void to_f2(float2 (&f)[1]) const { f[0] = r; }
    static __device__ __forceinline__ void store(float *p, const float2 (&f)[1]) {
        *reinterpret_cast<float2 *>(p) = f[0];
    }
    static __device__ __forceinline__ void store_zero(float *p) {
        *reinterpret_cast<float2 *>(p) = make_float2(0.f, 0.f);
    }
};

template <> struct Vec<float, 1> {
    float r;
    __device__ __forceinline__ void load(const float *p) { r = __ldg(p); }
    __device__ __forceinline__ void zero() { r = 0.f; }
    __device__ __forceinline__ void to_f2(float2 (&f)[1]) const { f[0] = make_float2(r, 0.f); }
    static __device__ __forceinline__ void store(float *p, const float2 (&f)[1]) { *p = f[0].x; }
    static __device__ __forceinline__ void store_zero(float *p) { *p = 0.f; }
};

// Number of float2 pairs that carry V channels.
template <int V> struct Pairs { static constexpr int n = V >= 2 ? V / 2 : 1; };

// Element type of a dtype code (0 float32, 1 bf16, 2 fp16): `f` is called with a value of it.
template <typename Fn>
inline auto with_dtype(int dtype, Fn &&fn) -> decltype(fn(float{})) {
    switch (dtype) {
        case 1: return fn(bf16{});
        case 2: return fn(f16{});
        default: return fn(float{});
    }
}

// V consecutive float32 parameters (weights or biases) starting at p, as float2 pairs.
// V >= 2 needs p 8-byte aligned; V == 1 reads one float.
template <int V>
__device__ __forceinline__ void load_param(const float *p, float2 (&f)[Pairs<V>::n]) {
    if constexpr (V == 1) {
        f[0] = make_float2(__ldg(p), 0.f);
    } else {
#pragma unroll
        for (int i = 0; i < V / 2; ++i) f[i] = __ldg(reinterpret_cast<const float2 *>(p) + i);
    }
}

__device__ __forceinline__ int64_t clamp_len(const int32_t *lengths, int64_t b, int64_t T) {
    if (lengths == nullptr) return T;
    int64_t L = __ldg(lengths + b);
    return L < 0 ? 0 : (L > T ? T : L);
}

}  // namespace dwk

// ---------------------------------------------------------------------------------------
// Bulk asynchronous copies (global -> shared, completion counted on an mbarrier) and
// mbarrier helpers, in hand-written PTX for sm_90+/sm_100a.  Every wait is bounded: after
// kSpinLimit failed polls the waiter records an error in dw_device_error_flag (read and
// cleared by the host through dw_device_error()) and gives up, so a kernel never hangs.
// ---------------------------------------------------------------------------------------
namespace dwk {

// One error word per translation unit (each .cu file reads and clears its own copy).
static __device__ unsigned int dw_device_error_flag = 0;
constexpr unsigned int kErrWaitTimeout = 1u;
constexpr uint32_t kSpinLimit = 1u << 24;

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Make initialised barriers visible to the asynchronous (bulk copy) proxy.
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete; false (and the error flag set) if
// it does not within kSpinLimit polls.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint32_t limit = kSpinLimit) {
    for (uint32_t i = 0; i < limit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    atomicOr(&dw_device_error_flag, kErrWaitTimeout);
    return false;
}

// size bytes from global src to shared dst (both 16-byte aligned, size a multiple of 16),
// completion reported to bar as transaction bytes.
__device__ __forceinline__ void bulk_copy_g2s(void *dst, const void *src, uint32_t size, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(size), "r"(smem_addr(bar))
        : "memory");
}

}  // namespace dwk

namespace dwk {

// One box of a 3-D tensor map (coordinates innermost first: channel, frame, item) into shared
// memory, completion counted on bar.  The channel coordinate must be a multiple of 16 bytes;
// frame coordinates may be negative or past the end (those rows arrive as zeros).
__device__ __forceinline__ void tma_load_3d(void *dst, const void *tmap, int c, int t, int b, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c), "r"(t), "r"(b), "r"(smem_addr(bar))
        : "memory");
}

// L2 prefetch of one tensor box (no shared-memory destination, no completion to wait for).  Safe
// before grid_dependency_wait for the same reason as prefetch_l2: it only fills the cache.
__device__ __forceinline__ void tma_prefetch_3d(const void *tmap, int c, int t, int b) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                     reinterpret_cast<uint64_t>(tmap)),
                 "r"(c), "r"(t), "r"(b)
                 : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void *tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

}  // namespace dwk

namespace dwk {

// Balanced tile order.  Tiles whose first frame is at or beyond len_b only store zeros, so a
// plain round robin deals some blocks far more real work than others.  Instead every block
// builds, in shared memory, the per-item prefix counts of valid tiles (first frame < len_b)
// and of masked tiles, and deals tiles in the order: all valid tiles, then all masked tiles,
// each run channel-tile fastest.  Block i takes positions i, i + G, i + 2G, ...: every block
// gets the same number of valid tiles to within one.  Used when B <= kOrderMaxItems.
// (With nC = 1 and only positions below V it deals the valid frame-runs of one channel tile.)
constexpr int kOrderMaxItems = 1024;

struct TileOrder {
    const int *pv;   // [B+1] valid tiles before item b (times nC)
    const int *pm;   // [B+1] masked tiles before item b (times nC)
    const int *len;  // [B] clamped lengths
    int B, nT, nC, V;

    // Builds the three arrays with warp 0 of the calling block (all threads must call it, then sync).
    __device__ void build(int *spv, int *spm, int *slen, const int32_t *lengths, int Tn, int TT) {
        if (threadIdx.x < 32) {
            const int lane = threadIdx.x;
            int run_v = 0, run_m = 0;
            if (lane == 0) {
                spv[0] = 0;
                spm[0] = 0;
            }
            for (int base = 0; base < B; base += 32) {
                const int bb = base + lane;
                int nv = 0, nm = 0;
                if (bb < B) {
                    const int L = static_cast<int>(clamp_len(lengths, bb, Tn));
                    slen[bb] = L;
                    nv = (L + TT - 1) / TT;
                    nm = nT - nv;
                }
                int iv = nv * nC, im = nm * nC;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int tv = __shfl_up_sync(0xffffffffu, iv, o), tm = __shfl_up_sync(0xffffffffu, im, o);
                    if (lane >= o) {
                        iv += tv;
                        im += tm;
                    }
                }
                if (bb < B) {
                    spv[bb + 1] = run_v + iv;
                    spm[bb + 1] = run_m + im;
                }
                run_v += __shfl_sync(0xffffffffu, iv, 31);
                run_m += __shfl_sync(0xffffffffu, im, 31);
            }
        }
    }

    // Last item b with a[b] <= g (a non-decreasing, a[0] = 0 <= g).
    static __device__ __forceinline__ int find(const int *a, int n, int g) {
        int lo = 0, hi = n;  // invariant: a[lo] <= g, answer in [lo, hi)
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (a[mid] <= g) lo = mid;
            else hi = mid;
        }
        return lo;
    }

    __device__ __forceinline__ void map(int g, int &b, int &tt, int &ct, int &L) const {
        if (g < V) {
            b = find(pv, B, g);
            const int local = g - pv[b];
            tt = local / nC;
            ct = local % nC;
        } else {
            const int m = g - V;
            b = find(pm, B, m);
            const int local = m - pm[b];
            tt = (pv[b + 1] - pv[b]) / nC + local / nC;
            ct = local % nC;
        }
        L = len[b];
    }
};

}  // namespace dwk

namespace dwk {

// Programmatic dependent launch: a kernel launched with programmatic stream serialization may
// start while the previous kernel in the stream drains; it must wait (grid_dependency_wait)
// before touching memory the previous kernel writes.  A kernel lets its dependents launch
// early with launch_dependents (they still wait for its completion before reading).
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
// Warm L2 with the line holding p.  Safe before grid_dependency_wait: a prefetch only fills the
// cache (L2 is where the previous kernel's writes land), so later reads still see those writes.
__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(__cvta_generic_to_global(p)));
}

}  // namespace dwk
