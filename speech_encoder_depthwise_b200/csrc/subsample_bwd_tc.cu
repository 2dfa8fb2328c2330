// Backward of the fused depthwise-striding subsampler front on the 5th-generation tensor cores
// (NeMo PR #16114, "Use Fused Kernels for Depthwise Striding Subsampler", section "What does
// this PR do ?": the fused kernels come with their backward passes).  Gradients of
// sum(out * dout) with respect to w0, b0, w1, b1; the mel input takes none.
//
// Per h pixel (r, s) and channel c (melpad, Pt as in the forward):
//   z  = b0 + sum_t w0[t] P[t],  P[3p+q] = melpad[2r+p, 2s+q]     (recomputed)
//   dh = sum over the taps (p, q) that map an output pixel (i, j) onto (r, s)
//        (2i + p - Pt = r, 2j + q - 1 = s) of doutm[i, j] w1[p, q]
//   dw1[p, q] += ReLU(z) doutm[i, j] over the same taps,   db1 = sum doutm
//   dz = [z > 0] dh,   dw0[t] += dz P[t],   db0 += dz
// Two of these are dense contractions over the taps or the pixels, and both run as tcgen05
// MMAs with the channels as M (128 per tile):
//   1. z:      D1[c, pixel] = A1[c, k] . B1[pixel, k]   (k: the forward's split patch layout, so
//              z is the forward's conv0 output, float32-accurate with the three-product split)
//   2. dw0/db0: D2[c, n] = A2[c, pixel] . B2[n, pixel] over the 32 pixels of a chunk,
//              A2 = dz (split hi | lo, two MMAs), B2 rows n: P_hi[0..8], P_lo[0..8], 1, 0...
//              so that dw0[t] = D2[t] + D2[9 + t] and db0 = D2[18].  Each chunk has its own
//              accumulator (two slots per group, read out two chunks later) and the chunk sums
//              are added in float32 registers: an accumulator carried over thousands of MMAs
//              loses the products' low bits against its own growing magnitude.
// The depthwise part (dh, dw1, db1) runs in float32 registers with packed FMAs, one channel per
// thread (its TMEM lane), two h rows per pair.
//
// Work unit: item b, h rows 4 rb + [0, 4), h columns 40 cb + [0, 40): 160 pixels, in five
// chunks of 8 columns; pixel (rl, 8 k + u) is row/column 32 k + 4 u + rl of the MMA operands.
// A chunk reads dout rows 2 rb + [0, 3) and columns 20 cb + 4 k + [0, 5) (one bulk tensor copy
// of 128 channels).  Units with every h row masked add nothing and are skipped; unit rb owns
// (adds to db1) the output rows 2 rb, 2 rb + 1 and columns 20 cb + [0, 20), so every output
// pixel is counted once.
//
// Roles (384 threads, one block per SM, persistent; three warps per SM sub-partition leave
// 168 registers a thread):
//   warps 0-3, 4-7  two epilogue groups; group g takes the block's units g, g + 2, ...;
//                   warp w reads TMEM lanes 32 (w % 4) + [0, 32) (its channel quarter).  Per
//                   chunk a warp reads z, computes dz, dh, dw1, writes its 32 rows of A2 and its
//                   taps' B2 rows, and arrives on the slot's mbarrier; the warps of a group never
//                   wait for one another
//   warps 8-10      patch builders: stage the unit's 9 x 81 mel window (even and odd columns
//                   apart, so that pixel-wise reads are free of bank conflicts) and build B1
//   warp 11         allocates tensor memory and lists the block's units; its lane 0 polls the
//                   ready-streams (conv0 per unit, dw0 per chunk of either group) and issues the
//                   MMAs and the dout copies, four chunks ahead per group
// Tensor memory: group g has D1 at columns 256 g + [0, 160) and its two D2 slots at
// 256 g + 192 + 32 s + [0, 32).
// Every mbarrier wait is bounded; a wait that gives up records an error (dw_device_error) and
// the block drains.  Each block writes one partial row (both groups added in a fixed order);
// the finalize kernel adds the rows in a fixed order, so results are reproducible for given
// sizes on a given GPU model.
#include "dw_internal.h"
#include "tc_common.cuh"

namespace dwk {
namespace {

constexpr int kUR = 4, kUC = 40;            // h rows and columns per unit
constexpr int kPix = kUR * kUC;             // MMA 1 N
constexpr int kChunks = 5, kCW = 8;         // chunks of 8 h columns (32 pixels)
constexpr int kWR = 2 * kUR + 1;            // mel window rows
constexpr int kWC = 2 * kUC + 1;            // mel window columns
constexpr int kWS = 44;                     // staged row stride of the even / odd column halves
constexpr int kWinFloats = 2 * kWR * kWS;   // one staged window
constexpr int kWinElems = kWR * kWC;
constexpr int kGroups = 2, kGroupThreads = 128;
constexpr int kBuildWarp0 = 8, kBuildThreads = 96;
constexpr int kMmaWarp = 11;
constexpr int kThreads = (kMmaWarp + 1) * 32;
constexpr int kWinLoads = (kWinElems + kBuildThreads - 1) / kBuildThreads;
constexpr int kTileA1 = 128 * 128;          // [128 channels][32 words]
constexpr int kTileB1 = kPix * 128;
constexpr int kTileA2 = 128 * 128;          // one of hi / lo for one chunk
constexpr int kTileB2 = 32 * 128;
constexpr int kDoutCols = 5, kDoutRows = 3;
constexpr int kDoutElems = 128 * kDoutCols * kDoutRows;
constexpr int kRing = 4;                    // dout chunks in flight per group
constexpr int kWinSlots = 4;
constexpr int kListCap = 768;
constexpr int kBarBuild = 1, kBarAll = 2;
constexpr int kTmemCols = 512;
constexpr int kD2Col = 192;

// Shared memory (offsets from a 1024-byte aligned base).
constexpr int kOffA1 = 0;
constexpr int kOffB1 = kOffA1 + kTileA1;
constexpr int kOffA2 = kOffB1 + kTileB1;                         // [group][slot][hi, lo]
constexpr int kOffB2 = kOffA2 + kGroups * 2 * 2 * kTileA2;       // [group][slot]
constexpr int kOffDout = kOffB2 + kGroups * 2 * kTileB2;         // [group][ring] 16-bit boxes
constexpr int kOffWin = kOffDout + kGroups * kRing * kDoutElems * 2;
constexpr int kOffList = kOffWin + kWinSlots * kWinFloats * 4;
constexpr int kOffBar = kOffList + kListCap * 4;
constexpr int kSmemBytes = kOffBar + 320;
constexpr int kSmemAlloc = kSmemBytes + 1024;

static_assert(kOffB1 % 1024 == 0 && kOffA2 % 1024 == 0 && kOffB2 % 1024 == 0, "swizzle atoms are 1024-byte aligned");
static_assert(kOffDout % 128 == 0 && (kDoutElems * 2) % 128 == 0, "bulk tensor destinations");
static_assert(kSmemAlloc <= 232448, "shared memory per block");
static_assert(kWS >= kUC + 1 && (2 * kWS) % 32 == 24, "window stride: four rows 2 rl apart hit distinct banks");
static_assert(kPix % 16 == 0 && kPix <= 256, "MMA N");

// Instruction descriptors: D float32, A and B TF32, both K-major, M = 128.
constexpr uint32_t idesc(int n) {
    return (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
}
constexpr uint32_t kIdescZ = idesc(kPix), kIdescW = idesc(32);

// Unit list entries: item (16 bits) | row block (12 bits) | column block (4 bits).
__device__ __forceinline__ int unit_b(uint32_t u) { return static_cast<int>(u >> 16); }
__device__ __forceinline__ int unit_rb(uint32_t u) { return static_cast<int>((u >> 4) & 0xfffu); }
__device__ __forceinline__ int unit_cb(uint32_t u) { return static_cast<int>(u & 15u); }

__device__ __forceinline__ void dout_box_load(void *dst, const void *tmap, int c, int j, int i, int b, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, "
        "%5}], [%6];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c), "r"(j), "r"(i), "r"(b), "r"(smem_addr(bar))
        : "memory");
}

// Whether the phase with the given parity has completed (does not wait).
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// 32 consecutive accumulator columns of this thread's lane, waited for.
__device__ __forceinline__ void tmem_ld32(uint32_t t, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(t)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Accumulator columns 0..19 of this thread's lane, waited for.
__device__ __forceinline__ void tmem_ld20(uint32_t t, float (&v)[20]) {
    uint32_t r[20];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%20];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%16, %17, %18, %19}, [%21];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19])
        : "r"(t), "r"(t + 16)
        : "memory");
#pragma unroll
    for (int i = 0; i < 20; ++i) v[i] = __uint_as_float(r[i]);
}

// Word w of row `row` of a K-major 128-byte-swizzled tile.
__device__ __forceinline__ float *swz_word(unsigned char *tile, int row, int w) {
    return reinterpret_cast<float *>(tile + row * 128 + ((((w >> 2) ^ (row & 7)) << 4) | ((w & 3) << 2)));
}

template <typename TD> __device__ __forceinline__ float dout_val(const TD *p) { return Half16<TD>::one(*reinterpret_cast<const unsigned short *>(p)); }

__device__ __forceinline__ float2 relu2(float2 z) { return make_float2(fmaxf(z.x, 0.f), fmaxf(z.y, 0.f)); }
__device__ __forceinline__ float2 pos_sel(float2 z, float2 v) {
    return make_float2(z.x > 0.f ? v.x : 0.f, z.y > 0.f ? v.y : 0.f);
}

}  // namespace

template <typename TD, bool PT1>
__global__ void __launch_bounds__(kThreads, 1)
dw_subsample_bwd_tc_kernel(const float *__restrict__ mel, const float *__restrict__ w0, const float *__restrict__ b0,
                           const float *__restrict__ w1, const int32_t *__restrict__ lengths,
                           const __grid_constant__ CUtensorMap dout_map, float *__restrict__ partials, int B,
                           int Tn, int F, int C, int F2, int nRB, int nCB, int nG) {
    constexpr int Pt = PT1 ? 1 : 2;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    unsigned char *tA1 = smem + kOffA1, *tB1 = smem + kOffB1, *tA2 = smem + kOffA2, *tB2 = smem + kOffB2;
    TD *ring = reinterpret_cast<TD *>(smem + kOffDout);
    float *win = reinterpret_cast<float *>(smem + kOffWin);
    uint32_t *ulist = reinterpret_cast<uint32_t *>(smem + kOffList);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
    uint64_t *b1_full = bars, *b1_empty = bars + 1, *d1_full = bars + 2 /* [group] */,
             *d1_empty = bars + 4 /* [group] */, *a2_empty = bars + 6 /* [group][slot] */,
             *dfull = bars + 10 /* [group][ring] */, *win_full = bars + 18, *win_free = bars + 22,
             *mma_done = bars + 26, *d2_done = bars + 27 /* [group] */;
    uint64_t *a2_full = bars + 29;  // [group][slot]: one arrival per warp of the group
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 33);
    int *count = reinterpret_cast<int *>(bars + 34);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int g = blockIdx.x % nG;                 // channel tile of this block
    const int q0 = blockIdx.x / nG, qs = gridDim.x / nG;
    const int perItem = nRB * nCB, nUnits = B * perItem;

    // ------------------------------------------------------------ set-up
    launch_dependents();  // the finalize may be scheduled now; it waits for this grid to finish
    if (threadIdx.x == 0) {
        mbar_init(b1_full, kBuildThreads);
        mbar_init(b1_empty, 1);
        for (int i = 0; i < kGroups; ++i) {
            mbar_init(&d1_full[i], 1);
            mbar_init(&d1_empty[i], kGroupThreads / 32);  // one arrival per warp of the group
            mbar_init(&a2_empty[2 * i], 1);
            mbar_init(&a2_empty[2 * i + 1], 1);
            mbar_init(&a2_full[2 * i], kGroupThreads / 32);
            mbar_init(&a2_full[2 * i + 1], kGroupThreads / 32);
            for (int r = 0; r < kRing; ++r) mbar_init(&dfull[i * kRing + r], 1);
            mbar_init(&d2_done[i], 1);
        }
        for (int s = 0; s < kWinSlots; ++s) {
            mbar_init(&win_full[s], kBuildThreads);
            mbar_init(&win_free[s], 1);
        }
        mbar_init(mma_done, 1);
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
        tc_fence_before();
        // This block's units: every qs-th of all units (item-major), those with an unmasked
        // h row only, in that order.
        const unsigned below = (1u << lane) - 1u;
        int n = 0;
        for (int base = q0; base < nUnits; base += 32 * qs) {
            const int q = base + lane * qs;
            bool act = false;
            uint32_t e = 0;
            if (q < nUnits) {
                const int b = q / perItem, rem = q - b * perItem, rb = rem / nCB, cb = rem - rb * nCB;
                const int L = static_cast<int>(clamp_len(lengths, b, Tn));
                act = kUR * rb < (L + 1) / 2;
                e = (static_cast<uint32_t>(b) << 16) | (static_cast<uint32_t>(rb) << 4) | static_cast<uint32_t>(cb);
            }
            const unsigned msk = __ballot_sync(0xffffffffu, act);
            if (act) ulist[n + __popc(msk & below)] = e;
            n += __popc(msk);
        }
        if (lane == 0) *count = n;
    }
    if (warp >= kBuildWarp0 && warp < kMmaWarp) {
        const int pt = threadIdx.x - kBuildWarp0 * 32;
        for (int r = pt; r < 128; r += kBuildThreads) {  // A1: split conv0 weights and bias, forward K layout
            const int c = g * 128 + r;
            float hi[9], lo[9];
#pragma unroll
            for (int t = 0; t < 9; ++t) {
                const float x = c < C ? __ldg(w0 + t * C + c) : 0.f;
                hi[t] = tf32_hi(x);
                lo[t] = x - hi[t];
            }
            const float bx = c < C ? __ldg(b0 + c) : 0.f;
            const float bhi = tf32_hi(bx);
            float4 q[8];
            q[0] = make_float4(hi[0], hi[1], hi[2], hi[3]);
            q[1] = make_float4(hi[4], hi[5], hi[6], hi[7]);
            q[2] = make_float4(lo[0], lo[1], lo[2], lo[3]);
            q[3] = make_float4(lo[4], lo[5], lo[6], lo[7]);
            q[4] = q[0];
            q[5] = q[1];
            q[6] = make_float4(hi[8], lo[8], hi[8], bhi);
            q[7] = make_float4(bx - bhi, 0.f, 0.f, 0.f);
            store_k_row(tA1, r, q);
        }
        // B2 rows 18 (ones: db0) and 19..31 (zeros) of every slot; chunks rewrite rows 0..17 only
        for (int e = pt; e < kGroups * 2 * 14; e += kBuildThreads) {
            const int slot = e / 14, row = 18 + e % 14;
            const float v = row == 18 ? 1.f : 0.f;
            float4 q[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) q[k] = make_float4(v, v, v, v);
            store_k_row(tB2 + slot * kTileB2, row, q);
        }
        fence_async_smem();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int nA = *count;

    if (warp < kBuildWarp0) {
        // ------------------------------------------------------------ epilogue groups
        const int grp = warp >> 2, qw = warp & 3, m = qw * 32 + lane;
        const int c = g * 128 + m;
        const uint32_t tl = tmem_base + (static_cast<uint32_t>(qw * 32) << 16) + grp * 256;
        const uint32_t d1 = tl, d2 = tl + kD2Col;
        float2 W[3][3], gw1[3][3];
#pragma unroll
        for (int t = 0; t < 9; ++t) {
            const float x = c < C ? __ldg(w1 + t * C + c) : 0.f;
            W[t / 3][t % 3] = make_float2(x, x);
            gw1[t / 3][t % 3] = make_float2(0.f, 0.f);
        }
        float gb1 = 0.f, gw0[9], gb0 = 0.f;
#pragma unroll
        for (int t = 0; t < 9; ++t) gw0[t] = 0.f;
        // adds chunk p's dw0 / db0 sums (its MMAs have completed) to the registers
        auto take_d2 = [&](int p) {
            float r[20];
            tmem_ld20(d2 + 32 * (p & 1), r);
#pragma unroll
            for (int t = 0; t < 9; ++t) gw0[t] += r[t] + r[9 + t];
            gb0 += r[18];
        };
        const int nU = (nA - grp + 1) / 2;            // units grp, grp + 2, ...
        unsigned char *a2 = tA2 + grp * (2 * 2 * kTileA2);
        unsigned char *b2 = tB2 + grp * (2 * kTileB2);
        TD *rg = ring + grp * kRing * kDoutElems;
        uint64_t *df = dfull + grp * kRing;
        // pixel pairs: rows eA, eA + 2 take the taps p = 0 and 2, rows oA, oA + 2 the tap p = 1
        constexpr int eA = PT1 ? 1 : 0, oA = PT1 ? 0 : 1;
        bool ok = true;
        int pos = 0, done = 0;                         // chunks started / finished (MMAs issued)
        for (int ul = 0; ul < nU && ok; ++ul) {
            const int idx = grp + 2 * ul;
            const uint32_t e = ulist[idx];
            const int rb = unit_rb(e);
            const int L = static_cast<int>(clamp_len(lengths, unit_b(e), Tn)), L4 = ((L + 1) / 2 + 1) / 2;
            const bool rv0 = 2 * rb < L4, rv1 = 2 * rb + 1 < L4, rv2 = 2 * rb + 2 < L4;
            const int ws = idx & (kWinSlots - 1);
            const float *wE = win + ws * kWinFloats, *wO = wE + kWR * kWS;
            bool wok = mbar_wait(&d1_full[grp], ul & 1);
            wok = wok && mbar_wait(&win_full[ws], (idx >> 2) & 1);
            ok = __all_sync(0xffffffffu, wok);
            if (!ok) break;
            tc_fence_after();
#pragma unroll 1
            for (int k = 0; k < kChunks; ++k, ++pos) {
                float v[32];
                tmem_ld32(d1 + 32 * k, v);
                if (k == kChunks - 1) {  // z read out: the next conv0 MMA may overwrite it
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&d1_empty[grp]);
                }
                wok = wok && mbar_wait(&df[pos & (kRing - 1)], (pos / kRing) & 1);
                // doutm of this chunk: rows 2 rb + bi, columns 20 cb + 4 k + j
                float D[3][5];
                {
                    const TD *dv = rg + (pos & (kRing - 1)) * kDoutElems + m;
#pragma unroll
                    for (int j = 0; j < 5; ++j) {
                        D[0][j] = rv0 ? dout_val(dv + j * 128) : 0.f;
                        D[1][j] = rv1 ? dout_val(dv + (5 + j) * 128) : 0.f;
                        D[2][j] = rv2 ? dout_val(dv + (10 + j) * 128) : 0.f;
                    }
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) gb1 += D[0][j] + D[1][j];  // the unit's own output pixels
                float2 X01[5], X12[5];
#pragma unroll
                for (int j = 0; j < 5; ++j) {
                    X01[j] = make_float2(D[0][j], D[1][j]);
                    X12[j] = make_float2(D[1][j], D[2][j]);
                }
#pragma unroll
                for (int u = 0; u < kCW; ++u) {
                    const float2 zE = make_float2(v[4 * u + eA], v[4 * u + eA + 2]);
                    const float2 zO = make_float2(v[4 * u + oA], v[4 * u + oA + 2]);
                    const float2 hE = relu2(zE), hO = relu2(zO);
                    float2 dhE = make_float2(0.f, 0.f), dhO = make_float2(0.f, 0.f);
                    // h column 8 k + u takes the tap q at output column (u + 1 - q) / 2 of the chunk
#pragma unroll
                    for (int q = 0; q < 3; ++q) {
                        if (((u + 1 - q) & 1) != 0) continue;
                        const int j = (u + 1 - q) / 2;
                        const float2 xo = PT1 ? X01[j] : X12[j];
                        dhE = ffma2(W[0][q], X12[j], dhE);
                        dhE = ffma2(W[2][q], X01[j], dhE);
                        dhO = ffma2(W[1][q], xo, dhO);
                        gw1[0][q] = ffma2(hE, X12[j], gw1[0][q]);
                        gw1[2][q] = ffma2(hE, X01[j], gw1[2][q]);
                        gw1[1][q] = ffma2(hO, xo, gw1[1][q]);
                    }
                    const float2 dzE = pos_sel(zE, dhE), dzO = pos_sel(zO, dhO);
                    v[4 * u + eA] = dzE.x;
                    v[4 * u + eA + 2] = dzE.y;
                    v[4 * u + oA] = dzO.x;
                    v[4 * u + oA + 2] = dzO.y;
                }
                // the slot's previous chunk (two back) has been read by its MMAs, and its sums
                // are complete: take them before this chunk's MMAs reuse the accumulator
                if (pos >= 2) {
                    wok = wok && mbar_wait(&a2_empty[2 * grp + (pos & 1)], ((pos - 2) >> 1) & 1);
                    tc_fence_after();
                    take_d2(pos - 2);
                    tc_fence_before();
                }
                unsigned char *ah = a2 + (pos & 1) * (2 * kTileA2), *al = ah + kTileA2;
                unsigned char *bt = b2 + (pos & 1) * kTileB2;
                {
                    float4 qh[8];
#pragma unroll
                    for (int u = 0; u < kCW; ++u)
                        qh[u] = make_float4(tf32_hi(v[4 * u]), tf32_hi(v[4 * u + 1]), tf32_hi(v[4 * u + 2]),
                                            tf32_hi(v[4 * u + 3]));
                    store_k_row(ah, m, qh);
#pragma unroll
                    for (int u = 0; u < kCW; ++u)
                        qh[u] = make_float4(v[4 * u] - qh[u].x, v[4 * u + 1] - qh[u].y, v[4 * u + 2] - qh[u].z,
                                            v[4 * u + 3] - qh[u].w);
                    store_k_row(al, m, qh);
                }
                {  // B2 rows t (hi) and 9 + t (lo) of pixel `lane` for this warp's taps t = qw + 4 i
                    const int u = lane >> 2, rl = lane & 3, sl = kCW * k + u;
#pragma unroll
                    for (int t = qw; t < 9; t += 4) {
                        const int p = t / 3, qq = t % 3;
                        const float x = qq == 1 ? wO[(2 * rl + p) * kWS + sl] : wE[(2 * rl + p) * kWS + sl + (qq >> 1)];
                        const float h = tf32_hi(x);
                        *swz_word(bt, t, lane) = h;
                        *swz_word(bt, 9 + t, lane) = x - h;
                    }
                }
                // this warp's rows of the chunk are written: hand them to the MMA thread
                fence_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&a2_full[2 * grp + (pos & 1)]);
                ok = __all_sync(0xffffffffu, wok);
                if (!ok) break;
                ++done;
            }
        }
        // slots 0..8 dw0, 9 db0, 10..18 dw1, 19 db1 (the partial row layout)
        float vals[20];
#pragma unroll
        for (int i = 0; i < 20; ++i) vals[i] = 0.f;
        if (done > 0) {  // the last two chunks' sums, once the group's last MMAs have completed
            const bool dok = mbar_wait(&d2_done[grp], 0);
            tc_fence_after();
            for (int p = done >= 2 ? done - 2 : 0; p < done; ++p) take_d2(p);
            if (dok && ok) {
#pragma unroll
                for (int t = 0; t < 9; ++t) vals[t] = gw0[t];
                vals[9] = gb0;
            }
        }
#pragma unroll
        for (int t = 0; t < 9; ++t) vals[10 + t] = gw1[t / 3][t % 3].x + gw1[t / 3][t % 3].y;
        vals[19] = gb1;
        // group 1 hands its sums to group 0 through its own (now idle) A2 area; fixed order
        float *xch = reinterpret_cast<float *>(tA2 + 2 * 2 * kTileA2);
        if (grp == 1) {
#pragma unroll
            for (int i = 0; i < 20; ++i) xch[i * 128 + m] = vals[i];
        }
        named_bar(kBarAll, kGroups * kGroupThreads);
        if (grp == 0 && c < C) {
            float *row = partials + static_cast<int64_t>(q0) * 20 * C + c;
#pragma unroll
            for (int i = 0; i < 20; ++i) row[static_cast<int64_t>(i) * C] = vals[i] + xch[i * 128 + m];
        }
    } else if (warp < kMmaWarp) {
        // ------------------------------------------------------------ patch builders
        const int pt = threadIdx.x - kBuildWarp0 * 32;
        // This thread's window elements are the same for every unit: element k sits at window
        // row wrc >> 8, column wrc & 255 (wrc = -1 past the window) and is staged at wofs.
        int wrc[kWinLoads], wofs[kWinLoads];
#pragma unroll
        for (int k = 0; k < kWinLoads; ++k) {
            const int e = pt + k * kBuildThreads;
            const int row = e / kWC, col = e % kWC;
            wrc[k] = e < kWinElems ? (row << 8) | col : -1;
            wofs[k] = ((col & 1) ? kWR * kWS : 0) + row * kWS + (col >> 1);
        }
        float mv[kWinLoads];
        auto load_win = [&](uint32_t e) {  // frames at or beyond len, and outside the plane, read as zero
            const int b = unit_b(e);
            const int L = static_cast<int>(clamp_len(lengths, b, Tn));
            const int mr0 = 2 * kUR * unit_rb(e) - Pt, mc0 = 2 * kUC * unit_cb(e) - 1;
            const float *base = mel + static_cast<int64_t>(b) * Tn * F;
#pragma unroll
            for (int k = 0; k < kWinLoads; ++k) {
                const int mr = mr0 + (wrc[k] >> 8), mc = mc0 + (wrc[k] & 255);
                const bool in = wrc[k] >= 0 && mr >= 0 && mr < L && mc >= 0 && mc < F;
                mv[k] = in ? __ldg(base + static_cast<int64_t>(mr) * F + mc) : 0.f;
            }
        };
        if (nA > 0) load_win(ulist[0]);
        bool ok = true;
        for (int idx = 0; idx < nA && ok; ++idx) {
            const uint32_t e = ulist[idx];
            const int ws = idx & (kWinSlots - 1);
            ok = named_bar_and(kBarBuild, kBuildThreads, mbar_wait(&win_free[ws], ((idx >> 2) & 1) ^ 1));
            if (!ok) break;
            float *S = win + ws * kWinFloats;
#pragma unroll
            for (int k = 0; k < kWinLoads; ++k)
                if (wrc[k] >= 0) S[wofs[k]] = mv[k];
            mbar_arrive(&win_full[ws]);
            if (idx + 1 < nA) load_win(ulist[idx + 1]);  // in flight while this unit's patches are built
            ok = named_bar_and(kBarBuild, kBuildThreads, mbar_wait(b1_empty, (idx & 1) ^ 1));
            if (!ok) break;
            const float *wE = S, *wO = S + kWR * kWS;
            const int L2 = (static_cast<int>(clamp_len(lengths, unit_b(e), Tn)) + 1) / 2;
            const int r0 = kUR * unit_rb(e), s0 = kUC * unit_cb(e);
#pragma unroll
            for (int n = pt; n < kPix; n += kBuildThreads) {
                const int k = n >> 5, w = n & 31, u = w >> 2, rl = w & 3, sl = kCW * k + u;
                float4 q[8];
                if (r0 + rl < L2 && s0 + sl < F2) {
                    float hi[9], lo[9];
#pragma unroll
                    for (int t = 0; t < 9; ++t) {
                        const int p = t / 3, qq = t % 3;
                        const float x = qq == 1 ? wO[(2 * rl + p) * kWS + sl] : wE[(2 * rl + p) * kWS + sl + (qq >> 1)];
                        hi[t] = tf32_hi(x);
                        lo[t] = x - hi[t];
                    }
                    q[0] = make_float4(hi[0], hi[1], hi[2], hi[3]);
                    q[1] = make_float4(hi[4], hi[5], hi[6], hi[7]);
                    q[2] = q[0];
                    q[3] = q[1];
                    q[4] = make_float4(lo[0], lo[1], lo[2], lo[3]);
                    q[5] = make_float4(lo[4], lo[5], lo[6], lo[7]);
                    q[6] = make_float4(hi[8], hi[8], lo[8], 1.f);
                    q[7] = make_float4(1.f, 0.f, 0.f, 0.f);
                } else {  // masked or outside the plane: z = 0 exactly, so h = dz = 0
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) q[kk] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
                store_k_row(tB1, n, q);
            }
            fence_async_smem();
            mbar_arrive(b1_full);
        }
    } else if (lane == 0) {
        // ------------------------------------------------------------ MMA and copy issuer
        // Three streams, served as their inputs become ready (polled, so that no stream waits
        // behind another): the conv0 MMAs of each unit (patch rows built, the group's z buffer
        // free), and per group the dw0 MMAs of each chunk (all four warps' rows written), each
        // followed by the dout copy of the group's chunk four ahead.
        const uint64_t ad = sw128_desc(smem_addr(tA1)), bd = sw128_desc(smem_addr(tB1));
        const int nP[2] = {(nA + 1) / 2 * kChunks, nA / 2 * kChunks};
        int cp[2] = {0, 0}, issued[2] = {0, 0}, zi = 0;
        auto prefetch = [&](int grp, int p) {
            const int ul = p / kChunks, k = p - ul * kChunks;
            const uint32_t e = ulist[grp + 2 * ul];
            uint64_t *bar = &dfull[grp * kRing + (p & (kRing - 1))];
            mbar_arrive_expect_tx(bar, kDoutElems * static_cast<uint32_t>(sizeof(TD)));
            dout_box_load(ring + (grp * kRing + (p & (kRing - 1))) * kDoutElems, &dout_map, g * 128,
                          20 * unit_cb(e) + 4 * k, 2 * unit_rb(e), unit_b(e), bar);
        };
        for (int grp = 0; grp < kGroups; ++grp)
            for (; issued[grp] < kRing && issued[grp] < nP[grp]; ++issued[grp]) prefetch(grp, issued[grp]);
        uint32_t idle = 0;
        while (zi < nA || cp[0] < nP[0] || cp[1] < nP[1]) {
            bool prog = false;
#pragma unroll
            for (int grp = 0; grp < kGroups; ++grp) {
                const int p = cp[grp];
                if (p < nP[grp] && mbar_test(&a2_full[2 * grp + (p & 1)], (p >> 1) & 1)) {
                    tc_fence_after();
                    unsigned char *ah = tA2 + grp * (2 * 2 * kTileA2) + (p & 1) * (2 * kTileA2);
                    const uint64_t b2d = sw128_desc(smem_addr(tB2 + grp * (2 * kTileB2) + (p & 1) * kTileB2));
                    const uint32_t d2 = tmem_base + grp * 256 + kD2Col + 32 * (p & 1);
#pragma unroll
                    for (int hl = 0; hl < 2; ++hl) {
                        const uint64_t a2d = sw128_desc(smem_addr(ah + hl * kTileA2));
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)  // 32 pixels = 4 K-steps of 8
                            mma_tf32(d2, a2d + 2 * ks, b2d + 2 * ks, kIdescW, (hl | ks) != 0 ? 1u : 0u);
                    }
                    mma_commit(&a2_empty[2 * grp + (p & 1)]);
                    if (p % kChunks == kChunks - 1)  // the group is done with the unit's window
                        mbar_arrive(&win_free[(grp + 2 * (p / kChunks)) & (kWinSlots - 1)]);
                    if (issued[grp] < nP[grp]) prefetch(grp, issued[grp]++);
                    cp[grp] = p + 1;
                    if (cp[grp] == nP[grp]) mma_commit(&d2_done[grp]);
                    prog = true;
                }
            }
            if (zi < nA && mbar_test(b1_full, zi & 1) && mbar_test(&d1_empty[zi & 1], ((zi >> 1) & 1) ^ 1)) {
                tc_fence_after();
                const uint32_t d = tmem_base + (zi & 1) * 256;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)  // K = 32 TF32 words = 4 steps of 8
                    mma_tf32(d, ad + 2 * ks, bd + 2 * ks, kIdescZ, ks > 0 ? 1u : 0u);
                mma_commit(&d1_full[zi & 1]);
                mma_commit(b1_empty);
                ++zi;
                prog = true;
            }
            if (prog) {
                idle = 0;
            } else {
                if (++idle > kSpinLimit) {  // nothing became ready for a long time: give up
                    atomicOr(&dw_device_error_flag, kErrWaitTimeout);
                    break;
                }
                __nanosleep(32);
            }
        }
        // the copies still in flight land before shared memory is released
        for (int grp = 0; grp < kGroups; ++grp)
            for (int p = issued[grp] > kRing ? issued[grp] - kRing : 0; p < issued[grp]; ++p)
                mbar_wait(&dfull[grp * kRing + (p & (kRing - 1))], (p / kRing) & 1, kSpinLimit >> 4);
        // every issued MMA has finished before tensor memory is released
        mma_commit(mma_done);
        mbar_wait(mma_done, 0);
    }
    tc_fence_before();
    __syncwarp();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// Tensor map over dout [B][T4][F4][C] (dims innermost first), box 128 x 5 x 3 x 1.
static cudaError_t make_dout_map(CUtensorMap *map, const void *dout, int dtype, int64_t B, int64_t T4, int64_t F4,
                                 int64_t C) {
    TensorMapEncodeTiledFn enc = tensor_map_encoder();
    if (enc == nullptr) return cudaErrorNotSupported;
    const int64_t es = dtype_bytes(dtype);
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(F4),
                                static_cast<cuuint64_t>(T4), static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(C * es), static_cast<cuuint64_t>(F4 * C * es),
                                   static_cast<cuuint64_t>(T4 * F4 * C * es)};
    const cuuint32_t box[4] = {128u, static_cast<cuuint32_t>(kDoutCols), static_cast<cuuint32_t>(kDoutRows), 1u};
    const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    const CUresult r = enc(map, tma_dtype(dtype), 4, const_cast<void *>(dout), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

int subsample_bwd_tc_blocks_per_group(int64_t C) {
    const int64_t nG = (C + 127) / 128;
    const int64_t per = sm_count() / nG;
    return static_cast<int>(per >= 1 ? per : 1);
}

cudaError_t subsample_bwd_tc_launch(const SubsampleBwdArgs &a, int max_rows, int *rows, cudaStream_t s) {
    auto s2 = [](int64_t n) -> int64_t { return n >= 1 ? (n - 1) / 2 + 1 : 0; };
    const int64_t T2 = s2(a.T), F2 = s2(a.F), T4 = s2(T2), F4 = s2(F2);
    const int64_t nRB = (T2 + kUR - 1) / kUR, nCB = (F2 + kUC - 1) / kUC;
    const int64_t nG = (a.C + 127) / 128;
    const int64_t units = a.B * nRB * nCB;
    if (a.dout_dtype != 1 && a.dout_dtype != 2) return cudaErrorNotSupported;
    if (a.C % 8 != 0 || reinterpret_cast<uintptr_t>(a.dout) % 16 != 0) return cudaErrorNotSupported;
    if (a.B > 65535 || nRB > 4096 || nCB > 16 || units >= (1LL << 26) || a.T * a.F >= (1LL << 31) ||
        9 * a.C >= (1LL << 31) || T4 == 0)
        return cudaErrorNotSupported;
    int64_t per = subsample_bwd_tc_blocks_per_group(a.C);
    if (per > max_rows) per = max_rows;
    if (per > units) per = units;
    if (per < 1) per = 1;
    // every block lists its units in shared memory; larger problems take the SIMT kernel
    if ((units + per - 1) / per > kListCap) return cudaErrorNotSupported;
    const int64_t grid = per * nG;
    if (grid > kMaxGrid) return cudaErrorNotSupported;
    CUtensorMap map;
    if (make_dout_map(&map, a.dout, a.dout_dtype, a.B, T4, F4, a.C) != cudaSuccess) return cudaErrorNotSupported;
    cudaError_t e = cudaSuccess;
#define DW_SBTC_LAUNCH(TD, P1)                                                                                \
    do {                                                                                                      \
        auto kern = dw_subsample_bwd_tc_kernel<TD, P1>;                                                       \
        e = ensure_smem_attr(reinterpret_cast<const void *>(kern), kSmemAlloc);                               \
        if (e != cudaSuccess) return e;                                                                       \
        kern<<<static_cast<unsigned>(grid), kThreads, kSmemAlloc, s>>>(                                       \
            a.mel, a.w0, a.b0, a.w1, a.lengths, map, a.partials, static_cast<int>(a.B), static_cast<int>(a.T), \
            static_cast<int>(a.F), static_cast<int>(a.C), static_cast<int>(F2), static_cast<int>(nRB),        \
            static_cast<int>(nCB), static_cast<int>(nG));                                                     \
    } while (0)
    if (a.dout_dtype == 1) {
        if (a.causal) DW_SBTC_LAUNCH(bf16, false);
        else DW_SBTC_LAUNCH(bf16, true);
    } else {
        if (a.causal) DW_SBTC_LAUNCH(f16, false);
        else DW_SBTC_LAUNCH(f16, true);
    }
#undef DW_SBTC_LAUNCH
    e = cudaGetLastError();
    if (e == cudaSuccess) *rows = static_cast<int>(per);
    return e;
}

}  // namespace dwk
