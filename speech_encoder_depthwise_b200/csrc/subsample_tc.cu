// Fused depthwise-striding subsampler front with conv0 on the 5th-generation tensor cores
// (NeMo PR #16114, "Use Fused Kernels for Depthwise Striding Subsampler", section "What does
// this PR do ?", first kernel: mel [B,T,F,1] -> conv0 -> ReLU -> masking -> conv_dw1).
//
// conv0 maps one input channel to C channels with a 3x3 stride-2 window, so for a block of
// h pixels it is a dense contraction: h[c, pixel] = sum over 9 taps of w0[tap, c] *
// patch[pixel, tap] + b0[c].  It runs as tcgen05 MMAs with the channels as M (128 per tile)
// and the h pixels of a unit as N, so the accumulator in tensor memory holds, in lane m,
// every h pixel of channel m.  Each epilogue thread owns one channel: it reads its lane,
// applies ReLU, and computes the depthwise conv_dw1 (3x3, stride 2) in float32 registers.
// The conv0 output never leaves the SM.
//
// Precision.  The MMA reads its operands as TF32 (10 explicit mantissa bits), so every
// float32 operand is split into x = hi + lo, hi = x with the low 13 mantissa bits cleared
// and lo = x - hi (exact), and the contraction sums w_hi*m_hi + w_lo*m_hi + w_hi*m_lo with
// float32 accumulation; the dropped w_lo*m_lo term and the truncation of lo are below 2^-20
// of each product.  This is the three-product emulation of float32 products on TF32 units.
// The bias b0 rides along as two more K columns (b0_hi, b0_lo against a 0/1 column that is 1
// exactly for unmasked h pixels, whose other columns are then zero too).  K layout, in 16-byte
// chunks of 4 words (patch | weights), taps t = 3 p + q:
//   0: m_hi[0..3] | w_hi[0..3]     1: m_hi[4..7] | w_hi[4..7]
//   2: m_hi[0..3] | w_lo[0..3]     3: m_hi[4..7] | w_lo[4..7]
//   4: m_lo[0..3] | w_hi[0..3]     5: m_lo[4..7] | w_hi[4..7]
//   6: m_hi[8], m_hi[8], m_lo[8], v | w_hi[8], w_lo[8], w_hi[8], b0_hi
//   7: v, 0, 0, 0 | b0_lo, 0, 0, 0
// so a patch row is six distinct register quads, two of them stored twice.
//
// Work unit: item b, output rows [i0, i0+2), output columns [j0, j0+20).  It needs h rows
// 2 i0 - Pt + [0, 5) and h columns 2 j0 - 1 + [0, 41): N = 5 x 41 = 205 pixels (208 with
// the pad to a multiple of 16), K = 32 TF32 words per pixel.  Padding pixels, masked h rows
// (at or beyond ceil(len/2)) and pixels outside the h plane get an all-zero patch, so their
// h is exactly zero.
//
// Roles (448 threads, one block per SM, persistent):
//   warps 0-7   epilogue, two groups of four: warp w reads TMEM lanes 32 (w % 4) + [0, 32)
//               (its channel quarter); group w / 4 takes every other job (unit x channel
//               tile); results are staged in shared memory and written with one bulk tensor
//               store per job
//   warps 8-11  patch builders: stage the unit's 11 x 83 mel window (frames at or beyond
//               len read as zero), build the split patch rows in the 128-byte-swizzled
//               K-major layout the MMA reads
//   warp 12     allocates tensor memory and lists the block's units; one thread issues the
//               MMAs (4 K-steps of 8)
//   warp 13     one thread issues every bulk tensor store (staged tiles, zero tiles)
// Pipelines: 2 patch stages (builders -> MMA), 2 accumulator buffers of 256 TMEM columns
// (MMA -> epilogue group; released as soon as the last column is read), two output staging
// tiles per group (epilogue group -> store thread -> back).  Every mbarrier wait
// is bounded; a wait that gives up records an error (dw_device_error) and the block drains.
#include "dw_internal.h"
#include "tc_common.cuh"

namespace dwk {
namespace {

constexpr int kRO = 2;                       // output rows per unit
constexpr int kJO = 20;                      // output columns per unit
constexpr int kHR = 2 * kRO + 1;             // h rows per unit
constexpr int kHC = 2 * kJO + 1;             // h columns per unit
constexpr int kNUsed = kHR * kHC;            // h pixels per unit
constexpr int kN = (kNUsed + 15) / 16 * 16;  // MMA N
constexpr int kMR = 2 * kHR + 1;             // mel rows per unit
constexpr int kMC = 2 * kHC + 1;             // mel columns per unit
constexpr int kMCP = kMC + 1;                // staged mel row stride (floats)
constexpr int kMelElems = kMR * kMC;
constexpr int kEpiWarps = 8, kPatchWarps = 4;
constexpr int kEpiThreads = kEpiWarps * 32, kPatchThreads = kPatchWarps * 32;
constexpr int kMmaWarp = kEpiWarps + kPatchWarps;  // then one warp whose lane 0 issues the bulk stores
constexpr int kThreads = (kMmaWarp + 2) * 32;
constexpr int kMelLoads = (kMelElems + kPatchThreads - 1) / kPatchThreads;
constexpr int kMelStages = 3;               // mel windows in shared memory: copies run two units ahead
constexpr int kRowBytes = 128;               // one K row: 32 TF32 words
constexpr int kTileA = 128 * kRowBytes;
constexpr int kTileB = kN * kRowBytes;
constexpr int kTmemCols = 512, kTmemBuf = 256;
constexpr int kHalfCols = kJO / 2;           // output columns per epilogue warp
constexpr int kChunk = 5;                    // output columns per tensor-memory read
constexpr int kRowsPer = (kN + kPatchThreads - 1) / kPatchThreads;  // patch rows per builder thread
constexpr int kBarPatch = 1;                // named barrier id of the patch builders
constexpr int kBarList = 2;                 // named barrier id: unit list ready (list warp + builders)
constexpr int kGroupThreads = 128;          // one epilogue group: 4 warps, one per lane quarter
constexpr int kListCap = 1024;              // units per block (the list lives in shared memory)
constexpr int kOrderItems = 4096;           // items up to which the unit deal is balanced

static_assert(kN <= 256 && kN % 16 == 0, "MMA N");
static_assert(kTileB % 1024 == 0 && kTileA % 1024 == 0, "swizzle atoms are 1024-byte aligned");
static_assert(3 * (kOrderItems + 1) * 4 <= 2 * kTileB, "unit-deal tables fit the patch tiles");
static_assert(kHalfCols % kChunk == 0 && 2 * kChunk * kHR == 50 && kHC == 41, "epilogue chunking");

template <typename TO, int CTG>
struct TcLayout {
    static constexpr int a_off = 0;
    static constexpr int b_off = CTG * kTileA;
    static constexpr int mel_bytes = (kMR * kMCP * 4 + 127) / 128 * 128;
    static constexpr int mel_off = b_off + 2 * kTileB;        // kMelStages staged mel windows
    static constexpr int st_bytes = kRO * kJO * 128 * static_cast<int>(sizeof(TO));
    static constexpr int st_off = mel_off + kMelStages * mel_bytes;  // 2 staging tiles per group, zero tile
    static constexpr int wt_off = st_off + 5 * st_bytes;      // conv_dw1 weight table
    static constexpr int list_off = wt_off + CTG * 10 * 128 * 4;  // unit list
    static constexpr int bar_off = list_off + kListCap * 16;
    static constexpr int bytes = bar_off + 256;
    // room to align the base to 1024; at least 120 KiB so that one block holds an SM (and all
    // of its tensor memory)
    static constexpr int alloc = bytes + 1024 > 120 * 1024 ? bytes + 1024 : 120 * 1024;
};

// Instruction descriptor: D float32, A and B TF32, both K-major, M = 128, N = kN.
constexpr uint32_t kIdesc = (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(kN >> 3) << 17) |
                            (static_cast<uint32_t>(128 >> 4) << 24);

// Accumulator column of h pixel (cc, rr) of a unit.  The 50 values an epilogue chunk reads
// (h columns 10k+1 .. 10k+10, 5 rows each) sit at columns 48k + [0, 48) and 192 + 2k + [0, 2),
// h column 0 at 200 + rr, so that every tensor-memory load starts at a multiple of its width.
__host__ __device__ constexpr int acc_col(int cc, int rr) {
    return cc == 0 ? 200 + rr
                   : (((cc - 1) % 10) * kHR + rr < 48 ? 48 * ((cc - 1) / 10) + ((cc - 1) % 10) * kHR + rr
                                                      : 192 + 2 * ((cc - 1) / 10) + ((cc - 1) % 10) * kHR + rr - 48);
}

// The 50 accumulator values of chunk k (h columns 10k+1 .. 10k+10) of this thread's lane, in
// (column, row) order, waited for.
__device__ __forceinline__ void tmem_ld_chunk(uint32_t tacc, int k, float (&v)[50]) {
    uint32_t r[50];
    const uint32_t a = tacc + 48 * k, t = tacc + 192 + 2 * k;
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%50];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%51];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, "
        "%44, %45, %46, %47}, [%52];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x2.b32 {%48, %49}, [%53];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]),
          "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]),
          "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49])
        : "r"(a), "r"(a + 16), "r"(a + 32), "r"(t)
        : "memory");
#pragma unroll
    for (int i = 0; i < 50; ++i) v[i] = __uint_as_float(r[i]);
}

// The 5 accumulator values (rows 0..4) of h column cc, one single-column load each, waited for.
__device__ __forceinline__ void tmem_ld_column(uint32_t tacc, int cc, float (&v)[5]) {
    uint32_t r[5];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%5];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x1.b32 {%1}, [%6];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x1.b32 {%2}, [%7];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x1.b32 {%3}, [%8];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x1.b32 {%4}, [%9];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4])
        : "r"(tacc + acc_col(cc, 0)), "r"(tacc + acc_col(cc, 1)), "r"(tacc + acc_col(cc, 2)),
          "r"(tacc + acc_col(cc, 3)), "r"(tacc + acc_col(cc, 4))
        : "memory");
#pragma unroll
    for (int i = 0; i < 5; ++i) v[i] = __uint_as_float(r[i]);
}

// Bulk tensor store of one staged box (coordinates innermost first: channel, column, row, item);
// the caller commits the bulk group.
__device__ __forceinline__ void tma_store_4d(const void *tmap, const void *src, int c, int j, int i, int b) {
    asm volatile(
        "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(tmap)),
        "r"(smem_addr(src)), "r"(c), "r"(j), "r"(i), "r"(b)
        : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N committed bulk groups of this thread still read shared memory.
template <int N> __device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// 4-byte asynchronous copy global -> shared; src_bytes = 0 writes a zero and reads nothing.
__device__ __forceinline__ void cp_async4(void *dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_addr(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <typename TO> __device__ __forceinline__ void stage_out(TO *p, float v);
template <> __device__ __forceinline__ void stage_out<float>(float *p, float v) { *p = v; }
template <> __device__ __forceinline__ void stage_out<bf16>(bf16 *p, float v) { *p = __float2bfloat16_rn(v); }
template <> __device__ __forceinline__ void stage_out<f16>(f16 *p, float v) { *p = __float2half_rn(v); }

// ReLU of two accumulator values as a pair, as fmaxf on the ALU pipe: the FMA pipe is the busier
// one here (conv_dw1's packed FMAs), so a ReLU there (x + |x| with halved weights) is slower.
__device__ __forceinline__ float2 relu_pair(float a, float b) { return make_float2(fmaxf(a, 0.f), fmaxf(b, 0.f)); }

}  // namespace

template <typename TO, int CTG>
__global__ void __launch_bounds__(kThreads, 1)
dw_subsample_tc_kernel(const float *__restrict__ mel, const float *__restrict__ w0, const float *__restrict__ b0,
                       const float *__restrict__ w1, const float *__restrict__ b1,
                       const int32_t *__restrict__ lengths, int32_t *__restrict__ out_lengths,
                       const __grid_constant__ CUtensorMap out_map, int B, int Tn, int F, int C, int F2, int Pt,
                       int nIP, int nJB, int nG) {
    using Lay = TcLayout<TO, CTG>;
    extern __shared__ unsigned char smem_raw[];
    // 1024-byte aligned base (the swizzled operand tiles need it), kept as a shared pointer
    unsigned char *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    unsigned char *tileA = smem + Lay::a_off;
    unsigned char *tileB = smem + Lay::b_off;
    float *mel_s_tile = reinterpret_cast<float *>(smem + Lay::mel_off);
    TO *stage = reinterpret_cast<TO *>(smem + Lay::st_off);       // [group][slot] tiles, zero tile
    float *wtab = reinterpret_cast<float *>(smem + Lay::wt_off);  // [CTG][10][128]: w1 taps, b1
    int4 *ulist = reinterpret_cast<int4 *>(smem + Lay::list_off); // units {b, i0, j0, len}
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Lay::bar_off);
    uint64_t *patch_full = bars, *patch_empty = bars + 2, *acc_full = bars + 4, *acc_empty = bars + 6,
             *staged = bars + 8, *stage_free = bars + 10 /* [group][slot] */, *mma_done = bars + 14;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 15);
    int *counts = reinterpret_cast<int *>(bars + 16);             // active units, masked units

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int g = blockIdx.x % nG;                 // channel group of this block
    const int q0 = blockIdx.x / nG, qs = gridDim.x / nG;
    const int nUnits = B * nIP * nJB;
    constexpr int kStElems = kRO * kJO * 128;

    // ------------------------------------------------------------ patch-builder constants
    // Builder thread pt takes rows pt, pt + 128 (< kN): the builder warps with two rows a lane
    // are the last ones (SM sub-partitions 2 and 3), because the MMA issuer and the store
    // thread share sub-partitions 0 and 1 with the first ones.  (Meaningless for other warps.)
    const int pt = kPatchThreads - 1 - (static_cast<int>(threadIdx.x) - kEpiThreads);
    // This thread's mel window elements and patch rows are the same for every unit:
    // element k sits at window row rs >> 8, column rs & 255 (rs = -1 past the window); rows
    // n = pt + i * kPatchThreads all share n % 8 (one swizzle pattern).
    int mel_rs[kMelLoads];
#pragma unroll
    for (int k = 0; k < kMelLoads; ++k) {
        const int e = pt + k * kPatchThreads;
        mel_rs[k] = e < kMelElems ? ((e / kMC) << 8) | (e % kMC) : -1;
    }
    int row_cc[kRowsPer], row_rr[kRowsPer];
#pragma unroll
    for (int i = 0; i < kRowsPer; ++i) {  // the h pixel whose accumulator column is n (inverse of acc_col)
        const int n = pt + i * kPatchThreads;
        if (n < 192) {
            const int v = n % 48;
            row_cc[i] = 10 * (n / 48) + 1 + v / kHR;
            row_rr[i] = v % kHR;
        } else if (n < 200) {
            const int v = 48 + (n - 192) % 2;
            row_cc[i] = 10 * ((n - 192) / 2) + 1 + v / kHR;
            row_rr[i] = v % kHR;
        } else {
            row_cc[i] = 0;
            row_rr[i] = n - 200;
        }
    }
    // The unit's mel window goes straight to shared memory with 4-byte asynchronous copies
    // (elements outside the window's valid frames and columns are written as zero without a
    // read), two units ahead of the one being built, in kMelStages rotating windows.
    auto load_mel = [&](int u) {
        const int4 e = ulist[u];  // {b, i0, j0, len}
        float *S = mel_s_tile + (u % kMelStages) * (Lay::mel_bytes / 4);
        const int mr0 = 4 * e.y - 3 * Pt, mc0 = 4 * e.z - 3;
        const float *base = mel + static_cast<int64_t>(e.x) * Tn * F;
        const bool rows_in = mr0 >= 0 && mr0 + kMR <= e.w;  // every window row is a valid frame
#pragma unroll
        for (int k = 0; k < kMelLoads; ++k) {
            if (mel_rs[k] < 0) continue;
            const int mr = mr0 + (mel_rs[k] >> 8), mc = mc0 + (mel_rs[k] & 255);
            const bool in = (rows_in || (mr >= 0 && mr < e.w)) && mc >= 0 && mc < F;
            cp_async4(S + (mel_rs[k] >> 8) * kMCP + (mel_rs[k] & 255), in ? base + mr * F + mc : base, in ? 4u : 0u);
        }
    };

    // ------------------------------------------------------------ set-up
    launch_dependents();  // the next kernel in the stream may start its own set-up
    {
        // Warm L2 with this block's parameters (w0, w1 rows and b0, b1 over its channels) and the
        // lengths while the previous kernel drains; the loads below then hit L2.
        constexpr int kLines = CTG * 4;  // 128-byte lines of one parameter row over CTG x 128 channels
        const int t = threadIdx.x, c = g * CTG * 128 + (t % kLines) * 32;
        if (t < 10 * kLines) {
            const int row = t / kLines;  // taps 0..8, then the bias
            if (c < C) {
                prefetch_l2(row < 9 ? w0 + row * C + c : b0 + c);
                prefetch_l2(row < 9 ? w1 + row * C + c : b1 + c);
            }
        } else if (lengths != nullptr && B <= kOrderItems) {
            for (int i = (t - 10 * kLines) * 32; i < B; i += (kThreads - 10 * kLines) * 32) prefetch_l2(lengths + i);
        }
    }
    grid_dependency_wait();  // launched programmatically: the previous kernel's writes are visible after this
    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&patch_full[i], kPatchThreads);
            mbar_init(&patch_empty[i], 1);
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], kGroupThreads / 32);  // one arrival per warp of the group
            mbar_init(&staged[i], kGroupThreads);
            mbar_init(&stage_free[2 * i], 1);
            mbar_init(&stage_free[2 * i + 1], 1);
        }
        mbar_init(mma_done, 1);
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
        tc_fence_before();
        // This block's units: the active ones from the front of the list, the fully masked ones
        // (zeros only) from the back, each in the order all blocks agree on.
        const int per_item = nIP * nJB;
        const unsigned below = (1u << lane) - 1u;
        int nA = 0, nZ = 0;
        auto push = [&](bool have, bool act, const int4 &e) {
            const unsigned ma = __ballot_sync(0xffffffffu, have && act), mz = __ballot_sync(0xffffffffu, have && !act);
            if (have && act) ulist[nA + __popc(ma & below)] = e;
            if (have && !act) ulist[kListCap - 1 - (nZ + __popc(mz & below))] = e;
            nA += __popc(ma);
            nZ += __popc(mz);
        };
        if (B <= kOrderItems) {
            // Balanced deal: number all active units item-major (then row pair, then column
            // block) and all masked units likewise; block k takes every qs-th of each, so the
            // blocks' active work differs by at most one unit.  The prefix tables live in the
            // patch-operand tile, which nobody touches before the main loops.
            int *pa = reinterpret_cast<int *>(tileB), *pz = pa + (B + 1), *pl = pz + (B + 1);
            int run_a = 0, run_z = 0;
            if (lane == 0) pa[0] = pz[0] = 0;
            for (int base = 0; base < B; base += 32) {
                const int b = base + lane;
                int ia = 0, iz = 0;
                if (b < B) {
                    const int L = static_cast<int>(clamp_len(lengths, b, Tn));
                    const int rows = (((L + 1) / 2 + 1) / 2 + kRO - 1) / kRO;  // row pairs with an unmasked row
                    ia = rows * nJB;
                    iz = (nIP - rows) * nJB;
                    pl[b] = L;
                }
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int ta = __shfl_up_sync(0xffffffffu, ia, o), tz = __shfl_up_sync(0xffffffffu, iz, o);
                    if (lane >= o) {
                        ia += ta;
                        iz += tz;
                    }
                }
                if (b < B) {
                    pa[b + 1] = run_a + ia;
                    pz[b + 1] = run_z + iz;
                }
                run_a += __shfl_sync(0xffffffffu, ia, 31);
                run_z += __shfl_sync(0xffffffffu, iz, 31);
            }
            __syncwarp();
            for (int k0 = 0;; k0 += 32) {  // active units q0 + k qs
                const int a = q0 + (k0 + lane) * qs;
                const bool have = a < run_a;
                if (!__any_sync(0xffffffffu, have)) break;
                int4 e = make_int4(0, 0, 0, 0);
                if (have) {
                    const int b = TileOrder::find(pa, B, a), local = a - pa[b], ip = local / nJB;
                    e = make_int4(b, ip * kRO, (local - ip * nJB) * kJO, pl[b]);
                }
                push(have, true, e);
            }
            for (int k0 = 0;; k0 += 32) {  // masked units q0 + k qs
                const int z = q0 + (k0 + lane) * qs;
                const bool have = z < run_z;
                if (!__any_sync(0xffffffffu, have)) break;
                int4 e = make_int4(0, 0, 0, 0);
                if (have) {
                    const int b = TileOrder::find(pz, B, z), local = z - pz[b], ip = local / nJB;
                    e = make_int4(b, ((pa[b + 1] - pa[b]) / nJB + ip) * kRO, (local - ip * nJB) * kJO, pl[b]);
                }
                push(have, false, e);
            }
        } else {  // many items: plain round robin over all units
            const int mine = q0 < nUnits ? (nUnits - q0 + qs - 1) / qs : 0;
            for (int base = 0; base < mine; base += 32) {
                const int k = base + lane;
                const bool have = k < mine;
                int4 e = make_int4(0, 0, 0, 0);
                bool act = false;
                if (have) {
                    const int q = q0 + k * qs;
                    const int b = q / per_item, rem = q - b * per_item, ip = rem / nJB;
                    e = make_int4(b, ip * kRO, (rem - ip * nJB) * kJO, static_cast<int>(clamp_len(lengths, b, Tn)));
                    act = e.y < ((e.w + 1) / 2 + 1) / 2;
                }
                push(have, act, e);
            }
        }
        if (lane == 0) {
            counts[0] = nA;
            counts[1] = nZ;
        }
        named_bar(kBarList, 32 + kPatchThreads);  // the list is ready for the builders' first copies
    }
    if (warp >= kEpiWarps && warp < kMmaWarp) {
        // A operand: split conv0 weights and bias of this block's channel tiles (K layout above);
        // row r of tile i is channel (g CTG + i) 128 + r, every load issued before the first use
        const int r = threadIdx.x - kEpiThreads;
        float xw[CTG][10];
#pragma unroll
        for (int i = 0; i < CTG; ++i) {
            const int c = (g * CTG + i) * 128 + r;
#pragma unroll
            for (int t = 0; t < 10; ++t) xw[i][t] = c < C ? __ldg(t < 9 ? w0 + t * C + c : b0 + c) : 0.f;
        }
#pragma unroll
        for (int i = 0; i < CTG; ++i) {
            float hi[9], lo[9];
#pragma unroll
            for (int t = 0; t < 9; ++t) {
                hi[t] = tf32_hi(xw[i][t]);
                lo[t] = xw[i][t] - hi[t];
            }
            const float bx = xw[i][9];
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
            store_k_row(tileA + i * kTileA, r, q);
        }
        fence_async_smem();
        // the first two units' mel windows start copying before the block-wide barrier
        named_bar(kBarList, 32 + kPatchThreads);
        const int nA0 = counts[0];
        if (nA0 > 0) load_mel(0);
        cp_async_commit();
        if (nA0 > 1) load_mel(1);
        cp_async_commit();
    }
    if (warp < kEpiWarps) {
        // conv_dw1 weights and bias: every load issued first, the zero tile written meanwhile
        constexpr int kWtPer = CTG * 10 * 128 / kEpiThreads;
        static_assert(CTG * 10 * 128 % kEpiThreads == 0, "weight table split");
        float wv[kWtPer];
#pragma unroll
        for (int j = 0; j < kWtPer; ++j) {
            const int e = threadIdx.x + j * kEpiThreads;
            const int ct = e / 1280, t = (e / 128) % 10, c = (g * CTG + ct) * 128 + e % 128;
            wv[j] = c < C ? __ldg(t < 9 ? w1 + t * C + c : b1 + c) : 0.f;
        }
        TO *z = stage + 4 * kStElems;  // the zero tile stored for fully masked units
        for (int e = threadIdx.x; e < kStElems; e += kEpiThreads) stage_out<TO>(z + e, 0.f);
        fence_async_smem();
#pragma unroll
        for (int j = 0; j < kWtPer; ++j) wtab[threadIdx.x + j * kEpiThreads] = wv[j];
        if (blockIdx.x == 0 && out_lengths != nullptr)
            for (int q = threadIdx.x; q < B; q += kEpiThreads) {
                const int Lq = static_cast<int>(clamp_len(lengths, q, Tn));
                out_lengths[q] = ((Lq + 1) / 2 + 1) / 2;
            }
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int nA = counts[0], nZ = counts[1];

    if (warp < kEpiWarps) {
        // ------------------------------------------------------------ epilogue
        // Two groups of four warps (one per TMEM lane quarter) take the jobs (unit x channel
        // tile) in turn: group 0 the even ones in accumulator buffer 0, group 1 the odd ones in
        // buffer 1.  A group's jobs all have the same channel tile, so its conv_dw1 taps stay in
        // registers.  No named barriers: the group hands its staged tile to the store thread and
        // gets it back through mbarriers.
        const int grp = warp >> 2, qw = warp & 3;
        const int m = qw * 32 + lane;                     // channel within the tile = TMEM lane
        const int ct = CTG == 2 ? grp : 0;
        const uint32_t tacc = tmem_base + (static_cast<uint32_t>(qw * 32) << 16) + grp * kTmemBuf;
        // conv_dw1 taps as pairs
        float2 W[3][3], bias;
        {
            const float *wt = wtab + ct * 1280 + m;
#pragma unroll
            for (int t = 0; t < 9; ++t) {
                const float x = wt[t * 128];
                W[t / 3][t % 3] = make_float2(x, x);
            }
            bias = make_float2(wt[9 * 128], wt[9 * 128]);
        }
        const int first = CTG == 1 ? grp : 0, step = CTG == 1 ? 2 : 1;
        bool ok = true;
        for (int idx = first, n = 0; idx < nA && ok; idx += step, ++n) {
            const int4 e = ulist[idx];
            const bool row1 = e.y + 1 < ((e.w + 1) / 2 + 1) / 2;  // the second output row is unmasked
            ok = mbar_wait(&acc_full[grp], n & 1);
            if (!ok) break;
            tc_fence_after();
            TO *st = stage + (2 * grp + (n & 1)) * kStElems;
            // E[i][p]: h rows (p, p+2) of the even h column 2 jl0 + 2i; E[0] carries over
            float2 E[kChunk + 1][3];
            {
                float v[5];
                tmem_ld_column(tacc, 0, v);
                E[0][0] = relu_pair(v[0], v[2]);
                E[0][1] = relu_pair(v[1], v[3]);
                E[0][2] = relu_pair(v[2], v[4]);
            }
#pragma unroll
            for (int ch = 0; ch < kJO / kChunk; ++ch) {  // unrolled: the per-chunk branches resolve at compile time
                const int jl0 = ch * kChunk;                     // first output column (unit-local)
                float v[50];
                tmem_ld_chunk(tacc, ch, v);                      // h columns 2 jl0 + 1 .. 2 jl0 + 10
                if (ch == kJO / kChunk - 1) {  // accumulator read out: the next MMA may start
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&acc_empty[grp]);
                }
                // this slot's previous tile (two jobs back) has been read by its store
                if (ch == 0 && n > 1) {
                    ok = mbar_wait(&stage_free[2 * grp + (n & 1)], ((n >> 1) - 1) & 1);
                    if (!ok) break;
                }
#pragma unroll
                for (int i = 1; i <= kChunk; ++i) {
                    const float *x = v + (2 * i - 1) * kHR;
                    E[i][0] = relu_pair(x[0], x[2]);
                    E[i][1] = relu_pair(x[1], x[3]);
                    E[i][2] = relu_pair(x[2], x[4]);
                }
                float2 acc[kChunk];
#pragma unroll
                for (int p = 0; p < 3; ++p)
#pragma unroll
                    for (int jj = 0; jj < kChunk; ++jj)
                        acc[jj] = ffma2(E[jj][p], W[p][0], p == 0 ? bias : acc[jj]);
#pragma unroll
                for (int jj = 0; jj < kChunk; ++jj) {  // odd h column 2 jj + 1
                    const float *x = v + (2 * jj) * kHR;
                    acc[jj] = ffma2(relu_pair(x[0], x[2]), W[0][1], acc[jj]);
                    acc[jj] = ffma2(relu_pair(x[1], x[3]), W[1][1], acc[jj]);
                    acc[jj] = ffma2(relu_pair(x[2], x[4]), W[2][1], acc[jj]);
                }
#pragma unroll
                for (int p = 0; p < 3; ++p)
#pragma unroll
                    for (int jj = 0; jj < kChunk; ++jj) acc[jj] = ffma2(E[jj + 1][p], W[p][2], acc[jj]);
#pragma unroll
                for (int jj = 0; jj < kChunk; ++jj) {
                    stage_out<TO>(st + (jl0 + jj) * 128 + m, acc[jj].x);
                    stage_out<TO>(st + (kJO + jl0 + jj) * 128 + m, row1 ? acc[jj].y : 0.f);
                }
#pragma unroll
                for (int p = 0; p < 3; ++p) E[0][p] = E[kChunk][p];
            }
            // staged tile complete: hand it to the store thread
            fence_async_smem();
            mbar_arrive(&staged[grp]);
        }
    } else if (warp < kMmaWarp) {
        // ------------------------------------------------------------ patch builders
        // (the first two units' mel windows were requested during the set-up)
        bool ok = true;
        for (int idx = 0; idx < nA && ok; ++idx) {
            const int4 e = ulist[idx];
            const int L2 = (e.w + 1) / 2;
            const float *S = mel_s_tile + (idx % kMelStages) * (Lay::mel_bytes / 4);
            cp_async_wait<1>();  // this thread's copies of unit idx have landed (idx + 1 may be in flight)
            named_bar(kBarPatch, kPatchThreads);  // ... and every builder's; all are done with unit idx - 1
            if (idx + 2 < nA) load_mel(idx + 2);  // into the window unit idx - 1 used
            cp_async_commit();
            const int stage_i = idx & 1;
            ok = named_bar_and(kBarPatch, kPatchThreads, mbar_wait(&patch_empty[stage_i], ((idx >> 1) & 1) ^ 1));
            if (!ok) break;
            unsigned char *tb = tileB + stage_i * kTileB;
#pragma unroll
            for (int i = 0; i < kRowsPer; ++i) {
                const int n = pt + i * kPatchThreads;
                if (n >= kN) break;
                const int cc = row_cc[i], rr = row_rr[i];
                const int hr = 2 * e.y - Pt + rr, hc = 2 * e.z - 1 + cc;
                const bool valid = n < kNUsed && hr >= 0 && hr < L2 && hc >= 0 && hc < F2;
                float4 q[8];
                if (valid) {
                    const float *sp = S + (2 * rr) * kMCP + 2 * cc;
                    float hi[9], lo[9];
#pragma unroll
                    for (int t = 0; t < 9; ++t) {
                        const float x = sp[(t / 3) * kMCP + t % 3];
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
                } else {
#pragma unroll
                    for (int k = 0; k < 8; ++k) q[k] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
                store_k_row(tb, n, q);
            }
            fence_async_smem();
            mbar_arrive(&patch_full[stage_i]);
        }
        cp_async_wait<0>();  // no copy outlives the loop (it may have ended early)
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            // ------------------------------------------------------------ MMA issuer
            const uint32_t a_base = smem_addr(tileA), b_base = smem_addr(tileB);
            bool ok = true;
            for (int idx = 0; idx < nA && ok; ++idx) {
                const int stage_i = idx & 1;
                ok = mbar_wait(&patch_full[stage_i], (idx >> 1) & 1);
                if (!ok) break;
                tc_fence_after();
                const uint64_t bdesc = sw128_desc(b_base + stage_i * kTileB);
                for (int ct = 0; ct < CTG; ++ct) {
                    const int job = idx * CTG + ct, buf = job & 1;
                    ok = mbar_wait(&acc_empty[buf], ((job >> 1) & 1) ^ 1);
                    if (!ok) break;
                    tc_fence_after();
                    const uint64_t adesc = sw128_desc(a_base + ct * kTileA);
                    const uint32_t d = tmem_base + buf * kTmemBuf;
#pragma unroll
                    for (int k = 0; k < 4; ++k)  // K = 32 TF32 words = 4 steps of 8 (32 bytes)
                        mma_tf32(d, adesc + 2 * k, bdesc + 2 * k, kIdesc, k > 0 ? 1u : 0u);
                    mma_commit(&acc_full[buf]);
                }
                mma_commit(&patch_empty[stage_i]);
            }
            // every issued MMA has finished before tensor memory is released
            mma_commit(mma_done);
            mbar_wait(mma_done, 0);
        }
    } else if (lane == 0) {
        // ------------------------------------------------------------ bulk stores
        // Staged tiles of the two epilogue groups in job order, and the zero tile for every
        // fully masked unit (one masked unit per staged job, so neither kind waits long).  Each
        // iteration commits exactly two bulk groups (masked unit, staged tile; either may be
        // empty), so when at most four groups are pending the staged tile of two jobs back has
        // been read and its slot goes back to its epilogue group.
        const TO *zero = stage + 4 * kStElems;
        int z = 0;
        auto store_zero_unit = [&]() {
            const int4 e = ulist[kListCap - 1 - z];
            for (int ct = 0; ct < CTG; ++ct) {
                const int c0 = (g * CTG + ct) * 128;
                if (c0 < C) tma_store_4d(&out_map, zero, c0, e.z, e.y, e.x);
            }
            ++z;
        };
        for (int job = 0; job < nA * CTG; ++job) {
            if (z < nZ) store_zero_unit();
            bulk_commit();
            const int grp = job & 1, n = job >> 1;
            if (!mbar_wait(&staged[grp], n & 1)) break;
            const int4 e = ulist[job / CTG];
            const int c0 = (g * CTG + job % CTG) * 128;
            if (c0 < C) tma_store_4d(&out_map, stage + (2 * grp + (n & 1)) * kStElems, c0, e.z, e.y, e.x);
            bulk_commit();
            if (job >= 2) {
                bulk_wait_read<4>();
                const int np = (job - 2) >> 1;  // the same group's previous job
                mbar_arrive(&stage_free[2 * grp + (np & 1)]);
            }
        }
        while (z < nZ) store_zero_unit();
        bulk_commit();
        bulk_wait_all();
    }
    __syncwarp();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

unsigned int subsample_tc_take_error() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, dw_device_error_flag, sizeof(v)) != cudaSuccess) return 0;
    if (v != 0) cudaMemcpyToSymbol(dw_device_error_flag, &zero, sizeof(zero));
    return v;
}

// Tensor map over the output [B][T4][F4][C] (dims innermost first), box 128 x kJO x kRO x 1.
static cudaError_t make_out_map(CUtensorMap *map, void *out, int dtype, int64_t B, int64_t T4, int64_t F4,
                                int64_t C) {
    TensorMapEncodeTiledFn enc = tensor_map_encoder();
    if (enc == nullptr) return cudaErrorNotSupported;
    const int64_t es = dtype_bytes(dtype);
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(F4),
                                static_cast<cuuint64_t>(T4), static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(C * es), static_cast<cuuint64_t>(F4 * C * es),
                                   static_cast<cuuint64_t>(T4 * F4 * C * es)};
    const cuuint32_t box[4] = {128u, static_cast<cuuint32_t>(kJO), static_cast<cuuint32_t>(kRO), 1u};
    const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    const CUresult r = enc(map, tma_dtype(dtype), 4,
                           out, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                           CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

bool subsample_tc_eligible(const SubsampleArgs &a) {
    const int64_t es = dtype_bytes(a.out_dtype);
    auto s2 = [](int64_t n) -> int64_t { return n >= 1 ? (n - 1) / 2 + 1 : 0; };
    const int64_t T4 = s2(s2(a.T)), F4 = s2(s2(a.F));
    const int64_t nIP = (T4 + kRO - 1) / kRO, nJB = (F4 + kJO - 1) / kJO;
    return tensor_map_encoder() != nullptr && (a.C * es) % 16 == 0 &&
           reinterpret_cast<uintptr_t>(a.out) % 16 == 0 && a.T * a.F < (1LL << 31) &&
           9 * a.C < (1LL << 31) && a.B * nIP * nJB < (1LL << 31) && T4 > 0;
}

cudaError_t subsample_tc_launch(const SubsampleArgs &a, cudaStream_t s) {
    auto s2 = [](int64_t n) -> int64_t { return n >= 1 ? (n - 1) / 2 + 1 : 0; };
    const int64_t F2 = s2(a.F), T4 = s2(s2(a.T)), F4 = s2(F2);
    const int64_t nIP = (T4 + kRO - 1) / kRO, nJB = (F4 + kJO - 1) / kJO;
    const int64_t nCT = (a.C + 127) / 128;
    const int ctg = nCT >= 2 ? 2 : 1;
    const int64_t nG = (nCT + ctg - 1) / ctg;
    const int64_t units = a.B * nIP * nJB;
    CUtensorMap map;
    cudaError_t e = make_out_map(&map, a.out, a.out_dtype, a.B, T4, F4, a.C);
    if (e != cudaSuccess) return cudaErrorNotSupported;  // the caller takes the SIMT kernel
    int64_t grid = (sm_count() / nG) * nG;
    if (grid < nG) grid = nG;
    if (grid > units * nG) grid = units * nG;
    if (grid > kMaxGrid) return cudaErrorInvalidConfiguration;
    // every block keeps its unit list in shared memory; larger problems take the SIMT kernel
    if ((units + grid / nG - 1) / (grid / nG) + 1 > kListCap) return cudaErrorNotSupported;
    const int Pt = a.causal ? 2 : 1;
#define DW_TC_LAUNCH(TO, CTG)                                                                                  \
    do {                                                                                                       \
        auto kern = dw_subsample_tc_kernel<TO, CTG>;                                                           \
        const int bytes = TcLayout<TO, CTG>::alloc;                                                            \
        e = ensure_smem_attr(reinterpret_cast<const void *>(kern), bytes);                                    \
        if (e != cudaSuccess) return e;                                                                        \
        cudaLaunchConfig_t cfg = {};                                                                           \
        cfg.gridDim = dim3(static_cast<unsigned>(grid));                                                       \
        cfg.blockDim = dim3(kThreads);                                                                         \
        cfg.dynamicSmemBytes = bytes;                                                                          \
        cfg.stream = s;                                                                                        \
        cudaLaunchAttribute at[1];                                                                             \
        at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;                                        \
        at[0].val.programmaticStreamSerializationAllowed = 1;                                                 \
        cfg.attrs = at;                                                                                        \
        cfg.numAttrs = 1;                                                                                      \
        e = cudaLaunchKernelEx(&cfg, kern,                                                                     \
            a.mel, a.w0, a.b0, a.w1, a.b1, a.lengths, a.out_lengths, map, static_cast<int>(a.B),               \
            static_cast<int>(a.T), static_cast<int>(a.F), static_cast<int>(a.C), static_cast<int>(F2), Pt,     \
            static_cast<int>(nIP), static_cast<int>(nJB), static_cast<int>(nG));                               \
    } while (0)
    if (a.out_dtype == 1) {
        if (ctg == 2) DW_TC_LAUNCH(bf16, 2);
        else DW_TC_LAUNCH(bf16, 1);
    } else if (a.out_dtype == 2) {
        if (ctg == 2) DW_TC_LAUNCH(f16, 2);
        else DW_TC_LAUNCH(f16, 1);
    } else {
        if (ctg == 2) DW_TC_LAUNCH(float, 2);
        else DW_TC_LAUNCH(float, 1);
    }
#undef DW_TC_LAUNCH
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace dwk
