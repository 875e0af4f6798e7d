// gemm_prefill.cuh -- tcgen05 block-scaled FP8 GEMM for large M (prefill).
//
// Y[m, n] = BF16( sum_kb sa[m, kb] * sw[n/128, kb] * P_kb[m, n] ),
// P_kb[m, n] = sum_{k in kb} e4m3(qa[m, k]) * e4m3(qw[n, k])
// (page "ProCreations/Nanbeige4.3-33B-FP8", introduction: W8A8 FP8 linear
// layers with 128x128 weight blocks and per-token group-128 activation scales).
//
// The scales are arbitrary binary32 values per 128-wide K chunk, which the
// tensor core's block-scaled MMA formats (power-of-two scales per 32 elements)
// cannot carry, so every K chunk is a fresh tensor-core partial in TMEM that
// CUDA cores promote into a register accumulator:  acc = fma(P_kb, sa*sw, acc).
//
// Design (one persistent CTA per SM, 384 threads = 3 warpgroups):
//   warp 0      TMA producer: per K chunk one A tile (128 x 128 B) and one B tile
//               (BN x 128 B), 128-byte swizzle, into a kStages-deep ring.
//   warps 1, 2  MMA issuers (one thread each, one per TMEM buffer of BN FP32
//               columns): 4 x tcgen05.mma (K = 32 each) per chunk, chunk i
//               into buffer i mod 2 by warp 1 + (i mod 2).  A thread that waits
//               on shared memory after issuing MMAs loses ~0.1 us; with two
//               issuers those waits overlap (measured +6% on the whole GEMM).
//   warp 3      idle; warpgroup 0 gives its registers up (setmaxnreg 40).
//   warps 4..11 promotion + epilogue (setmaxnreg 232): warp w reads TMEM lanes
//               32*(w%4)..+31 (its hardware lane quarter); warpgroup 1 owns tile
//               columns [0, 128), warpgroup 2 columns [128, 256), so a thread
//               keeps the 128 FP32 accumulators of one output row in one
//               128-column weight block, whose scale is a single sw per chunk.
// Register budget: launched at 168 per thread (384 x 168 = 64512); after the
// split 128 x 40 + 256 x 232 = 64512, the same total.
// Tiles are walked in groups of group_m(K) m-tiles (m fastest within a group)
// so the tiles resident at one time share A and B rows in L2.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "ptx.cuh"
#include "quantize.cuh"
#include "silu_quant.cuh"

namespace fp8bq {
namespace prefill {

constexpr int BM = 128;
constexpr int BK = 128;  // one scale chunk of K per pipeline stage
// Three 48 KB stages: two starve the tensor pipe (-24%), four are 1-2% slower
// than three (the smaller ring leaves more L1 for the promotion's scale loads).
constexpr int kStages = 3;
constexpr int kNumThreads = 384;
constexpr int kLaunchRegs = 168;     // registers per thread the kernel must be built with
constexpr int kProducerRegs = 40;    // warpgroup 0 after setmaxnreg.dec
constexpr int kConsumerRegs = 232;   // warpgroups 1-2 after setmaxnreg.inc
static_assert(128 * kProducerRegs + 256 * kConsumerRegs <= kNumThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr int kFirstPromoWarp = 4;
constexpr int kPromoWarps = 8;
// m-tiles per raster group: each group streams every weight tile once, so
// larger groups re-read the weights less often (QKV 8192 x 9216 x 7168: 322 MB
// of DRAM reads with 16, 204 MB with 32, for 125 MB of operands), as long as
// the group's A rows (group x 128 x K bytes) leave L2 room for the weight tiles
// in flight: 32 up to K = 10240, i.e. KB = K / 128 <= 80 (at most 42 MB of A),
// 16 beyond (64 m-tiles, all of A, raised the reads instead).  A template
// parameter of the kernel (a run-time group size costs the 40-register
// producer warp a spill).
__host__ __device__ constexpr int group_m(int KB) { return KB <= 80 ? 32 : 16; }
constexpr int kScaleLookahead = 2;   // K chunks of scale prefetch in registers

template <int BN, bool kSilu = false>
struct Layout {
    static_assert(BN == 256, "tile width");
    static constexpr int kA = BM * BK;
    static constexpr int kB = BN * BK;
    static constexpr int kStage = kA + kB;
    static constexpr int kBarOff = kStages * kStage;
    static constexpr int kNumBars = 2 * kStages + 2 + 2 + 1;  // full, empty, tfull, tempty, drain
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    // SiLU epilogue: per-row group maxima of the two column halves, two tiles
    // deep, each a 64-bit word tagged with the tile's index
    static constexpr int kXchgOff = kMiscOff + 32;
    static constexpr int kXchgBytes = kSilu ? 2 * BM * 2 * 8 : 0;
    static constexpr int kBytes = kXchgOff + kXchgBytes;
    static constexpr int kDynamicSmem = kBytes + 1024;  // room to align the base to 1024 B
    static_assert(kDynamicSmem <= 227 * 1024, "shared memory");
    static constexpr uint32_t kTmemCols = 2 * BN;
};

// Split-K tail: when the tiles leave a last wave of at most kTailMaxTiles tiles
// on the persistent grid, each of those tiles is split K-wise into tail_parts
// parts run by different CTAs; each part's FP32 partial goes to the workspace
// and the part that finishes last sums all of them in part order
// (deterministic) and writes the tile.
constexpr int kTailMaxTiles = 16;
constexpr int kTailMaxParts = 4;
constexpr int64_t kTailPartialFloats = int64_t(BM) * 256;  // one part of a 128 x 256 tile

// The CTA's w-th work item: first its full tiles (blockIdx.x + w gridDim.x
// below full_tiles), then at most one tail part.  part < 0 for a full tile.
__device__ __forceinline__ bool work_item(int w, int num_tiles, int full_tiles, int tail_parts,
                                          int KB, int &tile, int &kb0, int &kb1, int &part) {
    const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
    const int t = c + w * G;
    if (t < full_tiles) {
        tile = t;
        kb0 = 0;
        kb1 = KB;
        part = -1;
        return true;
    }
    if (tail_parts == 0 || w != (full_tiles - c + G - 1) / G) return false;
    if (c >= (num_tiles - full_tiles) * tail_parts) return false;
    tile = full_tiles + c / tail_parts;
    part = c % tail_parts;
    kb0 = part * KB / tail_parts;
    kb1 = (part + 1) * KB / tail_parts;
    return true;
}

__device__ __forceinline__ void tile_coords(int t, int m_tiles, int n_tiles, int group_rows, int &tm,
                                            int &tn) {
    const int group = group_rows * n_tiles;
    const int g = t / group, r = t - g * group;
    const int first_m = g * group_rows;
    const int gm = min(group_rows, m_tiles - first_m);
    tm = first_m + r % gm;
    tn = r / gm;
}

// Waits (bounded, like mbar_wait) until the upper 32 bits of the shared word
// *p equal those of `tag`, and returns the word in `word`.
__device__ __forceinline__ bool smem_tag_wait(volatile unsigned long long *p,
                                              unsigned long long tag, unsigned long long &word,
                                              volatile int *abort, int *status) {
    word = *p;
    if ((word >> 32) == (tag >> 32)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        word = *p;
        if ((word >> 32) == (tag >> 32)) return true;
        if ((it & 255u) == 0) {
            if (*abort) return false;
            if (global_timer_ns() - t0 > kWaitLimitNs) {
                *abort = 1;
                atomicExch(status, 6 /* FP8BQ_ERR_TIMEOUT */);
                return false;
            }
        }
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// Promotes one K chunk of this thread's 128 TMEM columns into acc:
// acc[i] = fma(P[i], scale, acc[i]), with the columns taken as two runs of 64:
// acc[0..63] from TMEM columns taddr0 .. taddr0 + 63 with scale0, acc[64..127]
// from taddr1 .. taddr1 + 63 with scale1 (for a plain tile, taddr1 = taddr0 +
// 64 and scale1 = scale0).  The TMEM loads go in two batches of 64 columns,
// one 32x32b.x64 load and one wait each: the second batch is in flight while
// the FMAs of the first run, and it is returned in `last` after its wait, so
// the caller releases the TMEM buffer after two load waits (not four) and
// finishes those 64 FMAs afterwards (measured +3% on every prefill shape over
// four 32-column loads with a wait each; one .x64 load per batch instead of
// two .x32 gained another 0.7-1% on QKV, fc and long o_proj).  Loads and waits
// live in one asm statement so no register is read before its wait.
__device__ __forceinline__ void promote_chunk(uint32_t taddr0, uint32_t taddr1, float scale0,
                                              float scale1, float (&acc)[128], float (&last)[64]) {
    asm volatile(
        "{\n\t"
        ".reg .f32 ra<32>, rb<32>;\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {ra0,ra1,ra2,ra3,ra4,ra5,ra6,ra7,ra8,ra9,ra10,ra11,ra12,ra13,ra14,ra15,ra16,ra17,ra18,ra19,ra20,ra21,ra22,ra23,ra24,ra25,ra26,ra27,ra28,ra29,ra30,ra31,rb0,rb1,rb2,rb3,rb4,rb5,rb6,rb7,rb8,rb9,rb10,rb11,rb12,rb13,rb14,rb15,rb16,rb17,rb18,rb19,rb20,rb21,rb22,rb23,rb24,rb25,rb26,rb27,rb28,rb29,rb30,rb31}, [%129];\n\t"
        "tcgen05.wait::ld.sync.aligned;\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95,%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127}, [%131];\n\t"
        "fma.rn.f32 %0, ra0, %128, %0;\n\t"
        "fma.rn.f32 %1, ra1, %128, %1;\n\t"
        "fma.rn.f32 %2, ra2, %128, %2;\n\t"
        "fma.rn.f32 %3, ra3, %128, %3;\n\t"
        "fma.rn.f32 %4, ra4, %128, %4;\n\t"
        "fma.rn.f32 %5, ra5, %128, %5;\n\t"
        "fma.rn.f32 %6, ra6, %128, %6;\n\t"
        "fma.rn.f32 %7, ra7, %128, %7;\n\t"
        "fma.rn.f32 %8, ra8, %128, %8;\n\t"
        "fma.rn.f32 %9, ra9, %128, %9;\n\t"
        "fma.rn.f32 %10, ra10, %128, %10;\n\t"
        "fma.rn.f32 %11, ra11, %128, %11;\n\t"
        "fma.rn.f32 %12, ra12, %128, %12;\n\t"
        "fma.rn.f32 %13, ra13, %128, %13;\n\t"
        "fma.rn.f32 %14, ra14, %128, %14;\n\t"
        "fma.rn.f32 %15, ra15, %128, %15;\n\t"
        "fma.rn.f32 %16, ra16, %128, %16;\n\t"
        "fma.rn.f32 %17, ra17, %128, %17;\n\t"
        "fma.rn.f32 %18, ra18, %128, %18;\n\t"
        "fma.rn.f32 %19, ra19, %128, %19;\n\t"
        "fma.rn.f32 %20, ra20, %128, %20;\n\t"
        "fma.rn.f32 %21, ra21, %128, %21;\n\t"
        "fma.rn.f32 %22, ra22, %128, %22;\n\t"
        "fma.rn.f32 %23, ra23, %128, %23;\n\t"
        "fma.rn.f32 %24, ra24, %128, %24;\n\t"
        "fma.rn.f32 %25, ra25, %128, %25;\n\t"
        "fma.rn.f32 %26, ra26, %128, %26;\n\t"
        "fma.rn.f32 %27, ra27, %128, %27;\n\t"
        "fma.rn.f32 %28, ra28, %128, %28;\n\t"
        "fma.rn.f32 %29, ra29, %128, %29;\n\t"
        "fma.rn.f32 %30, ra30, %128, %30;\n\t"
        "fma.rn.f32 %31, ra31, %128, %31;\n\t"
        "fma.rn.f32 %32, rb0, %128, %32;\n\t"
        "fma.rn.f32 %33, rb1, %128, %33;\n\t"
        "fma.rn.f32 %34, rb2, %128, %34;\n\t"
        "fma.rn.f32 %35, rb3, %128, %35;\n\t"
        "fma.rn.f32 %36, rb4, %128, %36;\n\t"
        "fma.rn.f32 %37, rb5, %128, %37;\n\t"
        "fma.rn.f32 %38, rb6, %128, %38;\n\t"
        "fma.rn.f32 %39, rb7, %128, %39;\n\t"
        "fma.rn.f32 %40, rb8, %128, %40;\n\t"
        "fma.rn.f32 %41, rb9, %128, %41;\n\t"
        "fma.rn.f32 %42, rb10, %128, %42;\n\t"
        "fma.rn.f32 %43, rb11, %128, %43;\n\t"
        "fma.rn.f32 %44, rb12, %128, %44;\n\t"
        "fma.rn.f32 %45, rb13, %128, %45;\n\t"
        "fma.rn.f32 %46, rb14, %128, %46;\n\t"
        "fma.rn.f32 %47, rb15, %128, %47;\n\t"
        "fma.rn.f32 %48, rb16, %128, %48;\n\t"
        "fma.rn.f32 %49, rb17, %128, %49;\n\t"
        "fma.rn.f32 %50, rb18, %128, %50;\n\t"
        "fma.rn.f32 %51, rb19, %128, %51;\n\t"
        "fma.rn.f32 %52, rb20, %128, %52;\n\t"
        "fma.rn.f32 %53, rb21, %128, %53;\n\t"
        "fma.rn.f32 %54, rb22, %128, %54;\n\t"
        "fma.rn.f32 %55, rb23, %128, %55;\n\t"
        "fma.rn.f32 %56, rb24, %128, %56;\n\t"
        "fma.rn.f32 %57, rb25, %128, %57;\n\t"
        "fma.rn.f32 %58, rb26, %128, %58;\n\t"
        "fma.rn.f32 %59, rb27, %128, %59;\n\t"
        "fma.rn.f32 %60, rb28, %128, %60;\n\t"
        "fma.rn.f32 %61, rb29, %128, %61;\n\t"
        "fma.rn.f32 %62, rb30, %128, %62;\n\t"
        "fma.rn.f32 %63, rb31, %128, %63;\n\t"
        "tcgen05.wait::ld.sync.aligned;\n\t"
        "}"
        : "+f"(acc[0]), "+f"(acc[1]), "+f"(acc[2]), "+f"(acc[3]), "+f"(acc[4]), "+f"(acc[5]), "+f"(acc[6]), "+f"(acc[7]), "+f"(acc[8]), "+f"(acc[9]), "+f"(acc[10]), "+f"(acc[11]), "+f"(acc[12]), "+f"(acc[13]), "+f"(acc[14]), "+f"(acc[15]), "+f"(acc[16]), "+f"(acc[17]), "+f"(acc[18]), "+f"(acc[19]), "+f"(acc[20]), "+f"(acc[21]), "+f"(acc[22]), "+f"(acc[23]), "+f"(acc[24]), "+f"(acc[25]), "+f"(acc[26]), "+f"(acc[27]), "+f"(acc[28]), "+f"(acc[29]), "+f"(acc[30]), "+f"(acc[31]), "+f"(acc[32]), "+f"(acc[33]), "+f"(acc[34]), "+f"(acc[35]), "+f"(acc[36]), "+f"(acc[37]), "+f"(acc[38]), "+f"(acc[39]), "+f"(acc[40]), "+f"(acc[41]), "+f"(acc[42]), "+f"(acc[43]), "+f"(acc[44]), "+f"(acc[45]), "+f"(acc[46]), "+f"(acc[47]), "+f"(acc[48]), "+f"(acc[49]), "+f"(acc[50]), "+f"(acc[51]), "+f"(acc[52]), "+f"(acc[53]), "+f"(acc[54]), "+f"(acc[55]), "+f"(acc[56]), "+f"(acc[57]), "+f"(acc[58]), "+f"(acc[59]), "+f"(acc[60]), "+f"(acc[61]), "+f"(acc[62]), "+f"(acc[63]), "=f"(last[0]), "=f"(last[1]), "=f"(last[2]), "=f"(last[3]), "=f"(last[4]), "=f"(last[5]), "=f"(last[6]), "=f"(last[7]), "=f"(last[8]), "=f"(last[9]), "=f"(last[10]), "=f"(last[11]), "=f"(last[12]), "=f"(last[13]), "=f"(last[14]), "=f"(last[15]), "=f"(last[16]), "=f"(last[17]), "=f"(last[18]), "=f"(last[19]), "=f"(last[20]), "=f"(last[21]), "=f"(last[22]), "=f"(last[23]), "=f"(last[24]), "=f"(last[25]), "=f"(last[26]), "=f"(last[27]), "=f"(last[28]), "=f"(last[29]), "=f"(last[30]), "=f"(last[31]), "=f"(last[32]), "=f"(last[33]), "=f"(last[34]), "=f"(last[35]), "=f"(last[36]), "=f"(last[37]), "=f"(last[38]), "=f"(last[39]), "=f"(last[40]), "=f"(last[41]), "=f"(last[42]), "=f"(last[43]), "=f"(last[44]), "=f"(last[45]), "=f"(last[46]), "=f"(last[47]), "=f"(last[48]), "=f"(last[49]), "=f"(last[50]), "=f"(last[51]), "=f"(last[52]), "=f"(last[53]), "=f"(last[54]), "=f"(last[55]), "=f"(last[56]), "=f"(last[57]), "=f"(last[58]), "=f"(last[59]), "=f"(last[60]), "=f"(last[61]), "=f"(last[62]), "=f"(last[63])
        : "f"(scale0), "r"(taddr0), "f"(scale1), "r"(taddr1)
        : "memory");
}

// Outputs of the SiLU-gated epilogue (kSilu): for the fused gate/up weight
// [2I, K] (gate rows [0, I), up rows [I, 2I)), tile column block tn holds gate
// channels [128 tn, 128 tn + 128) in TMEM columns [0, 128) and the up channels
// of the same indices in [128, 256); the tile's output is
// h = BF16(silu(BF16 gate) * BF16 up) for those 128 channels, quantized as one
// activation group: codes q [M, I], scales s [M, I/128], h [M, I] if h != null.
struct SiluOut {
    uint8_t *q;
    float *s;
    __nv_bfloat16 *h;
};

template <int BN, bool kSilu, int kGroupRows>
__global__ void __launch_bounds__(kNumThreads, 1)
gemm_prefill_kernel(const __grid_constant__ CUtensorMap tmap_a,
                    const __grid_constant__ CUtensorMap tmap_b, const float *__restrict__ sa,
                    const float *__restrict__ sw, __nv_bfloat16 *__restrict__ y, int M, int N,
                    int K, int *status, int tail_parts, float *tail_partials, int *tail_counters,
                    SiluOut silu) {
    using L = Layout<BN, kSilu>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kBarOff);
    uint64_t *empty = full + kStages;
    uint64_t *tfull = empty + kStages;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMiscOff);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOff + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = K / BK;
    const int m_tiles = (M + BM - 1) / BM;
    // kSilu: N = 2I weight rows, one tile per 128 output channels of h
    const int I = N / 2;
    const int n_tiles = kSilu ? I / 128 : (N + BN - 1) / BN;
    const int num_tiles = m_tiles * n_tiles;
    // with a split-K tail, the last wave's tiles are split into parts
    const int full_tiles =
        tail_parts > 0 ? num_tiles - num_tiles % static_cast<int>(gridDim.x) : num_tiles;

    allow_dependent_launch();
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], kPromoWarps);
        }
        mbar_init(drain, 2);
        *abort_flag = 0;
        reinterpret_cast<uint32_t *>(smem + L::kMiscOff + 8)[0] = 0;  // tail verdict
        reinterpret_cast<uint32_t *>(smem + L::kMiscOff + 8)[1] = 0;  // tail arrivals
        fence_barrier_init();
    }
    if constexpr (kSilu) {
        // no tile index matches this tag
        unsigned long long *xchg = reinterpret_cast<unsigned long long *>(smem + L::kXchgOff);
        for (int i = threadIdx.x; i < L::kXchgBytes / 8; i += kNumThreads) xchg[i] = ~0ull;
    }
    if (threadIdx.x == 0) {
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_b);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, L::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    // Everything above overlaps the previous kernel in the stream; every global
    // memory access below happens after it has completed.
    grid_dependency_wait();

    if (warp < kFirstPromoWarp) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
        if (warp == 0) {
            // ------------------------------------------------------------ TMA producer
            if (lane == 0) {
                uint32_t stage = 0, phase = 0;
                int64_t issued = 0;
                bool ok = true;
                int t, kb0, kb1, part;
                for (int w = 0; ok && work_item(w, num_tiles, full_tiles, tail_parts, KB, t, kb0, kb1, part);
                     ++w) {
                    int tm, tn;
                    tile_coords(t, m_tiles, n_tiles, kGroupRows, tm, tn);
                    for (int kb = kb0; kb < kb1; ++kb) {
                        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, status)) {
                            ok = false;
                            break;
                        }
                        uint8_t *st = smem + stage * L::kStage;
                        mbar_arrive_expect_tx(&full[stage], L::kStage);
                        tma_load_2d(st, &tmap_a, &full[stage], kb * BK, tm * BM);
                        if constexpr (kSilu) {
                            // gate block tn above up block tn (128-row boxes)
                            tma_load_2d(st + L::kA, &tmap_b, &full[stage], kb * BK, tn * 128);
                            tma_load_2d(st + L::kA + 128 * BK, &tmap_b, &full[stage], kb * BK,
                                        I + tn * 128);
                        } else {
                            tma_load_2d(st + L::kA, &tmap_b, &full[stage], kb * BK, tn * BN);
                        }
                        ++issued;
                        if (++stage == kStages) {
                            stage = 0;
                            phase ^= 1;
                        }
                    }
                }
                // Before the CTA may exit, every load it issued must have landed.
                for (int64_t i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
                    mbar_wait(&full[i % kStages], static_cast<uint32_t>((i / kStages) & 1), nullptr,
                              status);
            }
        } else if (warp == 1 || warp == 2) {
            // ------------------------------------------------------------ MMA issuers
            // Two threads, one per TMEM buffer: chunk i (counted over all of the
            // CTA's tiles) goes to buffer i mod 2 and is issued by warp 1 + (i mod 2).
            if (lane == 0) {
                const uint32_t idesc = umma_idesc_e4m3(BM, BN);
                const uint32_t buf = static_cast<uint32_t>(warp - 1);
                int64_t i = 0;
                bool ok = true;
                int t, kb0, kb1, part;
                for (int w = 0; ok && work_item(w, num_tiles, full_tiles, tail_parts, KB, t, kb0, kb1, part);
                     ++w) {
                    for (int kb = kb0; kb < kb1; ++kb, ++i) {
                        if ((i & 1) != buf) continue;
                        const uint32_t stage = static_cast<uint32_t>(i % kStages);
                        const uint32_t phase = static_cast<uint32_t>((i / kStages) & 1);
                        const uint32_t bphase = static_cast<uint32_t>((i >> 1) & 1);
                        if (!mbar_wait(&tempty[buf], bphase ^ 1, abort_flag, status) ||
                            !mbar_wait(&full[stage], phase, abort_flag, status)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after_sync();
                        const uint32_t a_addr = smem_addr(smem + stage * L::kStage);
                        const uint32_t b_addr = a_addr + L::kA;
                        const uint32_t d_tmem = tmem_base + buf * BN;
#pragma unroll
                        for (int j = 0; j < BK / 32; ++j)
                            umma_e4m3(d_tmem, umma_desc_sw128(a_addr + 32 * j),
                                      umma_desc_sw128(b_addr + 32 * j), idesc, j > 0 ? 1u : 0u);
                        umma_commit(&empty[stage]);
                        umma_commit(&tfull[buf]);
                    }
                }
                // Wait for every MMA either thread issued before TMEM is released.
                umma_commit(drain);
                mbar_wait(drain, 0, nullptr, status);
            }
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kConsumerRegs));
        // ------------------------------------------------------------ promotion + epilogue
        const int pw = warp - kFirstPromoWarp;
        const int quarter = warp & 3;  // TMEM lane quarter accessible to this warp
        const int half = pw >> 2;      // which 128-column weight block of the tile
        const int row_in_tile = quarter * 32 + lane;
        const int pt = threadIdx.x - kFirstPromoWarp * 32;  // 0..255
        // tail part hand-shake: arrivals of the promotion warps, then the verdict
        volatile uint32_t *tail_last = reinterpret_cast<volatile uint32_t *>(smem + L::kMiscOff + 8);
        uint32_t *tail_arrived = reinterpret_cast<uint32_t *>(smem + L::kMiscOff + 12);
        uint32_t buf = 0, bphase = 0;
        bool ok = true;
        int t, kb0, kb1, part;
        for (int w = 0; ok && work_item(w, num_tiles, full_tiles, tail_parts, KB, t, kb0, kb1, part);
             ++w) {
            int tm, tn;
            tile_coords(t, m_tiles, n_tiles, kGroupRows, tm, tn);
            const int grow = tm * BM + row_in_tile;
            // plain: this thread's 128 output columns, one weight block; SiLU:
            // 64 gate and the same 64 up channels, two weight blocks
            const int gcol = kSilu ? tn * 128 + half * 64 : tn * BN + half * 128;
            const bool row_ok = grow < M;
            const bool col_ok = gcol < N;
            const float *sa_row = sa + static_cast<int64_t>(row_ok ? grow : 0) * KB;
            const float *sw_row =
                sw + static_cast<int64_t>(kSilu ? tn : (col_ok ? gcol / 128 : 0)) * KB;
            const float *swu_row = sw + static_cast<int64_t>(I / 128 + tn) * KB;  // kSilu: up block

            float acc[128];
#pragma unroll
            for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
            // scales of the next kScaleLookahead chunks, in a register ring
            float sa_q[kScaleLookahead], sw_q[kScaleLookahead], swu_q[kScaleLookahead];
#pragma unroll
            for (int j = 0; j < kScaleLookahead; ++j) {
                sa_q[j] = (row_ok && kb0 + j < kb1) ? __ldg(sa_row + kb0 + j) : 0.0f;
                sw_q[j] = (col_ok && kb0 + j < kb1) ? __ldg(sw_row + kb0 + j) : 0.0f;
                if constexpr (kSilu) swu_q[j] = kb0 + j < kb1 ? __ldg(swu_row + kb0 + j) : 0.0f;
            }
            for (int kbb = kb0; kbb < kb1 && ok; kbb += kScaleLookahead) {
#pragma unroll
                for (int j = 0; j < kScaleLookahead; ++j) {
                    const int kb = kbb + j;
                    if (kb >= kb1) break;
                    const float sa_v = sa_q[j];
                    const float scale = sa_v * sw_q[j];
                    const float scale1 = kSilu ? sa_v * swu_q[j] : scale;
                    const int kn = kb + kScaleLookahead;
                    if (kn < kb1) {
                        sa_q[j] = row_ok ? __ldg(sa_row + kn) : 0.0f;
                        sw_q[j] = col_ok ? __ldg(sw_row + kn) : 0.0f;
                        if constexpr (kSilu) swu_q[j] = __ldg(swu_row + kn);
                    }
                    if (!mbar_wait(&tfull[buf], bphase, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                           buf * BN;
                    const uint32_t taddr0 = tbase + (kSilu ? half * 64 : half * 128);
                    const uint32_t taddr1 = kSilu ? tbase + 128 + half * 64 : taddr0 + 64;
                    float last[64];
                    promote_chunk(taddr0, taddr1, scale, scale1, acc, last);
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tempty[buf]);
#pragma unroll
                    for (int i = 0; i < 64; ++i) acc[64 + i] = fmaf(last[i], scale1, acc[64 + i]);
                    buf ^= 1;
                    if (buf == 0) bphase ^= 1;
                }
            }
            if (!ok) break;
            if constexpr (kSilu) {
                // h = BF16(silu(g) * u) with g, u the BF16-rounded accumulators
                // (what the plain GEMM would store), by the standalone SiLU
                // kernel's arithmetic; then one activation group of 128
                // channels per row, split over the two column halves, whose
                // maxima meet in shared memory.
                uint32_t hb[32];
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    const uint4 gv = make_uint4(pack_bf16x2(acc[8 * v + 0], acc[8 * v + 1]),
                                                pack_bf16x2(acc[8 * v + 2], acc[8 * v + 3]),
                                                pack_bf16x2(acc[8 * v + 4], acc[8 * v + 5]),
                                                pack_bf16x2(acc[8 * v + 6], acc[8 * v + 7]));
                    const uint4 uv = make_uint4(pack_bf16x2(acc[64 + 8 * v + 0], acc[64 + 8 * v + 1]),
                                                pack_bf16x2(acc[64 + 8 * v + 2], acc[64 + 8 * v + 3]),
                                                pack_bf16x2(acc[64 + 8 * v + 4], acc[64 + 8 * v + 5]),
                                                pack_bf16x2(acc[64 + 8 * v + 6], acc[64 + 8 * v + 7]));
                    const uint4 h8 = silu_mul8(gv, uv);
                    hb[4 * v + 0] = h8.x;
                    hb[4 * v + 1] = h8.y;
                    hb[4 * v + 2] = h8.z;
                    hb[4 * v + 3] = h8.w;
                }
                uint32_t amax = 0;
#pragma unroll
                for (int v = 0; v < 8; ++v)
                    amax = max(amax, amax_bits8(make_uint4(hb[4 * v], hb[4 * v + 1], hb[4 * v + 2],
                                                           hb[4 * v + 3])));
                // The partner thread (same row, other half) is in the other
                // promotion warpgroup.  Each publishes (tile index, amax) in one
                // 64-bit word and waits, bounded, for the partner's word of this
                // tile; slots alternate by tile parity, so a slot is rewritten
                // only after the partner has read it.
                volatile unsigned long long *xchg =
                    reinterpret_cast<volatile unsigned long long *>(smem + L::kXchgOff) +
                    (w & 1) * (2 * BM);
                const unsigned long long tag = static_cast<unsigned long long>(w) << 32;
                xchg[row_in_tile * 2 + half] = tag | amax;
                unsigned long long other;
                if (!smem_tag_wait(&xchg[row_in_tile * 2 + (half ^ 1)], tag, other, abort_flag,
                                   status)) {
                    ok = false;
                    break;
                }
                amax = max(amax, static_cast<uint32_t>(other));
                const float scale = scale_from_amax_bits(amax);
                if (row_ok) {
                    const int64_t c0 = static_cast<int64_t>(grow) * I + tn * 128 + half * 64;
                    uint4 *qd = reinterpret_cast<uint4 *>(silu.q + c0);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const uint2 lo = encode8(make_uint4(hb[8 * v], hb[8 * v + 1], hb[8 * v + 2],
                                                            hb[8 * v + 3]), scale);
                        const uint2 hi = encode8(make_uint4(hb[8 * v + 4], hb[8 * v + 5],
                                                            hb[8 * v + 6], hb[8 * v + 7]), scale);
                        qd[v] = make_uint4(lo.x, lo.y, hi.x, hi.y);
                    }
                    if (half == 0) silu.s[static_cast<int64_t>(grow) * (I / 128) + tn] = scale;
                    if (silu.h != nullptr) {
                        uint4 *hd = reinterpret_cast<uint4 *>(silu.h + c0);
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            hd[v] = make_uint4(hb[4 * v], hb[4 * v + 1], hb[4 * v + 2], hb[4 * v + 3]);
                    }
                }
                continue;
            }
            const bool write = part < 0;  // full tile: write its output from registers
            if (part >= 0) {
                // Tail part: publish the FP32 partial [128 rows][256 cols] of
                // this part; the part that arrives last sums them all.
                const int r = t - full_tiles;
                const int64_t unit = static_cast<int64_t>(r) * tail_parts + part;
                float4 *dst = reinterpret_cast<float4 *>(tail_partials + unit * kTailPartialFloats +
                                                         row_in_tile * 256 + half * 128);
#pragma unroll
                for (int c = 0; c < 32; ++c)
                    __stcg(dst + c, make_float4(acc[4 * c], acc[4 * c + 1], acc[4 * c + 2], acc[4 * c + 3]));
                // Every promotion warp's stores are published, then one thread
                // takes the tile's counter: 2 in *tail_last if this part is the
                // last to arrive, 1 otherwise.  (Flags in shared memory with
                // the usual bounded waits, so an abandoned wait elsewhere can
                // never leave a warp stuck here.)
                __threadfence();
                __syncwarp();
                if (lane == 0) atomicAdd(tail_arrived, 1u);
                if (pt == 0) {
                    if (smem_flag_wait(tail_arrived, static_cast<uint32_t>(kPromoWarps), abort_flag, status)) {
                        __threadfence();  // the CTA's partial stores before the counter increment
                        *tail_last = atomicAdd(&tail_counters[r], 1) == tail_parts - 1 ? 2u : 1u;
                    }
                }
                if (!smem_flag_wait(tail_last, 1u, abort_flag, status)) break;
                if (*tail_last == 2u && row_ok && col_ok) {
                    // Last part: sum every part's partial (this one's included,
                    // re-read from L2) in part order and write the tile's BF16
                    // output, four columns at a time.
                    __threadfence();
                    const float4 *base = reinterpret_cast<const float4 *>(
                        tail_partials + static_cast<int64_t>(r) * tail_parts * kTailPartialFloats +
                        row_in_tile * 256 + half * 128);
                    uint2 *yrow = reinterpret_cast<uint2 *>(y + static_cast<int64_t>(grow) * N + gcol);
                    // (eight column groups at a time, so their loads overlap)
#pragma unroll 8
                    for (int c = 0; c < 32; ++c) {
                        float4 s4 = __ldcg(base + c);
#pragma unroll
                        for (int pp = 1; pp < kTailMaxParts; ++pp) {
                            if (pp >= tail_parts) break;
                            const float4 v = __ldcg(base + pp * (kTailPartialFloats / 4) + c);
                            s4.x += v.x;
                            s4.y += v.y;
                            s4.z += v.z;
                            s4.w += v.w;
                        }
                        yrow[c] = make_uint2(pack_bf16x2(s4.x, s4.y), pack_bf16x2(s4.z, s4.w));
                    }
                }
                if (*tail_last == 2u && pt == 0) tail_counters[r] = 0;  // zeroed for the next call
            }
            if (write && row_ok && col_ok) {
                uint4 *dst = reinterpret_cast<uint4 *>(y + static_cast<int64_t>(grow) * N + gcol);
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    uint4 pk;
                    pk.x = pack_bf16x2(acc[8 * c + 0], acc[8 * c + 1]);
                    pk.y = pack_bf16x2(acc[8 * c + 2], acc[8 * c + 3]);
                    pk.z = pack_bf16x2(acc[8 * c + 4], acc[8 * c + 5]);
                    pk.w = pack_bf16x2(acc[8 * c + 6], acc[8 * c + 7]);
                    dst[c] = pk;
                }
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, L::kTmemCols);
    }
}

}  // namespace prefill
}  // namespace fp8bq
