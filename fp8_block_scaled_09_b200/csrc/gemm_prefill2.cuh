// gemm_prefill2.cuh -- the prefill GEMM on CTA pairs (tcgen05 cta_group::2).
//
// Same result as gemm_prefill.cuh (page "ProCreations/Nanbeige4.3-33B-FP8",
// introduction: W8A8 FP8 linear layers, 128x128 weight blocks, per-token
// group-128 activation scales), with one 256 x 256 output tile per pair of
// CTAs (a cluster of two SMs).  Each CTA loads its own 128 rows of A and one
// half (128 rows) of the tile's 256 weight rows; one pair MMA
// (M = 256, N = 256, K = 32) reads both CTAs' shared memory and leaves each
// CTA's 128 x 256 FP32 partial in its own TMEM.  Per output element this
// moves 2/3 of the operand bytes the single-CTA 128 x 256 tile moves from L2
// into shared memory.
//
// Roles per CTA (384 threads, the same register split as the single-CTA
// kernel: launch 168, warpgroup 0 -> 40, warpgroups 1-2 -> 232):
//   warp 0      TMA producer (both CTAs): its A and B halves of each K chunk;
//               the bytes complete on the even CTA's `full` barrier, which the
//               even CTA's producer arms for both CTAs' bytes.
//   warps 1, 2  even CTA: MMA issuers, one per TMEM buffer (chunk i into buffer
//               i mod 2 by warp 1 + (i mod 2), 4 pair MMAs per chunk), commits
//               multicast to both CTAs' `empty` and `tfull` barriers.  Odd CTA:
//               warp 1 allocates TMEM.
//   warps 4-11  promotion + epilogue of the CTA's own 128 rows, exactly as in
//               the single-CTA kernel; they release a TMEM buffer by arriving
//               on the even CTA's `tempty` barrier (16 arrivals: 8 warps x 2),
//               the odd CTA's warps with a relaxed remote arrive.
// Measured equal to the single-CTA kernel (QKV 8192x9216x7168: 543 us on the
// same GPU, 1.99 PFLOP/s) and not faster under the power cap; it is built and
// off (see fp8bq.cu).
#pragma once

#include "gemm_prefill.cuh"

namespace fp8bq {
namespace prefill2 {

using prefill::kConsumerRegs;
using prefill::kFirstPromoWarp;
using prefill::kLaunchRegs;
using prefill::kNumThreads;
using prefill::kProducerRegs;
using prefill::kScaleLookahead;
using prefill::pack_bf16x2;
using prefill::promote_chunk;

constexpr int BM = 256;       // rows per pair tile (128 per CTA)
constexpr int BN = 256;       // columns per tile (128 weight rows loaded per CTA)
constexpr int BK = 128;       // one scale chunk of K per stage
constexpr int kHalf = 128;
constexpr int kStages = 6;
constexpr int kPromoWarps = 8;
constexpr int kGroupM = 8;    // pair m-tiles per raster group

struct Layout {
    static constexpr int kA = kHalf * BK;  // this CTA's 128 A rows
    static constexpr int kB = kHalf * BK;  // this CTA's 128 weight rows
    static constexpr int kStage = kA + kB;
    static constexpr int kBarOff = kStages * kStage;
    static constexpr int kNumBars = 2 * kStages + 2 + 2 + 1;  // full, empty, tfull, tempty, drain
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kBytes = kMiscOff + 16;
    static constexpr int kDynamicSmem = kBytes + 1024;
    static constexpr uint32_t kTmemCols = 2 * BN;
};

__device__ __forceinline__ void tile_coords(int t, int m_tiles, int n_tiles, int &tm, int &tn) {
    const int group = kGroupM * n_tiles;
    const int g = t / group, r = t - g * group;
    const int first_m = g * kGroupM;
    const int gm = min(kGroupM, m_tiles - first_m);
    tm = first_m + r % gm;
    tn = r / gm;
}

__global__ void __launch_bounds__(kNumThreads, 1)
gemm_prefill_pair_kernel(const __grid_constant__ CUtensorMap tmap_a,
                         const __grid_constant__ CUtensorMap tmap_b,
                         const float *__restrict__ sa, const float *__restrict__ sw,
                         __nv_bfloat16 *__restrict__ y, int M, int N, int K, int *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Layout::kBarOff);
    uint64_t *empty = full + kStages;
    uint64_t *tfull = empty + kStages;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Layout::kMiscOff);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Layout::kMiscOff + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_cta_rank();  // 0: issues the pair MMAs
    const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
    const int KB = K / BK;
    const int m_tiles = (M + BM - 1) / BM;
    const int n_tiles = (N + BN - 1) / BN;
    const int num_tiles = m_tiles * n_tiles;

    allow_dependent_launch();
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 2 * kPromoWarps);
        }
        mbar_init(drain, 2);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_b);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, Layout::kTmemCols);
        tmem_relinquish_pair();
    }
    // Both CTAs' barriers exist and TMEM is allocated before either CTA
    // signals the other.
    tc_fence_before_sync();
    cluster_sync();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    grid_dependency_wait();

    if (warp < kFirstPromoWarp) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
        if (warp == 0) {
            // ------------------------------------------------------------ TMA producer
            if (lane == 0) {
                uint32_t stage = 0, phase = 0;
                int64_t issued = 0;
                bool ok = true;
                for (int t = pair; t < num_tiles && ok; t += num_pairs) {
                    int tm, tn;
                    tile_coords(t, m_tiles, n_tiles, tm, tn);
                    for (int kb = 0; kb < KB; ++kb) {
                        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, status)) {
                            ok = false;
                            break;
                        }
                        uint8_t *st = smem + stage * Layout::kStage;
                        const uint32_t full0 = map_to_cta(smem_addr(&full[stage]), 0);
                        if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * Layout::kStage);
                        tma_load_2d_pair(st, &tmap_a, full0, kb * BK, tm * BM + rank * kHalf);
                        tma_load_2d_pair(st + Layout::kA, &tmap_b, full0, kb * BK,
                                         tn * BN + rank * kHalf);
                        ++issued;
                        if (++stage == kStages) {
                            stage = 0;
                            phase ^= 1;
                        }
                    }
                }
                // A stage's loads have landed once the MMA that read it finished,
                // which its `empty` barrier records in both CTAs.
                for (int64_t i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
                    mbar_wait(&empty[i % kStages], static_cast<uint32_t>((i / kStages) & 1),
                              nullptr, status);
            }
        } else if ((warp == 1 || warp == 2) && rank == 0) {
            // ------------------------------------------------------------ pair MMA issuers
            if (lane == 0) {
                const uint32_t idesc = umma_idesc_e4m3(BM, BN);
                const uint32_t buf = static_cast<uint32_t>(warp - 1);
                int64_t i = 0;
                bool ok = true;
                for (int t = pair; t < num_tiles && ok; t += num_pairs) {
                    for (int kb = 0; kb < KB; ++kb, ++i) {
                        if ((i & 1) != buf) continue;
                        const uint32_t stage = static_cast<uint32_t>(i % kStages);
                        const uint32_t phase = static_cast<uint32_t>((i / kStages) & 1);
                        const uint32_t bphase = static_cast<uint32_t>((i >> 1) & 1);
                        // tempty gathers arrivals from both CTAs of the pair
                        if (!mbar_wait<true>(&tempty[buf], bphase ^ 1, abort_flag, status) ||
                            !mbar_wait(&full[stage], phase, abort_flag, status)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after_sync();
                        const uint32_t a_addr = smem_addr(smem + stage * Layout::kStage);
                        const uint32_t b_addr = a_addr + Layout::kA;
                        const uint32_t d_tmem = tmem_base + buf * BN;
#pragma unroll
                        for (int j = 0; j < BK / 32; ++j)
                            umma_e4m3_pair(d_tmem, umma_desc_sw128(a_addr + 32 * j),
                                           umma_desc_sw128(b_addr + 32 * j), idesc, j > 0 ? 1u : 0u);
                        umma_commit_pair_multicast(&empty[stage], 0x3);
                        umma_commit_pair_multicast(&tfull[buf], 0x3);
                    }
                }
                // every pair MMA either thread issued has finished before TMEM is released
                umma_commit_pair_multicast(drain, 0x1);
                mbar_wait(drain, 0, nullptr, status);
            }
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kConsumerRegs));
        // ------------------------------------------------------------ promotion + epilogue
        const int pw = warp - kFirstPromoWarp;
        const int quarter = warp & 3;
        const int half = pw >> 2;
        const int row_in_tile = quarter * 32 + lane;
        const uint32_t tempty0_b0 = map_to_cta(smem_addr(&tempty[0]), 0);
        const uint32_t tempty0_b1 = map_to_cta(smem_addr(&tempty[1]), 0);
        uint32_t buf = 0, bphase = 0;
        bool ok = true;
        for (int t = pair; t < num_tiles && ok; t += num_pairs) {
            int tm, tn;
            tile_coords(t, m_tiles, n_tiles, tm, tn);
            const int grow = tm * BM + static_cast<int>(rank) * kHalf + row_in_tile;
            const int gcol = tn * BN + half * 128;
            const bool row_ok = grow < M;
            const bool col_ok = gcol < N;
            const float *sa_row = sa + static_cast<int64_t>(row_ok ? grow : 0) * KB;
            const float *sw_row = sw + static_cast<int64_t>(col_ok ? gcol / 128 : 0) * KB;

            float acc[128];
#pragma unroll
            for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
            float sa_q[kScaleLookahead], sw_q[kScaleLookahead];
#pragma unroll
            for (int j = 0; j < kScaleLookahead; ++j) {
                sa_q[j] = (row_ok && j < KB) ? __ldg(sa_row + j) : 0.0f;
                sw_q[j] = (col_ok && j < KB) ? __ldg(sw_row + j) : 0.0f;
            }
            for (int kb0 = 0; kb0 < KB && ok; kb0 += kScaleLookahead) {
#pragma unroll
                for (int j = 0; j < kScaleLookahead; ++j) {
                    const int kb = kb0 + j;
                    if (kb >= KB) break;
                    const float scale = sa_q[j] * sw_q[j];
                    const int kn = kb + kScaleLookahead;
                    if (kn < KB) {
                        sa_q[j] = row_ok ? __ldg(sa_row + kn) : 0.0f;
                        sw_q[j] = col_ok ? __ldg(sw_row + kn) : 0.0f;
                    }
                    if (!mbar_wait(&tfull[buf], bphase, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t taddr = tmem_base +
                                           (static_cast<uint32_t>(quarter * 32) << 16) +
                                           buf * BN + half * 128;
                    float last[64];
                    promote_chunk(taddr, taddr + 64, scale, scale, acc, last);
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) {
                        if (rank == 0)
                            mbar_arrive(&tempty[buf]);
                        else
                            mbar_arrive_remote_relaxed(buf ? tempty0_b1 : tempty0_b0);
                    }
#pragma unroll
                    for (int i = 0; i < 64; ++i) acc[64 + i] = fmaf(last[i], scale, acc[64 + i]);
                    buf ^= 1;
                    if (buf == 0) bphase ^= 1;
                }
            }
            if (ok && row_ok && col_ok) {
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

    // Both CTAs are done with TMEM and the even CTA's MMAs have drained before
    // the pair's TMEM is released; neither CTA exits while the other may still
    // signal its barriers.
    tc_fence_before_sync();
    __syncthreads();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc_pair(tmem_base, Layout::kTmemCols);
    }
}

}  // namespace prefill2
}  // namespace fp8bq
