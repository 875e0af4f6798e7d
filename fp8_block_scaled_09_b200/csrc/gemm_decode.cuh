// gemm_decode.cuh -- block-scaled FP8 GEMM for small M (decode and mid-size
// batches, M <= 128), swap-AB and stream-K over the weight blocks.
//
// Same result as the prefill kernel (page "ProCreations/Nanbeige4.3-33B-FP8",
// introduction: W8A8 FP8 linear layers), shaped for the weight-bandwidth-bound
// regime: every weight byte is read from HBM exactly once, and the grid streams
// the N/128 x K/128 weight blocks (16 KB each) evenly over all SMs.
//
// Roles (224 threads; 352 with eight promotion warps):
//   warp 0      TMA producer: per unit (n-block nb, k-block kb) the 128 x 128 B
//               weight block and the MT x 128 B activation tile (rows >= M are
//               zero-filled by TMA).  Units travel in steps of kStep = 2: one
//               ring slot, one full/empty barrier pair and one TMEM group per
//               step, so the MMA thread touches shared memory (barrier waits)
//               once per two units; each such access after issued MMAs costs
//               it ~0.1 us, about the time a unit's data takes to arrive.
//   warp 1      MMA issuer: swap-AB, D[n, m] = W_blk[n, :] . X_tile[m, :] with
//               M_mma = 128 (weight rows) and N_mma = MT (the token tile: 16,
//               32, 64 or 128 rows, the smallest >= M), 4 MMAs of K = 32 per
//               unit, each unit into its own TMEM slot.
//   warps 2..   promotion (4 warps, or 8 from MT = 64): thread = one weight row
//               n of the block (its TMEM lane) and MT or MT/2 token columns,
//               one FP32 accumulator each; per unit
//               acc[m] = fma(P[n, m], sa[m, kb] * sw[nb, kb], acc[m]), scales read
//               from shared memory where they are staged once per CTA.
//   last warp   split-K: publishes this CTA's partial sums (device-wide fence and
//               counter increment), so promotion never waits on either; if the
//               CTA was an n-block's last contributor, all warps reduce it after
//               the main loop.
// Two ways to spread the units over CTAs, chosen per launch:
// Cluster split (cluster_s >= 1, when N/128 <= the SM count): CTA c works on
// n-block c / S, k-blocks [r KB / S, (r+1) KB / S) with r = c mod S, and the S
// CTAs of an n-block form a thread-block cluster.  At the end each stores its
// partial in its own shared memory; after a cluster barrier CTA r sums slice r
// of the n-block's output over the S partials (in rank order, read through
// distributed shared memory), writes it in BF16, and a second barrier keeps the
// partials alive until every peer has read them.  No global workspace is used.
// Stream-K (cluster_s == 0): units u = nb * KB + kb are split into gridDim.x
// contiguous ranges.
// An n-block whose K range lies inside one CTA is written straight to Y in
// BF16.  Otherwise each contributing CTA c stores its FP32 partial in slot
// nb + c of the workspace and increments counter[nb]; the last to arrive sums
// the slots in increasing c (a fixed order, so results are deterministic),
// writes BF16 and resets the counter to zero for the next call.  A CTA has at
// most two such split n-blocks: the first and the last of its range.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "ptx.cuh"

namespace fp8bq {
namespace decode {

constexpr int BNW = 128;  // weight rows per unit (one scale block)
// Suspend hint of this kernel's barrier waits (see mbar_wait).
constexpr uint32_t kDecodeSuspendNs = 10000;
constexpr int BK = 128;
constexpr int kMaxMT = 128;
constexpr int kMaxGrid = 256;  // workspace is sized for at most this many CTAs

// Warp roles for a token tile of MT rows: 4 promotion warps (one per TMEM lane
// quarter) up to MT = 32, 8 from MT = 64 on (two per quarter, each owning half
// of the token columns, so two warps per scheduler hide each other's TMEM and
// shared-memory latency and each holds MT/2 accumulators).
template <int MT>
struct Roles {
    static constexpr int kPromoWarps = MT >= 64 ? 8 : 4;
    static constexpr int kPromoThreads = 32 * kPromoWarps;
    static constexpr int kCols = MT * 4 / kPromoWarps;  // token columns per promotion thread
    static constexpr int kSplitWarp = 2 + kPromoWarps;
    static constexpr int kNumThreads = 32 * (kSplitWarp + 1);  // 224 or 352
};

// Smallest supported token tile holding M rows.
__host__ __device__ constexpr int token_tile(int64_t M) {
    return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128;
}

// Units per ring slot / barrier / TMEM group, by token tile.
__host__ __device__ constexpr int step_units_of(int /*MT*/) { return 2; }
constexpr int kMaxRingUnits = 8;    // ring slots x units per slot, at most (measured: 8 beats 4, 6 ~ 8, 10 and 12 lose 2-4% on the decode step)
constexpr int kMinStages = 2;
constexpr int kMaxSmem = 227 * 1024;

// Shared memory: `stages` ring slots of kStep (weight block, activation tile), then
// the barriers, a few words of CTA state, the activation scales [KB][MT + 4]
// (transposed, so one thread reads four tokens' scales at once; the 4 extra
// words per row make the transposing stores bank-conflict free) and the
// weight scales of the CTA's unit range.  The stage count is chosen per launch
// from what the scales leave of the 227 KB.
template <int MT>
struct Layout {
    static_assert(MT == 16 || MT == 32 || MT == 64 || MT == 128, "token tile");
    static constexpr int kStep = step_units_of(MT);
    static constexpr int kMaxStages = kMaxRingUnits / kStep;
    static constexpr int kTmemSlots = (512 / MT) < 8 ? (512 / MT) : 8;  // one unit each
    static constexpr int kGroups = kTmemSlots / kStep;                   // one step each
    static_assert(kGroups * kStep == kTmemSlots, "TMEM slots per group");
    static constexpr uint32_t kTmemCols = static_cast<uint32_t>(kTmemSlots * MT);  // 128..512
    static constexpr int kW = BNW * BK;  // 16 KB
    static constexpr int kX = MT * BK;   // 2-16 KB
    static constexpr int kUnit = kW + kX;
    static constexpr int kStage = kStep * kUnit;
    static constexpr int kSaRow = MT + 4;  // floats per staged activation-scale row
    __host__ __device__ static constexpr int bar_off(int stages) { return stages * kStage; }
    // full, empty (per stage), tfull, tempty (per TMEM group), drain, 2 split-K flushes
    __host__ __device__ static constexpr int misc_off(int stages) {
        return bar_off(stages) + (2 * stages + 2 * kGroups + 3) * 8;
    }
    __host__ __device__ static constexpr int scale_off(int stages) {
        return (misc_off(stages) + 16 + 15) & ~15;  // float4 reads of the scales
    }
};

// Rows of the staged activation-scale table: one per K block the CTA's unit
// range touches, i.e. min(KB, units); the range's K blocks form one cyclic
// interval starting at u_begin mod KB.
__host__ __device__ inline int64_t scale_rows(int64_t KB, int64_t units_per_cta_max) {
    return units_per_cta_max < KB ? units_per_cta_max : KB;
}

// Dynamic shared memory for a launch (1 KB of it for the alignment of the ring).
template <int MT>
__host__ __device__ inline int64_t smem_bytes(int stages, int64_t KB, int64_t units_per_cta_max) {
    return Layout<MT>::scale_off(stages) + Layout<MT>::kSaRow * scale_rows(KB, units_per_cta_max) * 4 +
           (units_per_cta_max + 1) * 4 + 1024;
}

// Bytes of one ring slot for a token tile.
__host__ __device__ constexpr int64_t kStageBytes(int MT) {
    return step_units_of(MT) * (int64_t(BNW) * BK + int64_t(MT) * BK);
}

// Most ring stages (<= kMaxStages) that fit, or 0 when fewer than kMinStages do.
template <int MT>
__host__ __device__ inline int pick_stages(int64_t KB, int64_t units_per_cta_max) {
    for (int s = Layout<MT>::kMaxStages; s >= kMinStages; --s)
        if (smem_bytes<MT>(s, KB, units_per_cta_max) <= kMaxSmem) return s;
    return 0;
}

// Workspace: a fixed header of kMaxCounters int32 split-K counters, then float
// partials [NB + kMaxGrid][MT][128].  The header has the same size for every
// shape, so partial sums never land on counters a later call (of any shape)
// expects to be zero: every successful call leaves the whole header zeroed.
constexpr int64_t kMaxCounters = 4096;  // n-blocks, i.e. N <= 524288 on this path
constexpr int64_t kCounterBytes = kMaxCounters * 4;
__host__ __device__ inline int64_t workspace_bytes(int64_t NB, int64_t MT) {
    return kCounterBytes + (NB + kMaxGrid) * MT * BNW * 4;
}

// CTA whose unit range [floor(c U / G), floor((c+1) U / G)) contains unit u.
__device__ __forceinline__ int cta_of_unit(int64_t u, int64_t U, int64_t G) {
    return static_cast<int>(((u + 1) * G - 1) / U);
}

// The split n-blocks of one CTA's unit range (at most two, in order): those
// whose K range the CTA covers only in part.
struct SplitPlan {
    int count = 0;
    int nb[2] = {0, 0};
};

__device__ __forceinline__ SplitPlan split_plan(int64_t u_begin, int64_t u_end, int KB) {
    SplitPlan p;
    if (u_end <= u_begin) return p;
    const int first_nb = static_cast<int>(u_begin / KB);
    const int last_nb = static_cast<int>((u_end - 1) / KB);
    const bool first_split = (u_begin % KB != 0) || (first_nb == last_nb && u_end % KB != 0);
    if (first_split) p.nb[p.count++] = first_nb;
    if (last_nb != first_nb && u_end % KB != 0) p.nb[p.count++] = last_nb;
    return p;
}

template <int MT>
__global__ void __launch_bounds__(Roles<MT>::kNumThreads, 1)
gemm_decode_kernel(const __grid_constant__ CUtensorMap tmap_w,
                   const __grid_constant__ CUtensorMap tmap_x, const float *__restrict__ sa,
                   const float *__restrict__ sw, __nv_bfloat16 *__restrict__ y, int M, int N,
                   int K, int *counters, float *partials, int *status, int early_weights,
                   int stages, int cluster_s) {
    using Layout = decode::Layout<MT>;
    const int kStages = stages;
    constexpr int kStep = Layout::kStep;
    constexpr int kGroups = Layout::kGroups;
    constexpr uint32_t kTmemCols = Layout::kTmemCols;
    constexpr int kPromoWarps = Roles<MT>::kPromoWarps;
    constexpr int kPromoThreads = Roles<MT>::kPromoThreads;
    constexpr int kCols = Roles<MT>::kCols;
    constexpr int kSplitWarp = Roles<MT>::kSplitWarp;
    constexpr int kNumThreads = Roles<MT>::kNumThreads;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Layout::bar_off(kStages));
    uint64_t *empty = full + kStages;
    uint64_t *tfull = empty + kStages;
    uint64_t *tempty = tfull + kGroups;
    uint64_t *drain = tempty + kGroups;
    uint64_t *flushed = drain + 1;  // [2]: promotion -> split-K warp, one per split n-block
    uint8_t *misc = smem + Layout::misc_off(kStages);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 4);
    float *sa_s = reinterpret_cast<float *>(smem + Layout::scale_off(kStages));  // [KB][kSaRow]
    // n-blocks this CTA must reduce (it was their last contributor), or -1
    volatile int *reduce_nb = reinterpret_cast<volatile int *>(misc + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = K / BK, NB = N / BNW;
    const int64_t U = static_cast<int64_t>(NB) * KB;
    const int64_t G = gridDim.x;
    int64_t u_begin, u_end;
    if (cluster_s > 0) {
        const int64_t nb = blockIdx.x / cluster_s, r = blockIdx.x % cluster_s;
        u_begin = nb * KB + r * KB / cluster_s;
        u_end = nb * KB + (r + 1) * KB / cluster_s;
    } else {
        u_begin = blockIdx.x * U / G;
        u_end = (blockIdx.x + 1) * U / G;
    }
    const int64_t n_steps = (u_end - u_begin + kStep - 1) / kStep;
    constexpr int kSaRow = Layout::kSaRow;
    // staged activation scales: row r holds K block (kb_first + r) mod KB
    const int kb_first = static_cast<int>(u_begin % KB);
    const int sa_rows = static_cast<int>(scale_rows(KB, u_end - u_begin));
    float *sw_s = sa_s + kSaRow * sa_rows;  // sw[u] for u in [u_begin, u_end): sw is [NB, KB] row-major

    allow_dependent_launch();
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < kGroups; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], kPromoWarps);
        }
        mbar_init(drain, 1);
        mbar_init(&flushed[0], kPromoWarps);
        mbar_init(&flushed[1], kPromoWarps);
        *abort_flag = 0;
        reduce_nb[0] = -1;
        reduce_nb[1] = -1;
        fence_barrier_init();
        prefetch_tmap(&tmap_w);
        prefetch_tmap(&tmap_x);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    // Everything above overlaps the previous kernel in the stream.  With
    // early_weights the first kStages weight blocks are requested too: only
    // the linear layer sets it, when the previous kernel is its own activation
    // quantizer, which writes activation codes and scales only.  No kernel of
    // this library that writes weights lets its successor start before it
    // completes, so every such kernel earlier in the stream has completed by
    // the time this one starts.  Every other global access happens after the
    // previous kernel has completed.
    // Units of step i: [u_begin + kStep i, min(u_end, u_begin + kStep (i + 1))).
    auto step_units = [&](int64_t i) {
        const int64_t left = u_end - (u_begin + kStep * i);
        return static_cast<int>(left < kStep ? left : kStep);
    };
    int64_t n_early = 0;
    if (early_weights && warp == 0 && lane == 0) {
        const uint64_t evict_first = l2_policy_evict_first();
        for (; n_early < n_steps && n_early < kStages; ++n_early) {
            const int cnt = step_units(n_early);
            mbar_arrive_expect_tx(&full[n_early], cnt * Layout::kUnit);
            for (int j = 0; j < cnt; ++j) {
                const int64_t u = u_begin + kStep * n_early + j;
                tma_load_2d_hint(smem + n_early * Layout::kStage + j * Layout::kUnit, &tmap_w,
                                 &full[n_early], static_cast<int>(u % KB) * BK,
                                 static_cast<int>(u / KB) * BNW, evict_first);
            }
        }
    }
    grid_dependency_wait();

    if (warp == 0) {
        if (lane == 0) {
            // activation tiles of the steps whose weight blocks went out early
            for (int64_t i = 0; i < n_early; ++i)
                for (int j = 0; j < step_units(i); ++j)
                    tma_load_2d(smem + i * Layout::kStage + j * Layout::kUnit + Layout::kW, &tmap_x,
                                &full[i], static_cast<int>((u_begin + kStep * i + j) % KB) * BK, 0);
            const uint64_t evict_first = l2_policy_evict_first();
            uint32_t stage = static_cast<uint32_t>(n_early % kStages);
            uint32_t phase = n_early == kStages ? 1u : 0u;
            int64_t issued = n_early;
            for (int64_t i = n_early; i < n_steps; ++i) {
                if (!mbar_wait<false, kDecodeSuspendNs>(&empty[stage], phase ^ 1, abort_flag, status)) break;
                const int cnt = step_units(i);
                uint8_t *st = smem + stage * Layout::kStage;
                mbar_arrive_expect_tx(&full[stage], cnt * Layout::kUnit);
                for (int j = 0; j < cnt; ++j) {
                    const int64_t u = u_begin + kStep * i + j;
                    const int nb = static_cast<int>(u / KB), kb = static_cast<int>(u % KB);
                    tma_load_2d_hint(st + j * Layout::kUnit, &tmap_w, &full[stage], kb * BK, nb * BNW,
                                     evict_first);
                    tma_load_2d(st + j * Layout::kUnit + Layout::kW, &tmap_x, &full[stage], kb * BK, 0);
                }
                ++issued;
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            for (int64_t i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
                mbar_wait<false, kDecodeSuspendNs>(&full[i % kStages], static_cast<uint32_t>((i / kStages) & 1), nullptr,
                          status);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = umma_idesc_e4m3(BNW, MT);
            uint32_t stage = 0, phase = 0, grp = 0, gphase = 0;
            for (int64_t i = 0; i < n_steps; ++i) {
                if (!mbar_wait<false, kDecodeSuspendNs>(&tempty[grp], gphase ^ 1, abort_flag, status) ||
                    !mbar_wait<false, kDecodeSuspendNs>(&full[stage], phase, abort_flag, status))
                    break;
                tc_fence_after_sync();
                const int cnt = step_units(i);
                for (int j = 0; j < cnt; ++j) {
                    const uint32_t w_addr = smem_addr(smem + stage * Layout::kStage + j * Layout::kUnit);
                    const uint32_t x_addr = w_addr + Layout::kW;
                    const uint32_t d_tmem = tmem_base + (grp * kStep + j) * MT;
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k)
                        umma_e4m3(d_tmem, umma_desc_sw128(w_addr + 32 * k),
                                  umma_desc_sw128(x_addr + 32 * k), idesc, k > 0 ? 1u : 0u);
                }
                umma_commit(&empty[stage]);
                umma_commit(&tfull[grp]);
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1;
                }
                if (++grp == kGroups) {
                    grp = 0;
                    gphase ^= 1;
                }
            }
            umma_commit(drain);
            mbar_wait<false, kDecodeSuspendNs>(drain, 0, nullptr, status);
        }
    } else if (warp < kSplitWarp) {
        const int quarter = warp & 3;                 // TMEM lane quarter this warp may access
        const int col0 = ((warp - 2) >> 2) * kCols;   // first token column of this thread
        const int n_local = quarter * 32 + lane;      // weight row within the block = TMEM lane
        const int ptid = threadIdx.x - 64;            // 0 .. kPromoThreads-1
        // Stage the scales once: every activation scale (rows past M as 0,
        // transposed to [KB][kSaRow]) and the weight scales of this CTA's
        // units, so the per-unit promotion reads shared memory only.  4-byte
        // async copies keep all of them in flight at once.  A warp copies a
        // tile of 8 k-blocks x 4 tokens: four 32-byte global segments, and 32
        // distinct shared-memory banks since kSaRow is 4 times an odd number.
        const int kb_tiles = (sa_rows + 7) / 8;
        for (int t = ptid >> 5; t < kb_tiles * (MT / 4); t += kPromoWarps) {
            const int r = (t % kb_tiles) * 8 + (lane & 7);
            const int m = (t / kb_tiles) * 4 + (lane >> 3);
            if (r < sa_rows) {
                const int kb = kb_first + r < KB ? kb_first + r : kb_first + r - KB;
                float *dst = sa_s + r * kSaRow + m;
                if (m < M)
                    cp_async_4(dst, sa + static_cast<int64_t>(m) * KB + kb);
                else
                    *dst = 0.0f;
            }
        }
        const int n_units = static_cast<int>(u_end - u_begin);
        for (int i = ptid; i < n_units; i += kPromoThreads) cp_async_4(sw_s + i, sw + u_begin + i);
        cp_async_wait_all();
        named_barrier(1, kPromoThreads);

        uint32_t grp = 0, gphase = 0;
        float acc[kCols];
#pragma unroll
        for (int m = 0; m < kCols; ++m) acc[m] = 0.0f;
        int seg_kb0 = static_cast<int>(u_begin % KB);
        int split_idx = 0;
        for (int64_t u = u_begin; u < u_end; ++u) {
            const int nb = static_cast<int>(u / KB), kb = static_cast<int>(u % KB);
            const float swv = sw_s[u - u_begin];
            const int j = static_cast<int>((u - u_begin) % kStep);  // unit within its step
            const bool last_of_step = j == kStep - 1 || u == u_end - 1;
            if (j == 0) {
                if (!mbar_wait<false, kDecodeSuspendNs>(&tfull[grp], gphase, abort_flag, status)) break;
                tc_fence_after_sync();
            }
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   (grp * kStep + j) * MT + col0;
            float v[kCols];
            if constexpr (kCols == 16)
                tmem_load16(taddr, v);
            else if constexpr (kCols == 32)
                tmem_load32(taddr, v);
            else
                tmem_load64(taddr, v);
            if (last_of_step) {
                // all of this thread's TMEM columns of the step are in registers
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[grp]);
                if (++grp == kGroups) {
                    grp = 0;
                    gphase ^= 1;
                }
            }
            const int sa_r = kb >= kb_first ? kb - kb_first : kb - kb_first + KB;
            const float4 *sa4 = reinterpret_cast<const float4 *>(sa_s + sa_r * kSaRow + col0);
#pragma unroll
            for (int i = 0; i < kCols / 4; ++i) {
                const float4 a = sa4[i];
                acc[4 * i + 0] = fmaf(v[4 * i + 0], a.x * swv, acc[4 * i + 0]);
                acc[4 * i + 1] = fmaf(v[4 * i + 1], a.y * swv, acc[4 * i + 1]);
                acc[4 * i + 2] = fmaf(v[4 * i + 2], a.z * swv, acc[4 * i + 2]);
                acc[4 * i + 3] = fmaf(v[4 * i + 3], a.w * swv, acc[4 * i + 3]);
            }

            if (kb == KB - 1 || u == u_end - 1) {
                // end of this CTA's segment of n-block nb
                const int col = nb * BNW + n_local;
                if (seg_kb0 == 0 && kb == KB - 1) {
#pragma unroll
                    for (int m = 0; m < kCols; ++m)
                        if (col0 + m < M)
                            y[static_cast<int64_t>(col0 + m) * N + col] = __float2bfloat16_rn(acc[m]);
                } else if (cluster_s > 0) {
                    // the CTA's whole range is this one segment, and every MMA
                    // that read the ring has completed: the ring holds the
                    // partial [MT][128] for the cluster reduction
                    float *red = reinterpret_cast<float *>(smem);
#pragma unroll
                    for (int m = 0; m < kCols; ++m) red[(col0 + m) * BNW + n_local] = acc[m];
                } else {
                    // hand the partial to the split-K warp
                    float *slot = partials + (static_cast<int64_t>(nb) + blockIdx.x) * (MT * BNW);
#pragma unroll
                    for (int m = 0; m < kCols; ++m)
                        __stcg(slot + (col0 + m) * BNW + n_local, acc[m]);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&flushed[split_idx]);
                    ++split_idx;
                }
#pragma unroll
                for (int m = 0; m < kCols; ++m) acc[m] = 0.0f;
                seg_kb0 = 0;
            }
        }
    } else {
        // ------------------------------------------------------------ split-K warp
        // Publishes each split n-block's partial and learns whether this CTA was
        // the last contributor; the reduction itself runs after the main loop on
        // all threads of the CTA.
        const SplitPlan plan = cluster_s > 0 ? SplitPlan{} : split_plan(u_begin, u_end, KB);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            if (i >= plan.count) break;
            const int nb = plan.nb[i];
            if (!mbar_wait<false, kDecodeSuspendNs>(&flushed[i], 0, abort_flag, status)) break;
            if (lane == 0) {
                const int c_first = cta_of_unit(static_cast<int64_t>(nb) * KB, U, G);
                const int c_last = cta_of_unit(static_cast<int64_t>(nb) * KB + KB - 1, U, G);
                // The promotion warps' partial stores are ordered before this
                // thread by the barrier; the fence publishes them device-wide
                // before the counter increment.
                __threadfence();
                reduce_nb[i] = (atomicAdd(&counters[nb], 1) == c_last - c_first) ? nb : -1;
            }
        }
    }

    if (cluster_s > 1) {
        // ------------------------------------------------------------ cluster reduction
        __syncwarp();
        cluster_sync();
        const int S = cluster_s;
        const int r = static_cast<int>(blockIdx.x % S);
        const int64_t nb = blockIdx.x / S;
        const uint32_t red = smem_addr(smem);
        const int items = M * (BNW / 4);  // float4 columns of the n-block's output
        const int i0 = r * items / S, i1 = (r + 1) * items / S;
        for (int item = i0 + static_cast<int>(threadIdx.x); item < i1; item += kNumThreads) {
            const int m = item / (BNW / 4), c4 = item % (BNW / 4);
            const uint32_t off = static_cast<uint32_t>((m * BNW + 4 * c4) * 4);
            float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int p = 0; p < S; ++p) {  // rank order = K order
                const float4 v = ld_shared_cluster_v4(map_to_cta(red + off, static_cast<uint32_t>(p)));
                sum.x += v.x;
                sum.y += v.y;
                sum.z += v.z;
                sum.w += v.w;
            }
            __nv_bfloat162 lo = __floats2bfloat162_rn(sum.x, sum.y);
            __nv_bfloat162 hi = __floats2bfloat162_rn(sum.z, sum.w);
            uint2 pk;
            pk.x = *reinterpret_cast<uint32_t *>(&lo);
            pk.y = *reinterpret_cast<uint32_t *>(&hi);
            *reinterpret_cast<uint2 *>(y + static_cast<int64_t>(m) * N + nb * BNW + 4 * c4) = pk;
        }
        __syncwarp();
        cluster_sync();  // peers may still be reading this CTA's partial until here
    }

    // ---------------------------------------------------------------- split-K reduction
    // Every thread of the CTA joins; partial sums are added in increasing
    // contributor order (deterministic).  A thread takes kItems float4 columns
    // at once and up to four contributors of each, so 32 loads are in flight.
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int nb = reduce_nb[i];
        if (nb < 0) continue;
        __threadfence();
        const int c_first = cta_of_unit(static_cast<int64_t>(nb) * KB, U, G);
        const int c_last = cta_of_unit(static_cast<int64_t>(nb) * KB + KB - 1, U, G);
        const float4 *base = reinterpret_cast<const float4 *>(
            partials + static_cast<int64_t>(nb) * (MT * BNW));
        constexpr int kSlot4 = MT * BNW / 4;  // float4s per partial slot
        constexpr int kItems = 8;
        const int items = M * (BNW / 4);
        for (int item0 = threadIdx.x; item0 < items; item0 += kItems * kNumThreads) {
            float4 sum[kItems];
#pragma unroll
            for (int r = 0; r < kItems; ++r) sum[r] = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int c = c_first; c <= c_last; c += 4) {
                float4 p[kItems][4];
#pragma unroll
                for (int r = 0; r < kItems; ++r) {
                    const int item = item0 + r * kNumThreads;
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        p[r][j] = (c + j <= c_last && item < items)
                                      ? __ldcg(base + static_cast<int64_t>(c + j) * kSlot4 + item)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int r = 0; r < kItems; ++r)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        sum[r].x += p[r][j].x;
                        sum[r].y += p[r][j].y;
                        sum[r].z += p[r][j].z;
                        sum[r].w += p[r][j].w;
                    }
            }
#pragma unroll
            for (int r = 0; r < kItems; ++r) {
                const int item = item0 + r * kNumThreads;
                if (item >= items) break;
                const int m = item / (BNW / 4), c4 = item % (BNW / 4);
                __nv_bfloat162 lo = __floats2bfloat162_rn(sum[r].x, sum[r].y);
                __nv_bfloat162 hi = __floats2bfloat162_rn(sum[r].z, sum[r].w);
                uint2 pk;
                pk.x = *reinterpret_cast<uint32_t *>(&lo);
                pk.y = *reinterpret_cast<uint32_t *>(&hi);
                *reinterpret_cast<uint2 *>(y + static_cast<int64_t>(m) * N + nb * BNW + 4 * c4) = pk;
            }
        }
        if (threadIdx.x == 0) atomicExch(&counters[nb], 0);
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace decode
}  // namespace fp8bq
