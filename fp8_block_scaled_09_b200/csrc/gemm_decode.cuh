// gemm_decode.cuh -- block-scaled FP8 GEMM for small M (decode, M <= 16).
//
// Same result as the prefill kernel (page "ProCreations/Nanbeige4.3-33B-FP8",
// introduction: W8A8 FP8 linear layers), shaped for the weight-bandwidth-bound
// regime: every weight byte is read from HBM exactly once, and the grid streams
// the N/128 x K/128 weight blocks (16 KB each) evenly over all SMs.
//
// Roles (224 threads):
//   warp 0      TMA producer: per unit (n-block nb, k-block kb) the 128 x 128 B
//               weight block and the 16 x 128 B activation tile (rows >= M are
//               zero-filled by TMA), kStages deep.
//   warp 1      MMA issuer: swap-AB, D[n, m] = W_blk[n, :] . X_tile[m, :] with
//               M_mma = 128 (weight rows) and N_mma = 16 (tokens), 4 MMAs of K = 32,
//               into one of kTmemBufs TMEM buffers.
//   warps 2..5  promotion: thread = one weight row n of the block (its TMEM
//               lane), 16 FP32 accumulators (one per token); per unit
//               acc[m] = fma(P[n, m], sa[m, kb] * sw[nb, kb], acc[m]), scales read
//               from shared memory where they are staged once per CTA.
//   warp 6      split-K: publishes this CTA's partial sums (device-wide fence and
//               counter increment), so promotion never waits on either; if the
//               CTA was an n-block's last contributor, all warps reduce it after
//               the main loop.
// Stream-K: units u = nb * KB + kb are split into gridDim.x contiguous ranges.
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
constexpr int BK = 128;
constexpr int MT = 16;    // token tile (MMA N)
constexpr int kStages = 8;
constexpr int kNumThreads = 224;
constexpr int kSplitWarp = 6;
constexpr int kTmemBufs = 8;
constexpr uint32_t kTmemCols = 128;  // kTmemBufs x MT columns
constexpr int kMaxGrid = 256;        // workspace is sized for at most this many CTAs

struct Layout {
    static constexpr int kW = BNW * BK;  // 16 KB
    static constexpr int kX = MT * BK;   // 2 KB
    static constexpr int kStage = kW + kX;
    static constexpr int kBarOff = kStages * kStage;
    // full, empty (per stage), tfull, tempty (per TMEM buffer), drain, 2 split-K flushes
    static constexpr int kNumBars = 2 * kStages + 2 * kTmemBufs + 1 + 2;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kScaleOff = kMiscOff + 16;  // then sa[MT][KB], then sw[units of this CTA]
    static constexpr int kMaxSmem = 227 * 1024;
};

// Dynamic shared memory for a launch: stages, barriers, the activation scales
// of all M rows and the weight scales of one CTA's unit range.
__host__ __device__ inline int64_t smem_bytes(int64_t KB, int64_t units_per_cta_max) {
    return Layout::kScaleOff + MT * KB * 4 + (units_per_cta_max + 1) * 4 + 1024;
}

// Workspace: a fixed header of kMaxCounters int32 split-K counters, then float
// partials [NB + kMaxGrid][MT][128].  The header has the same size for every
// shape, so partial sums never land on counters a later call (of any shape)
// expects to be zero: every successful call leaves the whole header zeroed.
constexpr int64_t kMaxCounters = 4096;  // n-blocks, i.e. N <= 524288 on this path
constexpr int64_t kCounterBytes = kMaxCounters * 4;
__host__ __device__ inline int64_t workspace_bytes(int64_t NB) {
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

__global__ void __launch_bounds__(kNumThreads, 1)
gemm_decode_kernel(const __grid_constant__ CUtensorMap tmap_w,
                   const __grid_constant__ CUtensorMap tmap_x, const float *__restrict__ sa,
                   const float *__restrict__ sw, __nv_bfloat16 *__restrict__ y, int M, int N,
                   int K, int *counters, float *partials, int *status, int early_weights) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Layout::kBarOff);
    uint64_t *empty = full + kStages;
    uint64_t *tfull = empty + kStages;
    uint64_t *tempty = tfull + kTmemBufs;
    uint64_t *drain = tempty + kTmemBufs;
    uint64_t *flushed = drain + 1;  // [2]: promotion -> split-K warp, one per split n-block
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Layout::kMiscOff);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Layout::kMiscOff + 4);
    float *sa_s = reinterpret_cast<float *>(smem + Layout::kScaleOff);  // [MT][KB]
    // n-blocks this CTA must reduce (it was their last contributor), or -1
    volatile int *reduce_nb = reinterpret_cast<volatile int *>(smem + Layout::kMiscOff + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = K / BK, NB = N / BNW;
    const int64_t U = static_cast<int64_t>(NB) * KB;
    const int64_t G = gridDim.x;
    const int64_t u_begin = blockIdx.x * U / G;
    const int64_t u_end = (blockIdx.x + 1) * U / G;
    float *sw_s = sa_s + MT * KB;  // sw[u] for u in [u_begin, u_end): sw is [NB, KB] row-major

    allow_dependent_launch();
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < kTmemBufs; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);
        }
        mbar_init(drain, 1);
        mbar_init(&flushed[0], 4);
        mbar_init(&flushed[1], 4);
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
    // quantizer, which writes activation codes and scales only and lets this
    // kernel start after its own dependency wait.  Every other global access
    // happens after the previous kernel has completed.
    int64_t n_early = 0;
    if (early_weights && warp == 0 && lane == 0) {
        const uint64_t evict_first = l2_policy_evict_first();
        for (int64_t u = u_begin; u < u_end && n_early < kStages; ++u, ++n_early) {
            const int nb = static_cast<int>(u / KB), kb = static_cast<int>(u % KB);
            mbar_arrive_expect_tx(&full[n_early], Layout::kStage);
            tma_load_2d_hint(smem + n_early * Layout::kStage, &tmap_w, &full[n_early], kb * BK,
                             nb * BNW, evict_first);
        }
    }
    grid_dependency_wait();

    if (warp == 0) {
        if (lane == 0) {
            // activation tiles of the stages whose weight blocks went out early
            for (int64_t i = 0; i < n_early; ++i)
                tma_load_2d(smem + i * Layout::kStage + Layout::kW, &tmap_x, &full[i],
                            static_cast<int>((u_begin + i) % KB) * BK, 0);
            const uint64_t evict_first = l2_policy_evict_first();
            uint32_t stage = static_cast<uint32_t>(n_early % kStages);
            uint32_t phase = n_early == kStages ? 1u : 0u;
            int64_t issued = n_early;
            for (int64_t u = u_begin + n_early; u < u_end; ++u) {
                const int nb = static_cast<int>(u / KB), kb = static_cast<int>(u % KB);
                if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, status)) break;
                uint8_t *st = smem + stage * Layout::kStage;
                mbar_arrive_expect_tx(&full[stage], Layout::kStage);
                tma_load_2d_hint(st, &tmap_w, &full[stage], kb * BK, nb * BNW, evict_first);
                tma_load_2d(st + Layout::kW, &tmap_x, &full[stage], kb * BK, 0);
                ++issued;
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            for (int64_t i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
                mbar_wait(&full[i % kStages], static_cast<uint32_t>((i / kStages) & 1), nullptr,
                          status);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = umma_idesc_e4m3(BNW, MT);
            uint32_t stage = 0, phase = 0, buf = 0, bphase = 0;
            for (int64_t u = u_begin; u < u_end; ++u) {
                if (!mbar_wait(&tempty[buf], bphase ^ 1, abort_flag, status) ||
                    !mbar_wait(&full[stage], phase, abort_flag, status))
                    break;
                tc_fence_after_sync();
                const uint32_t w_addr = smem_addr(smem + stage * Layout::kStage);
                const uint32_t x_addr = w_addr + Layout::kW;
                const uint32_t d_tmem = tmem_base + buf * MT;
#pragma unroll
                for (int j = 0; j < BK / 32; ++j)
                    umma_e4m3(d_tmem, umma_desc_sw128(w_addr + 32 * j),
                              umma_desc_sw128(x_addr + 32 * j), idesc, j > 0 ? 1u : 0u);
                umma_commit(&empty[stage]);
                umma_commit(&tfull[buf]);
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1;
                }
                if (++buf == kTmemBufs) {
                    buf = 0;
                    bphase ^= 1;
                }
            }
            umma_commit(drain);
            mbar_wait(drain, 0, nullptr, status);
        }
    } else if (warp < kSplitWarp) {
        const int quarter = warp & 3;
        const int n_local = quarter * 32 + lane;  // weight row within the block = TMEM lane
        const int ptid = threadIdx.x - 64;        // 0..127 among the promotion threads
        // Stage the scales once: every activation scale (M <= 16 rows) and the
        // weight scales of this CTA's units, so the per-unit promotion reads
        // shared memory only.  Loads are issued in batches so their latencies
        // overlap.
        constexpr int kBatch = 8;
        const int sa_total = MT * KB, sa_valid = M * KB;
        for (int base = ptid; base < sa_total; base += 128 * kBatch) {
            float v[kBatch];
#pragma unroll
            for (int j = 0; j < kBatch; ++j) {
                const int i = base + 128 * j;
                v[j] = (i < sa_valid) ? __ldg(sa + i) : 0.0f;
            }
#pragma unroll
            for (int j = 0; j < kBatch; ++j) {
                const int i = base + 128 * j;
                if (i < sa_total) sa_s[i] = v[j];
            }
        }
        const int n_units = static_cast<int>(u_end - u_begin);
        for (int base = ptid; base < n_units; base += 128 * kBatch) {
            float v[kBatch];
#pragma unroll
            for (int j = 0; j < kBatch; ++j) {
                const int i = base + 128 * j;
                v[j] = (i < n_units) ? __ldg(sw + u_begin + i) : 0.0f;
            }
#pragma unroll
            for (int j = 0; j < kBatch; ++j) {
                const int i = base + 128 * j;
                if (i < n_units) sw_s[i] = v[j];
            }
        }
        named_barrier(1, 128);

        uint32_t buf = 0, bphase = 0;
        float acc[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
        int seg_kb0 = static_cast<int>(u_begin % KB);
        int split_idx = 0;
        for (int64_t u = u_begin; u < u_end; ++u) {
            const int nb = static_cast<int>(u / KB), kb = static_cast<int>(u % KB);
            const float swv = sw_s[u - u_begin];
            float s[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) s[m] = sa_s[m * KB + kb] * swv;
            if (!mbar_wait(&tfull[buf], bphase, abort_flag, status)) break;
            tc_fence_after_sync();
            float v[MT];
            tmem_load16(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + buf * MT, v);
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[buf]);
            if (++buf == kTmemBufs) {
                buf = 0;
                bphase ^= 1;
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[m] = fmaf(v[m], s[m], acc[m]);

            if (kb == KB - 1 || u == u_end - 1) {
                // end of this CTA's segment of n-block nb
                const int col = nb * BNW + n_local;
                if (seg_kb0 == 0 && kb == KB - 1) {
#pragma unroll
                    for (int m = 0; m < MT; ++m)
                        if (m < M) y[static_cast<int64_t>(m) * N + col] = __float2bfloat16_rn(acc[m]);
                } else {
                    // hand the partial to the split-K warp
                    float *slot = partials + (static_cast<int64_t>(nb) + blockIdx.x) * (MT * BNW);
#pragma unroll
                    for (int m = 0; m < MT; ++m) __stcg(slot + m * BNW + n_local, acc[m]);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&flushed[split_idx]);
                    ++split_idx;
                }
#pragma unroll
                for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
                seg_kb0 = 0;
            }
        }
    } else {
        // ------------------------------------------------------------ split-K warp
        // Publishes each split n-block's partial and learns whether this CTA was
        // the last contributor; the reduction itself runs after the main loop on
        // all threads of the CTA.
        const SplitPlan plan = split_plan(u_begin, u_end, KB);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            if (i >= plan.count) break;
            const int nb = plan.nb[i];
            if (!mbar_wait(&flushed[i], 0, abort_flag, status)) break;
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

    // ---------------------------------------------------------------- split-K reduction
    // Every thread of the CTA joins; partial sums are added in increasing
    // contributor order (deterministic) with the loads of up to four
    // contributors in flight at once.
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
        for (int item = threadIdx.x; item < M * (BNW / 4); item += kNumThreads) {
            const int m = item / (BNW / 4), c4 = item % (BNW / 4);
            float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int c = c_first; c <= c_last; c += 4) {
                float4 p[4];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    p[j] = (c + j <= c_last)
                               ? __ldcg(base + static_cast<int64_t>(c + j) * kSlot4 + m * (BNW / 4) + c4)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    sum.x += p[j].x;
                    sum.y += p[j].y;
                    sum.z += p[j].z;
                    sum.w += p[j].w;
                }
            }
            __nv_bfloat162 lo = __floats2bfloat162_rn(sum.x, sum.y);
            __nv_bfloat162 hi = __floats2bfloat162_rn(sum.z, sum.w);
            uint2 pk;
            pk.x = *reinterpret_cast<uint32_t *>(&lo);
            pk.y = *reinterpret_cast<uint32_t *>(&hi);
            *reinterpret_cast<uint2 *>(y + static_cast<int64_t>(m) * N + nb * BNW + 4 * c4) = pk;
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
