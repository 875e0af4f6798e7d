// gemm_decode.cuh -- block-scaled FP8 GEMM for small M (decode, M <= 16).
//
// Same result as the prefill kernel (page "ProCreations/Nanbeige4.3-33B-FP8",
// introduction: W8A8 FP8 linear layers), shaped for the weight-bandwidth-bound
// regime: every weight byte is read from HBM exactly once, and the grid streams
// the N/128 x K/128 weight blocks (16 KB each) evenly over all SMs.
//
// Roles (192 threads):
//   warp 0      TMA producer: per unit (n-block nb, k-block kb) the 128 x 128 B
//               weight block and, for the GEMM, the 16 x 128 B activation tile
//               (rows >= M are zero-filled by TMA), kStages deep.
//   warp 1      MMA issuer: swap-AB, D[n, m] = W_blk[n, :] . X_tile[m, :] with
//               M_mma = 128 (weight rows) and N_mma = 16 (tokens), 4 MMAs of K = 32.
//   warps 2..5  promotion: thread = one weight row n of the block (its TMEM
//               lane), 16 FP32 accumulators (one per token); per unit
//               acc[m] = fma(P[n, m], sa[m, kb] * sw[nb, kb], acc[m]).
// Stream-K: units u = nb * KB + kb are split into gridDim.x contiguous ranges.
// An n-block whose K range lies inside one CTA is written straight to Y in
// BF16.  Otherwise each contributing CTA c stores its FP32 partial in slot
// nb + c of the workspace and increments counter[nb]; the last to arrive sums
// the slots in increasing c (a fixed order, so results are deterministic),
// writes BF16 and resets the counter to zero for the next call.
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
constexpr int kNumThreads = 192;
constexpr int kTmemBufs = 4;
constexpr uint32_t kTmemCols = 64;  // kTmemBufs x MT columns, rounded to a power of two
constexpr int kMaxGrid = 256;       // workspace is sized for at most this many CTAs

struct Layout {
    static constexpr int kW = BNW * BK;  // 16 KB
    static constexpr int kX = MT * BK;   // 2 KB
    static constexpr int kStage = kW + kX;
    static constexpr int kBarOff = kStages * kStage;
    static constexpr int kNumBars = 2 * kStages + 2 * kTmemBufs + 1;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kBytes = kMiscOff + 16;
    static constexpr int kDynamicSmem = kBytes + 1024;
};

// Workspace: int32 counters[NB] (padded to 256 B), then float partials
// [NB + kMaxGrid][MT][128].
__host__ __device__ inline int64_t counters_bytes(int64_t NB) { return ((NB * 4 + 255) / 256) * 256; }
__host__ __device__ inline int64_t workspace_bytes(int64_t NB) {
    return counters_bytes(NB) + (NB + kMaxGrid) * MT * BNW * 4;
}

// CTA whose unit range [floor(c U / G), floor((c+1) U / G)) contains unit u.
__device__ __forceinline__ int cta_of_unit(int64_t u, int64_t U, int64_t G) {
    return static_cast<int>(((u + 1) * G - 1) / U);
}

__global__ void __launch_bounds__(kNumThreads, 1)
gemm_decode_kernel(const __grid_constant__ CUtensorMap tmap_w,
                   const __grid_constant__ CUtensorMap tmap_x, const float *__restrict__ sa,
                   const float *__restrict__ sw, __nv_bfloat16 *__restrict__ y, int M, int N,
                   int K, int *counters, float *partials, int *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Layout::kBarOff);
    uint64_t *empty = full + kStages;
    uint64_t *tfull = empty + kStages;
    uint64_t *tempty = tfull + kTmemBufs;
    uint64_t *drain = tempty + kTmemBufs;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Layout::kMiscOff);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Layout::kMiscOff + 4);
    volatile int *is_last = reinterpret_cast<volatile int *>(smem + Layout::kMiscOff + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = K / BK, NB = N / BNW;
    const int64_t U = static_cast<int64_t>(NB) * KB;
    const int64_t G = gridDim.x;
    const int64_t u_begin = blockIdx.x * U / G;
    const int64_t u_end = (blockIdx.x + 1) * U / G;

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
        *abort_flag = 0;
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

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t evict_first = l2_policy_evict_first();
            uint32_t stage = 0, phase = 0;
            int64_t issued = 0;
            for (int64_t u = u_begin; u < u_end; ++u) {
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
    } else {
        const int quarter = warp & 3;
        const int n_local = quarter * 32 + lane;  // weight row within the block = TMEM lane
        const int ptid = threadIdx.x - 64;        // 0..127 among the promotion threads
        uint32_t buf = 0, bphase = 0;
        float acc[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
        int seg_kb0 = static_cast<int>(u_begin % KB);
        for (int64_t u = u_begin; u < u_end; ++u) {
            const int nb = static_cast<int>(u / KB), kb = static_cast<int>(u % KB);
            const float swv = __ldg(sw + static_cast<int64_t>(nb) * KB + kb);
            float s[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m)
                s[m] = (m < M) ? __ldg(sa + static_cast<int64_t>(m) * KB + kb) * swv : 0.0f;
            // No abort check here: the four promotion warps must leave this loop at
            // the same unit (they meet at named barriers below), and they all wait
            // on the same barrier phase, so the time limit alone keeps them together.
            if (!mbar_wait(&tfull[buf], bphase, nullptr, status)) break;
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
                    float *slot = partials + (static_cast<int64_t>(nb) + blockIdx.x) * (MT * BNW);
#pragma unroll
                    for (int m = 0; m < MT; ++m) __stcg(slot + m * BNW + n_local, acc[m]);
                    __threadfence();
                    named_barrier(1, 128);
                    const int c_first = cta_of_unit(static_cast<int64_t>(nb) * KB, U, G);
                    const int c_last = cta_of_unit(static_cast<int64_t>(nb) * KB + KB - 1, U, G);
                    if (ptid == 0) {
                        const int prev = atomicAdd(&counters[nb], 1);
                        *is_last = (prev == c_last - c_first) ? 1 : 0;
                    }
                    named_barrier(1, 128);
                    if (*is_last) {
                        __threadfence();
                        float sum[MT];
#pragma unroll
                        for (int m = 0; m < MT; ++m) sum[m] = 0.0f;
                        for (int c = c_first; c <= c_last; ++c) {
                            const float *src = partials + (static_cast<int64_t>(nb) + c) * (MT * BNW);
#pragma unroll
                            for (int m = 0; m < MT; ++m) sum[m] += __ldcg(src + m * BNW + n_local);
                        }
#pragma unroll
                        for (int m = 0; m < MT; ++m)
                            if (m < M)
                                y[static_cast<int64_t>(m) * N + col] = __float2bfloat16_rn(sum[m]);
                        if (ptid == 0) atomicExch(&counters[nb], 0);
                    }
                    named_barrier(1, 128);  // is_last is reused by the next segment
                }
#pragma unroll
                for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
                seg_kb0 = 0;
            }
        }
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
