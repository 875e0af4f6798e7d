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
// Design (one persistent CTA per SM, 320 threads):
//   warp 0      TMA producer: per K chunk one A tile (128 x 128 B) and one B tile
//               (BN x 128 B), 128-byte swizzle, into a kStages-deep ring.
//   warp 1      MMA issuer (one thread): 4 x tcgen05.mma (K = 32 each) per chunk
//               into one of two TMEM buffers of BN FP32 columns.
//   warps 2..9  promotion + epilogue: warp w reads TMEM lanes 32*(w%4)..+31
//               (its hardware lane quarter); warps 2-5 own tile columns
//               [0, 128), warps 6-9 columns [128, 256), so each thread keeps the
//               128 FP32 accumulators of one output row and one 128-column
//               weight block, whose scale is a single sw value per chunk.
// Tiles are walked in groups of kGroupM m-tiles so the tiles resident at one
// time share A and B rows in L2.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "ptx.cuh"

namespace fp8bq {
namespace prefill {

constexpr int BM = 128;
constexpr int BK = 128;  // one scale chunk of K per pipeline stage
constexpr int kStages = 4;
constexpr int kNumThreads = 320;
constexpr int kPromoWarps = 8;
constexpr int kGroupM = 16;

template <int BN>
struct Layout {
    static_assert(BN == 256, "tile width");
    static constexpr int kA = BM * BK;
    static constexpr int kB = BN * BK;
    static constexpr int kStage = kA + kB;
    static constexpr int kBarOff = kStages * kStage;
    static constexpr int kNumBars = 2 * kStages + 2 + 2 + 1;  // full, empty, tfull, tempty, drain
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kBytes = kMiscOff + 16;
    static constexpr int kDynamicSmem = kBytes + 1024;  // room to align the base to 1024 B
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

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

template <int BN>
__global__ void __launch_bounds__(kNumThreads, 1)
gemm_prefill_kernel(const __grid_constant__ CUtensorMap tmap_a,
                    const __grid_constant__ CUtensorMap tmap_b, const float *__restrict__ sa,
                    const float *__restrict__ sw, __nv_bfloat16 *__restrict__ y, int M, int N,
                    int K, int *status) {
    using L = Layout<BN>;
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
    const int n_tiles = (N + BN - 1) / BN;
    const int num_tiles = m_tiles * n_tiles;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], kPromoWarps);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
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

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            int64_t issued = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                int tm, tn;
                tile_coords(t, m_tiles, n_tiles, tm, tn);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sa_tile = smem + stage * L::kStage;
                    mbar_arrive_expect_tx(&full[stage], L::kStage);
                    tma_load_2d(sa_tile, &tmap_a, &full[stage], kb * BK, tm * BM);
                    tma_load_2d(sa_tile + L::kA, &tmap_b, &full[stage], kb * BK, tn * BN);
                    ++issued;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            // Before the CTA may exit, every load it issued must have landed.
            for (int64_t i = (issued > kStages ? issued - kStages : 0); i < issued; ++i) {
                const uint32_t s = static_cast<uint32_t>(i % kStages);
                const uint32_t p = static_cast<uint32_t>((i / kStages) & 1);
                mbar_wait(&full[s], p, nullptr, status);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = umma_idesc_e4m3(BM, BN);
            uint32_t stage = 0, phase = 0, buf = 0, bphase = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                for (int kb = 0; kb < KB; ++kb) {
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
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1;
                    }
                    buf ^= 1;
                    if (buf == 0) bphase ^= 1;
                }
            }
            // Wait for every MMA this thread issued before TMEM is released.
            umma_commit(drain);
            mbar_wait(drain, 0, nullptr, status);
        }
    } else {
        // ------------------------------------------------------------ promotion + epilogue
        const int pw = warp - 2;
        const int quarter = warp & 3;  // TMEM lane quarter accessible to this warp
        const int half = pw >> 2;      // which 128-column weight block of the tile
        const int row_in_tile = quarter * 32 + lane;
        uint32_t buf = 0, bphase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
            int tm, tn;
            tile_coords(t, m_tiles, n_tiles, tm, tn);
            const int grow = tm * BM + row_in_tile;
            const int gcol = tn * BN + half * 128;
            const bool row_ok = grow < M;
            const bool col_ok = gcol < N;
            const float *sa_row = sa + static_cast<int64_t>(row_ok ? grow : 0) * KB;
            const float *sw_row = sw + static_cast<int64_t>(col_ok ? gcol / 128 : 0) * KB;

            float acc[128];
#pragma unroll
            for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
            float sa_next = row_ok ? __ldg(sa_row) : 0.0f;
            float sw_next = col_ok ? __ldg(sw_row) : 0.0f;
            for (int kb = 0; kb < KB; ++kb) {
                const float scale = sa_next * sw_next;
                if (kb + 1 < KB) {
                    sa_next = row_ok ? __ldg(sa_row + kb + 1) : 0.0f;
                    sw_next = col_ok ? __ldg(sw_row + kb + 1) : 0.0f;
                }
                if (!mbar_wait(&tfull[buf], bphase, abort_flag, status)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                       buf * BN + half * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    float v[16];
                    tmem_load16(taddr + c * 16, v);
#pragma unroll
                    for (int i = 0; i < 16; ++i) acc[c * 16 + i] = fmaf(v[i], scale, acc[c * 16 + i]);
                }
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[buf]);
                buf ^= 1;
                if (buf == 0) bphase ^= 1;
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

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, L::kTmemCols);
    }
}

}  // namespace prefill
}  // namespace fp8bq
