// quantize.cuh -- E4M3 quantizers of the W8A8 FP8 block-scaled scheme (page
// "ProCreations/Nanbeige4.3-33B-FP8", introduction and "Recipe and
// calibration"): dynamic activation scales per token and 128-channel group,
// and offline min-max weight scales per 128x128 block.
//
// Both kernels are bit-exact with the definition: amax of the group/block (an
// integer max over BF16 magnitude bits, exact for finite values), scale =
// amax / 448 as the IEEE binary32 quotient (1.0 when amax is 0), and each code
// the saturating round-to-nearest-even E4M3 conversion of fl32(x / scale).
// Neither division is executed as such: both quotients come from a correctly
// rounded reciprocal and one FMA correction step (below), which reproduces
// them on this input domain.
// The build uses no fast-math and no flush-to-zero, so subnormal scales and
// quotients follow IEEE arithmetic.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "ptx.cuh"

namespace fp8bq {

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b16) {
    return __uint_as_float(b16 << 16);
}

// RN(1 / 448) = 8/7 * 2^-9 rounded to binary32.
constexpr float kRcp448 = 0x1.24924ap-9f;

// amax / 448, correctly rounded, by the corrected quotient with the constant
// reciprocal (the method of corrected_quotient below): q = RN(a / 448'),
// r = a - 448 q exactly, scale = RN(q + r / 448').  Equal to the IEEE quotient
// for every finite BF16 amax, subnormal results included (checked for all
// 32639 positive finite values).
__device__ __forceinline__ float scale_from_amax_bits(uint32_t amax_bits) {
    // amax_bits: BF16 magnitude bits (sign cleared) of the group maximum
    const float a = bf16_bits_to_float(amax_bits);
    const float q = __fmul_rn(a, kRcp448);
    const float scale = __fmaf_rn(__fmaf_rn(-q, 448.0f, a), kRcp448, q);
    return amax_bits == 0 ? 1.0f : scale;
}

// Smallest scale for which the corrected quotient below reproduces the E4M3
// code of fl32(x / scale) for every BF16 x with |x| <= 448 scale (checked for
// every BF16 amax down to this bound and every such x; below about 2^-110 the
// residual r is no longer exact).  Smaller scales use the IEEE division.
constexpr float kCorrectedQuotientMinScale = 0x1p-92f;

// x / s from y = RN(1/s) by one FMA correction step (Markstein's theorem,
// IBM J. Res. Dev. 34(1), 1990; Muller et al., "Handbook of Floating-Point
// Arithmetic", on division with a fused multiply-add): with q = RN(x y), the
// residual r = x - q s is exact, and RN(q + r y) is the correctly rounded
// quotient while no intermediate underflows.  The residual is formed negated,
// n = q s - x = -r, and the result as RN(q - n y): the same value, and for
// x = -0 (q = -0, n = +0) the sum -0 + -0 keeps the sign, so -0 / s gives the
// code 0x80 without a separate sign fix-up.
__device__ __forceinline__ float corrected_quotient(float x, float s, float y) {
    const float q = __fmul_rn(x, y);
    const float n = __fmaf_rn(q, s, -x);
    return __fmaf_rn(-n, y, q);
}

// Eight BF16 values (one 16-byte vector) -> eight E4M3 codes (8 bytes): each
// code is the saturating round-to-nearest conversion of the IEEE quotient
// fl32(x / scale).  The quotient comes from one reciprocal per call and three
// FP operations per element (corrected_quotient), which gives fl32(x / scale)
// bit for bit wherever |x / scale| >= 2^-11 or x = +-0, and the same code
// everywhere else; tiny scales take the IEEE division.
// encode8 with the reciprocal y = RN(1 / scale) supplied by the caller (used
// only when scale >= kCorrectedQuotientMinScale), for callers that encode many
// vectors with one scale.
__device__ __forceinline__ uint2 encode8_y(uint4 v, float scale, float y) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t c[4];
    if (scale >= kCorrectedQuotientMinScale) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            c[i] = e4m3x2_satfinite(corrected_quotient(__uint_as_float(w[i] << 16), scale, y),
                                    corrected_quotient(__uint_as_float(w[i] & 0xFFFF0000u), scale, y));
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            c[i] = e4m3x2_satfinite(__fdiv_rn(__uint_as_float(w[i] << 16), scale),
                                    __fdiv_rn(__uint_as_float(w[i] & 0xFFFF0000u), scale));
    }
    return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

__device__ __forceinline__ uint2 encode8(uint4 v, float scale) {
    return encode8_y(v, scale, __frcp_rn(scale));
}

__device__ __forceinline__ uint32_t amax_bits8(uint4 v) {
    uint32_t m = 0;
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        m = max(m, w[i] & 0x7FFFu);
        m = max(m, (w[i] >> 16) & 0x7FFFu);
    }
    return m;
}

// Both halves' magnitude maxima of 16 BF16 values, as two 16-bit lanes
// (packed per-halfword unsigned max; max_halves() finishes the reduction).
__device__ __forceinline__ uint32_t amax_bits16_packed(uint4 a, uint4 b) {
    constexpr uint32_t kMag = 0x7FFF7FFFu;
    uint32_t m = __vmaxu2(a.x & kMag, a.y & kMag);
    m = __vmaxu2(m, a.z & kMag);
    m = __vmaxu2(m, a.w & kMag);
    m = __vmaxu2(m, b.x & kMag);
    m = __vmaxu2(m, b.y & kMag);
    m = __vmaxu2(m, b.z & kMag);
    return __vmaxu2(m, b.w & kMag);
}

__device__ __forceinline__ uint32_t max_halves(uint32_t m) {
    return max(m & 0xFFFFu, m >> 16);
}

// ------------------------------------------------------------------ activations

// The activation [M, K] is a flat sequence of M K / 128 groups of 256 bytes
// (group g = row g / (K/128), channels 128 (g mod K/128) ...).  Persistent CTAs
// (two per SM) stream chunks of kActChunkGroups groups through a kActStages-deep
// shared-memory ring with untiled bulk copies, so the bytes in flight do not
// depend on registers; sixteen consumer warps encode from shared memory, one
// 8-lane team per group, and store codes and scales straight to global
// memory.  Lane `sub` of a team takes channels [8 sub, 8 sub + 8) and
// [64 + 8 sub, 64 + 8 sub + 8): each of its two 16-byte loads has the team
// read 128 contiguous bytes (no bank conflicts), and the per-group work (the
// shuffles, the scale and its reciprocal) is shared by 16 elements per lane.
constexpr int kActConsumerWarps = 16;
constexpr int kActThreads = 32 * (kActConsumerWarps + 1);  // + one producer warp
constexpr int kActChunkGroups = 64;                         // 16 KB of BF16 per chunk
constexpr int kActChunkBytes = kActChunkGroups * 256;
constexpr int kActStages = 6;
constexpr int kActCtasPerSm = 2;

struct ActLayout {
    static constexpr int kBarOff = kActStages * kActChunkBytes;
    static constexpr int kBytes = kBarOff + 2 * kActStages * 8 + 16;
};

__global__ void __launch_bounds__(kActThreads, kActCtasPerSm)
quantize_act_kernel(const uint8_t *__restrict__ x, int64_t num_groups, uint2 *__restrict__ q,
                    float *__restrict__ sa, int *status) {
    extern __shared__ __align__(128) uint8_t act_smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(act_smem + ActLayout::kBarOff);
    uint64_t *empty = full + kActStages;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + kActStages);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t num_chunks = (num_groups + kActChunkGroups - 1) / kActChunkGroups;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kActStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kActConsumerWarps);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    // The next kernel (typically the GEMM this feeds) may start at once, so
    // it can set up and stream its weights while this one runs: this kernel
    // writes activation codes only, and no kernel of this library that writes
    // weights lets its successor start before it completes.
    allow_dependent_launch();
    __syncthreads();
    grid_dependency_wait();

    if (warp == kActConsumerWarps) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t evict_first = l2_policy_evict_first();
            int64_t i = 0;
            for (int64_t c = blockIdx.x; c < num_chunks; c += gridDim.x, ++i) {
                const int s = static_cast<int>(i % kActStages);
                if (!mbar_wait(&empty[s], static_cast<uint32_t>(((i / kActStages) & 1) ^ 1),
                               abort_flag, status))
                    break;
                const int64_t g0 = c * kActChunkGroups;
                const int64_t left = num_groups - g0;
                const int64_t ng = left < kActChunkGroups ? left : kActChunkGroups;
                const uint32_t bytes = static_cast<uint32_t>(ng * 256);
                mbar_arrive_expect_tx(&full[s], bytes);
                bulk_load(act_smem + s * kActChunkBytes, x + g0 * 256, bytes, &full[s], evict_first);
            }
        }
    } else {
        // ------------------------------------------------------------ consumers
        static_assert(kActChunkGroups == kActConsumerWarps * 4, "one 8-lane team per group");
        const int gl = threadIdx.x >> 3;  // the team's group within a chunk, 0..63
        const int sub = threadIdx.x & 7;
        int64_t i = 0;
        for (int64_t c = blockIdx.x; c < num_chunks; c += gridDim.x, ++i) {
            const int s = static_cast<int>(i % kActStages);
            if (!mbar_wait(&full[s], static_cast<uint32_t>((i / kActStages) & 1), abort_flag, status))
                break;
            const int64_t g0 = c * kActChunkGroups;
            const uint8_t *st = act_smem + s * kActChunkBytes + gl * 256 + sub * 16;
            const bool ok = g0 + gl < num_groups;
            const uint4 v0 = ok ? *reinterpret_cast<const uint4 *>(st) : make_uint4(0, 0, 0, 0);
            const uint4 v1 = ok ? *reinterpret_cast<const uint4 *>(st + 128) : make_uint4(0, 0, 0, 0);
            uint32_t m = amax_bits16_packed(v0, v1);
#pragma unroll
            for (int off = 4; off > 0; off >>= 1) m = __vmaxu2(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
            // every lane has read its vectors: the slot can be refilled
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            const float scale = scale_from_amax_bits(max_halves(m));
            if (ok) {
                const float y = __frcp_rn(scale);
                q[(g0 + gl) * 16 + sub] = encode8_y(v0, scale, y);
                q[(g0 + gl) * 16 + 8 + sub] = encode8_y(v1, scale, y);
                if (sub == 0) sa[g0 + gl] = scale;
            }
        }
    }
}

// Small activations (decode batches): one 16-lane team per group, each lane
// one 16-byte load straight from global memory.  With no shared memory and
// 256 threads its CTAs fit on an SM beside a running decode GEMM CTA, so the
// kernel is resident, and past its dependency wait, as soon as the previous
// kernel completes.
constexpr int kSmallActThreads = 256;
constexpr int kSmallActGroupsPerCta = kSmallActThreads / 16;

__global__ void __launch_bounds__(kSmallActThreads)
quantize_act_small_kernel(const uint4 *__restrict__ x, int64_t num_groups, uint2 *__restrict__ q,
                          float *__restrict__ sa) {
    allow_dependent_launch();  // as in quantize_act_kernel
    grid_dependency_wait();
    const int64_t g = static_cast<int64_t>(blockIdx.x) * kSmallActGroupsPerCta + (threadIdx.x >> 4);
    const int sub = threadIdx.x & 15;
    const bool ok = g < num_groups;
    const uint4 v = ok ? x[g * 16 + sub] : make_uint4(0, 0, 0, 0);
    uint32_t m = amax_bits8(v);
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
    const float scale = scale_from_amax_bits(m);
    if (ok) {
        q[g * 16 + sub] = encode8(v, scale);
        if (sub == 0) sa[g] = scale;
    }
}

// ------------------------------------------------------------------ weights

// One CTA per 128x128 block: 256 threads, each holding 8 of the block's 2048
// 16-byte vectors (a vector is 8 consecutive elements of one row).
constexpr int kWeightThreads = 256;

__global__ void __launch_bounds__(kWeightThreads)
quantize_weight_kernel(const uint16_t *__restrict__ w, int64_t K, uint8_t *__restrict__ q,
                       float *__restrict__ sw) {
    __shared__ uint32_t warp_max[kWeightThreads / 32];
    // This kernel writes weights, so it never lets the next kernel start
    // early: a decode GEMM may read its weights before its dependency wait.
    grid_dependency_wait();
    const int64_t bj = blockIdx.x;  // K block
    const int64_t bi = blockIdx.y;  // N block
    const int64_t KB = K / 128;

    uint4 v[8];
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int vec = i * kWeightThreads + threadIdx.x;  // 0..2047
        const int r = vec >> 4, c = (vec & 15) * 8;
        const uint16_t *src = w + (bi * 128 + r) * K + bj * 128 + c;
        v[i] = __ldg(reinterpret_cast<const uint4 *>(src));
        m = max(m, amax_bits8(v[i]));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
    __syncthreads();
    m = 0;
#pragma unroll
    for (int i = 0; i < kWeightThreads / 32; ++i) m = max(m, warp_max[i]);
    const float scale = scale_from_amax_bits(m);
    if (threadIdx.x == 0) sw[bi * KB + bj] = scale;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int vec = i * kWeightThreads + threadIdx.x;
        const int r = vec >> 4, c = (vec & 15) * 8;
        *reinterpret_cast<uint2 *>(q + (bi * 128 + r) * K + bj * 128 + c) = encode8(v[i], scale);
    }
}

}  // namespace fp8bq
