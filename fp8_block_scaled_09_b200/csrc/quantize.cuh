// quantize.cuh -- E4M3 quantizers of the W8A8 FP8 block-scaled scheme (page
// "ProCreations/Nanbeige4.3-33B-FP8", introduction and "Recipe and
// calibration"): dynamic activation scales per token and 128-channel group,
// and offline min-max weight scales per 128x128 block.
//
// Both kernels are bit-exact with the definition: amax of the group/block (an
// integer max over BF16 magnitude bits, exact for finite values), scale =
// amax / 448 as an IEEE binary32 division (1.0 when amax is 0), and each code
// the saturating round-to-nearest-even E4M3 conversion of fl32(x / scale).
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

__device__ __forceinline__ float scale_from_amax_bits(uint32_t amax_bits) {
    // amax_bits: BF16 magnitude bits (sign cleared) of the group maximum
    return amax_bits == 0 ? 1.0f : __fdiv_rn(bf16_bits_to_float(amax_bits), 448.0f);
}

// Eight BF16 values (one 16-byte vector) -> eight E4M3 codes (8 bytes).
__device__ __forceinline__ uint2 encode8(uint4 v, float scale) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const float a0 = __fdiv_rn(bf16_bits_to_float(w[2 * h] & 0xFFFFu), scale);
        const float a1 = __fdiv_rn(bf16_bits_to_float(w[2 * h] >> 16), scale);
        const float a2 = __fdiv_rn(bf16_bits_to_float(w[2 * h + 1] & 0xFFFFu), scale);
        const float a3 = __fdiv_rn(bf16_bits_to_float(w[2 * h + 1] >> 16), scale);
        out[h] = static_cast<uint32_t>(e4m3x2_satfinite(a0, a1)) |
                 (static_cast<uint32_t>(e4m3x2_satfinite(a2, a3)) << 16);
    }
    return make_uint2(out[0], out[1]);
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

// ------------------------------------------------------------------ activations

// One 128-element group is handled by 16 consecutive lanes, each holding one
// 16-byte vector (8 BF16).  Each thread takes kActUnroll groups per pass so
// that several independent loads are in flight.
constexpr int kActThreads = 256;
constexpr int kActUnroll = 2;

__global__ void __launch_bounds__(kActThreads)
quantize_act_kernel(const uint4 *__restrict__ x, int64_t num_groups, uint2 *__restrict__ q,
                    float *__restrict__ sa) {
    allow_dependent_launch();
    grid_dependency_wait();
    const int sub = threadIdx.x & 15;  // lane within the 16-lane group team
    const int64_t team = (static_cast<int64_t>(blockIdx.x) * kActThreads + threadIdx.x) >> 4;
    const int64_t num_teams = (static_cast<int64_t>(gridDim.x) * kActThreads) >> 4;

    // The loop bound uses the warp's first team so both teams of a warp iterate
    // together (the shuffles below use the full warp mask).
    const int64_t warp_team = team & ~static_cast<int64_t>(1);
    for (int64_t it = warp_team; it < num_groups; it += num_teams * kActUnroll) {
        const int64_t g0 = it + (team & 1);
        uint4 v[kActUnroll];
        bool ok[kActUnroll];
#pragma unroll
        for (int u = 0; u < kActUnroll; ++u) {
            const int64_t g = g0 + u * num_teams;
            ok[u] = g < num_groups;
            v[u] = ok[u] ? __ldcs(x + g * 16 + sub) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kActUnroll; ++u) {
            uint32_t m = amax_bits8(v[u]);
            // reduce over the 16 lanes of the team (xor offsets < 16 stay inside it)
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
            const float scale = scale_from_amax_bits(m);
            if (ok[u]) {
                const int64_t g = g0 + u * num_teams;
                q[g * 16 + sub] = encode8(v[u], scale);
                if (sub == 0) sa[g] = scale;
            }
        }
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
    allow_dependent_launch();
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
