// silu_quant.cuh -- SiLU-gated product of the MLP, quantized for the down
// projection in the same pass.
//
// Page "ProCreations/Nanbeige4.3-33B-FP8", introduction: every linear layer,
// the MLP's down projection included, takes dynamically quantized activations
// (per token, groups of 128 channels, scale = amax / 448).  The down
// projection's input is h = silu(gate) * up of the fused gate/up output
// gu [M, 2I] (gate = columns [0, I), up = [I, 2I)), rounded to BF16 as the
// unfused path would store it.  This kernel computes h, rounds it to BF16 and
// quantizes it exactly as quantize_act_kernel would quantize that BF16 tensor,
// so the BF16 h never travels through HBM (it is written only when asked for).
//
// silu(g) = g * sigmoid(g), sigmoid from e = exp(-|g|) (in (0, 1], so nothing
// overflows): 1 / (1 + e) for g >= 0, e / (1 + e) otherwise.  exp and the
// divide are the fast hardware approximations (a few binary32 ulps), far below
// half a BF16 step of h.  Only the quantization divide h / scale must be the
// IEEE one, since the codes must equal fp8bq_quantize_act's on the same h.
//
// Two layouts, chosen per call:
// - silu_mul_quantize_kernel: a half-warp per 128-channel group, 8 channels per
//   lane, warps striding over the flat group index (any I, any M; the lower
//   latency per warp suits small problems).
// - silu_mul_quantize_wide_kernel: grid (chunks of 32 groups of a row, rows);
//   a warp takes four consecutive groups of one row, an 8-lane team each,
//   lane `sub` channels [8 sub, 8 sub + 8) and [64 + 8 sub, 64 + 8 sub + 8) of
//   gate and of up, so every 16-byte load has the team read 128 contiguous
//   bytes and the per-group work (the shuffle reduction of the maximum, the
//   scale and its reciprocal) is shared by 16 elements per lane, with no
//   integer division per group.  For large problems whose rows hold a
//   multiple of 4 groups.
// HBM: 4 bytes read (gate, up) and ~1 byte written (code, plus 4 bytes of scale
// per 128) per output element.
#pragma once

#include <stdint.h>

#include "ptx.cuh"
#include "quantize.cuh"

namespace fp8bq {

constexpr int kSiluThreads = 256;
constexpr int kSiluWarps = kSiluThreads / 32;
constexpr int kSiluWideGroupsPerCta = 4 * kSiluWarps;  // groups of one row per CTA iteration

__device__ __forceinline__ float silu_f32(float g) {
    const float e = __expf(-fabsf(g));
    const float den = 1.0f + e;  // in [1, 2]: the fast reciprocal-based divide is accurate here
    const float sig = __fdividef(g >= 0.0f ? 1.0f : e, den);
    return g * sig;
}

// Eight gate and eight up values -> eight BF16 h values (packed like the input).
__device__ __forceinline__ uint4 silu_mul8(uint4 gv, uint4 uv) {
    const uint32_t g[4] = {gv.x, gv.y, gv.z, gv.w};
    const uint32_t u[4] = {uv.x, uv.y, uv.z, uv.w};
    uint32_t h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float lo = silu_f32(__uint_as_float(g[i] << 16)) * __uint_as_float(u[i] << 16);
        const float hi =
            silu_f32(__uint_as_float(g[i] & 0xFFFF0000u)) * __uint_as_float(u[i] & 0xFFFF0000u);
        const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
        h[i] = *reinterpret_cast<const uint32_t *>(&p);
    }
    return make_uint4(h[0], h[1], h[2], h[3]);
}

// q: codes [M, I] as 8-byte vectors; s: scales [M, I/128]; h_out: optional BF16
// h [M, I] as 16-byte vectors.
__global__ void __launch_bounds__(kSiluThreads)
silu_mul_quantize_kernel(const uint4 *__restrict__ gu, int64_t M, int64_t I, uint2 *__restrict__ q,
                         float *__restrict__ s, uint4 *__restrict__ h_out) {
    grid_dependency_wait();
    allow_dependent_launch();
    const int lane = threadIdx.x & 31, sub = lane & 15;
    const int64_t G = I / 128, groups = M * G;
    const int64_t row_vec = 2 * I / 8;  // 16-byte vectors per gu row
    const int64_t warps = static_cast<int64_t>(gridDim.x) * kSiluWarps;
    // A warp takes two groups per iteration (one per half); the trip count is
    // uniform across the warp so the full-mask shuffles below are safe.
    for (int64_t w = static_cast<int64_t>(blockIdx.x) * kSiluWarps + (threadIdx.x >> 5);
         2 * w < groups; w += warps) {
        const int64_t g = 2 * w + (lane >> 4);
        const bool valid = g < groups;
        uint4 hv = make_uint4(0, 0, 0, 0);
        if (valid) {
            const int64_t m = g / G, gi = g % G;
            const uint4 *row = gu + m * row_vec;
            const uint4 gv = __ldcs(row + gi * 16 + sub);
            const uint4 uv = __ldcs(row + I / 8 + gi * 16 + sub);
            hv = silu_mul8(gv, uv);
        }
        uint32_t amax = amax_bits8(hv);
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if (valid) {
            const float scale = scale_from_amax_bits(amax);
            q[g * 16 + sub] = encode8(hv, scale);
            if (sub == 0) s[g] = scale;
            if (h_out != nullptr) h_out[g * 16 + sub] = hv;
        }
    }
}

// Same output; I / 128 a multiple of 4.  blockIdx.x: chunk of
// kSiluWideGroupsPerCta groups of a row; blockIdx.y: first row, rows advance by
// gridDim.y.
__global__ void __launch_bounds__(kSiluThreads)
silu_mul_quantize_wide_kernel(const uint4 *__restrict__ gu, int64_t M, int64_t I,
                              uint2 *__restrict__ q, float *__restrict__ s,
                              uint4 *__restrict__ h_out) {
    grid_dependency_wait();
    allow_dependent_launch();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane & 7;
    const int G = static_cast<int>(I / 128);
    const int gi0 = static_cast<int>(blockIdx.x) * kSiluWideGroupsPerCta + 4 * warp;
    if (gi0 >= G) return;  // the whole warp (G is a multiple of 4)
    const int gi = gi0 + (lane >> 3);
    const int64_t row_vec = I / 4;  // 16-byte vectors per gu row (2I BF16 values)
    for (int64_t m = blockIdx.y; m < M; m += gridDim.y) {
        const uint4 *gate = gu + m * row_vec + gi * 16 + sub;
        const uint4 *up = gate + I / 8;
        const uint4 g0 = __ldcs(gate), g1 = __ldcs(gate + 8);
        const uint4 u0 = __ldcs(up), u1 = __ldcs(up + 8);
        const uint4 h0 = silu_mul8(g0, u0), h1 = silu_mul8(g1, u1);
        uint32_t mx = amax_bits16_packed(h0, h1);
#pragma unroll
        for (int o = 4; o >= 1; o >>= 1) mx = __vmaxu2(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const int64_t g = m * G + gi;
        const float scale = scale_from_amax_bits(max_halves(mx));
        const float y = __frcp_rn(scale);
        q[g * 16 + sub] = encode8_y(h0, scale, y);
        q[g * 16 + 8 + sub] = encode8_y(h1, scale, y);
        if (sub == 0) s[g] = scale;
        if (h_out != nullptr) {
            h_out[g * 16 + sub] = h0;
            h_out[g * 16 + 8 + sub] = h1;
        }
    }
}

}  // namespace fp8bq
