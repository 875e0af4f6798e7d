// kv_cache.cuh -- FP8 E4M3 KV-cache write with unit scales.
//
// Page "ProCreations/Nanbeige4.3-33B-FP8", "Serving" and the "Speed on Vega"
// table: with --kv-cache-dtype fp8_e4m3 the K and V projections are stored in
// E4M3 with unit cache scales.  A code is the saturating round-to-nearest-even
// conversion of fl32(x / 1) = x, the same rule as every activation and weight
// code of the linear layers; NaN stays NaN and +-infinity saturates to +-448.
//
// One warp per (token, K or V) row: the row is read as 16-byte vectors of 8
// BF16 values straight out of the projection output (any row stride, e.g. the
// K and V column ranges of the fused QKV output) and written as 8-byte vectors
// of codes to its cache slot loc[t].  HBM-bound: 2 bytes read and 1 written
// per element.
#pragma once

#include <stdint.h>

#include "ptx.cuh"

namespace fp8bq {

constexpr int kKvThreads = 256;
constexpr int kKvWarps = kKvThreads / 32;

// Eight BF16 values -> eight E4M3 codes at unit scale: x / 1 is exactly x, so
// the code is the saturating conversion of x itself.
__device__ __forceinline__ uint2 encode8_unit(uint4 v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        c[i] = e4m3x2_satfinite(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
    return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

// Rows r = 2 t (K of token t) and 2 t + 1 (V); width8 = row width / 8.
__global__ void __launch_bounds__(kKvThreads)
kv_write_e4m3_kernel(const uint16_t *__restrict__ k, const uint16_t *__restrict__ v,
                     int64_t row_stride, int64_t T, int width8, const int64_t *__restrict__ loc,
                     uint8_t *__restrict__ k_cache, uint8_t *__restrict__ v_cache,
                     int64_t num_slots, int64_t slot_stride, int *status) {
    // The projections come from the previous kernel in the stream.
    grid_dependency_wait();
    allow_dependent_launch();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t rows = 2 * T;
    const int64_t step = static_cast<int64_t>(gridDim.x) * kKvWarps;
    for (int64_t r = static_cast<int64_t>(blockIdx.x) * kKvWarps + warp; r < rows; r += step) {
        const int64_t t = r >> 1;
        const bool is_v = (r & 1) != 0;
        const int64_t s = __ldg(loc + t);
        if (s < 0 || s >= num_slots) {
            if (lane == 0 && !is_v) atomicExch(status, 8 /* FP8BQ_ERR_INDEX */);
            continue;
        }
        const uint4 *src = reinterpret_cast<const uint4 *>((is_v ? v : k) + t * row_stride);
        uint2 *dst = reinterpret_cast<uint2 *>((is_v ? v_cache : k_cache) + s * slot_stride);
        // four 16-byte loads in flight per lane
        for (int c0 = lane; c0 < width8; c0 += 4 * 32) {
            uint4 x[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = c0 + 32 * j;
                if (c < width8) x[j] = __ldcs(src + c);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = c0 + 32 * j;
                if (c < width8) dst[c] = encode8_unit(x[j]);
            }
        }
    }
}

}  // namespace fp8bq
