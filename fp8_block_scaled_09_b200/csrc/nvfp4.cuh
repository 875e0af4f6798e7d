// nvfp4.cuh -- NVFP4 weight-only linear layer with BF16 activations (A16).
//
// Page "ProCreations/Nanbeige4.3-33B-NVFP4-A16", recipe paragraph: FP4 E2M1
// weights in groups of 16 consecutive k with E4M3 block scales and one global
// FP32 scale per tensor; activations stay BF16.  A weight is
//     w[n, k] = e2m1(q[n, k]) * e4m3(sb[n, k/16]) * g.
// Layouts: packed [N, K/2] bytes (element 2j in the low nibble), sb [N, K/16]
// E4M3 codes, g one float in device memory.
//
// Quantizer (offline, plain min-max; the page's own scales come from a
// data-driven search): g = amax(W) / 2688 (2688 = 6 * 448), sb = E4M3 of
// fl32(amax_group / fl32(6 g)), q = E2M1 of fl32(w / fl32(e4m3(sb) * g)).
//
// GEMM: e2m1 * e4m3 products are exact in BF16 (at most 6 significant bits,
// |value| in [2^-10, 2688]), so the weights are expanded to BF16 in shared
// memory with their block scale folded in and multiplied by the BF16
// activations on the tensor cores (tcgen05 kind::f16, FP32 accumulation in
// TMEM over the CTA's whole K range, in four accumulators that consecutive
// K steps rotate through so the MMAs overlap instead of forming one dependent
// chain); g scales the summed accumulators once in the epilogue.  Swap-AB as in the FP8 decode kernel: the weight rows are the MMA's
// M = 128, the tokens its N = 16.  Units are 128 weight rows x 256 k.
//   warp 0      TMA producer: per unit the packed rows (128 x 128 B, 128-byte
//               swizzle), their 16 scale bytes (128 x 16 B) and the activation
//               tile (16 tokens x 256 k as four 128-byte-swizzled chunks).
//   warp 1      MMA issuer: per unit 16 MMAs of K = 16, after one wait on the
//               unit's A tile and one on its raw stage.
//   warps 2..17 dequant: per unit, thread (row, 64-k chunk) turns 32 code
//               bytes and 4 block scales into 64 BF16 values of the A tile
//               (128 rows x 256 k, four 128-byte-swizzled K-major chunks; two
//               tiles in flight); then the epilogue reads TMEM.
// Split: as the FP8 decode kernel's cluster mode -- n-block nb on a cluster of
// S CTAs, each a contiguous k range, partials summed in rank order through
// distributed shared memory.  Token tiles beyond 16 rows are separate grid
// rows (blockIdx.y), each streaming the weights again.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "ptx.cuh"

namespace fp8bq {
namespace nvfp4 {

constexpr int BNW = 128;       // weight rows per n-block
constexpr int BKU = 256;       // k per unit
constexpr int MT = 16;         // token tile
constexpr int kStages = 3;     // raw TMA ring
constexpr int kABufs = 2;      // BF16 A tiles (whole units of 256 k)
constexpr int kDqWarps = 16;
constexpr int kNumThreads = 32 * (2 + kDqWarps);  // 576
constexpr int kNumAcc = 4;                        // accumulators, rotated over K steps
constexpr uint32_t kTmemCols = 64;                // kNumAcc x 16 FP32 columns

struct Layout {
    static constexpr int kW = BNW * BKU / 2;       // 16 KB packed
    static constexpr int kS = BNW * BKU / 16;      // 2 KB of scales
    static constexpr int kXChunk = MT * 128;       // 64 k of 16 tokens, BF16
    static constexpr int kX = 4 * kXChunk;         // 8 KB
    static constexpr int kStage = kW + kS + kX;    // 26 KB
    static constexpr int kAChunk = BNW * 128;      // 16 KB: 64 k of 128 rows in BF16
    static constexpr int kA = 4 * kAChunk;         // 64 KB BF16 tile of a whole unit
    static constexpr int kAOff = kStages * kStage;
    static constexpr int kBarOff = kAOff + kABufs * kA;
    // full, empty (per stage), afull, aempty (per A tile), done
    static constexpr int kNumBars = 2 * kStages + 2 * kABufs + 1;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kBytes = kMiscOff + 16 + 1024;  // + alignment slack
};
static_assert(Layout::kStage % 1024 == 0 && Layout::kW % 1024 == 0, "swizzled tiles 1 KB aligned");
static_assert(Layout::kA * kABufs >= MT * BNW * 4, "the cluster partial fits in the A tiles");

// ---------------------------------------------------------------- quantizer

// Pass 1: amax(|W|) as BF16 magnitude bits, atomically maxed into *amax_bits.
__global__ void __launch_bounds__(256)
nvfp4_amax_kernel(const uint4 *__restrict__ w, int64_t n_vec, unsigned int *amax_bits) {
    uint32_t m = 0;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_vec;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const uint4 v = __ldcs(w + i);
        const uint32_t a[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) m = max(m, max(a[j] & 0x7FFFu, (a[j] >> 16) & 0x7FFFu));
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, m);
}

__device__ __forceinline__ float nvfp4_global_scale(uint32_t amax_bits) {
    return amax_bits == 0 ? 1.0f : __fdiv_rn(__uint_as_float(amax_bits << 16), 2688.0f);
}

// Pass 2: one thread per 16-element group.  g_word holds the amax bits.
__global__ void __launch_bounds__(256)
nvfp4_quantize_kernel(const uint4 *__restrict__ w, int64_t groups, const unsigned int *g_word,
                      uint2 *__restrict__ packed, uint8_t *__restrict__ sb) {
    grid_dependency_wait();  // the amax pass
    // (no early start for the next kernel: this one writes weights)
    const float g = nvfp4_global_scale(*g_word);
    const float six_g = 6.0f * g;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < groups;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const uint4 v0 = __ldcs(w + 2 * i), v1 = __ldcs(w + 2 * i + 1);
        const uint32_t a[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        uint32_t ab = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) ab = max(ab, max(a[j] & 0x7FFFu, (a[j] >> 16) & 0x7FFFu));
        const float t = __fdiv_rn(__uint_as_float(ab << 16), six_g);
        const uint32_t code = e4m3x2_satfinite(t, 0.0f) & 0xFFu;
        const float sig = e4m3_to_float(code) * g;
        float x[16];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            x[2 * j] = __uint_as_float(a[j] << 16);
            x[2 * j + 1] = __uint_as_float(a[j] & 0xFFFF0000u);
        }
        float lo[8], hi[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            lo[j] = sig != 0.0f ? __fdiv_rn(x[j], sig) : 0.0f;
            hi[j] = sig != 0.0f ? __fdiv_rn(x[8 + j], sig) : 0.0f;
        }
        packed[i] = make_uint2(e2m1x8_satfinite(lo), e2m1x8_satfinite(hi));
        sb[i] = static_cast<uint8_t>(code);
    }
}

// Pass 3: the global scale itself.
__global__ void nvfp4_global_kernel(unsigned int *g_word) {
    grid_dependency_wait();  // every quantize block has read the amax bits
    const float g = nvfp4_global_scale(*g_word);
    *reinterpret_cast<float *>(g_word) = g;
}

// ---------------------------------------------------------------- GEMM

// Eight E2M1 codes (one 32-bit word, element 0 in the low nibble) -> eight BF16
// values scaled by s (a BF16 pair (s, s)): magnitude bytes from two 8-entry
// byte tables, sign from the code's top bit; the product by s is exact.
__device__ __forceinline__ uint4 e2m1x8_to_bf16_scaled(uint32_t w, __nv_bfloat162 s) {
    // high and low bytes of the BF16 values 0, 0.5, 1, 1.5, 2, 3, 4, 6
    constexpr uint32_t kHi0 = 0x3F3F3F00u, kHi1 = 0x40404040u;
    constexpr uint32_t kLo0 = 0xC0800000u, kLo1 = 0xC0804000u;
    const uint32_t mags = w & 0x77777777u;
    uint32_t out[4];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const uint32_t sel = (mags >> (16 * half)) & 0xFFFFu;
        const uint32_t hb = __byte_perm(kHi0, kHi1, sel);
        const uint32_t lb = __byte_perm(kLo0, kLo1, sel);
        const uint32_t wh = w >> (16 * half);
        // elements 4 half + {0, 1} and {2, 3}: bytes (lo, hi, lo, hi), sign bits at 15 and 31
        const uint32_t p01 = __byte_perm(lb, hb, 0x5140) | ((wh << 12) & 0x8000u) | ((wh << 24) & 0x80000000u);
        const uint32_t p23 = __byte_perm(lb, hb, 0x7362) | ((wh << 4) & 0x8000u) | ((wh << 16) & 0x80000000u);
        const __nv_bfloat162 a = __hmul2(*reinterpret_cast<const __nv_bfloat162 *>(&p01), s);
        const __nv_bfloat162 b = __hmul2(*reinterpret_cast<const __nv_bfloat162 *>(&p23), s);
        out[2 * half] = *reinterpret_cast<const uint32_t *>(&a);
        out[2 * half + 1] = *reinterpret_cast<const uint32_t *>(&b);
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

// grid (N/128 * S, ceil(M/16)); cluster (S, 1, 1) when S >= 2.
__global__ void __launch_bounds__(kNumThreads, 1)
nvfp4_gemm_a16_kernel(const __grid_constant__ CUtensorMap tmap_w,
                      const __grid_constant__ CUtensorMap tmap_s,
                      const __grid_constant__ CUtensorMap tmap_x, const float *__restrict__ g_ptr,
                      __nv_bfloat16 *__restrict__ y, int M, int N, int K, int cluster_s,
                      int *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Layout::kBarOff);
    uint64_t *empty = full + kStages;
    uint64_t *afull = empty + kStages;
    uint64_t *aempty = afull + kABufs;
    uint64_t *done = aempty + kABufs;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Layout::kMiscOff);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Layout::kMiscOff + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = K / BKU;
    const int S = cluster_s;
    const int nb = static_cast<int>(blockIdx.x) / S, r = static_cast<int>(blockIdx.x) % S;
    const int kb_begin = r * KB / S, kb_end = (r + 1) * KB / S;
    const int n_units = kb_end - kb_begin;
    const int m0 = static_cast<int>(blockIdx.y) * MT;

    allow_dependent_launch();
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < kABufs; ++a) {
            mbar_init(&afull[a], kDqWarps);
            mbar_init(&aempty[a], 1);
        }
        mbar_init(done, 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tmap(&tmap_w);
        prefetch_tmap(&tmap_s);
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
    grid_dependency_wait();

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t evict_first = l2_policy_evict_first();
            uint32_t stage = 0, phase = 0;
            for (int u = 0; u < n_units; ++u) {
                if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, status)) break;
                const int kb = kb_begin + u;
                uint8_t *st = smem + stage * Layout::kStage;
                mbar_arrive_expect_tx(&full[stage], Layout::kStage);
                tma_load_2d_hint(st, &tmap_w, &full[stage], kb * (BKU / 2), nb * BNW, evict_first);
                tma_load_2d_hint(st + Layout::kW, &tmap_s, &full[stage], kb * (BKU / 16), nb * BNW,
                                 evict_first);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    tma_load_2d(st + Layout::kW + Layout::kS + c * Layout::kXChunk, &tmap_x,
                                &full[stage], kb * BKU + c * 64, m0);
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            const int first = n_units > kStages ? n_units - kStages : 0;
            for (int u = first; u < n_units; ++u)
                mbar_wait(&full[u % kStages], static_cast<uint32_t>((u / kStages) & 1), nullptr, status);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = umma_idesc_bf16(BNW, MT);
            uint32_t stage = 0, phase = 0, abuf = 0, aphase = 0;
            uint32_t fresh = (1u << kNumAcc) - 1;  // accumulators not yet written
            for (int u = 0; u < n_units; ++u) {
                // one barrier pair and 16 back-to-back MMAs per unit: every shared-
                // memory wait after issued MMAs costs this thread ~0.1 us
                if (!mbar_wait(&afull[abuf], aphase, abort_flag, status) ||
                    !mbar_wait(&full[stage], phase, abort_flag, status))
                    break;
                tc_fence_after_sync();
                const uint32_t a_addr = smem_addr(smem + Layout::kAOff + abuf * Layout::kA);
                const uint32_t x_addr =
                    smem_addr(smem + stage * Layout::kStage + Layout::kW + Layout::kS);
#pragma unroll
                for (int c = 0; c < 4; ++c)        // four 64-k chunks
#pragma unroll
                    for (int k = 0; k < 4; ++k) {  // four K = 16 steps of 32 bytes
                        // consecutive steps go to different accumulators, so the
                        // MMAs are not one dependent chain over the whole K range
                        const int a = k % kNumAcc;
                        umma_bf16(tmem_base + a * MT,
                                  umma_desc_sw128(a_addr + c * Layout::kAChunk + 32 * k),
                                  umma_desc_sw128(x_addr + c * Layout::kXChunk + 32 * k), idesc,
                                  (fresh >> a) & 1u ? 0u : 1u);
                        fresh &= ~(1u << a);
                    }
                umma_commit(&aempty[abuf]);
                umma_commit(&empty[stage]);
                if (++abuf == kABufs) {
                    abuf = 0;
                    aphase ^= 1;
                }
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            umma_commit(done);
        }
    } else {
        // ------------------------------------------------------------ dequant
        // Thread (row r = dt mod 128, chunk q = dt / 128) of each unit: the 32
        // code bytes of k range [64 q, 64 q + 64) (two swizzled 16-byte pieces of
        // the packed row) and their 4 block scales -> 64 BF16 values, the row's
        // 8 pieces of A chunk q.  A warp covers 32 consecutive rows of one chunk,
        // so each store instruction fills all banks.
        const int dt = threadIdx.x - 64;  // 0..511
        const int row = dt & 127, q = dt >> 7;
        uint32_t stage = 0, phase = 0, abuf = 0, aphase = 0;
        for (int u = 0; u < n_units; ++u) {
            if (!mbar_wait(&full[stage], phase, abort_flag, status) ||
                !mbar_wait(&aempty[abuf], aphase ^ 1, abort_flag, status))
                break;
            const uint8_t *st = smem + stage * Layout::kStage;
            const uint4 *prow = reinterpret_cast<const uint4 *>(st + row * 128);
            const uint4 p0 = prow[(2 * q) ^ (row & 7)];
            const uint4 p1 = prow[(2 * q + 1) ^ (row & 7)];
            const uint32_t sc = *reinterpret_cast<const uint32_t *>(st + Layout::kW + row * 16 + 4 * q);
            __nv_bfloat162 s2[4];
#pragma unroll
            for (int gi = 0; gi < 4; ++gi) {
                const float sf = e4m3_to_float((sc >> (8 * gi)) & 0xFFu);
                s2[gi] = __floats2bfloat162_rn(sf, sf);
            }
            const uint32_t pw[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
            uint8_t *arow = smem + Layout::kAOff + abuf * Layout::kA + q * Layout::kAChunk + row * 128;
#pragma unroll
            for (int i = 0; i < 8; ++i)  // 8 codes -> one 16-byte piece of the A row
                *reinterpret_cast<uint4 *>(arow + ((i ^ (row & 7)) << 4)) =
                    e2m1x8_to_bf16_scaled(pw[i], s2[i >> 1]);
            fence_proxy_async_smem();  // generic writes -> tensor-core reads
            __syncwarp();
            if (lane == 0) mbar_arrive(&afull[abuf]);
            if (++abuf == kABufs) {
                abuf = 0;
                aphase ^= 1;
            }
            if (++stage == kStages) {
                stage = 0;
                phase ^= 1;
            }
        }
        // ------------------------------------------------------------ epilogue
        // warps 2..17: lanes of TMEM quarter (warp & 3); each of the 4 warps of
        // a quarter takes 4 of the 16 token columns
        const bool got = mbar_wait(done, 0, abort_flag, status);
        tc_fence_after_sync();
        const int quarter = warp & 3, col0 = ((warp - 2) >> 2) * 4;
        const int n_local = quarter * 32 + lane;
        float v[16];
        if (got) {
            // the accumulators summed in a fixed order (deterministic)
            tmem_load16(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16), v);
#pragma unroll
            for (int a = 1; a < kNumAcc; ++a) {
                float t[16];
                tmem_load16(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + a * MT, t);
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] += t[i];
            }
        }
        const float g = __ldg(g_ptr);
        float *red = reinterpret_cast<float *>(smem + Layout::kAOff);  // [MT][128], A tiles are idle
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int m = col0 + i;
            // static indices only, so v stays in registers
            const float vm = col0 == 0 ? v[i] : col0 == 4 ? v[4 + i] : col0 == 8 ? v[8 + i] : v[12 + i];
            const float acc = got ? vm * g : 0.0f;
            if (S == 1) {
                if (m0 + m < M)
                    y[static_cast<int64_t>(m0 + m) * N + nb * BNW + n_local] = __float2bfloat16_rn(acc);
            } else {
                red[m * BNW + n_local] = acc;
            }
        }
    }

    if (S > 1) {
        // ------------------------------------------------------------ cluster reduction
        __syncwarp();
        cluster_sync();
        const uint32_t red = smem_addr(smem + Layout::kAOff);
        const int rows = min(MT, M - m0);
        const int items = rows * (BNW / 4);
        const int i0 = r * items / S, i1 = (r + 1) * items / S;
        for (int item = i0 + static_cast<int>(threadIdx.x); item < i1; item += kNumThreads) {
            const int m = item / (BNW / 4), c4 = item % (BNW / 4);
            const uint32_t off = static_cast<uint32_t>((m * BNW + 4 * c4) * 4);
            float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int p = 0; p < S; ++p) {
                const float4 t = ld_shared_cluster_v4(map_to_cta(red + off, static_cast<uint32_t>(p)));
                sum.x += t.x;
                sum.y += t.y;
                sum.z += t.z;
                sum.w += t.w;
            }
            __nv_bfloat162 lo = __floats2bfloat162_rn(sum.x, sum.y);
            __nv_bfloat162 hi = __floats2bfloat162_rn(sum.z, sum.w);
            uint2 pk;
            pk.x = *reinterpret_cast<uint32_t *>(&lo);
            pk.y = *reinterpret_cast<uint32_t *>(&hi);
            *reinterpret_cast<uint2 *>(y + static_cast<int64_t>(m0 + m) * N + nb * BNW + 4 * c4) = pk;
        }
        __syncwarp();
        cluster_sync();
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}


// ---------------------------------------------------------------- GEMV (M <= 2)
//
// For a handful of tokens the tensor-core path above is bound by shared-memory
// traffic (a 4 KB BF16 tile per 512 codes, written and read again).  This
// kernel keeps the codes packed: each thread decodes its codes in registers
// (hardware E2M1 -> f16 conversion, then f32) and multiplies them with the
// activations on the CUDA cores, two k at a time (packed FP32 FMA), per
// 16-element group then times the block scale.  Same units, TMA ring, split
// and cluster reduction as the tensor-core kernel.
//   warp 0      TMA producer (codes 128-byte swizzled, scales, activation tile)
//   warp 1      converts each stage's BF16 activation tile to FP32 [MB][256]
//   warps 2..17 thread (row r = t mod 128, 64-k quarter q = t / 128): 64 codes
//               of its row per unit; a warp's lanes are 32 rows at the same k,
//               so the activation reads are shared-memory broadcasts.
template <int MB>
struct GemvLayout {
    static constexpr int kStages = 8;
    static constexpr int kW = BNW * BKU / 2;             // 16 KB codes
    static constexpr int kS = BNW * BKU / 16;            // 2 KB scales
    static constexpr int kXb = 2048;                     // BF16 [MB][256] (<= 2 KB)
    static constexpr int kXf = 4096;                     // FP32 [MB][256] (<= 4 KB)
    static constexpr int kStage = kW + kS + kXb + kXf;   // 24 KB
    static constexpr int kRedOff = kStages * kStage;     // [4][MB][128] FP32 quarter sums
    static constexpr int kBarOff = kRedOff + 4 * MB * BNW * 4;
    static constexpr int kNumBars = 3 * kStages;         // full, xready, empty
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kBytes = kMiscOff + 16 + 1024;
};
constexpr int kGemvComputeWarps = 16;
constexpr int kGemvThreads = 32 * (2 + kGemvComputeWarps);  // 576

template <int MB>
__global__ void __launch_bounds__(kGemvThreads, 1)
nvfp4_gemv_a16_kernel(const __grid_constant__ CUtensorMap tmap_w,
                      const __grid_constant__ CUtensorMap tmap_s,
                      const __grid_constant__ CUtensorMap tmap_x, const float *__restrict__ g_ptr,
                      __nv_bfloat16 *__restrict__ y, int M, int N, int K, int cluster_s,
                      int *status) {
    static_assert(MB == 1 || MB == 2, "token count bucket");
    using L = GemvLayout<MB>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kBarOff);
    uint64_t *xready = full + L::kStages;
    uint64_t *empty = xready + L::kStages;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOff);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = K / BKU;
    const int S = cluster_s;
    const int nb = static_cast<int>(blockIdx.x) / S, r = static_cast<int>(blockIdx.x) % S;
    const int kb_begin = r * KB / S, kb_end = (r + 1) * KB / S;
    const int n_units = kb_end - kb_begin;

    allow_dependent_launch();
    if (threadIdx.x == 0) {
        for (int st = 0; st < L::kStages; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&xready[st], 1);
            mbar_init(&empty[st], kGemvComputeWarps);
        }
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tmap(&tmap_w);
        prefetch_tmap(&tmap_s);
        prefetch_tmap(&tmap_x);
    }
    __syncthreads();
    grid_dependency_wait();

    float acc[MB];
#pragma unroll
    for (int m = 0; m < MB; ++m) acc[m] = 0.0f;
    const int ct = threadIdx.x - 64;  // compute thread 0..511
    const int row = ct & 127, q = ct >> 7;

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t evict_first = l2_policy_evict_first();
            uint32_t stage = 0, phase = 0;
            for (int u = 0; u < n_units; ++u) {
                if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, status)) break;
                const int kb = kb_begin + u;
                uint8_t *st = smem + stage * L::kStage;
                mbar_arrive_expect_tx(&full[stage], L::kW + L::kS + MB * BKU * 2);
                tma_load_2d_hint(st, &tmap_w, &full[stage], kb * (BKU / 2), nb * BNW, evict_first);
                tma_load_2d_hint(st + L::kW, &tmap_s, &full[stage], kb * (BKU / 16), nb * BNW,
                                 evict_first);
                tma_load_2d(st + L::kW + L::kS, &tmap_x, &full[stage], kb * BKU, 0);
                if (++stage == L::kStages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
    } else if (warp == 1) {
        uint32_t stage = 0, phase = 0;
        for (int u = 0; u < n_units; ++u) {
            if (!mbar_wait(&full[stage], phase, abort_flag, status)) break;
            uint8_t *st = smem + stage * L::kStage;
            const uint32_t *xb = reinterpret_cast<const uint32_t *>(st + L::kW + L::kS);
            float2 *xf = reinterpret_cast<float2 *>(st + L::kW + L::kS + L::kXb);
            for (int i = lane; i < MB * BKU / 2; i += 32) {  // BF16 pairs -> float pairs
                const uint32_t w = xb[i];
                xf[i] = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&xready[stage]);
            if (++stage == L::kStages) {
                stage = 0;
                phase ^= 1;
            }
        }
    } else {
        uint32_t stage = 0, phase = 0;
        for (int u = 0; u < n_units; ++u) {
            if (!mbar_wait(&xready[stage], phase, abort_flag, status)) break;
            const uint8_t *st = smem + stage * L::kStage;
            const uint4 *prow = reinterpret_cast<const uint4 *>(st + row * 128);
            const uint4 p0 = prow[(2 * q) ^ (row & 7)];
            const uint4 p1 = prow[(2 * q + 1) ^ (row & 7)];
            const uint32_t sc = *reinterpret_cast<const uint32_t *>(st + L::kW + row * 16 + 4 * q);
            const float *xf = reinterpret_cast<const float *>(st + L::kW + L::kS + L::kXb);
            const uint32_t pw[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
            for (int g = 0; g < 4; ++g) {  // 16-element groups, one block scale each
                float2 part[MB];
#pragma unroll
                for (int m = 0; m < MB; ++m) part[m] = make_float2(0.f, 0.f);
#pragma unroll
                for (int h = 0; h < 2; ++h) {  // two code words of 8
                    const uint32_t w = pw[2 * g + h];
                    const int k0 = 64 * q + 16 * g + 8 * h;
#pragma unroll
                    for (int b = 0; b < 4; ++b) {  // bytes: elements k0 + 2b, k0 + 2b + 1
                        const float2 wv = e2m1x2_to_float2(w >> (8 * b));
#pragma unroll
                        for (int m = 0; m < MB; ++m) {
                            const float2 xv = *reinterpret_cast<const float2 *>(xf + m * BKU + k0 + 2 * b);
                            part[m] = ffma2(wv, xv, part[m]);
                        }
                    }
                }
                const float s = e4m3_to_float((sc >> (8 * g)) & 0xFFu);
#pragma unroll
                for (int m = 0; m < MB; ++m) acc[m] = fmaf(s, part[m].x + part[m].y, acc[m]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (++stage == L::kStages) {
                stage = 0;
                phase ^= 1;
            }
        }
        // quarter sums of this row -> shared memory
        float *qs = reinterpret_cast<float *>(smem + L::kRedOff);
#pragma unroll
        for (int m = 0; m < MB; ++m) qs[(q * MB + m) * BNW + row] = acc[m];
    }
    __syncthreads();

    // the CTA's partial [MB][128]: quarters summed in order, times g
    const float g = __ldg(g_ptr);
    float *part = reinterpret_cast<float *>(smem);  // ring memory is idle now
    if (threadIdx.x < MB * BNW) {
        const int m = threadIdx.x / BNW, n = threadIdx.x % BNW;
        const float *qs = reinterpret_cast<const float *>(smem + L::kRedOff);
        float v = 0.0f;
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) v += qs[(qq * MB + m) * BNW + n];
        v *= g;
        if (S == 1) {
            if (m < M) y[static_cast<int64_t>(m) * N + nb * BNW + n] = __float2bfloat16_rn(v);
        } else {
            part[m * BNW + n] = v;
        }
    }
    if (S > 1) {
        __syncwarp();
        cluster_sync();
        const uint32_t red = smem_addr(part);
        const int items = M * (BNW / 4);
        const int i0 = r * items / S, i1 = (r + 1) * items / S;
        for (int item = i0 + static_cast<int>(threadIdx.x); item < i1; item += kGemvThreads) {
            const int m = item / (BNW / 4), c4 = item % (BNW / 4);
            const uint32_t off = static_cast<uint32_t>((m * BNW + 4 * c4) * 4);
            float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int p = 0; p < S; ++p) {
                const float4 t = ld_shared_cluster_v4(map_to_cta(red + off, static_cast<uint32_t>(p)));
                sum.x += t.x;
                sum.y += t.y;
                sum.z += t.z;
                sum.w += t.w;
            }
            __nv_bfloat162 lo = __floats2bfloat162_rn(sum.x, sum.y);
            __nv_bfloat162 hi = __floats2bfloat162_rn(sum.z, sum.w);
            uint2 pk;
            pk.x = *reinterpret_cast<uint32_t *>(&lo);
            pk.y = *reinterpret_cast<uint32_t *>(&hi);
            *reinterpret_cast<uint2 *>(y + static_cast<int64_t>(m) * N + nb * BNW + 4 * c4) = pk;
        }
        __syncwarp();
        cluster_sync();
    }
}

}  // namespace nvfp4
}  // namespace fp8bq
