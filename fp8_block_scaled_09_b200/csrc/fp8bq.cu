// fp8bq.cu -- the C ABI declared in include/fp8bq.h: host-side argument
// validation, per-device set-up, TMA descriptor encoding and kernel dispatch.
//
// All kernels live in this one translation unit so the device status word is a
// single per-device symbol.  Dispatch:
//   quantize_act     -> up to 8192 groups: quantize_act_small_kernel (no shared
//                       memory, fits beside a running GEMM); larger:
//                       quantize_act_kernel (HBM-bound, persistent, bulk-copy ring)
//   quantize_weight  -> quantize_weight_kernel (one CTA per 128x128 block)
//   gemm, M <= 128   -> decode::gemm_decode_kernel<MT> (token tile MT = 16, 32,
//                       64 or 128; each n-block split over a cluster of CTAs
//                       reduced in shared memory, or stream-K over all weight
//                       blocks with a global split-K reduction)
//   gemm, M > 128    -> prefill::gemm_prefill_kernel<256, false, 16|32> (persistent tcgen05;
//                       the CTA-pair kernel prefill2 only with FP8BQ_PREFILL_PAIRS=1)
//   kv_write_e4m3    -> kv_write_e4m3_kernel (warp per K/V row, slot scatter)
//   nvfp4_quantize_weight -> nvfp4 amax, quantize and global-scale kernels
//   nvfp4_gemm_a16   -> M <= 2: nvfp4::nvfp4_gemv_a16_kernel<1|2> (codes decoded in
//                       registers, CUDA-core FMA); larger M: nvfp4::nvfp4_gemm_a16_kernel
//                       (BF16 dequant into shared memory + tcgen05 kind::f16)
//   silu_mul_quantize-> silu_mul_quantize_kernel (half-warp per 128-channel group) or,
//                       for large problems, silu_mul_quantize_wide_kernel (8-lane teams)
//   gemm_silu_mul_quantize -> M > 128: prefill::gemm_prefill_kernel<256, true, 16|32>
//                       (gate/up GEMM whose epilogue quantizes silu(gate) * up);
//                       smaller M: the decode GEMM, then silu_mul_quantize
//   linear           -> quantize_act into the workspace, then the gemm path; the
//                       decode kernel then streams its first weight blocks while
//                       the quantizer still runs (programmatic dependent launch)
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <unordered_map>
#include <utility>

#include "fp8bq.h"
#include "gemm_decode.cuh"
#include "gemm_prefill.cuh"
#include "gemm_prefill2.cuh"
#include "ptx.cuh"
#include "kv_cache.cuh"
#include "nvfp4.cuh"
#include "quantize.cuh"
#include "silu_quant.cuh"

namespace fp8bq {

// Per-device status word: FP8BQ_OK or FP8BQ_ERR_TIMEOUT (set by a kernel that
// abandoned a wait).  Read and cleared by fp8bq_last_device_status().
__device__ int g_status;

// Waits on a barrier that nothing ever arrives on: the bounded wait gives up
// after limit_ns and records FP8BQ_ERR_TIMEOUT (exercises the failure path
// every kernel uses, without faulting or hanging the GPU).
__global__ void selftest_timeout_kernel(int *status, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
}

namespace {

constexpr int kMaxDevices = 64;
constexpr int kPrefillBN = 256;
// The CTA-pair prefill kernel is correct and, moving 2/3 of the operand bytes,
// runs exactly as fast as the single-CTA kernel (both are bound by the
// per-chunk TMEM hand-off, not by L2), and no faster under the power cap; the
// single-CTA kernel is the one dispatched unless the environment variable
// FP8BQ_PREFILL_PAIRS=1 selects the pair kernel (read once per device).
bool pair_prefill_requested() {
    const char *v = std::getenv("FP8BQ_PREFILL_PAIRS");
    return v != nullptr && v[0] == '1' && v[1] == '\0';
}
constexpr int64_t kDecodeMaxM = decode::kMaxMT;

std::atomic<uint64_t> g_launches{0};

struct DeviceInfo {
    int sm_count = 0;
    int pair_clusters = 0;  // co-resident 2-CTA clusters of the pair prefill kernel
    // co-resident decode clusters of each size 2..8 (one CTA per SM at full
    // shared memory); the decode plan only uses sizes whose clusters all fit
    int cluster_capacity[9] = {};
    int nvfp4_cluster_capacity[9] = {};  // the same for the NVFP4 A16 GEMM
    int *status = nullptr;  // device address of g_status
    bool supported = false;
};

DeviceInfo g_dev[kMaxDevices];
std::once_flag g_dev_once[kMaxDevices];

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

EncodeTiledFn encode_fn() {
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    });
    return g_encode;
}

// Sets the prefill kernel variant's shared-memory limit and checks that it was
// built with the register count its setmaxnreg split assumes.
template <bool kSilu>
bool prefill_instance_ready(void (*k)(CUtensorMap, CUtensorMap, const float *, const float *,
                                      __nv_bfloat16 *, int, int, int, int *, int, float *, int *,
                                      prefill::SiluOut)) {
    cudaFuncAttributes fa;
    return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                prefill::Layout<kPrefillBN, kSilu>::kDynamicSmem) == cudaSuccess &&
           cudaFuncGetAttributes(&fa, k) == cudaSuccess && fa.numRegs == prefill::kLaunchRegs;
}

// The prefill kernel instance for a K (raster group of prefill::group_m(K/128)
// m-tiles).
template <bool kSilu>
auto prefill_kernel_for(int64_t K) {
    return prefill::group_m(static_cast<int>(K / 128)) == 32
               ? prefill::gemm_prefill_kernel<kPrefillBN, kSilu, 32>
               : prefill::gemm_prefill_kernel<kPrefillBN, kSilu, 16>;
}

template <bool kSilu>
bool prefill_variant_ready() {
    return prefill_instance_ready<kSilu>(prefill::gemm_prefill_kernel<kPrefillBN, kSilu, 16>) &&
           prefill_instance_ready<kSilu>(prefill::gemm_prefill_kernel<kPrefillBN, kSilu, 32>);
}

// Current device's info, set up once per device (kernel attributes, status word).
const DeviceInfo *device_info() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::call_once(g_dev_once[dev], [dev] {
        DeviceInfo &d = g_dev[dev];
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return;
        if (major != 10 || minor != 0) return;  // built for sm_100a only
        if (cudaGetSymbolAddress(reinterpret_cast<void **>(&d.status), g_status) != cudaSuccess)
            return;
        if (cudaMemset(d.status, 0, sizeof(int)) != cudaSuccess) return;
        // The prefill kernel moves registers between warpgroups with setmaxnreg;
        // the split is only safe if the launch allocates exactly what it was
        // designed for (otherwise setmaxnreg.inc could wait forever).
        cudaFuncAttributes fa;
        if (!prefill_variant_ready<false>() || !prefill_variant_ready<true>()) return;
        // CTA-pair prefill kernel: optional; any failure here only leaves it off.
        d.pair_clusters = 0;
        if (pair_prefill_requested() &&
            cudaFuncSetAttribute(prefill2::gemm_prefill_pair_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 prefill2::Layout::kDynamicSmem) == cudaSuccess &&
            cudaFuncGetAttributes(&fa, prefill2::gemm_prefill_pair_kernel) == cudaSuccess &&
            fa.numRegs == prefill2::kLaunchRegs) {
            // how many 2-CTA clusters fit at once: the persistent pair grid size
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(2 * (d.sm_count / 2));
            cfg.blockDim = dim3(prefill2::kNumThreads);
            cfg.dynamicSmemBytes = prefill2::Layout::kDynamicSmem;
            cudaLaunchAttribute at[1];
            at[0].id = cudaLaunchAttributeClusterDimension;
            at[0].val.clusterDim.x = 2;
            at[0].val.clusterDim.y = 1;
            at[0].val.clusterDim.z = 1;
            cfg.attrs = at;
            cfg.numAttrs = 1;
            if (cudaOccupancyMaxActiveClusters(&d.pair_clusters, prefill2::gemm_prefill_pair_kernel,
                                               &cfg) != cudaSuccess)
                d.pair_clusters = 0;
            cudaGetLastError();  // clear a failed query
        }
        if (cudaFuncSetAttribute(quantize_act_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 ActLayout::kBytes) != cudaSuccess)
            return;
        if (cudaFuncSetAttribute(decode::gemm_decode_kernel<16>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 decode::kMaxSmem) != cudaSuccess ||
            cudaFuncSetAttribute(decode::gemm_decode_kernel<32>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 decode::kMaxSmem) != cudaSuccess ||
            cudaFuncSetAttribute(decode::gemm_decode_kernel<64>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 decode::kMaxSmem) != cudaSuccess ||
            cudaFuncSetAttribute(decode::gemm_decode_kernel<128>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 decode::kMaxSmem) != cudaSuccess)
            return;
        // How many clusters of decode CTAs (one per SM at full shared memory)
        // the GPU can hold at once, per cluster size.
        for (int c = 2; c <= 8; ++c) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(static_cast<unsigned>(c));
            cfg.blockDim = dim3(decode::Roles<128>::kNumThreads);
            cfg.dynamicSmemBytes = decode::kMaxSmem;
            cudaLaunchAttribute at[1];
            at[0].id = cudaLaunchAttributeClusterDimension;
            at[0].val.clusterDim.x = static_cast<unsigned>(c);
            at[0].val.clusterDim.y = 1;
            at[0].val.clusterDim.z = 1;
            cfg.attrs = at;
            cfg.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, decode::gemm_decode_kernel<128>, &cfg) != cudaSuccess)
                n = 0;
            cudaGetLastError();  // clear a failed query
            d.cluster_capacity[c] = n;
        }
        if (cudaFuncSetAttribute(nvfp4::nvfp4_gemm_a16_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 nvfp4::Layout::kBytes) != cudaSuccess ||
            cudaFuncSetAttribute(nvfp4::nvfp4_gemv_a16_kernel<1>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 nvfp4::GemvLayout<1>::kBytes) != cudaSuccess ||
            cudaFuncSetAttribute(nvfp4::nvfp4_gemv_a16_kernel<2>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 nvfp4::GemvLayout<2>::kBytes) != cudaSuccess)
            return;
        for (int c = 2; c <= 8; ++c) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(static_cast<unsigned>(c));
            cfg.blockDim = dim3(nvfp4::kNumThreads);
            cfg.dynamicSmemBytes = nvfp4::Layout::kBytes;
            cudaLaunchAttribute at[1];
            at[0].id = cudaLaunchAttributeClusterDimension;
            at[0].val.clusterDim.x = static_cast<unsigned>(c);
            at[0].val.clusterDim.y = 1;
            at[0].val.clusterDim.z = 1;
            cfg.attrs = at;
            cfg.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, nvfp4::nvfp4_gemm_a16_kernel, &cfg) != cudaSuccess)
                n = 0;
            cudaGetLastError();
            d.nvfp4_cluster_capacity[c] = n;
        }
        if (cudaDeviceSynchronize() != cudaSuccess) return;
        d.supported = true;
    });
    const DeviceInfo *d = &g_dev[dev];
    return d->supported ? d : nullptr;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int64_t kMaxDim = 0x7FFFFFFF;
constexpr int64_t kMaxBytes = int64_t(1) << 40;

fp8bq_status check_mk(int64_t M, int64_t K) {
    if (M < 0 || K <= 0) return FP8BQ_ERR_UNSUPPORTED_SHAPE;
    if (K % 128 != 0 || M > kMaxDim || K > kMaxDim) return FP8BQ_ERR_UNSUPPORTED_SHAPE;
    if (M > 0 && K > kMaxBytes / 2 / M) return FP8BQ_ERR_UNSUPPORTED_SHAPE;  // BF16 [M, K]
    return FP8BQ_OK;
}

fp8bq_status check_mnk(int64_t M, int64_t N, int64_t K) {
    fp8bq_status st = check_mk(M, K);
    if (st != FP8BQ_OK) return st;
    if (N <= 0 || N % 128 != 0 || N > kMaxDim) return FP8BQ_ERR_UNSUPPORTED_SHAPE;
    if (N > kMaxBytes / K) return FP8BQ_ERR_UNSUPPORTED_SHAPE;             // codes [N, K]
    if (M > 0 && N > kMaxBytes / 2 / M) return FP8BQ_ERR_UNSUPPORTED_SHAPE;  // BF16 [M, N]
    return FP8BQ_OK;
}

fp8bq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? FP8BQ_OK : FP8BQ_ERR_CUDA; }

// Every kernel is launched with programmatic stream serialization: it may be
// scheduled while the previous kernel in the stream finishes, runs its
// prologue (barrier set-up, TMEM allocation), and waits (griddepcontrol.wait)
// before touching global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_clustered(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t st, unsigned cluster_x, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cluster_x > 1) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = cluster_x;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.numAttrs = 2;
    }
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    if (e == cudaSuccess) g_launches.fetch_add(1, std::memory_order_relaxed);
    return e;
}

template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                   Args &&...args) {
    return launch_clustered(kernel, grid, block, smem, st, 1u, std::forward<Args>(args)...);
}

// Encoded tensor maps, keyed on everything the encoding depends on (address,
// shape, element type, box and swizzle): an entry is valid for any tensor that
// matches its key, whatever that memory held before, so entries never go stale.
// Bounded; fp8bq_clear_cache() empties it.
struct TmapKey {
    uintptr_t ptr;
    int64_t rows, cols;
    uint32_t box_cols, box_rows;
    int type, elem_bytes, swizzle;
    bool operator==(const TmapKey &o) const {
        return ptr == o.ptr && rows == o.rows && cols == o.cols && box_cols == o.box_cols &&
               box_rows == o.box_rows && type == o.type && elem_bytes == o.elem_bytes &&
               swizzle == o.swizzle;
    }
};
struct TmapKeyHash {
    size_t operator()(const TmapKey &k) const {
        uint64_t h = static_cast<uint64_t>(k.ptr) * 0x9E3779B97F4A7C15ull;
        const uint64_t parts[5] = {static_cast<uint64_t>(k.rows), static_cast<uint64_t>(k.cols),
                                   (static_cast<uint64_t>(k.box_cols) << 32) | k.box_rows,
                                   (static_cast<uint64_t>(k.type) << 16) |
                                       static_cast<uint64_t>(k.elem_bytes),
                                   static_cast<uint64_t>(k.swizzle)};
        for (uint64_t p : parts) h = (h ^ p) * 0x100000001B3ull;
        return static_cast<size_t>(h ^ (h >> 29));
    }
};
constexpr size_t kTmapCacheMax = 4096;
std::mutex g_tmap_mu;
std::unordered_map<TmapKey, CUtensorMap, TmapKeyHash> g_tmap_cache;

// 2-D tensor map over a row-major [rows, cols] matrix of `type` (elem_bytes each),
// box [box_rows, box_cols], zero fill out of bounds.
bool make_tmap_2d(CUtensorMap *map, const void *ptr, CUtensorMapDataType type, int elem_bytes,
                  int64_t rows, int64_t cols, uint32_t box_cols, uint32_t box_rows,
                  CUtensorMapSwizzle swizzle) {
    const TmapKey key{reinterpret_cast<uintptr_t>(ptr), rows, cols, box_cols, box_rows,
                      static_cast<int>(type), elem_bytes, static_cast<int>(swizzle)};
    {
        std::lock_guard<std::mutex> lk(g_tmap_mu);
        auto it = g_tmap_cache.find(key);
        if (it != g_tmap_cache.end()) {
            *map = it->second;
            return true;
        }
    }
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols * elem_bytes)};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t elem[2] = {1u, 1u};
    std::memset(map, 0, sizeof(*map));
    if (enc(map, type, 2, const_cast<void *>(ptr), dims, strides, box, elem,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    std::lock_guard<std::mutex> lk(g_tmap_mu);
    if (g_tmap_cache.size() >= kTmapCacheMax) g_tmap_cache.clear();
    g_tmap_cache.emplace(key, *map);
    return true;
}

// 2-D uint8 tensor map over a row-major [rows, cols] byte matrix, box
// [box_rows, 128 bytes], 128-byte swizzle, zero fill out of bounds.
bool make_tmap(CUtensorMap *map, const void *ptr, int64_t rows, int64_t cols, uint32_t box_rows) {
    return make_tmap_2d(map, ptr, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, rows, cols, 128u, box_rows,
                        CU_TENSOR_MAP_SWIZZLE_128B);
}

size_t round256(int64_t b) { return static_cast<size_t>(((b + 255) / 256) * 256); }

// The decode kernel takes M <= 128 as long as its staged scales leave room for
// at least kMinStages ring slots (for M <= 16, K up to roughly 1.4e5; for
// M > 64, up to roughly 2.6e4); anything else runs on the prefill kernel.
// Decode grid: one CTA per SM, but at least kMinUnitsPerCta weight blocks per
// CTA so small problems do not split every n-block across many CTAs.
constexpr int64_t kMinUnitsPerCta = 4;
int64_t decode_grid(int64_t units, int64_t sms) {
    const int64_t by_work = (units + kMinUnitsPerCta - 1) / kMinUnitsPerCta;
    return std::max<int64_t>(1, std::min<int64_t>(std::min<int64_t>(sms, decode::kMaxGrid), by_work));
}

// How the decode kernel runs one shape: grid, ring stages (0: the decode
// kernel does not apply) and cluster size (0: stream-K over the whole grid;
// S >= 1: n-block nb on CTAs [nb S, nb S + S), one cluster of S when S >= 2).
struct DecodePlan {
    int64_t grid = 0;
    int stages = 0;
    int cluster_s = 0;
};

template <int MT>
int pick_stages_for(int64_t KB, int64_t upc) {
    return decode::pick_stages<MT>(KB, upc);
}

int pick_stages_mt(int MT, int64_t KB, int64_t upc) {
    switch (MT) {
        case 16: return pick_stages_for<16>(KB, upc);
        case 32: return pick_stages_for<32>(KB, upc);
        case 64: return pick_stages_for<64>(KB, upc);
        default: return pick_stages_for<128>(KB, upc);
    }
}

// Chooses between the two modes with a cost model fitted to globaltimer traces
// of this kernel: a unit (one 16 KB weight block) takes ~0.35 us per CTA
// (~0.5 us with a 128-row token tile); stream-K adds ~4.4 us (~6 us) of tail
// for its global split-K reduction, the cluster mode ~1 us (0.3 us when each
// CTA owns a whole n-block).
DecodePlan decode_plan(const DeviceInfo &d, int64_t M, int64_t N, int64_t K) {
    DecodePlan p;
    if (M > kDecodeMaxM || N / 128 > decode::kMaxCounters) return p;
    const int64_t NB = N / 128, KB = K / 128, U = NB * KB, sms = d.sm_count;
    const int MT = decode::token_tile(M);
    const double t_unit = MT == 128 ? 0.5 : 0.35, tail_sk = MT == 128 ? 6.0 : 4.4;
    const int64_t g_sk = decode_grid(U, sms);
    const int64_t upc_sk = (U + g_sk - 1) / g_sk;
    const double cost_sk = upc_sk * t_unit + tail_sk;
    if (NB <= sms) {
        // largest S <= 8 whose NB clusters are all co-resident, with a unit each
        int64_t S = std::min<int64_t>(std::min<int64_t>(8, sms / NB), KB);
        while (S >= 2 && NB > d.cluster_capacity[S]) --S;
        S = std::max<int64_t>(S, 1);
        const int64_t upc_c = (KB + S - 1) / S;
        const double cost_c = upc_c * t_unit + (S > 1 ? 1.0 : 0.3);
        const int st_c = pick_stages_mt(MT, KB, upc_c);
        // the cluster reduction keeps the [MT][128] FP32 partial in the ring
        const bool ring_holds_partial =
            st_c > 0 && static_cast<int64_t>(st_c) * decode::kStageBytes(MT) >= int64_t(MT) * 128 * 4;
        if (ring_holds_partial && cost_c <= cost_sk) {
            p.grid = NB * S;
            p.stages = st_c;
            p.cluster_s = static_cast<int>(S);
            return p;
        }
    }
    p.grid = g_sk;
    p.stages = pick_stages_mt(MT, KB, upc_sk);
    p.cluster_s = 0;
    return p;
}

// Workspace the GEMM requires: the decode path's, whenever that path may be
// chosen (the choice needs the device's SM count; the size does not).
size_t gemm_ws_bytes(int64_t M, int64_t N) {
    if (M <= kDecodeMaxM && N / 128 <= decode::kMaxCounters)
        return round256(decode::workspace_bytes(N / 128, decode::token_tile(M)));
    return 0;
}

// Prefill split-K tail: the counter header, then kTailMaxTiles x kTailMaxParts
// FP32 partial tiles.  Optional: a smaller workspace runs without the split.
constexpr size_t kPrefillTailBytes =
    size_t(decode::kCounterBytes) +
    size_t(prefill::kTailMaxTiles) * prefill::kTailMaxParts * prefill::kTailPartialFloats * 4;

constexpr int64_t kPrefillTailMinKB = 128;  // K >= 16384

// Split-K tail parts of the prefill kernel for a grid over `tiles` tiles (0:
// no split): a last wave of at most kTailMaxTiles tiles leaves most SMs idle,
// so each of its tiles is split K-wise into up to kTailMaxParts parts.
// Measured: it pays for long K (M=4096, N=7168: K=21504 681 -> 631 us) but not
// for K=8192 (269 -> 278 us), where the partial hand-off outweighs it.
int prefill_tail_parts(int64_t tiles, int grid, int64_t KB, const void *ws, size_t ws_bytes) {
    const int64_t rest = tiles % grid;
    int parts = 0;
    if (ws != nullptr && aligned16(ws) && ws_bytes >= kPrefillTailBytes && tiles > grid && rest >= 1 &&
        rest <= prefill::kTailMaxTiles && KB >= kPrefillTailMinKB)
        parts = static_cast<int>(std::min<int64_t>(std::min<int64_t>(prefill::kTailMaxParts, grid / rest), KB));
    return parts < 2 ? 0 : parts;
}


// Workspace fp8bq_workspace_size reports: what the GEMM requires, or for the
// prefill path what its split-K tail can use (only at K >= 16384; whether the
// last wave is short enough to split also depends on the SM count, which the
// size query does not need).
size_t gemm_ws_bytes_full(int64_t M, int64_t N, int64_t K) {
    const size_t need = gemm_ws_bytes(M, N);
    const bool tail = M > kDecodeMaxM && K / 128 >= kPrefillTailMinKB;
    return tail ? std::max(need, round256(kPrefillTailBytes)) : need;
}

size_t act_ws_bytes(int64_t M, int64_t K) { return round256(M * K) + round256(M * (K / 128) * 4); }

// The fused linear's workspace holds the GEMM's part first, never shorter than
// the counter header, then the activation codes and scales (plain scratch).
// So the split-K counters sit at offset 0 of every workspace, whatever the
// operation and shape, and one workspace can serve any sequence of calls.
size_t linear_gemm_part(int64_t M, int64_t N, int64_t K, bool with_tail) {
    const size_t g = with_tail ? gemm_ws_bytes_full(M, N, K) : gemm_ws_bytes(M, N);
    return std::max(g, static_cast<size_t>(decode::kCounterBytes));
}

// ---------------------------------------------------------------- launches

// Up to this many groups (M <= 128 at K = 7168) the shared-memory-free
// quantizer runs instead of the bulk-copy one.
constexpr int64_t kSmallActMaxGroups = 8192;

cudaError_t launch_quantize_act(const DeviceInfo &d, const void *x, int64_t M, int64_t K,
                                uint8_t *q, float *sa, cudaStream_t st) {
    const int64_t groups = M * (K / 128);
    if (groups <= kSmallActMaxGroups)
        return launch(quantize_act_small_kernel,
                      dim3(static_cast<unsigned>((groups + kSmallActGroupsPerCta - 1) /
                                                 kSmallActGroupsPerCta)),
                      dim3(kSmallActThreads), 0, st, static_cast<const uint4 *>(x), groups,
                      reinterpret_cast<uint2 *>(q), sa);
    const int64_t chunks = (groups + kActChunkGroups - 1) / kActChunkGroups;
    const int64_t max_ctas = static_cast<int64_t>(d.sm_count) * kActCtasPerSm;
    const int blocks = static_cast<int>(std::min(chunks, max_ctas));
    return launch(quantize_act_kernel, dim3(blocks), dim3(kActThreads), ActLayout::kBytes, st,
                  static_cast<const uint8_t *>(x), groups, reinterpret_cast<uint2 *>(q), sa,
                  d.status);
}

template <int MT>
cudaError_t launch_decode(const DeviceInfo &d, const uint8_t *qa, const float *sa,
                          const uint8_t *qw, const float *sw, int64_t M, int64_t N, int64_t K,
                          void *y, void *ws, cudaStream_t st, fp8bq_status *err,
                          bool early_weights, const DecodePlan &plan) {
    CUtensorMap tw, tx;
    if (!make_tmap(&tw, qw, N, K, decode::BNW) || !make_tmap(&tx, qa, M, K, MT)) {
        *err = FP8BQ_ERR_CUDA;
        return cudaSuccess;
    }
    const int64_t KB = K / 128, units = (N / 128) * KB;
    const int64_t upc = plan.cluster_s > 0 ? (KB + plan.cluster_s - 1) / plan.cluster_s
                                           : (units + plan.grid - 1) / plan.grid;
    int *counters = static_cast<int *>(ws);
    float *partials =
        ws ? reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + decode::kCounterBytes) : nullptr;
    const int64_t smem = decode::smem_bytes<MT>(plan.stages, KB, upc);
    return launch_clustered(decode::gemm_decode_kernel<MT>, dim3(static_cast<unsigned>(plan.grid)),
                            dim3(decode::Roles<MT>::kNumThreads), static_cast<size_t>(smem), st,
                            plan.cluster_s > 1 ? static_cast<unsigned>(plan.cluster_s) : 1u, tw, tx,
                            sa, sw, static_cast<__nv_bfloat16 *>(y), static_cast<int>(M),
                            static_cast<int>(N), static_cast<int>(K), counters, partials, d.status,
                            early_weights ? 1 : 0, plan.stages, plan.cluster_s);
}

// early_weights: the decode kernel may request its first weight blocks before
// its dependency wait (only valid right after this library's activation
// quantizer, while the GEMM before it may still be running; see
// gemm_decode.cuh).
// ws_bytes: usable workspace bytes (the prefill path splits its last wave of
// tiles K-wise when they hold kPrefillTailBytes).
cudaError_t launch_gemm(const DeviceInfo &d, const uint8_t *qa, const float *sa,
                        const uint8_t *qw, const float *sw, int64_t M, int64_t N, int64_t K,
                        void *y, void *ws, size_t ws_bytes, cudaStream_t st, fp8bq_status *err,
                        bool early_weights = false, bool allow_decode = true) {
    *err = FP8BQ_OK;
    const DecodePlan plan = decode_plan(d, M, N, K);
    if (plan.stages > 0 && (allow_decode || plan.cluster_s > 0)) {
        switch (decode::token_tile(M)) {
            case 16:
                return launch_decode<16>(d, qa, sa, qw, sw, M, N, K, y, ws, st, err, early_weights, plan);
            case 32:
                return launch_decode<32>(d, qa, sa, qw, sw, M, N, K, y, ws, st, err, early_weights, plan);
            case 64:
                return launch_decode<64>(d, qa, sa, qw, sw, M, N, K, y, ws, st, err, early_weights, plan);
            default:
                return launch_decode<128>(d, qa, sa, qw, sw, M, N, K, y, ws, st, err, early_weights, plan);
        }
    } else if (d.pair_clusters > 0 && M > prefill::BM) {
        // CTA pairs: each CTA loads 128 rows of A and 128 of the 256 weight rows
        CUtensorMap ta, tb;
        if (!make_tmap(&ta, qa, M, K, prefill2::kHalf) || !make_tmap(&tb, qw, N, K, prefill2::kHalf)) {
            *err = FP8BQ_ERR_CUDA;
            return cudaSuccess;
        }
        const int64_t tiles = ((M + prefill2::BM - 1) / prefill2::BM) *
                              ((N + prefill2::BN - 1) / prefill2::BN);
        const int64_t pairs = std::min<int64_t>(tiles, d.pair_clusters);
        return launch_clustered(prefill2::gemm_prefill_pair_kernel, dim3(static_cast<unsigned>(2 * pairs)),
                                dim3(prefill2::kNumThreads), prefill2::Layout::kDynamicSmem, st, 2u,
                                ta, tb, sa, sw, static_cast<__nv_bfloat16 *>(y), static_cast<int>(M),
                                static_cast<int>(N), static_cast<int>(K), d.status);
    } else {
        CUtensorMap ta, tb;
        if (!make_tmap(&ta, qa, M, K, prefill::BM) || !make_tmap(&tb, qw, N, K, kPrefillBN)) {
            *err = FP8BQ_ERR_CUDA;
            return cudaSuccess;
        }
        const int64_t tiles = ((M + prefill::BM - 1) / prefill::BM) * ((N + kPrefillBN - 1) / kPrefillBN);
        const int grid = static_cast<int>(tiles < d.sm_count ? tiles : d.sm_count);
        const int tail_parts = prefill_tail_parts(tiles, grid, K / 128, ws, ws_bytes);
        int *tail_counters = tail_parts ? static_cast<int *>(ws) : nullptr;
        float *tail_partials =
            tail_parts ? reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + decode::kCounterBytes)
                       : nullptr;
        return launch(prefill_kernel_for<false>(K), dim3(grid),
                      dim3(prefill::kNumThreads), prefill::Layout<kPrefillBN, false>::kDynamicSmem,
                      st, ta, tb, sa, sw, static_cast<__nv_bfloat16 *>(y), static_cast<int>(M),
                      static_cast<int>(N), static_cast<int>(K), d.status, tail_parts,
                      tail_partials, tail_counters, prefill::SiluOut{nullptr, nullptr, nullptr});
    }
}

// Gate/up GEMM with the SiLU-gated product quantized in its epilogue (M > 128):
// the prefill kernel with tiles of 128 gate and the same 128 up channels.
cudaError_t launch_gemm_silu(const DeviceInfo &d, const uint8_t *qa, const float *sa,
                             const uint8_t *qw, const float *sw, int64_t M, int64_t I, int64_t K,
                             uint8_t *q, float *s, void *h, cudaStream_t st, fp8bq_status *err) {
    *err = FP8BQ_OK;
    CUtensorMap ta, tb;
    if (!make_tmap(&ta, qa, M, K, prefill::BM) || !make_tmap(&tb, qw, 2 * I, K, 128)) {
        *err = FP8BQ_ERR_CUDA;
        return cudaSuccess;
    }
    const int64_t tiles = ((M + prefill::BM - 1) / prefill::BM) * (I / 128);
    const int grid = static_cast<int>(tiles < d.sm_count ? tiles : d.sm_count);
    return launch(prefill_kernel_for<true>(K), dim3(grid),
                  dim3(prefill::kNumThreads), prefill::Layout<kPrefillBN, true>::kDynamicSmem, st,
                  ta, tb, sa, sw, static_cast<__nv_bfloat16 *>(nullptr), static_cast<int>(M),
                  static_cast<int>(2 * I), static_cast<int>(K), d.status, 0,
                  static_cast<float *>(nullptr), static_cast<int *>(nullptr),
                  prefill::SiluOut{q, s, static_cast<__nv_bfloat16 *>(h)});
}

// Workspace of the gate/up GEMM with the SiLU epilogue: none on the fused
// path (M > 128); otherwise the decode GEMM's, then the BF16 gate/up output
// [M, 2I] that the separate SiLU kernel reads.
size_t silu_ws_bytes(int64_t M, int64_t I) {
    if (M > kDecodeMaxM) return 0;
    return std::max(gemm_ws_bytes(M, 2 * I), static_cast<size_t>(decode::kCounterBytes)) +
           round256(M * 2 * I * 2);
}

}  // namespace
}  // namespace fp8bq

// ---------------------------------------------------------------- allocation-free GEMM
// Scratch for fp8bq_gemm_noalloc: a file-scope device array, so callers that
// cannot allocate device memory need not supply a workspace.  Every GPU that
// loads this library holds it until the process exits.
namespace fp8bq {
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];
// Device address of the array per device, kept once a lookup has succeeded; a
// failed lookup is not remembered, so a later call tries again.
std::atomic<void *> g_noalloc_ptr[kMaxDevices];
std::mutex g_noalloc_mu;

// The array's device address on device `dev` (current), or null.  In host code
// the array's name is only a host-side stand-in, never a device address.
void *noalloc_scratch(int dev) {
    void *p = g_noalloc_ptr[dev].load(std::memory_order_acquire);
    if (p != nullptr) return p;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    p = g_noalloc_ptr[dev].load(std::memory_order_relaxed);
    if (p == nullptr) {
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) == cudaSuccess && p != nullptr) {
            g_noalloc_ptr[dev].store(p, std::memory_order_release);
        } else {
            p = nullptr;
            cudaGetLastError();  // leave no error behind for the caller's next CUDA call
        }
    }
    return p;
}
}  // namespace
}  // namespace fp8bq

using namespace fp8bq;

extern "C" {

fp8bq_status fp8bq_quantize_act(const void *x_bf16, int64_t M, int64_t K, uint8_t *q_e4m3,
                                float *sa, void *stream) {
    fp8bq_status st = check_mk(M, K);
    if (st != FP8BQ_OK) return st;
    if (M == 0) return FP8BQ_OK;
    if (!x_bf16 || !q_e4m3 || !sa) return FP8BQ_ERR_INVALID_ARG;
    if (!aligned16(x_bf16) || !aligned16(q_e4m3) || !aligned16(sa)) return FP8BQ_ERR_MISALIGNED;
    const DeviceInfo *d = device_info();
    if (!d) return FP8BQ_ERR_NO_DEVICE;
    return from_cuda(launch_quantize_act(*d, x_bf16, M, K, q_e4m3, sa,
                                         static_cast<cudaStream_t>(stream)));
}

fp8bq_status fp8bq_quantize_weight(const void *w_bf16, int64_t N, int64_t K, uint8_t *q_e4m3,
                                   float *sw, void *stream) {
    fp8bq_status st = check_mk(N, K);
    if (st != FP8BQ_OK) return st;
    if (N <= 0 || N % 128 != 0) return FP8BQ_ERR_UNSUPPORTED_SHAPE;
    if (N / 128 > 65535) return FP8BQ_ERR_UNSUPPORTED_SHAPE;  // grid.y limit
    if (!w_bf16 || !q_e4m3 || !sw) return FP8BQ_ERR_INVALID_ARG;
    if (!aligned16(w_bf16) || !aligned16(q_e4m3) || !aligned16(sw)) return FP8BQ_ERR_MISALIGNED;
    const DeviceInfo *d = device_info();
    if (!d) return FP8BQ_ERR_NO_DEVICE;
    const dim3 grid(static_cast<unsigned>(K / 128), static_cast<unsigned>(N / 128));
    return from_cuda(launch(quantize_weight_kernel, grid, dim3(kWeightThreads), 0,
                            static_cast<cudaStream_t>(stream),
                            static_cast<const uint16_t *>(w_bf16), K, q_e4m3, sw));
}

fp8bq_status fp8bq_kv_write_e4m3(const void *k_bf16, const void *v_bf16, int64_t row_stride,
                                 int64_t T, int64_t width, const int64_t *loc, uint8_t *k_cache,
                                 uint8_t *v_cache, int64_t num_slots, int64_t slot_stride,
                                 void *stream) {
    if (T < 0 || width <= 0 || row_stride < width || slot_stride < width || num_slots < 0)
        return FP8BQ_ERR_INVALID_ARG;
    if (width % 8 != 0 || row_stride % 8 != 0 || slot_stride % 16 != 0 || width / 8 > kMaxDim)
        return FP8BQ_ERR_UNSUPPORTED_SHAPE;
    if (T > 0 && row_stride > kMaxBytes / 2 / T) return FP8BQ_ERR_UNSUPPORTED_SHAPE;
    if (num_slots > 0 && slot_stride > kMaxBytes / num_slots) return FP8BQ_ERR_UNSUPPORTED_SHAPE;
    if (T == 0) return FP8BQ_OK;
    if (!k_bf16 || !v_bf16 || !loc || !k_cache || !v_cache) return FP8BQ_ERR_INVALID_ARG;
    if (!aligned16(k_bf16) || !aligned16(v_bf16) || !aligned16(k_cache) || !aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(loc) & 7u) != 0)
        return FP8BQ_ERR_MISALIGNED;
    const DeviceInfo *d = device_info();
    if (!d) return FP8BQ_ERR_NO_DEVICE;
    const int64_t blocks = std::min<int64_t>((2 * T + kKvWarps - 1) / kKvWarps,
                                             static_cast<int64_t>(d->sm_count) * 8);
    return from_cuda(launch(kv_write_e4m3_kernel, dim3(static_cast<unsigned>(blocks)),
                            dim3(kKvThreads), 0, static_cast<cudaStream_t>(stream),
                            static_cast<const uint16_t *>(k_bf16),
                            static_cast<const uint16_t *>(v_bf16), row_stride, T,
                            static_cast<int>(width / 8), loc, k_cache, v_cache, num_slots,
                            slot_stride, d->status));
}

fp8bq_status fp8bq_silu_mul_quantize(const void *gu_bf16, int64_t M, int64_t I, uint8_t *q_e4m3,
                                     float *s, void *h_bf16, void *stream) {
    fp8bq_status st = check_mk(M, I);
    if (st != FP8BQ_OK) return st;
    if (M > 0 && 2 * I > kMaxBytes / 2 / M) return FP8BQ_ERR_UNSUPPORTED_SHAPE;  // gu [M, 2I]
    if (M == 0) return FP8BQ_OK;
    if (!gu_bf16 || !q_e4m3 || !s) return FP8BQ_ERR_INVALID_ARG;
    if (!aligned16(gu_bf16) || !aligned16(q_e4m3) || !aligned16(s) ||
        (h_bf16 != nullptr && !aligned16(h_bf16)))
        return FP8BQ_ERR_MISALIGNED;
    const DeviceInfo *d = device_info();
    if (!d) return FP8BQ_ERR_NO_DEVICE;
    const int64_t G = I / 128;
    const int64_t groups = M * G;
    if (G % 4 == 0 && groups >= static_cast<int64_t>(d->sm_count) * 512) {
        // large, rows of a multiple of 4 groups: (chunks of a row) x (rows,
        // strided), about 8 CTAs of 256 threads per SM
        const int64_t chunks = (G + kSiluWideGroupsPerCta - 1) / kSiluWideGroupsPerCta;
        const int64_t rows = std::max<int64_t>(
            1, std::min<int64_t>(M, (static_cast<int64_t>(d->sm_count) * 8 + chunks - 1) / chunks));
        return from_cuda(launch(silu_mul_quantize_wide_kernel,
                                dim3(static_cast<unsigned>(chunks), static_cast<unsigned>(rows)),
                                dim3(kSiluThreads), 0, static_cast<cudaStream_t>(stream),
                                static_cast<const uint4 *>(gu_bf16), M, I,
                                reinterpret_cast<uint2 *>(q_e4m3), s, static_cast<uint4 *>(h_bf16)));
    }
    const int64_t warps = (groups + 1) / 2;
    const int64_t blocks = std::min<int64_t>((warps + kSiluWarps - 1) / kSiluWarps,
                                             static_cast<int64_t>(d->sm_count) * 16);
    return from_cuda(launch(silu_mul_quantize_kernel, dim3(static_cast<unsigned>(blocks)),
                            dim3(kSiluThreads), 0, static_cast<cudaStream_t>(stream),
                            static_cast<const uint4 *>(gu_bf16), M, I,
                            reinterpret_cast<uint2 *>(q_e4m3), s, static_cast<uint4 *>(h_bf16)));
}

fp8bq_status fp8bq_nvfp4_quantize_weight(const void *w_bf16, int64_t N, int64_t K, uint8_t *packed,
                                         uint8_t *sb, float *g, void *stream) {
    if (N <= 0 || K <= 0 || K % 16 != 0 || N > kMaxDim || K > kMaxDim || K > kMaxBytes / 2 / N)
        return FP8BQ_ERR_UNSUPPORTED_SHAPE;
    if (!w_bf16 || !packed || !sb || !g) return FP8BQ_ERR_INVALID_ARG;
    if (!aligned16(w_bf16) || !aligned16(packed) || !aligned16(sb) ||
        (reinterpret_cast<uintptr_t>(g) & 3u) != 0)
        return FP8BQ_ERR_MISALIGNED;
    const DeviceInfo *d = device_info();
    if (!d) return FP8BQ_ERR_NO_DEVICE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t n_vec = N * K / 8, groups = N * K / 16;
    const int64_t cap = static_cast<int64_t>(d->sm_count) * 8;
    unsigned int *gw = reinterpret_cast<unsigned int *>(g);
    cudaError_t e = cudaMemsetAsync(g, 0, sizeof(float), st);
    if (e == cudaSuccess)
        e = launch(nvfp4::nvfp4_amax_kernel, dim3(static_cast<unsigned>(std::min((n_vec + 255) / 256, cap))),
                   dim3(256), 0, st, static_cast<const uint4 *>(w_bf16), n_vec, gw);
    if (e == cudaSuccess)
        e = launch(nvfp4::nvfp4_quantize_kernel,
                   dim3(static_cast<unsigned>(std::min((groups + 255) / 256, 2 * cap))), dim3(256), 0,
                   st, static_cast<const uint4 *>(w_bf16), groups, static_cast<const unsigned int *>(gw),
                   reinterpret_cast<uint2 *>(packed), sb);
    if (e == cudaSuccess) e = launch(nvfp4::nvfp4_global_kernel, dim3(1), dim3(1), 0, st, gw);
    return from_cuda(e);
}

fp8bq_status fp8bq_nvfp4_gemm_a16(const void *x_bf16, const uint8_t *packed, const uint8_t *sb,
                                  const float *g, int64_t M, int64_t N, int64_t K, void *y_bf16,
                                  void *stream) {
    if (M < 0 || N <= 0 || K <= 0 || N % 128 != 0 || K % nvfp4::BKU != 0 || M > kMaxDim ||
        N > kMaxDim || K > kMaxDim || (M > 0 && K > kMaxBytes / 2 / M) || N / 128 > 65535)
        return FP8BQ_ERR_UNSUPPORTED_SHAPE;
    if (M == 0) return FP8BQ_OK;
    if (!x_bf16 || !packed || !sb || !g || !y_bf16) return FP8BQ_ERR_INVALID_ARG;
    if (!aligned16(x_bf16) || !aligned16(packed) || !aligned16(sb) || !aligned16(y_bf16) ||
        (reinterpret_cast<uintptr_t>(g) & 3u) != 0)
        return FP8BQ_ERR_MISALIGNED;
    const DeviceInfo *d = device_info();
    if (!d) return FP8BQ_ERR_NO_DEVICE;
    const int64_t NB = N / 128, KB = K / nvfp4::BKU, sms = d->sm_count;
    int64_t S = 1;
    if (NB <= sms) {
        S = std::min<int64_t>(std::min<int64_t>(8, sms / NB), KB);
        while (S >= 2 && NB > d->nvfp4_cluster_capacity[S]) --S;
        S = std::max<int64_t>(S, 1);
    }
    const int64_t mtiles = (M + nvfp4::MT - 1) / nvfp4::MT;
    if (mtiles > 65535) return FP8BQ_ERR_UNSUPPORTED_SHAPE;
    CUtensorMap tw, ts, tx;
    if (M <= 2) {
        // one or two tokens: packed codes decoded in registers on the CUDA cores
        // (from M = 3 on the tensor-core kernel, whose time hardly depends on M
        // up to its 16-row tile, is faster: at M = 4 the CUDA-core kernel took
        // 37.9 us against 28.9 us on fused QKV [9216, 7168])
        const int MB = M <= 1 ? 1 : 2;
        if (!make_tmap_2d(&tw, packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K / 2, 128, 128,
                          CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_tmap_2d(&ts, sb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K / 16, 16, 128,
                          CU_TENSOR_MAP_SWIZZLE_NONE) ||
            !make_tmap_2d(&tx, x_bf16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, K, nvfp4::BKU,
                          static_cast<uint32_t>(MB), CU_TENSOR_MAP_SWIZZLE_NONE))
            return FP8BQ_ERR_CUDA;
        const dim3 grid(static_cast<unsigned>(NB * S)), block(nvfp4::kGemvThreads);
        const unsigned cl = S > 1 ? static_cast<unsigned>(S) : 1u;
        cudaStream_t st = static_cast<cudaStream_t>(stream);
        __nv_bfloat16 *yp = static_cast<__nv_bfloat16 *>(y_bf16);
        const int iM = static_cast<int>(M), iN = static_cast<int>(N), iK = static_cast<int>(K),
                  iS = static_cast<int>(S);
        cudaError_t e;
        if (MB == 1)
            e = launch_clustered(nvfp4::nvfp4_gemv_a16_kernel<1>, grid, block,
                                 nvfp4::GemvLayout<1>::kBytes, st, cl, tw, ts, tx, g, yp, iM, iN, iK,
                                 iS, d->status);
        else
            e = launch_clustered(nvfp4::nvfp4_gemv_a16_kernel<2>, grid, block,
                                 nvfp4::GemvLayout<2>::kBytes, st, cl, tw, ts, tx, g, yp, iM, iN, iK,
                                 iS, d->status);
        return from_cuda(e);
    }
    if (!make_tmap_2d(&tw, packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K / 2, 128, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_2d(&ts, sb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K / 16, 16, 128,
                      CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_tmap_2d(&tx, x_bf16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, K, 64, nvfp4::MT,
                      CU_TENSOR_MAP_SWIZZLE_128B))
        return FP8BQ_ERR_CUDA;
    return from_cuda(launch_clustered(
        nvfp4::nvfp4_gemm_a16_kernel, dim3(static_cast<unsigned>(NB * S), static_cast<unsigned>(mtiles)),
        dim3(nvfp4::kNumThreads), nvfp4::Layout::kBytes, static_cast<cudaStream_t>(stream),
        S > 1 ? static_cast<unsigned>(S) : 1u, tw, ts, tx, g, static_cast<__nv_bfloat16 *>(y_bf16),
        static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), static_cast<int>(S), d->status));
}

size_t fp8bq_workspace_size(int op, int64_t M, int64_t N, int64_t K) {
    if (check_mnk(M, N, K) != FP8BQ_OK || M == 0) return 0;
    if (op == FP8BQ_OP_GEMM) return gemm_ws_bytes_full(M, N, K);
    if (op == FP8BQ_OP_LINEAR) return act_ws_bytes(M, K) + linear_gemm_part(M, N, K, true);
    if (op == FP8BQ_OP_GEMM_SILU) return N % 256 == 0 ? silu_ws_bytes(M, N / 2) : 0;
    return 0;
}

fp8bq_status fp8bq_gemm(const uint8_t *qa, const float *sa, const uint8_t *qw, const float *sw,
                        int64_t M, int64_t N, int64_t K, void *y_bf16, void *workspace,
                        size_t ws_bytes, void *stream) {
    fp8bq_status st = check_mnk(M, N, K);
    if (st != FP8BQ_OK) return st;
    if (M == 0) return FP8BQ_OK;
    if (!qa || !sa || !qw || !sw || !y_bf16) return FP8BQ_ERR_INVALID_ARG;
    if (!aligned16(qa) || !aligned16(sa) || !aligned16(qw) || !aligned16(sw) || !aligned16(y_bf16))
        return FP8BQ_ERR_MISALIGNED;
    const size_t need = gemm_ws_bytes(M, N);
    if (need && (!workspace || ws_bytes < need)) return FP8BQ_ERR_WORKSPACE;
    if (need && !aligned16(workspace)) return FP8BQ_ERR_MISALIGNED;
    const DeviceInfo *d = device_info();
    if (!d) return FP8BQ_ERR_NO_DEVICE;
    fp8bq_status err;
    cudaError_t e = launch_gemm(*d, qa, sa, qw, sw, M, N, K, y_bf16, workspace,
                                workspace ? ws_bytes : 0, static_cast<cudaStream_t>(stream), &err);
    if (err != FP8BQ_OK) return err;
    return from_cuda(e);
}

fp8bq_status fp8bq_linear(const void *x_bf16, const uint8_t *qw, const float *sw, int64_t M,
                          int64_t N, int64_t K, void *y_bf16, void *workspace, size_t ws_bytes,
                          void *stream) {
    fp8bq_status st = check_mnk(M, N, K);
    if (st != FP8BQ_OK) return st;
    if (M == 0) return FP8BQ_OK;
    if (!x_bf16 || !qw || !sw || !y_bf16) return FP8BQ_ERR_INVALID_ARG;
    if (!aligned16(x_bf16) || !aligned16(qw) || !aligned16(sw) || !aligned16(y_bf16))
        return FP8BQ_ERR_MISALIGNED;
    const size_t act = act_ws_bytes(M, K);
    const size_t part_req = linear_gemm_part(M, N, K, false);
    if (!workspace || ws_bytes < act + part_req) return FP8BQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return FP8BQ_ERR_MISALIGNED;
    const DeviceInfo *d = device_info();
    if (!d) return FP8BQ_ERR_NO_DEVICE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // [GEMM part][activation codes][activation scales]; the GEMM part takes
    // the prefill split-K tail's size when the workspace holds it
    const size_t part_full = linear_gemm_part(M, N, K, true);
    const size_t part = ws_bytes >= act + part_full ? part_full : part_req;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint8_t *qa = ws + part;
    float *sa = reinterpret_cast<float *>(qa + round256(M * K));
    cudaError_t e = launch_quantize_act(*d, x_bf16, M, K, qa, sa, s);
    if (e != cudaSuccess) return FP8BQ_ERR_CUDA;
    fp8bq_status err;
    e = launch_gemm(*d, qa, sa, qw, sw, M, N, K, y_bf16, ws, part, s, &err,
                    /*early_weights=*/true);
    if (err != FP8BQ_OK) return err;
    return from_cuda(e);
}

fp8bq_status fp8bq_gemm_silu_mul_quantize(const uint8_t *qa, const float *sa, const uint8_t *qw,
                                           const float *sw, int64_t M, int64_t I, int64_t K,
                                           uint8_t *q_e4m3, float *s, void *h_bf16, void *workspace,
                                           size_t ws_bytes, void *stream) {
    if (I <= 0 || I % 128 != 0 || I > kMaxDim / 2) return FP8BQ_ERR_UNSUPPORTED_SHAPE;
    fp8bq_status st = check_mnk(M, 2 * I, K);
    if (st != FP8BQ_OK) return st;
    if (M == 0) return FP8BQ_OK;
    if (!qa || !sa || !qw || !sw || !q_e4m3 || !s) return FP8BQ_ERR_INVALID_ARG;
    if (!aligned16(qa) || !aligned16(sa) || !aligned16(qw) || !aligned16(sw) ||
        !aligned16(q_e4m3) || !aligned16(s) || (h_bf16 != nullptr && !aligned16(h_bf16)))
        return FP8BQ_ERR_MISALIGNED;
    const size_t need = silu_ws_bytes(M, I);
    if (need && (!workspace || ws_bytes < need)) return FP8BQ_ERR_WORKSPACE;
    if (need && !aligned16(workspace)) return FP8BQ_ERR_MISALIGNED;
    const DeviceInfo *d = device_info();
    if (!d) return FP8BQ_ERR_NO_DEVICE;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    fp8bq_status err;
    if (M > kDecodeMaxM) {
        cudaError_t e = launch_gemm_silu(*d, qa, sa, qw, sw, M, I, K, q_e4m3, s, h_bf16, cs, &err);
        if (err != FP8BQ_OK) return err;
        return from_cuda(e);
    }
    // Decode-sized M: the decode GEMM writes the BF16 gate/up output into the
    // workspace behind its own part, then the SiLU kernel quantizes it.
    const size_t part = need - round256(M * 2 * I * 2);
    void *gu = static_cast<uint8_t *>(workspace) + part;
    cudaError_t e = launch_gemm(*d, qa, sa, qw, sw, M, 2 * I, K, gu, workspace, part, cs, &err);
    if (err != FP8BQ_OK) return err;
    if (e != cudaSuccess) return FP8BQ_ERR_CUDA;
    return fp8bq_silu_mul_quantize(gu, M, I, q_e4m3, s, h_bf16, stream);
}

fp8bq_status fp8bq_workspace_init(void *workspace, size_t ws_bytes, void *stream) {
    if (ws_bytes == 0) return FP8BQ_OK;
    if (!workspace) return FP8BQ_ERR_INVALID_ARG;
    return from_cuda(cudaMemsetAsync(workspace, 0, ws_bytes, static_cast<cudaStream_t>(stream)));
}

fp8bq_status fp8bq_last_device_status(void *stream) {
    const DeviceInfo *d = device_info();
    if (!d) return FP8BQ_ERR_NO_DEVICE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return FP8BQ_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, d->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return FP8BQ_ERR_CUDA;
    if (v != 0 && cudaMemset(d->status, 0, sizeof(int)) != cudaSuccess) return FP8BQ_ERR_CUDA;
    return v == 0 ? FP8BQ_OK : static_cast<fp8bq_status>(v);
}

const char *fp8bq_status_string(fp8bq_status status) {
    switch (status) {
        case FP8BQ_OK: return "ok";
        case FP8BQ_ERR_INVALID_ARG: return "invalid argument (null pointer or negative size)";
        case FP8BQ_ERR_UNSUPPORTED_SHAPE: return "unsupported shape (N and K must be multiples of 128)";
        case FP8BQ_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case FP8BQ_ERR_WORKSPACE: return "workspace missing or too small";
        case FP8BQ_ERR_CUDA: return "CUDA runtime or driver call failed";
        case FP8BQ_ERR_TIMEOUT: return "a kernel abandoned a bounded wait (timeout)";
        case FP8BQ_ERR_NO_DEVICE: return "no sm_100 device is current";
        case FP8BQ_ERR_INDEX: return "a row's cache slot was out of range (the row was skipped)";
    }
    return "unknown status";
}

uint64_t fp8bq_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int fp8bq_version(void) { return 100; }

void fp8bq_clear_cache(void) {
    std::lock_guard<std::mutex> lk(g_tmap_mu);
    g_tmap_cache.clear();
}

fp8bq_status fp8bq_selftest_timeout(uint32_t limit_us, void *stream) {
    if (limit_us == 0 || limit_us > 2000000u) return FP8BQ_ERR_INVALID_ARG;
    const DeviceInfo *d = device_info();
    if (!d) return FP8BQ_ERR_NO_DEVICE;
    selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        d->status, static_cast<uint64_t>(limit_us) * 1000u);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return from_cuda(cudaGetLastError());
}

fp8bq_status fp8bq_gemm_noalloc(const uint8_t *qa, const float *sa, const uint8_t *qw,
                                const float *sw, int64_t M, int64_t N, int64_t K, void *y_bf16,
                                void *stream) {
    fp8bq_status st = check_mnk(M, N, K);
    if (st != FP8BQ_OK) return st;
    if (M == 0) return FP8BQ_OK;
    if (!qa || !sa || !qw || !sw || !y_bf16) return FP8BQ_ERR_INVALID_ARG;
    if (!aligned16(qa) || !aligned16(sa) || !aligned16(qw) || !aligned16(sw) || !aligned16(y_bf16))
        return FP8BQ_ERR_MISALIGNED;
    size_t need = gemm_ws_bytes(M, N);
    // Beyond the built-in scratch: M <= 16 is refused; larger M runs on the
    // prefill kernel, which needs no scratch.
    const bool fits = need <= kNoAllocScratchBytes;
    if (!fits && M <= 16) return FP8BQ_ERR_WORKSPACE;
    if (!fits) need = 0;
    const DeviceInfo *d = device_info();
    if (!d) return FP8BQ_ERR_NO_DEVICE;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FP8BQ_ERR_CUDA;
    // With the device current: the array's device address (looked up on the
    // first call that succeeds in doing so on this device).
    void *scratch = noalloc_scratch(dev);
    if (scratch == nullptr) return FP8BQ_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // The array keeps whatever the previous call left; the split-K counters
    // must start at zero, so clear them on this call's stream first.
    if (need && cudaMemsetAsync(scratch, 0, static_cast<size_t>(decode::kCounterBytes), s) !=
                    cudaSuccess)
        return FP8BQ_ERR_CUDA;
    fp8bq_status err;
    cudaError_t e = launch_gemm(*d, qa, sa, qw, sw, M, N, K, y_bf16, scratch,
                                /*ws_bytes (no prefill tail split)=*/0, s, &err,
                                /*early_weights=*/false, /*allow_decode=*/fits);
    if (err != FP8BQ_OK) return err;
    return from_cuda(e);
}

}  // extern "C"
