/*
 * fp8bq.h -- C ABI of the B200 (sm_100a) W8A8 FP8 block-scaled linear layer.
 *
 * The method (page "ProCreations/Nanbeige4.3-33B-FP8", introduction and section
 * "Recipe and calibration"): linear layers run in W8A8 FP8 -- E4M3 weights with
 * one scale per 128x128 block (standard min-max, data independent) and
 * activations quantized dynamically per token and per group of 128 channels;
 * embeddings and the output head stay BF16 and are not part of this library.
 *
 * Numerics fixed by this library (the page leaves them open):
 *   - E4M3 is the OCP "e4m3fn" format (largest finite value 448, no infinities).
 *   - scale = amax / 448 computed as one IEEE binary32 division (round to
 *     nearest even); a group or block whose amax is 0 gets scale 1.0.
 *   - code = E4M3 round-to-nearest-even of fl32(x / scale), saturating at
 *     +-448; the sign of zero is kept; finite input never yields the NaN code.
 *   - the GEMM multiplies E4M3 codes exactly, sums each 128-wide K chunk in
 *     FP32, promotes the chunk into an FP32 accumulator multiplied by
 *     act_scale[m, kb] * weight_scale[n/128, kb], and rounds the result to BF16
 *     (round to nearest even).  Y = X W^T (W stored out x in, nn.Linear layout).
 *
 * Layouts: every matrix is dense and row-major (leading dimension = number of
 * columns).  X, Y: BF16 [M, K] / [M, N].  Codes: one byte per element, E4M3
 * bit patterns.  Activation scales: FP32 [M, K/128].  Weight scales: FP32
 * [N/128, K/128].
 *
 * Ownership: the caller allocates and frees every buffer (inputs, outputs and
 * workspace) in device memory of the current device; the library never
 * allocates device memory.  The only host state is a bounded cache of encoded
 * TMA descriptors keyed on address, shape, element type, box and swizzle (an
 * entry describes any tensor with that key, whatever the memory holds, so it
 * never goes stale; fp8bq_clear_cache() empties it).  Descriptors are passed
 * by value to the kernels.
 *
 * Execution: every compute call is asynchronous on the given stream (a
 * cudaStream_t passed as void*; NULL = the legacy default stream) and returns
 * after enqueueing.  Argument errors are detected on the host before anything
 * is enqueued and reported synchronously.  A kernel that gives up on an
 * internal wait (FP8BQ_ERR_TIMEOUT) records it in a per-device status word,
 * read by fp8bq_last_device_status().
 *
 * Requirements checked on the host (else the listed status, nothing enqueued):
 *   M >= 0, N > 0, K > 0, N % 128 == 0, K % 128 == 0  (else UNSUPPORTED_SHAPE;
 *     M == 0 is a no-op returning FP8BQ_OK);
 *   M, N, K <= 2^31 - 1 and every tensor smaller than 2^40 bytes (UNSUPPORTED_SHAPE);
 *   non-NULL pointers for every non-empty tensor (INVALID_ARG);
 *   every pointer 16-byte aligned (MISALIGNED);
 *   where a workspace is required (decode GEMMs and the fused linear, see
 *     fp8bq_workspace_size), at least that many bytes (WORKSPACE).
 * Inputs must be finite; NaN or infinite inputs give unspecified codes.
 *
 * Thread safety: calls on different streams may run concurrently as long as
 * they use different output and workspace buffers.
 */
#ifndef FP8BQ_H
#define FP8BQ_H

#include <stddef.h>
#include <stdint.h>

/* Symbols of this ABI are the only ones the shared library exports. */
#if defined(__GNUC__)
#define FP8BQ_API __attribute__((visibility("default")))
#else
#define FP8BQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FP8BQ_OK = 0,
    FP8BQ_ERR_INVALID_ARG = 1,       /* NULL pointer or negative size */
    FP8BQ_ERR_UNSUPPORTED_SHAPE = 2, /* N or K not a multiple of 128, or too large */
    FP8BQ_ERR_MISALIGNED = 3,        /* a pointer is not 16-byte aligned */
    FP8BQ_ERR_WORKSPACE = 4,         /* workspace missing or smaller than required */
    FP8BQ_ERR_CUDA = 5,              /* a CUDA runtime or driver call failed */
    FP8BQ_ERR_TIMEOUT = 6,           /* a kernel abandoned a bounded wait */
    FP8BQ_ERR_NO_DEVICE = 7,         /* no sm_100 device is current */
    FP8BQ_ERR_INDEX = 8              /* device side: a row's slot index was out of range */
} fp8bq_status;

/* Operation selector for fp8bq_workspace_size. */
typedef enum { FP8BQ_OP_GEMM = 0, FP8BQ_OP_LINEAR = 1, FP8BQ_OP_GEMM_SILU = 2 } fp8bq_op;

/*
 * Dynamic per-token, group-128 activation quantization (page
 * "ProCreations/Nanbeige4.3-33B-FP8", introduction: activations get one scale
 * per token and per 128-channel group, computed at run time).
 *   x_bf16 : in,  BF16 [M, K]
 *   q_e4m3 : out, E4M3 codes [M, K]
 *   sa     : out, FP32 [M, K/128]; sa[m, g] = amax(|x[m, 128g : 128g+128]|) / 448, or 1
 * Codes and scales are bit-exact with the definition above.
 */
FP8BQ_API fp8bq_status fp8bq_quantize_act(const void *x_bf16, int64_t M, int64_t K, uint8_t *q_e4m3,
                                float *sa, void *stream);

/*
 * Offline 128x128-block min-max weight quantization (same page, section
 * "Recipe and calibration": one scale per 128x128 block of the E4M3 weights,
 * chosen by plain min-max without calibration data).
 *   w_bf16 : in,  BF16 [N, K] (out x in)
 *   q_e4m3 : out, E4M3 codes [N, K]
 *   sw     : out, FP32 [N/128, K/128]; sw[i, j] = amax of block (i, j) / 448, or 1
 * Codes and scales are bit-exact with the definition above.
 */
FP8BQ_API fp8bq_status fp8bq_quantize_weight(const void *w_bf16, int64_t N, int64_t K, uint8_t *q_e4m3,
                                   float *sw, void *stream);

/*
 * Block-scaled FP8 GEMM (same page, introduction: W8A8 FP8 linear layers with
 * BF16 activations in and out): Y[m, n] = BF16( sum_kb sa[m,kb] sw[n/128,kb]
 * sum_{k in kb} e4m3(qa[m,k]) e4m3(qw[n,k]) ).
 *   qa, sa : in, activation codes [M, K] and scales [M, K/128]
 *   qw, sw : in, weight codes [N, K] and scales [N/128, K/128]
 *   y_bf16 : out, BF16 [M, N]
 *   workspace, ws_bytes : device scratch of at least
 *       fp8bq_workspace_size(FP8BQ_OP_GEMM, M, N, K) bytes (may be NULL when
 *       that is 0; optional for M > 128, see fp8bq_workspace_size).  Its
 *       contents must be the state left by
 *       fp8bq_workspace_init() or by any previous successful fp8bq_gemm or
 *       fp8bq_linear call, of any shape (every successful call restores that
 *       state); calls that share a workspace must be ordered (same stream).
 * Output accuracy: |y - ref| <= 1e-2 |ref| + 2e-3 rms(ref) against the FP64 sum
 * of the dequantized operands; results are deterministic for a given shape.
 * Every operand is read only after the previous kernel in the stream has
 * completed; the call lets the next kernel launch early (programmatic
 * dependent launch) and that kernel waits for this one before reading its
 * output.
 */
FP8BQ_API fp8bq_status fp8bq_gemm(const uint8_t *qa, const float *sa, const uint8_t *qw, const float *sw,
                        int64_t M, int64_t N, int64_t K, void *y_bf16, void *workspace,
                        size_t ws_bytes, void *stream);

/*
 * Linear layer with the activation quantization fused into the call:
 * Y = gemm(quantize_act(X), qw, sw) with identical codes and scales.
 *   x_bf16 : in, BF16 [M, K]; qw / sw / y_bf16 as in fp8bq_gemm
 *   workspace : at least fp8bq_workspace_size(FP8BQ_OP_LINEAR, M, N, K) bytes,
 *               same state rule as fp8bq_gemm.
 * On the decode path the call starts reading qw / sw while earlier kernels in
 * the stream may still be running (programmatic dependent launch).  This is
 * safe against this library's weight quantizers, which never let a successor
 * start early; qw / sw must not be written by a foreign kernel that does.
 */
FP8BQ_API fp8bq_status fp8bq_linear(const void *x_bf16, const uint8_t *qw, const float *sw, int64_t M,
                          int64_t N, int64_t K, void *y_bf16, void *workspace, size_t ws_bytes,
                          void *stream);

/*
 * FP8 E4M3 KV-cache write with unit scales (page "ProCreations/Nanbeige4.3-33B-FP8",
 * "Serving" and the "Speed on Vega" table: --kv-cache-dtype fp8_e4m3 with unit
 * cache scales).  For every token t:
 *     k_cache[loc[t], i] = e4m3(k[t, i]),  v_cache[loc[t], i] = e4m3(v[t, i])
 * where e4m3(x) is the saturating round-to-nearest-even E4M3 code of x / 1 = x
 * (the same rule as every other code; NaN stays NaN, +-infinity gives +-448).
 *   k_bf16, v_bf16 : in, BF16 rows, row t at (element) offset t * row_stride;
 *       width elements per row (all KV heads of the token, e.g. the K and V
 *       column ranges of the fused QKV output, row_stride = its width).
 *   loc            : in, int64 [T] cache slot of each token (device memory).
 *   k_cache, v_cache : in/out, E4M3 codes, slot s at byte offset s * slot_stride;
 *       the first width bytes of each written slot are replaced, nothing else.
 *   num_slots      : slots in each cache.
 * Requirements: width and row_stride multiples of 8, slot_stride a multiple of
 * 16 and >= width, k/v/caches 16-byte and loc 8-byte aligned (MISALIGNED
 * otherwise).  Distinct tokens should have distinct slots (with duplicates,
 * which row a slot keeps is unspecified).  A token whose slot is outside
 * [0, num_slots) is skipped on the device and FP8BQ_ERR_INDEX is recorded in
 * the device status word (read with fp8bq_last_device_status).
 */
FP8BQ_API fp8bq_status fp8bq_kv_write_e4m3(const void *k_bf16, const void *v_bf16,
                                           int64_t row_stride, int64_t T, int64_t width,
                                           const int64_t *loc, uint8_t *k_cache,
                                           uint8_t *v_cache, int64_t num_slots,
                                           int64_t slot_stride, void *stream);

/*
 * SiLU-gated MLP product, quantized for the down projection (page
 * "ProCreations/Nanbeige4.3-33B-FP8", introduction: dynamic per-token group-128
 * activation quantization for every linear layer).  With gate = gu[:, :I] and
 * up = gu[:, I:],
 *     h = BF16( silu(gate) * up ),  silu(g) = g / (1 + exp(-g)),
 * and (q_e4m3, s) = the group-128 quantization of h, exactly what
 * fp8bq_quantize_act would produce from that BF16 h.  h itself differs from
 * the exactly rounded silu(gate) * up by at most one BF16 step (the
 * exponential is the hardware one).
 *   gu_bf16 : in, BF16 [M, 2I] row-major.
 *   q_e4m3  : out, E4M3 [M, I];  s : out, FP32 [M, I/128].
 *   h_bf16  : out, optional BF16 [M, I] (NULL: h is not stored).
 * I must be a multiple of 128; pointers 16-byte aligned.
 */
FP8BQ_API fp8bq_status fp8bq_silu_mul_quantize(const void *gu_bf16, int64_t M, int64_t I,
                                               uint8_t *q_e4m3, float *s, void *h_bf16,
                                               void *stream);

/*
 * Gate/up projection of the MLP with the SiLU-gated product quantized for the
 * down projection in the same pass (pages "ProCreations/Nanbeige4.3-33B-DFlash2",
 * "Architecture and checkpoint format": separate gate and up projections of the
 * MLP; "ProCreations/Nanbeige4.3-33B-FP8", introduction: every linear layer,
 * the down projection included, takes group-128 dynamically quantized
 * activations).  With gu = gemm(qa, sa, qw, sw) the BF16 [M, 2I] output of the
 * fused gate/up weight, this computes exactly
 *     fp8bq_silu_mul_quantize(gu, M, I, q_e4m3, s, h_bf16)
 * (same codes, scales and h, bit for bit) without gu ever reaching memory for
 * M > 128: there the GEMM's epilogue holds 128 gate channels and the same 128
 * up channels of a row and writes their h codes and scale directly.
 *   qa, sa : in, activation codes [M, K] and scales [M, K/128]
 *   qw, sw : in, the fused gate/up weight: codes [2I, K] (gate rows [0, I), up
 *            rows [I, 2I)) and scales [2I/128, K/128], e.g. from
 *            fp8bq_quantize_weight of the BF16 [2I, K] weight
 *   q_e4m3, s : out, the down projection's input codes [M, I], scales [M, I/128]
 *   h_bf16 : out, optional BF16 h [M, I] (NULL: not stored)
 *   workspace : at least fp8bq_workspace_size(FP8BQ_OP_GEMM_SILU, M, 2I, K)
 *       bytes (0 for M > 128; for M <= 128 the call runs the decode GEMM into
 *       the workspace and then the SiLU kernel), same state rule as fp8bq_gemm.
 * I a multiple of 128, K a multiple of 128; pointers 16-byte aligned.
 */
FP8BQ_API fp8bq_status fp8bq_gemm_silu_mul_quantize(const uint8_t *qa, const float *sa,
                                                    const uint8_t *qw, const float *sw, int64_t M,
                                                    int64_t I, int64_t K, uint8_t *q_e4m3,
                                                    float *s, void *h_bf16, void *workspace,
                                                    size_t ws_bytes, void *stream);

/*
 * NVFP4 weight-only format with BF16 activations (page
 * "ProCreations/Nanbeige4.3-33B-NVFP4-A16", recipe paragraph: FP4 E2M1 weights
 * in groups of 16 with E4M3 block scales and a global weight scale; activations
 * BF16).  A weight is w[n, k] = e2m1(q[n, k]) * e4m3(sb[n, k/16]) * g.
 * Layout: packed [N, K/2] bytes, element 2j in the low nibble and 2j+1 in the
 * high nibble of byte j of its row; sb [N, K/16] E4M3 codes; g one FP32 value.
 *
 * fp8bq_nvfp4_quantize_weight: plain min-max quantization (the page's own
 * scales come from a data-driven search, which needs calibration data):
 *   g  = fl32(amax(|W|) / 2688)   (2688 = 6 * 448; 1.0 when W is all zero)
 *   sb = E4M3_RNE_sat(fl32(amax_group / fl32(6 g)))
 *   q  = E2M1_RNE_sat(fl32(w / fl32(e4m3(sb) * g)))   (0 when that scale is 0)
 *   w_bf16 : in, BF16 [N, K], K a multiple of 16.
 *   packed : out, [N, K/2];  sb : out, [N, K/16];  g : out, one float (device).
 * Codes, block scales and g are bit-exact with that definition.  Pointers
 * 16-byte aligned (g: 4).  Three kernels and a 4-byte memset on `stream`.
 */
FP8BQ_API fp8bq_status fp8bq_nvfp4_quantize_weight(const void *w_bf16, int64_t N, int64_t K,
                                                   uint8_t *packed, uint8_t *sb, float *g,
                                                   void *stream);

/*
 * Y[m, n] = BF16( sum_k x[m, k] * w[n, k] ) for BF16 X [M, K] and an NVFP4 W
 * [N, K] in the layout above; g is read from device memory (e.g. as written by
 * fp8bq_nvfp4_quantize_weight).  N a multiple of 128, K a multiple of 256;
 * pointers 16-byte aligned (g: 4).  No workspace.  Accuracy as fp8bq_gemm:
 * |y - ref| <= 1e-2 |ref| + 2e-3 rms(ref) against the FP64 sum.  Built for
 * decode-sized M; every 16 rows of M stream the weights once.
 */
FP8BQ_API fp8bq_status fp8bq_nvfp4_gemm_a16(const void *x_bf16, const uint8_t *packed,
                                            const uint8_t *sb, const float *g, int64_t M,
                                            int64_t N, int64_t K, void *y_bf16, void *stream);

/*
 * fp8bq_gemm without a workspace argument, for callers that cannot allocate
 * device memory: code running where no allocator is reachable (an embedding
 * runtime that hands out only fixed buffers, or a context where cudaMalloc is
 * not permitted).  The pages describe no such call; it is a convenience of the
 * library.  Same arguments, results and accuracy as fp8bq_gemm, minus the
 * workspace.  Its scratch is a 4 MiB array inside the library (held on every
 * GPU that loads it until the process exits).  Problems whose split-K scratch
 * would exceed it are rejected with FP8BQ_ERR_WORKSPACE when M <= 16 (that
 * is, N > 32512); for 16 < M <= 128 they run on the prefill kernel instead,
 * which needs no scratch, and M > 128 never needs any.  It calls no allocator.
 *   - The first call on a device looks up the array's device address (a
 *     one-time set-up); make that first call before any stream capture.
 *   - All calls share the one array: calls that overlap on the GPU (other
 *     streams, other host threads) race and give wrong results; order them.
 *   - Each call first clears the part of the array that must start at zero
 *     (a memset on its stream).
 */
FP8BQ_API fp8bq_status fp8bq_gemm_noalloc(const uint8_t *qa, const float *sa, const uint8_t *qw,
                                          const float *sw, int64_t M, int64_t N, int64_t K,
                                          void *y_bf16, void *stream);

/* Bytes of workspace the operation uses for this shape (0 when none, and for
 * arguments the call would reject).  Always a multiple of 256.  For M <= 128
 * the call requires at least this much.  For M > 128 (the prefill GEMM) any
 * workspace is accepted, NULL included, and the size is 0 unless K >= 16384.
 * There, with at least this much, a last wave of at most 16 output tiles on
 * the persistent grid is split K-wise over more CTAs (FP32 partials summed in
 * a fixed order, so results stay deterministic and within the same
 * tolerance), which a smaller workspace goes without.  The fused linear
 * requires, besides the GEMM's part (never less than its 16 KB counter
 * header), its activation codes and scales.  FP8BQ_OP_GEMM_SILU takes N = 2I
 * (the fused gate/up weight's rows): 0 for M > 128, else the GEMM's part (at
 * least the header) and the BF16 gate/up output [M, 2I].
 * Every workspace starts with the same 16 KB header of split-K counters, at
 * offset 0 for every operation and shape, and every successful call leaves
 * them at zero: one workspace, large enough for each call, can serve any
 * sequence of fp8bq_gemm, fp8bq_linear and fp8bq_gemm_silu_mul_quantize calls
 * in stream order. */
FP8BQ_API size_t fp8bq_workspace_size(int op, int64_t M, int64_t N, int64_t K);

/* Put a workspace into its initial state (zero-fills ws_bytes bytes on the
 * stream).  Needed once after allocation and after a call that reported
 * FP8BQ_ERR_TIMEOUT. */
FP8BQ_API fp8bq_status fp8bq_workspace_init(void *workspace, size_t ws_bytes, void *stream);

/* Synchronizes the stream, then returns and clears the current device's status
 * word: FP8BQ_OK, or FP8BQ_ERR_TIMEOUT if a kernel abandoned a wait since the
 * last read.  A failed synchronize returns FP8BQ_ERR_CUDA. */
FP8BQ_API fp8bq_status fp8bq_last_device_status(void *stream);

/* Static description of a status code (never NULL). */
FP8BQ_API const char *fp8bq_status_string(fp8bq_status status);

/* Diagnostic for the failure path: launches a kernel whose only internal wait
 * can never complete, with the same bounded wait every kernel of the library
 * uses, limited to limit_us microseconds (1 .. 2e6).  It returns after
 * enqueueing; afterwards fp8bq_last_device_status() reports FP8BQ_ERR_TIMEOUT
 * (and clears it).  Nothing faults or hangs; the context stays usable. */
FP8BQ_API fp8bq_status fp8bq_selftest_timeout(uint32_t limit_us, void *stream);

/* Number of kernels this library has launched in this process (all devices). */
FP8BQ_API uint64_t fp8bq_launch_count(void);

/* ABI version: major * 10000 + minor * 100 + patch. */
FP8BQ_API int fp8bq_version(void);

/* The library keeps the TMA descriptors it encodes, keyed on everything an
 * encoding depends on (address, shape, element type, box, swizzle), so a
 * repeated call skips the encoding; an entry is valid for any tensor matching
 * its key, so entries never go stale.  The cache is bounded (it empties itself
 * when full); this call empties it now.  Host memory only; thread-safe. */
FP8BQ_API void fp8bq_clear_cache(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8BQ_H */
