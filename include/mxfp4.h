/*
 * mxfp4.h -- C ABI of the B200 (sm_100a) MXFP4 quantize / MoE expert-MLP library.
 *
 * MXFP4: every element is an E2M1 4-bit float (1 sign, 2 exponent, 1 mantissa bit)
 * and each block of 32 consecutive elements shares one scale (agentlenshq.com,
 * "Transformers 4.40 performance upgrades for OpenAI GPT-OSS: zero-build kernels,
 * MXFP4 quantization, parallelism, and faster loading", section "What MXFP4 Is").
 * The MoE expert MLP on MXFP4 expert weights is the layer that page runs through
 * its downloadable MoE kernel (section "Zero-Build Kernels from the Hub").
 *
 * Encoding used throughout (readings: the pages leave these open):
 *   - E2M1 with exponent bias 1: magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6};
 *     a 4-bit code is (sign << 3) | magnitude index;
 *   - one E8M0 scale byte S per block, value 2^(S-127), S = 0xFF is NaN;
 *   - packed codes: uint8 [rows, cols/2], element 2j in the low nibble of byte j;
 *   - scales: uint8 [rows, cols/32], row-major; blocks run along the last
 *     (contiguous) dimension, which for weights is the contraction dimension K.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     never allocates, frees or keeps them.  Row-major, densely packed.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = legacy default stream).  Nothing synchronizes except
 *     mxfp4_get_device_status().
 *   - Arguments are validated on the host before anything is launched; an invalid
 *     call launches nothing and returns a status.  Functions never print, abort
 *     or exit.  A failed launch returns MXFP4_ERR_CUDA and the cudaError_t is kept
 *     per host thread (mxfp4_last_cuda_error()).
 *   - Kernels that wait on barriers do so with a time limit; on expiry they record
 *     MXFP4_ERR_TIMEOUT in a per-device status word, clean up and return.  Read it
 *     with mxfp4_get_device_status().
 *   - The device must be compute capability 10.0 (B200, sm_100a), else MXFP4_ERR_ARCH.
 *   - Pointers must be 16-byte aligned (MXFP4_ERR_MISALIGNED).
 */
#ifndef MXFP4_H_
#define MXFP4_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MXFP4_API __attribute__((visibility("default")))
#else
#define MXFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MXFP4_OK = 0,
    MXFP4_ERR_INVALID_ARG = 1,       /* null pointer, non-positive size, bad enum   */
    MXFP4_ERR_UNSUPPORTED_SHAPE = 2, /* a dimension violates the stated multiples   */
    MXFP4_ERR_MISALIGNED = 3,        /* a pointer is not 16-byte aligned            */
    MXFP4_ERR_ARCH = 4,              /* current device is not sm_100                */
    MXFP4_ERR_WORKSPACE = 5,         /* workspace missing or smaller than required  */
    MXFP4_ERR_CUDA = 6,              /* a CUDA runtime/driver call failed           */
    MXFP4_ERR_TIMEOUT = 7            /* a device-side wait ran out of time          */
} mxfp4_status;

typedef enum { MXFP4_IN_BF16 = 0, MXFP4_IN_F32 = 1 } mxfp4_in_dtype;

/* Block scale exponent s (scale = 2^s):
 *   FLOOR: s = floor(log2(amax)) - 2 (OCP MX rule; |v|/2^s in (6, 8) saturates to 6);
 *   CEIL:  smallest s with amax / 2^s <= 6 (never saturates).
 * s is clamped to [-127, 127]; an all-zero block gets S = 0. */
typedef enum { MXFP4_SCALE_FLOOR = 0, MXFP4_SCALE_CEIL = 1 } mxfp4_scale_rule;

/* W4A16: bf16 activations x dequantized (bf16) MXFP4 weights, fp32 accumulation
 *        on tcgen05 kind::f16.
 * W4A4:  activations are MXFP4-quantized too (FLOOR rule, blocks along K) and the
 *        product runs on the block-scaled tcgen05 kind::mxf4 MMA. */
typedef enum { MXFP4_W4A16 = 0, MXFP4_W4A4 = 1 } mxfp4_mode;

/* ---------------------------------------------------------------- quantize
 * x [rows, cols] (bf16 or fp32 per `dt`) -> codes uint8 [rows, cols/2] and
 * scales uint8 [rows, cols/32].  Per 32-element block: amax, E8M0 scale (rule),
 * E2M1 round-to-nearest-even of |v|/2^s saturating at 6, input sign bit copied
 * (-0 gives code 8); a block containing Inf/NaN gets S = 0xFF and zero codes.
 * Requires cols % 32 == 0.  Bit-exact: exactly one correct output exists.
 * Source: agentlenshq.com, "Transformers 4.40 performance upgrades for OpenAI GPT-OSS ...", section "What MXFP4 Is"
 * (E2M1 elements with a 1/2/1 bit split; 32-element blocks share one scale), and
 * otomatix.tech, the E2M1 sentence.  The scale encoding, scale exponent rule,
 * rounding and packing are readings (listed above and in the encoding notes). */
MXFP4_API mxfp4_status mxfp4_quantize(const void* x, mxfp4_in_dtype dt, int64_t rows, int64_t cols,
                            uint8_t* codes, uint8_t* scales, mxfp4_scale_rule rule,
                            void* stream);

/* ---------------------------------------------------------------- dequantize
 * codes uint8 [rows, cols/2] + scales uint8 [rows, cols/32] -> out bf16 [rows, cols].
 * value = code_value * 2^(S-127) rounded once to bf16 (exact except overflow to
 * Inf); S = 0xFF gives NaN.  Requires cols % 32 == 0.
 * Source: the same section "What MXFP4 Is" (value = E2M1 element x block scale);
 * section "Native Support in transformers" names the bf16 form this produces (the
 * fallback at about four times the memory). */
MXFP4_API mxfp4_status mxfp4_dequantize(const uint8_t* codes, const uint8_t* scales,
                              int64_t rows, int64_t cols, void* out_bf16, void* stream);

/* ---------------------------------------------------------------- GEMM
 * y [M, N] bf16 = x [M, K] bf16 . dequant(W)^T, W = MXFP4 codes [N, K/2] +
 * scales [N, K/32]; fp32 accumulation, one rounding to bf16 at the end.
 * Requires K % 64 == 0 and K <= 7680 (the block scales of a 128-row weight tile
 * are staged whole in shared memory); any M >= 1, N >= 1.  Workspace: W4A16 needs none
 * (ws may be NULL); W4A4 needs mxfp4_gemm_workspace_size() bytes (x quantized to
 * MXFP4: codes and block scales).
 * Source: agentlenshq.com, "Transformers 4.40 performance upgrades for OpenAI GPT-OSS ...", section "MXFP4 4-Bit
 * Quantization" (MXFP4 weights multiplied by specialized kernels without a bf16 copy)
 * and "What MXFP4 Is"; W4A4 reads "the same quantised math" as quantizing the
 * activations with mxfp4_quantize's FLOOR rule. */
MXFP4_API mxfp4_status mxfp4_gemm(const void* x_bf16, int64_t M, int64_t K,
                        const uint8_t* w_codes, const uint8_t* w_scales, int64_t N,
                        void* y_bf16, mxfp4_mode mode, void* ws, size_t ws_bytes,
                        void* stream);
MXFP4_API size_t mxfp4_gemm_workspace_size(int64_t M, int64_t K, int64_t N, mxfp4_mode mode);

/* Token rows per work tile (the MMA's N side) that the grouped GEMMs take for `rows`
 * activation rows spread over `groups` groups: one group in mxfp4_gemm, the experts in
 * the MoE layer (rows = T * top_k).  W4A16: 16, 32, 64, 128 or 192, the size with the
 * least measured tile cost times tiles for a group one standard deviation above the
 * mean; W4A4: the smallest of 16, 32, 64, 128 that holds the mean.  A host query for
 * tests and tuning: no CUDA call.  Returns 0 when rows or groups is below 1 or at
 * least 2^62, or the mode is unknown.  No counterpart in the pages: the launch policy of the GEMMs above. */
MXFP4_API int32_t mxfp4_token_tile_rows(int64_t rows, int64_t groups, mxfp4_mode mode);

/* ---------------------------------------------------------------- routing
 * Per token t of router logits [T, E] fp32: the top_k experts ordered by
 * (logit descending, expert id ascending) -> ids int32 [T, top_k]; softmax over
 * those k logits in fp32 -> weights fp32 [T, top_k]; then the pairs p = t*top_k + j
 * grouped by expert: counts int32 [E], offsets int32 [E+1] (exclusive prefix
 * sum), perm int32 [P] (perm[offsets[e] + r] = the r-th pair routed to e in
 * ascending p) and inv int32 [P] (inv[perm[i]] = i), P = T*top_k.
 * Requires 1 <= top_k <= min(E, 8), E <= 256, T*top_k < 2^31.
 * A NaN logit ranks below every number (-inf included), NaNs among themselves by id.
 * ids/counts/offsets/perm/inv are bit-exact; weights match an fp64 softmax to
 * ~1e-6 relative.
 * Source: agentlenshq.com, "Transformers 4.40 performance upgrades for OpenAI GPT-OSS ...", section "Zero-Build Kernels
 * from the Hub" (the MoE layer runs as a MegaBlocks MoE kernel, which routes each
 * token to its top experts); the ordering, tie rule and softmax scope are readings. */
MXFP4_API mxfp4_status moe_mxfp4_route(const float* router_logits, int64_t T, int64_t E, int32_t top_k,
                             int32_t* ids, float* weights, int32_t* counts, int32_t* offsets,
                             int32_t* perm, int32_t* inv, void* ws, size_t ws_bytes,
                             void* stream);
/* ---------------------------------------------------------------- router projection + routing
 * The same routing computed from the tokens themselves: logits[t, e] = x[t] . W_r[e]
 * (x bf16 [T, H], router weights bf16 [E, H], products exact, fp32 accumulation on
 * the tensor cores), then exactly the ordering, softmax and tables of
 * moe_mxfp4_route applied to those fp32 logits, in the same launch: the logits are
 * not written to memory unless `logits_out` (fp32 [T, E], may be NULL) asks for a
 * copy.  Same outputs, workspace (moe_mxfp4_route_workspace_size) and errors as
 * moe_mxfp4_route; requires H % 64 == 0.  The logits agree with an fp64 dot product
 * to within fp32 accumulation error (H * 2^-24 * sum |x * w|), so ids can differ
 * from an fp64 router's only where two logits are that close.
 * Source: agentlenshq.com, "Transformers 4.40 performance upgrades for OpenAI
 * GPT-OSS ...", section "Zero-Build Kernels from the Hub" (the MoE kernel's routing;
 * a top-k kernel); the bias-free linear router is a reading. */
MXFP4_API mxfp4_status moe_mxfp4_route_project(const void* x_bf16, int64_t T, int64_t H,
                                               const void* w_router_bf16, int64_t E, int32_t top_k,
                                               int32_t* ids, float* weights, int32_t* counts,
                                               int32_t* offsets, int32_t* perm, int32_t* inv,
                                               float* logits_out, void* ws, size_t ws_bytes,
                                               void* stream);
/* Scratch bytes moe_mxfp4_route needs in `ws` (per-chunk counts and ranks). */
MXFP4_API size_t moe_mxfp4_route_workspace_size(int64_t T, int64_t E, int32_t top_k);

/* ---------------------------------------------------------------- MoE expert MLP
 * gpt-oss-style MoE expert MLP with MXFP4 expert weights, one layer:
 *   route (as moe_mxfp4_route) -> gather x rows per expert ->
 *   [g | u] = x . W13[e]^T   (W13 [E, 2I, H]: rows [0, I) gate, [I, 2I) up) ->
 *   h = bf16( SiLU(g) * u )  (SiLU(g) = g / (1 + e^-g), fp32) ->
 *   y = w_tj * (h . W2[e]^T) (W2 [E, H, I], weight applied in fp32) ->
 *   out[t] = bf16( sum_j y_tj ) in slot order (deterministic; no atomics).
 * x bf16 [T, H]; router_logits fp32 [T, E]; w13 codes uint8 [E, 2I, H/2] +
 * scales uint8 [E, 2I, H/32]; w2 codes uint8 [E, H, I/2] + scales [E, H, I/32];
 * out bf16 [T, H].  Requires H % 64 == 0, I % 64 == 0, H, I <= 7680, 1 <= top_k <= min(E, 8),
 * E <= 256, T*top_k < 2^31.  ws must hold moe_mxfp4_workspace_size() bytes
 * (routing tables and the per-pair activations h / y).
 * Source: agentlenshq.com, "Transformers 4.40 performance upgrades for OpenAI GPT-OSS ...", sections "Zero-Build
 * Kernels from the Hub" (the MoE expert MLP as one MegaBlocks MoE kernel) and "MXFP4
 * 4-Bit Quantization" (its expert weights in MXFP4); the gated-SiLU expert MLP,
 * gate/up row split and weighted combine are readings of "h = SiLU(gate) * up;
 * out = sum of weight x down(h)". */
MXFP4_API mxfp4_status moe_mxfp4_mlp(const void* x_bf16, int64_t T, int64_t H,
                           const float* router_logits, int64_t E, int32_t top_k,
                           const uint8_t* w13_codes, const uint8_t* w13_scales, int64_t I,
                           const uint8_t* w2_codes, const uint8_t* w2_scales,
                           void* out_bf16, mxfp4_mode mode, void* ws, size_t ws_bytes,
                           void* stream);
MXFP4_API size_t moe_mxfp4_workspace_size(int64_t T, int64_t H, int64_t I, int64_t E, int32_t top_k,
                                mxfp4_mode mode);

/* ---------------------------------------------------------------- the layer's parts, for composition
 * The MoE layer above is route -> experts -> combine.  These entry points expose the
 * parts after routing, so that a caller can move the expert-sorted rows between
 * GPUs in between (expert parallelism: each GPU runs the experts it holds on the
 * rows routed to them from every GPU, then sends the results back).
 * Source: agentlenshq.com, "Transformers 4.40 performance upgrades for OpenAI
 * GPT-OSS ...", section "Expert Parallelism (EP)" (MoE experts distributed across
 * GPUs); the split into these parts is this library's design.
 *
 * mxfp4_gather_rows: dst row i = src row (idx[i] / div) for i < n, rows of row_bytes
 * bytes (a multiple of 4); src [n_src rows], idx int32 [n], dst [n rows].  With
 * div = top_k and idx = the routing's perm, it gathers token rows into expert-sorted
 * order.  An index whose row is outside src leaves its dst row unwritten and
 * records MXFP4_ERR_INVALID_ARG in the device status word. */
MXFP4_API mxfp4_status mxfp4_gather_rows(const void* src, int64_t n_src, int64_t row_bytes,
                                         const int32_t* idx, int64_t n, int32_t div, void* dst,
                                         void* stream);
/* moe_mxfp4_experts: the experts of one layer on rows already grouped by expert:
 * x_sorted bf16 [P, H] with expert e's rows at offsets[e] .. offsets[e+1] (int32
 * [E+1], device), routing weight row_w fp32 [P] ->
 *   h = bf16(SiLU(x W13[e][0:I]^T) * (x W13[e][I:2I]^T)),  y = row_w * (h W2[e]^T)
 * into y_sorted fp32 [P, H] (W4A4: x and h MXFP4-quantized first, as in the layer).
 * Weights and requirements as moe_mxfp4_mlp; offsets must be non-decreasing with
 * offsets[0] = 0 and offsets[E] = P.  ws: moe_mxfp4_experts_workspace_size() bytes. */
MXFP4_API mxfp4_status moe_mxfp4_experts(const void* x_sorted_bf16, int64_t P, int64_t H,
                                         const int32_t* offsets, int64_t E, const uint8_t* w13_codes,
                                         const uint8_t* w13_scales, int64_t I, const uint8_t* w2_codes,
                                         const uint8_t* w2_scales, const float* row_w, float* y_sorted,
                                         mxfp4_mode mode, void* ws, size_t ws_bytes, void* stream);
MXFP4_API size_t moe_mxfp4_experts_workspace_size(int64_t P, int64_t H, int64_t I, int64_t E,
                                                  mxfp4_mode mode);
/* moe_mxfp4_combine: out[t] = bf16( sum_j y_sorted[inv[t*top_k + j]] ) summed in fp32 in
 * slot order j = 0 .. top_k-1 (deterministic); y_sorted fp32 [*, H], inv int32
 * [T*top_k], out bf16 [T, H].  Requires H % 8 == 0, top_k <= 8.  The sum is the
 * weighted combine of moe_mxfp4_mlp (the reading of "out = sum of weight x
 * down(h)"; the routing weight is already in y). */
MXFP4_API mxfp4_status moe_mxfp4_combine(const float* y_sorted, const int32_t* inv, int64_t T,
                                         int32_t top_k, int64_t H, void* out_bf16, void* stream);

/* ---------------------------------------------------------------- bf16-weight layer (comparison)
 * The same layer as moe_mxfp4_mlp in W4A16 arithmetic, with the expert weights in bf16
 * instead of MXFP4: w13 bf16 [E, 2I, H] (rows [0, I) gate, [I, 2I) up), w2 bf16
 * [E, H, I]; everything else (routing, SwiGLU, fp32 accumulation, weighted combine,
 * x, logits, out, ws = moe_bf16_workspace_size() bytes) as moe_mxfp4_mlp.  It exists to
 * measure what MXFP4 weights save on this GPU against the format they replace.
 * Requires H % 64 == 0 and I % 64 == 0.
 * Source: agentlenshq.com, "Transformers 4.40 performance upgrades for OpenAI
 * GPT-OSS ...", sections "Native Support in transformers" (without the MXFP4 path the
 * model runs in bfloat16 at roughly four times the memory) and "Memory Savings". */
MXFP4_API mxfp4_status moe_bf16_mlp(const void* x_bf16, int64_t T, int64_t H, const float* router_logits,
                                    int64_t E, int32_t top_k, const void* w13_bf16, int64_t I,
                                    const void* w2_bf16, void* out_bf16, void* ws, size_t ws_bytes,
                                    void* stream);
MXFP4_API size_t moe_bf16_workspace_size(int64_t T, int64_t H, int64_t I, int64_t E, int32_t top_k);

/* ---------------------------------------------------------------- allocation-free MoE layer
 * Not a step of the method: the pages have no counterpart of this entry point.
 *
 * The same layer as moe_mxfp4_mlp, for callers that cannot allocate a workspace:
 * cudaMalloc / cudaFree synchronize the whole device and can fail under memory
 * pressure, so latency-critical decode loops, plugin hosts that hand out no device
 * allocator, and code whose memory budget is owned by another framework must not
 * allocate per call.  This entry point takes no workspace and allocates nothing; its
 * scratch is one fixed array of MXFP4_NOALLOC_SCRATCH_BYTES in device memory, set
 * aside on every GPU that loads the library until the process exits.
 *   - Limit: calls whose moe_mxfp4_workspace_size(...) exceeds
 *     MXFP4_NOALLOC_SCRATCH_BYTES return MXFP4_ERR_WORKSPACE (with H = I = 2880,
 *     32 experts and top-4 that is up to 724 token-expert pairs, T * top_k, in W4A16
 *     and 808 in W4A4: decode batches).
 *   - The first call on each device looks up the array's device address (a host-side
 *     query, no allocation); make that first call before any stream capture.
 *   - All calls share the one array: calls that overlap on the GPU (other streams, or
 *     other host threads) race on it and must be serialized by the caller.  Nothing
 *     carries over between calls: each call writes every scratch byte it reads.
 * Arguments, layouts, results and the other errors are those of moe_mxfp4_mlp. */
#define MXFP4_NOALLOC_SCRATCH_BYTES (16u << 20)
MXFP4_API mxfp4_status moe_mxfp4_mlp_noalloc(const void* x_bf16, int64_t T, int64_t H,
                                             const float* router_logits, int64_t E, int32_t top_k,
                                             const uint8_t* w13_codes, const uint8_t* w13_scales,
                                             int64_t I, const uint8_t* w2_codes,
                                             const uint8_t* w2_scales, void* out_bf16,
                                             mxfp4_mode mode, void* stream);

/* ---------------------------------------------------------------- tracing
 * Optional stage timing for the calling host thread (no counterpart in the pages:
 * the benchmark's per-stage timing).  `events` points to
 * `n_events` cudaEvent_t handles (passed as void*) created by the caller; while
 * set, moe_mxfp4_mlp records events[i] on its stream at stage boundary i:
 *   0 start, 1 after routing + gather (W4A4: + activation quantization),
 *   2 after the gate/up GEMM + SwiGLU, 3 after the down GEMM (W4A4: + the
 *   quantization of h before it), 4 after the combine.
 * Boundaries beyond n_events are skipped.  Pass NULL / 0 to disable.  The
 * pointer array must stay valid while tracing is on.  Never fails. */
MXFP4_API void mxfp4_set_trace_events(void* const* events, int n_events);

/* ---------------------------------------------------------------- status
 * Error reporting (no counterpart in the pages).
 * Synchronizes `stream`, then returns and clears the current device's device-side
 * status word (MXFP4_OK, or MXFP4_ERR_TIMEOUT if a kernel gave up waiting).
 * Returns MXFP4_ERR_CUDA if the synchronization itself failed. */
MXFP4_API mxfp4_status mxfp4_get_device_status(void* stream);
/* cudaError_t of the last failed CUDA call on this host thread (0 if none). */
MXFP4_API int mxfp4_last_cuda_error(void);
/* Static, human-readable name of a status code. */
MXFP4_API const char* mxfp4_status_string(mxfp4_status s);
/* Failure-detection self-test (no counterpart in the pages): launches one CTA on
 * `stream` whose only thread waits on an mbarrier that nothing arrives on.  After
 * the library's wait limit (2 s of %globaltimer) the wait gives up, the kernel
 * records MXFP4_ERR_TIMEOUT in the device status word and returns, exactly as the
 * library's kernels do when a pipeline stalls.  No fault, trap or hang: the context
 * stays usable.  Returns MXFP4_OK once launched (read the outcome with
 * mxfp4_get_device_status), or MXFP4_ERR_ARCH / MXFP4_ERR_CUDA. */
MXFP4_API mxfp4_status mxfp4_selftest_wait_timeout(void* stream);
/* Tensor-pipe rate probe (no counterpart in the pages; it supplies the roofline
 * denominator of the block-scaled MMA, which no library figure gives for this box).
 * Launches one CTA per SM on `stream`; each issues iters x 4 back-to-back
 * tcgen05.mma of M = 128, N = 256 from shared memory: kind = 0 is kind::f16 (bf16
 * operands, K = 16 per MMA), kind = 1 is kind::mxf4.block_scale (E2M1 operands with
 * E8M0 scales, K = 64 per MMA).  Operands are pseudo-random finite values.  *flops
 * receives the launch's multiply-add count x 2; time the launch with events on
 * `stream` and divide.  Requires 1 <= iters <= 2^20.  Errors as the other entry
 * points (a completion wait that runs out records MXFP4_ERR_TIMEOUT). */
MXFP4_API mxfp4_status mxfp4_selftest_mma_rate(int32_t kind, int32_t iters, double* flops, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MXFP4_H_ */
