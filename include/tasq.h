/*
 * tasq.h - C ABI of the timestep-adaptive masked INT8 linear layer (B200, sm_100a).
 *
 * One shared INT8 weight buffer per layer serves every denoising step; at step t the layer
 * runs with the k = 8 - bits[layer][step] least-significant bit planes of every weight
 * cleared, as in TASQ's Temporal-Spatial LSB Mask (TASQ technical summary, section 2,
 * "Representacao de Peso Compartilhada e Mascaramento de LSB", equation
 * Q^(t,l) = Q_n - (1 - M_t,l) * LSB; TASQ abstract: "one shared maximum-precision weight
 * buffer", no per-stage weight copies, no runtime search, switching costs nothing).
 * Activations are smoothed by a block Hadamard transform and quantized per token to INT8
 * before an integer GEMM whose result is dequantized by FP scales (HQ-DM technical summary,
 * sections 2.1 "Mecanismo" / "Eficiencia de Hardware" and 2.2 "Quantizacao Simetrica";
 * 6Bit-Diffusion section 2.A, Block Hadamard Transform).
 *
 * Conventions for every entry point:
 *   - Pointers marked "device" must be CUDA device (or managed) memory of the device that was
 *     current when the context was created; "host" pointers are ordinary host memory.
 *   - `stream` is a cudaStream_t passed as void*; NULL means the legacy default stream.
 *     Work is enqueued on that stream and the call returns without synchronising unless
 *     stated otherwise.
 *   - Every argument is validated on the host before anything is enqueued. On error the call
 *     enqueues nothing, returns a non-zero tasq_status and records a message readable with
 *     tasq_last_error() on the calling thread. No call aborts, throws or traps.
 *   - Layouts are row-major. Alignment: every device pointer 16-byte aligned; every row
 *     stride (in elements) a multiple of 8 (16 bytes for FP16), so rows stay 16-byte aligned.
 *   - A context is not thread-safe: one thread (or external locking) per context.
 */
#ifndef TASQ_H_
#define TASQ_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TASQ_OK = 0,
  TASQ_ERR_INVALID_ARG = 1,      /* a pointer, size, index, alignment or bit width is invalid */
  TASQ_ERR_CUDA = 2,             /* a CUDA runtime / driver call failed (message has details) */
  TASQ_ERR_UNSUPPORTED_ARCH = 3, /* the current device is not compute capability 10.0 */
  TASQ_ERR_WORKSPACE = 4,        /* M exceeds the max_tokens the context was created with */
  TASQ_ERR_TIMEOUT = 5,          /* a bounded device-side wait gave up (see device status) */
} tasq_status;

typedef enum {
  TASQ_OUT_F16 = 0,   /* IEEE binary16 outputs */
  TASQ_OUT_BF16 = 1,  /* bfloat16 outputs */
} tasq_out_dtype;

/* Device status bits written by bounded waits that ran out (see tasq_get_device_status). */
#define TASQ_DEVICE_TIMEOUT_PRODUCER 0x1u
#define TASQ_DEVICE_TIMEOUT_MMA 0x2u
#define TASQ_DEVICE_TIMEOUT_MASK 0x4u
#define TASQ_DEVICE_TIMEOUT_EPILOGUE 0x8u
#define TASQ_DEVICE_TIMEOUT_DRAIN 0x10u
#define TASQ_DEVICE_TIMEOUT_PROLOGUE 0x20u
#define TASQ_DEVICE_BAD_BITS 0x100u

/* Limits of this implementation. */
#define TASQ_MAX_KP 16384           /* Kp = ceil(K / n) * n must not exceed this */
#define TASQ_DMPQ_MAX_LAYERS 32     /* table rows one tasq_dmpq_update call may write */
#define TASQ_GROUP_MAX 4            /* layers one tasq_linear_forward_group call may run */

/*
 * One linear layer y = x W^T, described for tasq_linear_create.
 *   N   : out-features (rows of W), N >= 1.
 *   K   : in-features (columns of the activations), K >= 8 and K % 8 == 0.
 *   w   : INT8 weight codes [N, Kp], row-major, Kp = ceil(K / n) * n (n = hadamard_n). The
 *         codes are read in the Hadamard-rotated input basis (the basis the activations are
 *         transformed into), so every one of the Kp columns takes part. Host or device
 *         memory; copied by tasq_linear_create, the caller keeps ownership.
 *   s_w : FP32 per-output-channel weight scales [N]. Host or device; copied.
 */
typedef struct {
  int32_t N;
  int32_t K;
  const int8_t* w;
  const float* s_w;
} tasq_layer_desc;

typedef struct tasq_ctx tasq_ctx;

/*
 * Create a context owning one shared weight buffer for `num_layers` layers, a device schedule
 * table bits[num_layers][num_steps] (every entry initialised to 8 = full precision), an
 * activation workspace for up to `max_tokens` tokens, and a transient weight buffer of
 * min(num_layers, TASQ_GROUP_MAX) slots of the largest layer: an NVFP4 step's converted weights
 * live there, and so do the masked copies that mask mode 2 (tasq_debug_set_mask_mode) makes.
 *   out         : receives the context; *out is set to NULL on failure.
 *   layers      : host array [num_layers] of layer descriptors.
 *   hadamard_n  : block size of the Hadamard transform along K, 64 or 128.
 *   max_tokens  : largest M any later forward may use, >= 1.
 *   out_dtype   : a tasq_out_dtype for the outputs of tasq_linear_forward.
 *   stream      : stream used for the copies; tasq_linear_create synchronises it before
 *                 returning, so the caller may free its weight copies afterwards.
 * Requires the current device to be sm_100 (B200). Allocates device memory with cudaMalloc.
 */
tasq_status tasq_linear_create(tasq_ctx** out, const tasq_layer_desc* layers, int32_t num_layers,
                               int32_t num_steps, int32_t hadamard_n, int64_t max_tokens,
                               int32_t out_dtype, void* stream);

/*
 * Replace the schedule table with bits_host [num_layers * num_steps] (host, row-major by layer,
 * every entry in [0, 8]; bits = 8 keeps all bit planes, bits = b keeps the top b planes, and
 * TASQ_NVFP4 (0) selects the NVFP4 step described below tasq_dmpq_update).
 * Stream-ordered: forwards enqueued on `stream` after this call see the new table. The host
 * array may be reused as soon as the call returns. No kernel is launched and the weight
 * buffer is never touched: the table is the only thing that changes between steps.
 */
tasq_status tasq_set_schedule(tasq_ctx* ctx, const uint8_t* bits_host, void* stream);

/*
 * y = dequant( Q(x H) . mask(W_layer, bits[layer][step])^T )  for one layer at one step.
 *   x     : device FP16 activations [M, K_layer], row stride ldx (elements, >= K, % 8 == 0).
 *   M     : tokens, 0 <= M <= max_tokens (M == 0 enqueues nothing).
 *   layer : 0 <= layer < num_layers.   step : 0 <= step < num_steps.
 *   y     : device outputs [M, N_layer] in the context's out_dtype, row stride ldy
 *           (elements, >= N, % 8 == 0).
 * Two kernels run on `stream`: the prologue (block Hadamard of size n along K with zero
 * padding to Kp, per-token absmax, s_x = absmax / (127 sqrt(n)), codes RNE(z * 127 / absmax)
 * in [-127, 127]) into the context workspace, then the GEMM, which accumulates exactly in INT32
 * and writes y = acc * s_x[m] * s_w[n]. The weights' low bit planes are cleared in flight,
 * according to bits[layer][step] read from the device table: the GEMM loads every weight tile of
 * the one stored buffer into shared memory and, when the step drops bits, its mask warps AND the
 * tile with 0xFF << (8 - bits) there, before the tensor cores read it, so no masked copy of the
 * weights is ever written. Uses the context workspace: forwards of one context must not overlap in
 * time on different streams.
 */
tasq_status tasq_linear_forward(tasq_ctx* ctx, const void* x, int64_t M, int64_t ldx, int32_t layer,
                                int32_t step, void* y, int64_t ldy, void* stream);

/*
 * Several linears on one input: one prologue (block Hadamard + INT8 codes of x, computed once)
 * feeds one GEMM per layer, e.g. separate q, k and v projections of the same hidden states.
 * Output i is computed exactly as tasq_linear_forward(ctx, x, M, ldx, layers[i], step, ys[i],
 * ldys[i], stream) would compute it.
 *   layers : host array [count] of layer indices sharing the same K, 1 <= count <=
 *            min(num_layers, TASQ_GROUP_MAX).
 *   ys     : host array [count] of device output pointers; ldys : host array [count] of their
 *            row strides (elements, >= N of the layer, % 8 == 0).
 * Each GEMM masks its layer's weights in flight as tasq_linear_forward does (with mask mode 2 the
 * prologue launch masks them ahead instead, each member into its own slot of the context's
 * masked-weight buffer, which holds min(num_layers, TASQ_GROUP_MAX) slots). The same overlap rule
 * as tasq_linear_forward applies.
 */
tasq_status tasq_linear_forward_group(tasq_ctx* ctx, const void* x, int64_t M, int64_t ldx,
                                      const int32_t* layers, int32_t count, int32_t step, void* const* ys,
                                      const int64_t* ldys, void* stream);

/* Free every device allocation of the context (synchronises the device first). NULL is a no-op. */
tasq_status tasq_linear_destroy(tasq_ctx* ctx);

/* Message of the last failing call on this thread ("" if none). Valid until the next call. */
const char* tasq_last_error(void);

/*
 * Read the context's device status word (0 = healthy; otherwise TASQ_DEVICE_* bits of bounded
 * waits that ran out or of invalid table entries). Synchronises `stream`. If `clear` is
 * non-zero the word is reset to 0 afterwards.
 */
tasq_status tasq_get_device_status(tasq_ctx* ctx, uint32_t* status_out, int32_t clear, void* stream);

/*
 * Bound for every device-side wait of the context's kernels, in nanoseconds (default 1e9).
 * A wait that runs out sets a status bit and makes its kernel wind down and return.
 */
tasq_status tasq_set_wait_limit(tasq_ctx* ctx, uint64_t limit_ns);

/* Hadamard block size, padded K and N of a layer (host queries, no device work). */
tasq_status tasq_layer_info(const tasq_ctx* ctx, int32_t layer, int32_t* N, int32_t* K, int32_t* Kp);

/*
 * Test hooks: the same kernels as tasq_linear_forward, with caller-owned buffers.
 *
 * tasq_debug_quantize: prologue only. x as in tasq_linear_forward (layer selects K); writes
 *   xq [M, Kp] INT8 (device, row stride Kp) and s_x [M] FP32 (device).
 *
 * tasq_debug_gemm_s32: GEMM only, raw INT32 accumulators. xq [M, Kp] INT8 (device, stride Kp);
 *   acc [M, N] INT32 (device, row stride ld_acc >= N, % 8 == 0).
 *
 * tasq_debug_gemm: GEMM only with the dequantizing epilogue. xq as above, s_x [M] FP32
 *   (device), y [M, N] in out_dtype (a tasq_out_dtype, independent of the context's).
 */
tasq_status tasq_debug_quantize(tasq_ctx* ctx, const void* x, int64_t M, int64_t ldx, int32_t layer,
                                int8_t* xq, float* s_x, void* stream);
tasq_status tasq_debug_gemm_s32(tasq_ctx* ctx, const int8_t* xq, int64_t M, int32_t layer, int32_t step,
                                int32_t* acc, int64_t ld_acc, void* stream);
tasq_status tasq_debug_gemm(tasq_ctx* ctx, const int8_t* xq, const float* s_x, int64_t M, int32_t layer,
                            int32_t step, void* y, int64_t ldy, int32_t out_dtype, void* stream);

/*
 * Copy the device schedule table [num_layers * num_steps] (row-major by layer) into bits_host
 * (host). Stream-ordered after everything enqueued on `stream` before it; synchronises `stream`.
 */
tasq_status tasq_get_schedule(tasq_ctx* ctx, uint8_t* bits_host, void* stream);

/*
 * On-device precision predictor: the DMPQ rule of 6Bit-Diffusion (technical summary, section
 * 2.A, "Quantizacao de Precisao Mista Dinamica"). The relative L1 change of a transformer block
 * over the previous step, Gamma = ||out - in||_1 / ||in||_1, picks the bit width of the block's
 * linears for `step`: bits[layer][step] = Gamma > tau ? bits_unstable : bits_stable for every
 * layer in `layers`. When ||in||_1 = 0, Gamma is +inf (or 0 if the output is zero as well) and
 * the layers take bits_unstable. Each width is an INT8 width 1..8 or TASQ_NVFP4 (0): the pages
 * keep unstable layers in INT8 and compress stable ones to NVFP4 (bits_unstable = 8,
 * bits_stable = TASQ_NVFP4). When one of the two is NVFP4, later forwards of these (layer, step)
 * entries launch both the INT8 and the NVFP4 kernels; each reads the device table and the one
 * whose format was not chosen returns at once, so the choice needs no host round trip and holds
 * inside a captured CUDA graph as well.
 *   block_in, block_out : device FP16 [M, D], the block's input and output at the previous
 *                         step, row strides ld_in / ld_out (elements, >= D, % 8 == 0), 16-byte
 *                         aligned; D % 8 == 0. Neither is modified.
 *   layers              : host array [num_block_layers] (1 .. TASQ_DMPQ_MAX_LAYERS) of layer
 *                         indices; read before the call returns.
 *   gamma_out           : optional device double that receives Gamma.
 * Both L1 sums are exact (integer arithmetic in units of 2^-24); Gamma is their IEEE double
 * quotient, each sum rounded once to nearest-even. One kernel runs on `stream` (using
 * context-owned partial sums: calls of one context must not overlap on different streams),
 * and the table
 * entries change in stream order: forwards enqueued later on `stream` use the new widths,
 * with no host round trip. Returns TASQ_ERR_INVALID_ARG for bad arguments (checked on the
 * host before anything is enqueued), including M * D so large that a per-thread 64-bit partial
 * sum could overflow. Non-finite inputs give an undefined decision.
 */
tasq_status tasq_dmpq_update(tasq_ctx* ctx, const void* block_in, int64_t ld_in, const void* block_out,
                             int64_t ld_out, int64_t M, int32_t D, const int32_t* layers,
                             int32_t num_block_layers, int32_t step, double tau, int32_t bits_unstable,
                             int32_t bits_stable, double* gamma_out, void* stream);

/*
 * NVFP4 steps (6Bit-Diffusion, technical summary section 2.A: stable layers compressed to NVFP4,
 * Blackwell's native 4-bit format, unstable ones kept in INT8). A schedule entry of TASQ_NVFP4
 * (0) makes that (layer, step) an NVFP4 step: the forward's prologue launch quantizes the
 * block-Hadamard activations to E2M1 codes with one UE4M3 scale per 16 elements along K and a
 * per-token FP32 scale, and converts the layer's shared INT8 weights the same way (per output
 * channel, s_w unchanged); a block-scaled tcgen05 GEMM (kind::mxf4nvf4) with FP32 accumulation
 * and the same dequantizing epilogue follows. Entries 1..8 keep the INT8 path with that many
 * weight bits. NVFP4 codes are packed two per byte along K, the lower-indexed element in the low
 * nibble; block scales use 512-byte chunks, one per 128 rows x 64 elements of K, in which row r
 * and 16-block j sit at byte (r % 32) * 16 + ((r % 128) / 32) * 4 + j, the chunks of a 128-row
 * group in K order; K is padded with zero scales to a multiple of 256.
 * tasq_linear_forward_noalloc stays INT8-only.
 */
#define TASQ_NVFP4 0
#define TASQ_NVFP4_RAW_ACC 2   /* out_kind of tasq_debug_gemm_nvfp4: raw FP32 accumulators */

/* Host-only: bytes of the NVFP4 block scales of `rows` rows with Kp in-features (a multiple of 64). */
tasq_status tasq_nvfp4_scale_bytes(int64_t rows, int32_t Kp, int64_t* bytes);

/*
 * Test hook: the NVFP4 prologue alone. x FP16 [M, K] (row stride ldx), codes [M, Kp / 2] bytes,
 * scales tasq_nvfp4_scale_bytes(M, Kp) bytes (both 16-byte aligned, caller-owned device memory),
 * s_x [M] FP32. Scales of padding rows and of K past Kp are left as they were.
 */
tasq_status tasq_debug_quantize_nvfp4(tasq_ctx* ctx, const void* x, int64_t M, int64_t ldx, int32_t layer,
                                      void* codes, void* scales, float* s_x, void* stream);

/* Test hook: the NVFP4 conversion of a layer's shared INT8 weights into codes [N, Kp / 2] and
 * scales (tasq_nvfp4_scale_bytes(N, Kp) bytes), the K padding written as zero scales. */
tasq_status tasq_debug_nvfp4_weights(tasq_ctx* ctx, int32_t layer, void* codes, void* scales, void* stream);

/*
 * Test hook: the NVFP4 GEMM on given activation codes, scales (as tasq_debug_quantize_nvfp4 writes
 * them, with zero or finite scales wherever the layout has no row or no K) and s_x, against the
 * layer's converted weights. out_kind TASQ_OUT_F16 / TASQ_OUT_BF16 write y = acc * s_x * s_w;
 * TASQ_NVFP4_RAW_ACC writes the FP32 accumulators acc themselves (y float32 [M, ldy], ldy a
 * multiple of 4).
 */
tasq_status tasq_debug_gemm_nvfp4(tasq_ctx* ctx, const void* codes, const void* scales, const float* s_x, int64_t M,
                                  int32_t layer, void* y, int64_t ldy, int32_t out_kind, void* stream);

/*
 * Test hook: which GEMM kernel later forwards of this context use. 0 (default) lets the library
 * choose per launch from the wave count of each kernel's tiles (tasq_gemm_choice), 1 forces one
 * CTA per 128 x 256 tile (tcgen05 cta_group::1), 2 forces CTA pairs on 256 x 256 tiles (tcgen05
 * cta_group::2). Both compute identical results. Any other mode is TASQ_ERR_INVALID_ARG.
 * The mode also selects the NVFP4 GEMM (forwards of NVFP4 steps and tasq_debug_gemm_nvfp4): 0
 * chooses by wave count (tasq_nvfp4_gemm_choice), 1 forces one CTA per 128 x 128 tile, 2 forces
 * CTA pairs on tiles of 256 channels x 192 tokens. Both NVFP4 kernels read the same code and
 * scale layouts; their FP32
 * accumulators may differ in rounding order, each within the bound documented for
 * tasq_debug_gemm_nvfp4's raw accumulators.
 */
tasq_status tasq_debug_set_gemm_mode(tasq_ctx* ctx, int32_t mode);

/*
 * Host-only query (no device, no context): whether a forward with the automatic choice runs the
 * GEMM of M tokens and N output channels on a device with num_sms SMs on CTA pairs (*pair = 1,
 * tiles of 256 channels x 256 tokens) or on one CTA per tile (*pair = 0, 128 x 256). The choice
 * depends on these three numbers only. TASQ_ERR_INVALID_ARG for a NULL output, M or N <= 0, or
 * num_sms < 2.
 */
tasq_status tasq_gemm_choice(int64_t M, int32_t N, int32_t num_sms, int32_t* pair);

/*
 * Host-only query (no device, no context), the NVFP4 counterpart of tasq_gemm_choice: whether an
 * NVFP4 step with the automatic choice runs its block-scaled GEMM of M tokens and N output
 * channels on CTA pairs (*pair = 1, tiles of 256 channels x 192 tokens) or on one CTA per tile
 * (*pair = 0, 128 x 128). The pair is taken unless it needs more than 1/1.1 as many waves of
 * tiles as the one-CTA kernel: a pair tile holds 1.5x the MACs per SM and runs them about 1.37x
 * faster (6Bit-Diffusion's NVFP4 stable-layer step; see tasq_set_schedule). TASQ_ERR_INVALID_ARG
 * for a NULL output, M or N <= 0, or num_sms < 2.
 */
tasq_status tasq_nvfp4_gemm_choice(int64_t M, int32_t N, int32_t num_sms, int32_t* pair);

/*
 * Test hook: where later forwards (and tasq_debug_gemm / tasq_debug_gemm_s32) apply the step's
 * LSB mask to the weights (TASQ, "LSB masking" of the stored INT8 weights).
 *   0 (default) and 1: in flight, inside the GEMM: its mask warps AND every weight tile of the
 *     stored buffer with the step's byte mask in shared memory as it lands (no pass when the device
 *     table keeps all 8 bits).
 *   2: ahead of the GEMM, in the prologue launch, into a context-owned masked copy of the layer's
 *     weights (2 N Kp bytes of extra traffic per forward) that the GEMM loads as it is; kept to
 *     measure the in-flight mask against.
 * Every mode reads the bit width from the device schedule table, so all give identical results
 * for every table. Any other mode is TASQ_ERR_INVALID_ARG.
 */
tasq_status tasq_debug_set_mask_mode(tasq_ctx* ctx, int32_t mode);

/*
 * Test hook: which prologue kernel later forwards and tasq_debug_quantize use. 1: the direct-load
 * kernel (each thread loads its 32 channels straight from global memory, one block of rows per
 * CTA); 2: the bulk-fed kernel (one persistent CTA per SM, rows streamed into a ring of
 * shared-memory stages by 1-D bulk copies) wherever its layout fits, else the direct one; 3: the
 * direct-load kernel with 64 channels a thread; 0 (default): the 64-channel kernel for rows longer
 * than 9216 channels (Kp), else the bulk-fed kernel when every SM gets many blocks of rows, else the
 * direct one. All produce bit-identical codes and scales. Any other mode is TASQ_ERR_INVALID_ARG.
 */
tasq_status tasq_debug_set_prologue_mode(tasq_ctx* ctx, int32_t mode);

/*
 * Failure-detection hook: launch one CTA that waits, with the context's wait limit, on a
 * shared-memory barrier that nothing ever arrives on. The wait must run out, set
 * TASQ_DEVICE_TIMEOUT_MMA in the status word and return. Used by tests to check that a
 * stuck wait ends with a status the host can read and leaves the context usable.
 */
tasq_status tasq_debug_stuck_wait(tasq_ctx* ctx, void* stream);

/*
 * Kernel timing trace (native instrumentation). When enabled with capacity > 0, every forward
 * records CUDA events around its prologue and GEMM kernels on the forward's stream, for up to
 * `capacity` forwards (later forwards are not recorded). tasq_trace_read synchronises the
 * recorded events and returns, per kernel kind, the number of launches and the summed
 * duration in milliseconds, then clears the trace. capacity 0 disables tracing. Any output
 * pointer may be NULL.
 *   gemm_ops          : 2 M N K integer ops of the recorded GEMMs (K unpadded).
 *   prologue_bytes    : the prologue launches' activation bytes, M (2 K + Kp + 4) per launch
 *                       (FP16 read, INT8 codes and FP32 scale written); NVFP4 steps count their
 *                       codes and block scales instead.
 *   weight_pass_bytes : bytes the same launches moved for weights: 2 N Kp per masked copy made
 *                       ahead of the GEMM (tasq_debug_set_mask_mode 2 only), and the NVFP4 steps'
 *                       weight conversion.
 */
tasq_status tasq_trace_enable(tasq_ctx* ctx, int32_t capacity);
tasq_status tasq_trace_read(tasq_ctx* ctx, int32_t* prologue_launches, double* prologue_ms,
                            int32_t* gemm_launches, double* gemm_ms, double* gemm_ops, double* prologue_bytes,
                            double* weight_pass_bytes);

/*
 * Allocation-free variant of tasq_linear_forward, for callers that cannot call cudaMalloc:
 * code that runs inside a custom allocator or memory-pool callback, a host that hands every byte
 * of device memory to its own arena up front, or a capture harness that forbids allocation.
 * The pages have no counterpart; this is a deployment entry point around the same two kernels.
 *
 * No context is needed: the caller passes the layer's weights directly (the mask is applied to
 * them in flight, they are never copied or modified) and this call allocates nothing. The
 * activation codes and scales go to one fixed device array of TASQ_NOALLOC_SCRATCH_BYTES that
 * every GPU loading this library reserves until the process exits.
 *   x          : device FP16 [M, K], row stride ldx (>= K, % 8 == 0), 16-byte aligned.
 *   K          : in-features, >= 8 and % 8 == 0; Kp = ceil(K / hadamard_n) * hadamard_n.
 *   w          : device INT8 [N, Kp] row-major, 16-byte aligned (caller-owned, read only).
 *   s_w        : device FP32 [N].
 *   bits       : bit width for this call, 1..8 (8 = all bit planes kept).
 *   y          : device [M, N] in out_dtype, row stride ldy (>= N, % 8 == 0), 16-byte aligned.
 *   device_status : optional device uint32 that receives TASQ_DEVICE_* bits (OR-ed in; the
 *                caller clears it). With NULL the bits go to a status word inside the fixed array
 *                instead, which the call clears first and tasq_noalloc_device_status reads.
 * Limits: round_up(256 + 4 * M, 1024) + M * Kp bytes must not exceed TASQ_NOALLOC_SCRATCH_BYTES
 * (a 256-byte control block and the M FP32 scales, rounded up to 1 KiB, then the M x Kp INT8
 * codes); larger sizes return TASQ_ERR_WORKSPACE before anything is enqueued.
 * The first call on each device, made with that device current, looks the array's device
 * address up (cudaGetSymbolAddress) and caches it with the CUDA context that was current; a
 * later call under another context of the device (a non-primary driver context, or the primary
 * context created again after cudaDeviceReset) looks it up again. Make the first call under each
 * context before any stream capture. Every call uses the same array and leaves its contents
 * behind for the next one, so calls that overlap on the GPU (on different streams, or from
 * different threads without ordering) race on it and must be serialised by the caller.
 */
#define TASQ_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
tasq_status tasq_linear_forward_noalloc(const void* x, int64_t M, int64_t ldx, int32_t K, const int8_t* w,
                                        const float* s_w, int32_t N, int32_t bits, int32_t hadamard_n, void* y,
                                        int64_t ldy, int32_t out_dtype, uint32_t* device_status, void* stream);

/*
 * The status word that tasq_linear_forward_noalloc calls made with device_status == NULL write
 * on the current device: TASQ_DEVICE_* bits of the last such call (each one clears the word
 * first), so that a caller without a device word of its own can still learn that a bounded wait
 * ran out. Stream-ordered after the work enqueued on `stream`, which it synchronises; with clear
 * non-zero the word is reset to 0 afterwards. Allocates nothing. The pages have no counterpart.
 */
tasq_status tasq_noalloc_device_status(uint32_t* status_out, int32_t clear, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TASQ_H_ */
