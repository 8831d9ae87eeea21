/*
 * moemx.h - C ABI of libmoemx: the expert MLP of one mixture-of-experts layer on one
 * NVIDIA B200 (sm_100a), forward and backward, with MXFP8 or BF16 GEMM operands.
 *
 * What the library computes is the chain the pages describe as
 *   GroupedLinear(gate_up) -> ScaledSwiGLU -> GroupedLinear(down)
 * (ai4snews, paragraph 3; sitech.ge, "Memory and quantization overhead"), with the tokens
 * of every expert gathered by the per-expert counts ``split_sizes`` into one grouped call
 * (sitech.ge, "Grouped experts instead of a Python loop"; andresseo.expert, "Fragmented
 * Expert Kernels"), and operands in MXFP8: 8-bit E4M3 elements with one power-of-two
 * E8M0 scale per block of 32 consecutive values along the GEMM's K (sitech.ge, "Memory and
 * quantization overhead"; ai4snews, paragraph 2), quantised every step from 16-bit masters.
 *
 * Conventions for every entry point
 *  - Pointers are DEVICE pointers unless the comment says host.  The caller allocates and
 *    owns every buffer; the library never allocates device memory inside a call (the only
 *    allocation is the small status block made by moe_ctx_create).
 *  - Tensors are row-major and contiguous.  bf16 = IEEE bfloat16 (2 bytes).  E4M3 codes and
 *    E8M0 scale bytes are uint8.  Device buffers must be 16-byte aligned.
 *  - ``stream`` is a cudaStream_t (NULL = legacy default stream).  Every call only enqueues
 *    work and returns; nothing synchronises except moe_get_status.
 *  - Host-side checks return an error code and enqueue nothing.  Errors found on the device
 *    (an expert index out of range, a split_sizes that disagrees with topk_idx, a bounded
 *    wait that expired) are recorded in the context's device status word; the kernels that
 *    find them stop early without trapping.  moe_get_status reads and clears that word.
 *  - Calls that share a context may run on different streams; they share only the status word.
 */
#ifndef MOEMX_H
#define MOEMX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Rows of the permuted (expert-sorted) token space are grouped into per-expert segments
 * padded to a multiple of this many rows.  128 is one tensor-core tile and a multiple of the
 * 32-row MXFP8 block, so token-axis scale blocks never straddle two experts. */
#define MOE_ROW_ALIGN 128

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* null pointer, negative or zero size, bad flag              */
  MOE_ERR_SHAPE = 2,        /* a size breaks an alignment rule stated below               */
  MOE_ERR_UNSUPPORTED = 3,  /* device is not sm_100, or E/k beyond the stated maxima      */
  MOE_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed (launch, tensor map)    */
  MOE_ERR_DEVICE = 5,       /* device-detected: expert index out of range or a caller
                               split_sizes that does not match topk_idx                   */
  MOE_ERR_TIMEOUT = 6,      /* a bounded in-kernel wait expired; the kernel gave up       */
  MOE_ERR_WORKSPACE = 7     /* a workspace / saved buffer is smaller than required        */
} moe_status_t;

/* GEMM operand precision of the fused layer.  FP8 is per-tensor FP8 with current scaling (ai4snews
 * paragraph 2: FP8 and MXFP8 training; MXFP8 being the format that adds a scale per block of 32,
 * plain FP8 keeps one scale per tensor): see "Per-tensor FP8" at the fused layer below. */
typedef enum { MOE_PREC_BF16 = 0, MOE_PREC_MXFP8 = 1, MOE_PREC_FP8 = 2 } moe_precision_t;

/* flags of mxfp8_quantize */
#define MXFP8_ROWWISE 1        /* blocks of 32 along each row                              */
#define MXFP8_COLWISE_T 2      /* blocks of 32 down each column, written transposed        */
#define MXFP8_SF_MMA_LAYOUT 4  /* scales in the tensor-core tile layout instead of row-major */
#define MXFP8_FLAG_SCALE_FLOOR 8 /* shared exponent by the OCP floor rule instead of round-up   */
#define MXFP8_FLAG_E5M2 16       /* E5M2 elements (max 57344) instead of E4M3                   */

/* flags of fp8_quantize */
#define FP8_ROWWISE 1        /* codes in the source layout (required)                      */
#define FP8_COLWISE_T 2      /* the same codes transposed as well                          */
#define FP8_FLAG_E5M2 16     /* E5M2 elements (max 57344) instead of E4M3 (max 448)         */

/* Element format of the gradient operands (dy, dh) of the backward GEMMs (moe_ctx_set_grad_format). */
#define MOE_GRAD_E4M3 0
#define MOE_GRAD_E5M2 1

/* Shared-exponent rules (moe_ctx_set_scale_rule).  ROUND_UP: e = the smallest integer with
 * amax <= 448 * 2^e, so no element saturates (this library's default reading of "a scaling factor
 * per block of 32 values" that protects the range: sitech.ge "Memory and quantization overhead").
 * FLOOR: e = floor(log2 amax) - 8, the OCP MX v1.0 rule; the block maximum scales into [256, 512)
 * and elements above 448 saturate to 448. */
#define MXFP8_SCALE_ROUND_UP 0
#define MXFP8_SCALE_FLOOR 1

#define MOE_MAX_EXPERTS 256
#define MOE_MAX_TOPK 8

typedef struct moe_ctx_s* moe_ctx_t;

/* Create a context bound to CUDA device ``device`` (allocates a 256-byte device status block).
 * Returns MOE_ERR_UNSUPPORTED unless the device is compute capability 10.0. */
moe_status_t moe_ctx_create(moe_ctx_t* ctx, int device);
moe_status_t moe_ctx_destroy(moe_ctx_t ctx);

/* Synchronise ``stream``, then read and clear the device status word.  Returns MOE_OK,
 * MOE_ERR_DEVICE or MOE_ERR_TIMEOUT (device errors), or MOE_ERR_CUDA if the stream itself
 * reported an error. */
moe_status_t moe_get_status(moe_ctx_t ctx, void* stream);

/* Debug hooks (tests only).  When set, the gate_up GEMM epilogue writes the fp32 value of
 * a = silu(g)*u*p it quantises into ``a_f32`` [capacity, f], and the down-projection dgrad
 * epilogue writes the fp32 dh = [dg, du] it quantises into ``dh_f32`` [capacity, 2f]; pass
 * NULL to switch off.  The buffers must outlive every call that runs while set. */
moe_status_t moe_ctx_set_debug_dump(moe_ctx_t ctx, float* a_f32, float* dh_f32);

/* Shared-exponent rule of every MXFP8 quantisation the fused layer makes with this context
 * (weights, x, dy and the epilogue requantisations of a and dh): MXFP8_SCALE_ROUND_UP (default) or
 * MXFP8_SCALE_FLOOR.  Calls already enqueued are not affected. */
moe_status_t moe_ctx_set_scale_rule(moe_ctx_t ctx, int rule);

/* Element format of the MXFP8 (or per-tensor FP8) gradient operands of the fused layer's backward
 * with this context (ai4snews paragraph 2: FP8 and MXFP8 training): MOE_GRAD_E4M3 (default) or
 * MOE_GRAD_E5M2.  Per-tensor FP8 takes it the same way: dy and dh get E5M2 codes with scales
 * computed against 57344.
 * With E5M2, dy (quantised along d and along the tokens) and the requantised dh take E5M2
 * elements (round to nearest even, saturating at 57344) with the same E8M0 scales per 32 values,
 * the shared exponent computed against 57344 (round-up: the smallest e with amax <= 57344 * 2^e;
 * floor rule: floor(log2 amax) - 15); every backward GEMM then multiplies an E5M2 A operand by an
 * E4M3 B operand (weights, a, x).  The forward is unchanged. */
moe_status_t moe_ctx_set_grad_format(moe_ctx_t ctx, int fmt);

/* Format of the gate/up pre-activations h that a training forward with this context saves for the
 * backward (the backward must run with the same setting).  Long sequences make h the largest saved
 * tensor (4*T*k*f bytes in bf16; andresseo.expert "Memory Pressure From Long Sequences", sitech.ge
 * "Memory and quantization overhead"):
 *   MOE_SAVED_H_BF16  (default) bf16 h [capacity, 2f];
 *   MOE_SAVED_H_MXFP8 MXFP8 h: E4M3 codes [capacity, 2f] with one E8M0 scale per 32 values along
 *                     2f (row-major [capacity, 2f/32]), quantised in the gate_up GEMM's epilogue with
 *                     the context's scale rule; the dSwiGLU epilogue reads g and u dequantised from
 *                     it.  About half the bytes; MXFP8 precision only (MOE_ERR_UNSUPPORTED otherwise).
 *   MOE_SAVED_H_RECOMPUTE no h at all: the forward keeps x's gate_up operand instead (MXFP8 row-wise
 *                     codes and scales, or the BF16 gathered rows, [capacity, d]); the backward
 *                     quantises W1 again (MXFP8), re-runs the gate_up GEMM with an epilogue that only
 *                     writes h into its workspace (moe_bwd_workspace_size_ex), and goes on as with a
 *                     saved bf16 h, giving the same results bit for bit.  Costs one more gate_up GEMM
 *                     (and W1 quantisation) per backward.  MXFP8 and BF16 only.
 * Per-tensor FP8 saves h in bf16 only (MOE_ERR_UNSUPPORTED for the other two).
 * moe_saved_size_ex / moe_bwd_workspace_size_ex give the buffer sizes for a mode (0 for an
 * unsupported combination). */
#define MOE_SAVED_H_BF16 0
#define MOE_SAVED_H_MXFP8 1
#define MOE_SAVED_H_RECOMPUTE 2
moe_status_t moe_ctx_set_saved_h(moe_ctx_t ctx, int mode);

/* Forward GEMMs in one launch (hyper.ai: gate-up projection, SwiGLU, routing-weight scaling and the
 * down projection fused into a single GroupedMLP kernel).  With ``on`` non-zero the fused layer's
 * forward runs one persistent kernel that walks the gate_up tiles and then the down tiles; each
 * down tile's loads wait (bounded, MOE_ERR_TIMEOUT on expiry) until every gate_up tile of its
 * 128-row block has written its rows of a, which the gate_up epilogues release through one
 * counter per row block in the forward workspace.  The kernel keeps one CTA on every SM for its
 * whole run and its CTAs wait on one another, so it needs the GPU to itself: kernels of other
 * streams that hold SMs meanwhile can make those waits expire.  Default off.  Per-tensor FP8 keeps
 * two launches whatever the setting: a is quantised only once its expert's maximum is complete. */
moe_status_t moe_ctx_set_fused_forward(moe_ctx_t ctx, int on);

/* Test hook for the bounded in-kernel waits (tests only).  With ``stall`` non-zero, every CTA of
 * the persistent kernels (the grouped GEMMs and the TMA-fed quantiser) makes one extra wait on a
 * word of the context's status block that nothing ever sets, bounded by ``limit_cycles`` SM clock
 * cycles (1 .. about 2e9): the GEMM producer after it has issued the first stages of its first tile
 * (operand loads and MMAs in flight), the quantiser with its first source tiles in flight.  The
 * wait expires as any wait would: the CTA raises its abort flag, every role stops, the copies and
 * MMAs already issued are waited for (full-length bounded waits), TMEM is freed, and the call's
 * moe_get_status returns MOE_ERR_TIMEOUT.  Outputs of calls made while it is set are undefined.
 * stall = 0 switches it off; the context stays usable. */
moe_status_t moe_ctx_set_test_stall(moe_ctx_t ctx, int stall, int64_t limit_cycles);

const char* moe_status_string(moe_status_t s);

/* Launch hook (profiling).  When set, the fused-layer and codec entry points call
 * hook(user, kernel_name, 0, stream) just before and hook(user, kernel_name, 1, stream) just
 * after enqueueing each of their kernels, on the host thread that made the call, so a caller can
 * record CUDA events around every kernel on the stream it runs on.  NULL switches it off. */
typedef void (*moe_launch_hook_t)(void* user, const char* kernel, int after, void* stream);
moe_status_t moe_ctx_set_launch_hook(moe_ctx_t ctx, moe_launch_hook_t hook, void* user);

/* ---------------------------------------------------------------------------------------
 * mxfp8_quantize: bf16 -> MXFP8 (sitech.ge "Memory and quantization overhead": one scale per
 * block of 32 consecutive values; ai4snews paragraph 2).
 *
 * x        bf16 [batch, rows, cols]
 * flags    MXFP8_ROWWISE and/or MXFP8_COLWISE_T, optionally | MXFP8_SF_MMA_LAYOUT and
 *          | MXFP8_FLAG_SCALE_FLOOR (the OCP floor rule below instead of round-up)
 *          | MXFP8_FLAG_E5M2 (E5M2 element codes; 57344 replaces 448 and 15 replaces 8 below)
 * q_row    uint8 [batch, rows, cols] E4M3 codes, blocks of 32 along each row   (ROWWISE)
 * s_row    uint8 E8M0 bytes, [batch, rows, cols/32] row-major, or the MMA layout (ROWWISE)
 * q_colT   uint8 [batch, cols, rows] codes of blocks of 32 down each column, transposed
 * s_colT   uint8 E8M0 bytes, [batch, cols, rows/32] row-major, or the MMA layout
 *
 * Scale rule: e = the smallest integer with amax <= 448 * 2^e over the block (clamped to
 * [-127, 127]), byte = e + 127; element code = E4M3(v * 2^-e) rounded to nearest-even,
 * saturating (no element can exceed 448 under this rule); all-zero blocks get byte 0.
 * With MXFP8_FLAG_SCALE_FLOOR: e = floor(log2 amax) - 8, elements above 448 after scaling
 * saturate to 448.
 *
 * MMA layout (MXFP8_SF_MMA_LAYOUT): a scale matrix S[R][KB] (R rows, KB = K/32 blocks) is
 * stored as 512-byte tiles, tile (R/128 index rb, KB/4 index kb4) at byte (rb*KB/4 + kb4)*512,
 * and inside a tile S[r][kb] sits at 16*(r%32) + 4*((r/32)%4) + kb%4.  It needs R and K to be
 * multiples of 128 for each batch; a batch's tiles follow the previous batch's.
 *
 * Shapes: cols % 32 == 0; rows % 32 == 0 when COLWISE_T is set; with the MMA layout rows and
 * cols must be multiples of 128.  Returns MOE_ERR_SHAPE otherwise.
 */
moe_status_t mxfp8_quantize(moe_ctx_t ctx, const void* x, int64_t batch, int64_t rows, int64_t cols,
                            int flags, uint8_t* q_row, uint8_t* s_row, uint8_t* q_colT, uint8_t* s_colT,
                            void* stream);

/* Inverse of mxfp8_quantize for row-wise E4M3 data (tests): out[r][c] = decode(q[r][c]) * 2^(s-127),
 * fp32 [rows, cols]; ``sf_mma_layout`` says how ``s`` is laid out.  cols % 32 == 0. */
moe_status_t mxfp8_dequantize(moe_ctx_t ctx, const uint8_t* q, const uint8_t* s, int64_t rows, int64_t cols,
                              int sf_mma_layout, float* out, void* stream);

/* ---------------------------------------------------------------------------------------
 * fp8_quantize: bf16 -> per-tensor FP8 with current scaling (ai4snews paragraph 2: FP8 and MXFP8
 * training; plain FP8 has no block scales, so one scale serves the whole tensor).
 *
 * x        bf16 [batch, rows, cols], each batch one tensor
 * flags    FP8_ROWWISE (required), optionally | FP8_COLWISE_T, | FP8_FLAG_E5M2
 * q_row    uint8 [batch, rows, cols] codes
 * q_colT   uint8 [batch, cols, rows] the same codes transposed (FP8_COLWISE_T)
 * scale    fp32 [batch] out: the scale s of each tensor (also used as scratch during the call)
 *
 * s = vmax / amax rounded to nearest in fp32, amax the tensor's largest magnitude, vmax 448 (E4M3)
 * or 57344 (E5M2); s = 1 for an all-zero tensor; the largest finite fp32 when the quotient
 * overflows.  Code = E4M3 (E5M2) of the fp32 product v * s, rounded to nearest even, saturating;
 * the value it stands for is code / s.
 * Shapes: rows % 128 == 0, cols % 128 == 0 (MOE_ERR_SHAPE otherwise); batch <= MOE_MAX_EXPERTS
 * (MOE_ERR_UNSUPPORTED); x, q_row, q_colT 16-byte aligned (MOE_ERR_INVALID_ARG). */
moe_status_t fp8_quantize(moe_ctx_t ctx, const void* x, int64_t batch, int64_t rows, int64_t cols, int flags,
                          uint8_t* q_row, uint8_t* q_colT, float* scale, void* stream);

/* ---------------------------------------------------------------------------------------
 * Routing bookkeeping and token permutation (sitech.ge "Grouped experts instead of a Python
 * loop": GroupedLinear gathers each expert's tokens and takes per-expert counts).
 *
 * capacity = moe_capacity_rows(T, k, E): the padded row count for the worst-case routing.
 * Slot s = t*k + j (token t, choice j) goes to expert topk_idx[t][j]; experts keep their slots
 * in increasing s (a stable counting sort); expert e owns rows [poffsets[e], poffsets[e+1])
 * of the permuted space, its split_sizes[e] slots first, then zero padding up to a multiple
 * of MOE_ROW_ALIGN.  Rows past poffsets[E] up to capacity are padding as well.
 */
int64_t moe_capacity_rows(int64_t T, int k, int E);

/* x            bf16 [T, d] or NULL (routing only)
 * topk_idx     int32 [T, k], values in [0, E)
 * topk_prob    fp32 [T, k] or NULL
 * split_sizes_in int32 [E] or NULL: if given it must equal the histogram of topk_idx
 *              (MOE_ERR_DEVICE otherwise, reported by moe_get_status)
 * outputs      split_sizes int32 [E]; poffsets int32 [E+1]; sorted_to_src int32 [capacity]
 *              (slot of each row, -1 for padding); src_to_sorted int32 [T*k] (row of each slot);
 *              prob_perm fp32 [capacity] or NULL (topk_prob of each row, 0 for padding);
 *              x_perm bf16 [capacity, d] or NULL (x[slot/k] per row, zeros for padding)
 * Limits: 1 <= k <= MOE_MAX_TOPK, 1 <= E <= MOE_MAX_EXPERTS, d % 32 == 0. */
moe_status_t moe_permute(moe_ctx_t ctx, const void* x, const int32_t* topk_idx, const float* topk_prob,
                         int64_t T, int k, int E, int64_t d, const int32_t* split_sizes_in,
                         int32_t* split_sizes, int32_t* poffsets, int32_t* sorted_to_src,
                         int32_t* src_to_sorted, float* prob_perm, void* x_perm, void* stream);

/* Combine rows back to tokens: y[t] = bf16( sum_{j<k} w_j * fp32(y_perm[src_to_sorted[t*k+j]]) )
 * summed in fp32 in order j = 0..k-1, with w_j = probs[t][j] (fp32 products) or 1 if probs is
 * NULL (the fused layer applies the probability inside ScaledSwiGLU, so it combines with NULL).
 * An entry of src_to_sorted equal to -1 (a slot moe_permute rejected for its expert index) is
 * skipped; every other entry must be a row of y_perm.
 * y_perm bf16 [capacity, d]; y bf16 [T, d]; d % 8 == 0. */
moe_status_t moe_unpermute(moe_ctx_t ctx, const void* y_perm, const int32_t* src_to_sorted, const float* probs,
                           int64_t T, int k, int64_t d, void* y, void* stream);

/* ---------------------------------------------------------------------------------------
 * The fused layer (ai4snews paragraph 3: Sequential(GroupedLinear(gate_up), ScaledSwiGLU(),
 * GroupedLinear(down)) with a matching fused backward; sitech.ge "Memory and quantization
 * overhead").  For slot (t, j), e = topk_idx[t][j], p = topk_prob[t][j]:
 *   h = x_t W1_e^T,  g = h[0:f], u = h[f:2f],  a = silu(g) * u * p,  y_t += a W2_e^T
 * W1_e = w_gate_up[e] bf16 [2f, d] (gate rows first), W2_e = w_down[e] bf16 [d, f].
 * MXFP8: every GEMM operand is quantised along that GEMM's K with blocks of 32; the weights
 * are quantised from the bf16 masters inside each call.  a is requantised straight from the
 * gate_up GEMM's epilogue into the down GEMM's operand; h never goes to memory except the bf16
 * copy saved for the backward when ``training`` is set.  Products accumulate in fp32.
 *
 * Per-tensor FP8 (MOE_PREC_FP8): every GEMM operand of every expert is one tensor with one scale
 * (fp8_quantize's rule): W1_e, W2_e, expert e's rows of x, of a, of dy and of dh.  The weights and
 * the gathered rows of x / dy are quantised after a pass that finds their maxima; a and dh leave
 * their GEMM epilogues as bf16 rows together with their per-expert maxima and are quantised in a
 * pass of their own.  One set of codes serves both GEMMs that read a tensor (the transposed copy
 * holds the same codes).  The GEMMs run on the kind::f8f6f4 tensor-core instructions and multiply
 * each expert's fp32 accumulator by 1/s_A * 1/s_B.  E4M3 elements; dy and dh take the context's
 * gradient format.
 *
 * w_gate_up, w_down, dw_gate_up, dw_down are HOST arrays of E device pointers (each expert
 * keeps its own weight tensor, ai4snews paragraph 1).
 * Shapes: d % 256 == 0, f % 256 == 0, 1 <= k <= MOE_MAX_TOPK, 1 <= E <= MOE_MAX_EXPERTS.
 *
 * saved: written by a training forward, read by the backward; moe_saved_size bytes.
 * workspace: scratch for one call; moe_fwd_workspace_size / moe_bwd_workspace_size bytes.
 * Neither may be shared by two calls in flight at once.
 */
size_t moe_saved_size(int64_t T, int k, int E, int64_t d, int64_t f, moe_precision_t prec);
/* Saved-buffer size when h is saved in format ``saved_h`` (see moe_ctx_set_saved_h); 0 for an
 * unsupported combination. */
size_t moe_saved_size_ex(int64_t T, int k, int E, int64_t d, int64_t f, moe_precision_t prec, int saved_h);
size_t moe_fwd_workspace_size(int64_t T, int k, int E, int64_t d, int64_t f, moe_precision_t prec, int training);
size_t moe_bwd_workspace_size(int64_t T, int k, int E, int64_t d, int64_t f, moe_precision_t prec);
size_t moe_bwd_workspace_size_ex(int64_t T, int k, int E, int64_t d, int64_t f, moe_precision_t prec, int saved_h);

/* x bf16 [T, d]; topk_idx int32 [T, k]; topk_prob fp32 [T, k]; split_sizes int32 [E] or NULL
 * (checked against topk_idx on the device when given); y bf16 [T, d]. */
moe_status_t moe_grouped_mlp_fwd(moe_ctx_t ctx, const void* x, const int32_t* topk_idx, const float* topk_prob,
                                 const int32_t* split_sizes, const void* const* w_gate_up,
                                 const void* const* w_down, int64_t T, int64_t d, int64_t f, int E, int k,
                                 moe_precision_t prec, int training, void* y, void* saved, size_t saved_bytes,
                                 void* workspace, size_t workspace_bytes, void* stream);

/* dy bf16 [T, d]; saved from a training forward with the same arguments; outputs dx bf16 [T, d],
 * dw_gate_up[e] bf16 [2f, d], dw_down[e] bf16 [d, f] (overwritten, zeros for experts with no
 * tokens), d_topk_prob fp32 [T, k] (gradient of topk_prob). */
moe_status_t moe_grouped_mlp_bwd(moe_ctx_t ctx, const void* dy, const void* saved, size_t saved_bytes,
                                 const void* const* w_gate_up, const void* const* w_down, int64_t T, int64_t d,
                                 int64_t f, int E, int k, moe_precision_t prec, void* dx, void* const* dw_gate_up,
                                 void* const* dw_down, float* d_topk_prob, void* workspace, size_t workspace_bytes,
                                 void* stream);

/* ---------------------------------------------------------------------------------------
 * Inference forward without any device allocation (no counterpart on the pages; this is a
 * deployment convenience).  Some callers cannot allocate device memory when they run the layer:
 * a serving loop whose device memory is entirely owned by its own pool allocator, or a host
 * framework whose extensions may not call cudaMalloc / cudaFree on the hot path (those calls can
 * synchronise the device and fail once the pool has taken the memory).  This entry point computes
 * exactly what moe_grouped_mlp_fwd computes with training = 0, but takes no context and no
 * workspace: its scratch is one file-scope device array of MOE_NOALLOC_SCRATCH_BYTES that every
 * GPU which loads the library holds until the process exits.
 *  - It runs on the current CUDA device.  The first call on a device looks up that array's device
 *    address (and checks the device); make that first call before any stream capture.
 *  - Sizes whose forward workspace (moe_fwd_workspace_size with training = 0) exceeds
 *    MOE_NOALLOC_SCRATCH_BYTES are rejected with MOE_ERR_WORKSPACE before anything is enqueued.
 *  - It calls no cudaMalloc, cudaFree or allocating library routine.
 *  - Every call uses the same array, so calls that overlap on the GPU (different streams, or
 *    different host threads) race and must be serialised by the caller.  Nothing in the array
 *    needs to start at zero: each call writes every scratch byte it later reads.
 *  - device_status: optional device int the kernels OR their findings into: the value 1 (bit 0)
 *    for a bad expert index or a split_sizes mismatch, the value 2 (bit 1) for a bounded wait that
 *    expired.  The caller zeroes it and reads it after synchronising.  NULL drops the findings.
 * Arguments and layouts are those of moe_grouped_mlp_fwd. */
#define MOE_NOALLOC_SCRATCH_BYTES (64u << 20)
moe_status_t moe_grouped_mlp_fwd_noalloc(const void* x, const int32_t* topk_idx, const float* topk_prob,
                                         const int32_t* split_sizes, const void* const* w_gate_up,
                                         const void* const* w_down, int64_t T, int64_t d, int64_t f, int E, int k,
                                         moe_precision_t prec, void* y, int* device_status, void* stream);

/* ---------------------------------------------------------------------------------------
 * Tensor-core peak loop (measurement; the denominator of the GEMMs' roofline fractions).  The
 * MXFP8 GEMMs run on Blackwell's block-scaled tensor-core instructions (ai4snews, paragraph 2);
 * this measures what those instructions deliver on this GPU with nothing else in the way.
 * Enqueues one kernel: one CTA per SM, each issuing ``iters`` groups of four tcgen05 MMAs of
 * M = 128, N = 256 (K = 32 E4M3 with E8M0 scales per MMA for MXFP8, kind::mxf8f6f4; K = 32 E4M3
 * for per-tensor FP8, kind::f8f6f4; K = 16 bf16 for BF16, kind::f16) on operands resident in
 * shared memory, into one TMEM accumulator.  It
 * reads and writes no global memory except the context's status word.  ``scale_refresh``
 * (MXFP8 only) also copies the scale tiles shared memory -> TMEM before every group, as the
 * grouped GEMM mainloop does per 128-wide K step.  The caller times it (CUDA events on
 * ``stream``); moe_tensor_peak_flops gives the FLOPs of one launch (0 on bad arguments).
 * 1 <= iters <= 1000000 (MOE_ERR_INVALID_ARG otherwise). */
moe_status_t moe_tensor_peak_loop(moe_ctx_t ctx, moe_precision_t prec, int64_t iters, int scale_refresh,
                                  void* stream);
double moe_tensor_peak_flops(moe_ctx_t ctx, moe_precision_t prec, int64_t iters);

/* Inspection hook (tests): address of a named intermediate inside a saved buffer (which = 0),
 * a forward workspace (which = 1) or a backward workspace (which = 2) laid out for these
 * dimensions, given the buffer's base address ``base``; NULL for an unknown name.  Names:
 * saved: split_sizes poffsets sorted_to_src src_to_sorted prob_perm w1c_q w1c_s w2c_q w2c_s
 *        xT_q xT_s aT_q aT_s xT aT h (with moe_buffer_address_ex: h_q h_s for MOE_SAVED_H_MXFP8,
 *        xr_q xr_s xr for MOE_SAVED_H_RECOMPUTE); per-tensor FP8: pt_amax, the [4][E] maxima
 *        (fp32) of x, W1, W2 and a
 * forward workspace: w1_q w1_s w2_q w2_s x_q x_s a_q a_s x_perm a y_perm (+ the routing names
 *        when training == 0; per-tensor FP8 inference: pt_amax)
 * backward workspace: dy_q dy_s dyT_q dyT_s dh_q dh_s dhT_q dhT_s dy_perm dyT dh dhT w1T w2T
 *        dx_perm dp_part (+ hr w1r_q w1r_s for MOE_SAVED_H_RECOMPUTE; per-tensor FP8: pt_amax,
 *        the [2][E] maxima of dy and dh)
 * Scales (*_s) are in the tensor-core tile layout described at mxfp8_quantize. */
void* moe_buffer_address(int64_t T, int k, int E, int64_t d, int64_t f, moe_precision_t prec, int training,
                         int which, void* base, const char* name);
/* The same for a saved buffer laid out for the saved-h format ``saved_h``. */
void* moe_buffer_address_ex(int64_t T, int k, int E, int64_t d, int64_t f, moe_precision_t prec, int training,
                            int saved_h, int which, void* base, const char* name);

#ifdef __cplusplus
}
#endif

#endif /* MOEMX_H */
