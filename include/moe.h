/*
 * moe.h - C ABI of the sparse Mixture-of-Experts layer forward pass (sm_100a).
 *
 * The layer is the one defined on the page "Mixture of experts"
 * (rayaq.ca/ml-models/mixture-of-experts), sections "Replacing the
 * feed-forward block", "Top-k gating", "The load-balancing loss",
 * "Capacity and dropped tokens" and "Implementation":
 *
 *   h = W_r x (+ b)            router logits, fp32
 *   p = softmax(h)             full softmax over the E experts
 *   TopK(h)                    k largest logits, largest first, ties -> lower index
 *   g                          SWITCH: g_j = p[idx_j]; RENORM: softmax over the k chosen logits
 *   capacity                   C = ceil(capacity_factor * T * k / E); slots filled in
 *                              token order; overflow assignments dropped (contribute 0)
 *   y_t = sum_j kept g_tj * E_{idx_tj}(x_t)   summed in slot order j
 *   E_e(x) = W2_e relu(W1_e x)            (ReLU experts)
 *   E_e(x) = W2_e (silu(W1_e x) * W3_e x)  (SwiGLU experts)
 *   aux = E * sum_i f_i P_i    f_i: share of first choices (before capacity),
 *                              P_i: mean of p_i over the T tokens (unscaled: the
 *                              caller multiplies by alpha = 0.01)
 *   z   = mean_t (log sum_j exp h_tj)^2   (unscaled: the caller multiplies by 1e-3)
 *
 * Conventions for every entry point:
 *   - Tensor arguments are DEVICE pointers owned by the caller, row-major,
 *     16-byte aligned, and not aliased with one another.
 *   - bf16 layers: x, W1, W3, W2 and y are bf16; W_r and b_r are fp32.
 *     fp32 layers: everything is fp32.
 *   - Weights use the nn.Linear (out, in) layout: W_r [E][d], W1 and W3
 *     [E][d_ff][d], W2 [E][d][d_ff].
 *   - Every call is asynchronous on the given CUDA stream (a cudaStream_t
 *     passed as void*; NULL = the legacy default stream).  moe_forward never
 *     synchronises and never allocates device memory.
 *   - Errors detectable on the host are returned before any launch and leave
 *     the outputs untouched; a message is kept for moe_last_error().
 *     Errors raised on the device (a bounded wait that ran out) are sticky
 *     per device and reported by moe_status().
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct moe_layer* moe_handle;

enum { MOE_ACT_RELU = 0, MOE_ACT_SWIGLU = 1 };
enum { MOE_GATE_SWITCH = 0, MOE_GATE_RENORM = 1 };
enum { MOE_F32 = 0, MOE_BF16 = 1 };
enum { MOE_HIDDEN_BF16X2 = 0, MOE_HIDDEN_BF16 = 1, MOE_HIDDEN_F16 = 2, MOE_HIDDEN_AUTO = 3 };
enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* bad shape, mode, null pointer or too small workspace */
  MOE_ERR_UNSUPPORTED = 2, /* valid layer this build cannot run (alignment, limits) */
  MOE_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
  MOE_ERR_TIMEOUT = 4,     /* a device-side bounded wait ran out (kernel gave up) */
  MOE_ERR_RANGE = 5        /* MOE_HIDDEN_F16: a hidden value (or W2) beyond the fp16 range */
};

/* Kernel stages of one forward call, in launch order (see moe_debug.events). */
enum {
  MOE_STAGE_ROUTER = 0,   /* logits, softmax, top-k, gates, per-block counts      */
  MOE_STAGE_SCAN = 1,     /* per-expert scan, capacity, offsets, losses            */
  MOE_STAGE_DISPATCH = 2, /* slot ranks, drop mask, permute of x into expert order */
  MOE_STAGE_GEMM1 = 3,    /* grouped x W1^T (|| x W3^T) with ReLU / SwiGLU         */
  MOE_STAGE_GEMM2 = 4,    /* grouped h W2^T with the gate                          */
  MOE_STAGE_COMBINE = 5,  /* slot-order sum per token                              */
  MOE_NUM_STAGES = 6
};

/*
 * Optional debug / profiling hooks for moe_forward.  Every pointer may be
 * NULL.  Output arrays are device memory of the stated shape:
 *   logits_in   [T][E] fp32, read : route from these logits instead of W_r x + b
 *                                   (the "identical logits" parity mode)
 *   logits_out  [T][E] fp32, write: the fp32 router logits used for routing
 *   lse_out     [T]    fp32, write: log-sum-exp of each token's logits
 *   topk_idx    [T][k] int32      : chosen experts, largest logit first
 *   topk_gate   [T][k] fp32       : gate of each choice
 *   dest_row    [T][k] int32      : row of (t, j) in the expert-sorted buffer, -1 if dropped
 *   drop_mask   [T][k] uint8      : 1 if assignment (t, j) was dropped
 *   expert_offsets [E+1] int32    : first row of each expert in the sorted buffer
 *   y_f32       [T][d] fp32, write: the output in fp32, before its final rounding to
 *                                   the layer dtype (y is its round-to-nearest-even image)
 *   events[2*s], events[2*s+1]    : cudaEvent_t recorded on the stream right before
 *                                   and after the launches of stage s (MOE_STAGE_*)
 */
typedef struct moe_debug {
  const float* logits_in;
  float* logits_out;
  float* lse_out;
  int32_t* topk_idx;
  float* topk_gate;
  int32_t* dest_row;
  uint8_t* drop_mask;
  int32_t* expert_offsets;
  float* y_f32;
  void* events[2 * MOE_NUM_STAGES];
} moe_debug;

/*
 * Create a layer description (host memory only; no device work).
 *   num_experts E in [1, 256]; 1 <= k <= E and k <= 8; d >= 1; d_ff >= 1;
 *   act MOE_ACT_*; gate_mode MOE_GATE_*; dtype MOE_F32 or MOE_BF16;
 *   capacity_factor <= 0 means dropless (no capacity limit).
 * bf16 layers need d and d_ff to be multiples of 8 (16-byte rows for the
 * tensor-memory-accelerator loads): otherwise MOE_ERR_UNSUPPORTED.
 * Returns MOE_OK and *out, or MOE_ERR_INVALID_ARG (out untouched).
 */
MOE_API int moe_create(int num_experts, int k, int d, int d_ff, int act, int gate_mode,
               double capacity_factor, int dtype, moe_handle* out);

/*
 * bf16 layers: how the hidden activation between the two expert projections
 * is held (no counterpart on the pages, which fix only the router at fp32):
 *   MOE_HIDDEN_BF16X2: as the sum of two bf16 numbers hi + lo (about 16
 *     significant bits); the second projection runs its tensor-core MMAs on
 *     both planes, twice the tensor work of that projection.
 *   MOE_HIDDEN_F16: as one fp16 number (11 significant bits); the second
 *     projection multiplies it by an fp16 image of W2 that each call makes
 *     in the workspace while the first projection runs (bf16 -> fp16 is exact
 *     for |w| in [2^-17, 65504]; smaller weights move by at most 2^-25).  One
 *     plane of MMAs.  |hidden| and |W2| must stay below 65504: a larger value
 *     makes moe_status() report MOE_ERR_RANGE and that call's outputs are
 *     undefined.
 *   MOE_HIDDEN_AUTO (default): MOE_HIDDEN_F16 when the batch averages at least
 *     1024 rows per expert (shared experts counted), where the second
 *     projection is bound by the tensor cores; MOE_HIDDEN_BF16X2 otherwise,
 *     where it is bound by the weight stream and the pair costs no time.
 *   MOE_HIDDEN_BF16: one bf16 number (8 significant bits, unit roundoff 2^-8).
 *     OUTSIDE THE PARITY BAR: against an fp32 reference on the same bf16
 *     inputs, the rounding of the hidden activation alone gives max|dy| of
 *     about 1.5e-2 * RMS(y) on layers with millions of outputs (the bar is
 *     1e-2 * RMS) and a mean relative error of about 1.6e-3 before the final
 *     cast, which the cast to bf16 raises to about 2.3e-3 in the returned y
 *     (the bar is 2e-3).  Use it only where that is acceptable.
 * Changes moe_workspace_bytes() (MOE_HIDDEN_F16 and the automatic mode at
 * large batches add the W2 image: (E + n_shared) * d * d_ff * 2 bytes).
 * fp32 layers ignore it.  Returns MOE_OK or MOE_ERR_INVALID_ARG.
 */
MOE_API int moe_set_hidden_precision(moe_handle h, int mode);

/*
 * Shared experts ("Mixture of experts", rayaq.ca, section "Total versus
 * active parameters": shared experts every token visits).  With n_shared > 0
 * the layer adds, for every token, the outputs of n_shared more experts of
 * the same shape and activation, each with weight 1, after the gated routed
 * sum:  y_t = sum_j g_tj E_{idx_tj}(x_t) + sum_s S_s(x_t).  Their weights
 * follow the routed experts' in W1, W3 and W2, which then hold E + n_shared
 * experts (index E + s is shared expert s).  Shared experts take no part in
 * routing, capacity, expert_counts, dropped or the losses; a token whose
 * routed choices were all dropped still gets them.  0 <= n_shared <= 8 and
 * E + n_shared <= 256, else MOE_ERR_INVALID_ARG.  Changes
 * moe_workspace_bytes().  Default 0.
 */
MOE_API int moe_set_shared_experts(moe_handle h, int n_shared);

/* Free a handle created by moe_create.  NULL is accepted. */
MOE_API int moe_destroy(moe_handle h);

/*
 * Expert capacity for a batch of T tokens: ceil(capacity_factor * T * k / E)
 * evaluated in double, or -1 for a dropless layer.  Host only.
 */
MOE_API int64_t moe_capacity(moe_handle h, int64_t T);

/*
 * Bytes of device workspace moe_forward needs for T tokens (0 on bad args).
 * The workspace holds the routing tables and the expert-sorted activations;
 * it must be 256-byte aligned and is fully rewritten by every call.
 */
MOE_API size_t moe_workspace_bytes(moe_handle h, int64_t T);

/*
 * One forward pass of the layer over T tokens (T >= 0).
 *   x            [T][d]        layer input (bf16 or fp32)
 *   W_r          [E][d]  fp32  router weight;   b_r [E] fp32 bias or NULL
 *   W1           [E][d_ff][d]  first expert projection ([E + n_shared] rows of
 *                              experts with shared experts, see moe_set_shared_experts)
 *   W3           [E][d_ff][d]  SwiGLU value projection; must be NULL for ReLU
 *   W2           [E][d][d_ff]  second expert projection
 *   y            [T][d]        output (same dtype as x); 0 for fully dropped tokens
 *   expert_counts[E]     int32 assignments routed to each expert, before capacity
 *   dropped      [1]     int32 number of dropped (token, choice) assignments
 *   aux_loss     [1]     fp32  E * sum_i f_i P_i (unscaled)
 *   z_loss       [1]     fp32  mean_t lse_t^2 (unscaled)
 *   workspace, workspace_bytes: device scratch of at least moe_workspace_bytes(h, T)
 *   dbg          optional hooks (may be NULL)
 *   stream       cudaStream_t as void*
 * T = 0 writes zero counts, dropped = 0, aux = z = 0 and launches nothing else.
 */
MOE_API int moe_forward(moe_handle h, int64_t T, const void* x, const float* W_r, const float* b_r,
                const void* W1, const void* W3, const void* W2, void* y,
                int32_t* expert_counts, int32_t* dropped, float* aux_loss, float* z_loss,
                void* workspace, size_t workspace_bytes, const moe_debug* dbg, void* stream);

/*
 * 4-bit expert weights for serving ("Mixture of Experts (MoE)", inferensys.com,
 * inference-optimization glossary, model quantization: post-training 4-bit
 * quantization of a trained MoE's weights; "Mixture of experts", rayaq.ca,
 * "Total versus active parameters": small-batch decoding is bound by reading
 * the experts' weights, which quantization eases).  The pages fix no scheme;
 * this library's format:
 *   - each weight row [K] (K a multiple of 128) is cut into groups of 128
 *     consecutive elements; group g has a bf16 scale s_g with at most 5
 *     significant bits, and element k is w_k = (u_k - 8) * s_{k / 128} with a
 *     4-bit code u_k in [0, 15] (so w_k is exact in bf16);
 *   - a word holds 8 consecutive elements 8m .. 8m+7 of a row, element
 *     8m + 2j in bits 4j .. 4j+3 and element 8m + 2j + 1 in bits
 *     4j+16 .. 4j+19 (j = 0 .. 3);
 *   - codes are stored in tiles of 128 rows x 64 elements (rows a multiple of
 *     128), each tile 4 KB contiguous with its row r at byte 32 r:
 *     uint32 [rows / 128][K / 64][128][8]; the word of (row, 8m) is at index
 *     ((row / 128) (K / 64) + 8m / 64) 1024 + (row % 128) 8 + (m % 8);
 *   - scales: bf16 [rows / 128][K / 128][128], the scale of (row, group g) at
 *     ((row / 128) (K / 128) + g) 128 + row % 128.
 * The tiles make each 64-element slice of 128 rows one contiguous read.  Rows
 * are the rows of the nn.Linear weights: W1 / W3 [E (+ n_shared)][d_ff] rows of
 * K = d, W2 [E (+ n_shared)][d] rows of K = d_ff, so an expert's codes and
 * scales are contiguous.
 *
 * moe_quantize_int4: codes and scales of a bf16 weight W [rows][K] (device
 * pointers; W and codes 16-byte aligned, scales 2-byte aligned), by
 * s = max|w| / 7 over the group in fp32, rounded up to 5 significant bits,
 * and u = round-half-even(w / s) + 8 in fp32 (u = 8 when s = 0).  Asynchronous
 * on `stream`.  rows and K must be multiples of 128, else MOE_ERR_UNSUPPORTED.
 *
 * moe_forward_w4: moe_forward of a bf16 layer (d and d_ff multiples of 128)
 * whose expert weights are given in that format; the result is the layer
 * with the dequantized weights.  The expert products run on the tensor
 * cores with the weights dequantized on the fly (HBM carries the codes and
 * scales only); the hidden activation is held as a hi + lo bf16 pair.
 * Batches of T <= 64 tokens take warp-level MMAs fed from registers, larger
 * ones the tcgen05 grouped GEMM.  Codes and scales must be 16-byte aligned.
 * The workspace is moe_workspace_bytes_w4(h, T) bytes (256-byte aligned).
 * Arguments, results and errors as moe_forward; W3_codes / W3_scales are
 * NULL for ReLU layers.  moe_backward does not serve layers run this way.
 */
MOE_API int moe_quantize_int4(const void* W, int64_t rows, int64_t K, uint32_t* codes, void* scales, void* stream);
MOE_API size_t moe_workspace_bytes_w4(moe_handle h, int64_t T);
MOE_API int moe_forward_w4(moe_handle h, int64_t T, const void* x, const float* W_r, const float* b_r,
                           const uint32_t* W1_codes, const void* W1_scales, const uint32_t* W3_codes,
                           const void* W3_scales, const uint32_t* W2_codes, const void* W2_scales, void* y,
                           int32_t* expert_counts, int32_t* dropped, float* aux_loss, float* z_loss, void* workspace,
                           size_t workspace_bytes, const moe_debug* dbg, void* stream);

/*
 * The alternative load-balancing statistics of the last moe_forward that used
 * `workspace` with T tokens (stream-ordered on `stream`), unscaled, written as
 * three fp32 values to the device pointer `out`:
 *   out[0]  E * sum_i (c_i / (T k)) P_i: the Switch loss with f_i counted over
 *           all k choices ("Mixture of experts", rayaq.ca, section "The
 *           load-balancing loss");
 *   out[1]  the coefficient of variation std(c) / mean(c) of the assignment
 *           counts c_i (= expert_counts) over the E experts ("Mixture of
 *           Experts (MoE)", inferensys.com: 0.01 times the coefficient of
 *           variation of expert assignment counts);
 *   out[2]  the squared coefficient of variation var(P) / mean(P)^2 of the
 *           mean router probabilities P_i ("Mixture of Experts (MoE) Language
 *           Models", chipfoundryservices.com: cv^2 of the router probabilities).
 * Moments are over the E values (divided by E).  The forward pass computes
 * them in its reduction at no extra launch; this call copies them (T = 0
 * writes zeros).  Returns MOE_OK, MOE_ERR_INVALID_ARG or MOE_ERR_CUDA.
 */
MOE_API int moe_balance_losses(moe_handle h, int64_t T, const void* workspace, float* out, void* stream);

/*
 * moe_forward for callers that cannot allocate device memory (no counterpart
 * on the pages): for example a plug-in inside a host framework that owns every
 * device allocation and offers its extensions no workspace, or a serving loop
 * that must not enter an allocator on its hot path.  Same arguments and
 * results as moe_forward, without the workspace and the debug hooks: the
 * scratch is a 32 MiB array compiled into the library, resident on every GPU
 * that loads it until the process exits.
 *   - A call needing more than 32 MiB (moe_workspace_bytes(h, T) > 32 MiB;
 *     e.g. the 8-expert top-2 d 4096 / d_ff 14336 SwiGLU layer up to T = 116)
 *     is rejected with MOE_ERR_UNSUPPORTED before any launch.
 *   - The first call on a device looks up the array's address on that device
 *     (with it current); make that first call before any stream capture.
 *   - Every call shares the array and leaves its contents there; calls that
 *     overlap on the GPU (other streams, other host threads) race on it.
 *     Nothing in it needs to start at zero.
 *   - The looked-up address is kept for the life of the process.  A
 *     cudaDeviceReset (or any other teardown of the device's primary
 *     context) invalidates it, like the device error word every entry point
 *     uses: make no further call of this library on that device afterwards.
 *   - Allocates nothing (no cudaMalloc / cudaFree or allocating routine).
 */
MOE_API int moe_forward_static(moe_handle h, int64_t T, const void* x, const float* W_r, const float* b_r,
                               const void* W1, const void* W3, const void* W2, void* y,
                               int32_t* expert_counts, int32_t* dropped, float* aux_loss, float* z_loss,
                               void* stream);

/*
 * Backward pass ("Mixture of experts", rayaq.ca: section "Replacing the
 * feed-forward block", the router learns through the gate values only, the
 * choice of experts being discrete; section "The load-balancing loss", f_i
 * is a count without gradient, P_i and the z-loss's lse have one).
 *
 * Gradients of L = sum_t <dy_t, y_t> + aux_coef * aux_loss + z_coef * z_loss
 * (aux_loss and z_loss unscaled, as moe_forward reports them) with respect to
 * x, W_r, b_r, W1, W3 and W2, the routing of the forward pass held fixed: the
 * top-k choices, the capacity drops and the slots come from `workspace`,
 * which must hold the moe_forward call of the same handle, T and inputs,
 * issued earlier on `stream` with nothing written to it since (the
 * moe_forward_static scratch cannot serve).  A dropped assignment passes no
 * gradient; shared experts get gate 1.  bf16 layers: every product on the
 * tensor cores (bf16 operands, fp32-derived ones as hi + lo bf16 pairs, fp32
 * accumulation); fp32 layers: fp32 on CUDA cores.  Every sum runs in a fixed
 * order (deterministic).
 *   x, W1, W3, W2, dy in the layer's dtype (dy [T][d] like y); W_r, b_r fp32.
 *   Outputs, fp32, overwritten: dx [T][d], dW_r [E][d], db_r [E] (NULL: not
 *   wanted), dW1 / dW3 [E + n_shared][d_ff][d] (dW3 NULL for ReLU),
 *   dW2 [E + n_shared][d][d_ff].
 *   bw_workspace: device scratch of moe_backward_workspace_bytes(h, T) bytes,
 *   256-byte aligned (never shrinks as T grows).
 * Errors as moe_forward; T = 0 zeroes the weight gradients.  Asynchronous.
 */
MOE_API size_t moe_backward_workspace_bytes(moe_handle h, int64_t T);
MOE_API int moe_backward(moe_handle h, int64_t T, const void* x, const float* W_r, const float* b_r,
                         const void* W1, const void* W3, const void* W2, const void* dy, float aux_coef,
                         float z_coef, float* dx, float* dW_r, float* db_r, float* dW1, float* dW3, float* dW2,
                         const void* workspace, size_t workspace_bytes, void* bw_workspace,
                         size_t bw_workspace_bytes, void* stream);

/*
 * Synchronise `stream` and report the device error word of the current device:
 * MOE_OK, MOE_ERR_TIMEOUT (a kernel's bounded wait ran out and it returned
 * early; outputs of that call are undefined), MOE_ERR_RANGE (fp16 hidden mode:
 * a value beyond the fp16 range; outputs of that call are undefined) or
 * MOE_ERR_CUDA.  The error word stays set until moe_clear_status().
 */
MOE_API int moe_status(void* stream);

/* Clear the device error word of the current device (synchronous). */
MOE_API int moe_clear_status(void);

/* Message of the last host-side error of the calling thread ("" if none). */
MOE_API const char* moe_last_error(void);

/* Kernels launched by this library in the calling process so far. */
MOE_API uint64_t moe_launch_count(void);

/*
 * Self-test of the device-side failure path (no counterpart on the pages):
 * launches one thread that waits on a device flag nothing ever sets, with the
 * same bounded wait the pipelined kernels use, limited to `limit_ns`
 * nanoseconds (clamped to [1e3, 2e9]).  When the wait runs out the kernel
 * records MOE_ERR_TIMEOUT in the device error word and returns, so a
 * following moe_status() reports MOE_ERR_TIMEOUT and the context stays usable.
 */
MOE_API int moe_selftest_timeout(int64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
