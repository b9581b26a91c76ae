/*
 * moe.h -- C ABI of the B200 (sm_100a) MoE FFN forward library (libmoe.so).
 *
 * One call computes the FFN half of a DeepSeek-V3.2-style MoE transformer block:
 *
 *     x, residual = ffn_norm(x, residual)        RMSNorm with the residual add fused in
 *     out         = ffn(x)                       routed SwiGLU experts + shared expert
 *
 * as defined on the DeepSeek-V3.2-Exp model-atlas pages:
 *   - "MoE update" page, Block excerpt: x, residual = self.ffn_norm(x, residual); x = self.ffn(x).
 *   - "MoE update" page, RMSNorm.forward excerpt: s = x.float() + residual.float();
 *     var = mean(s^2); s * rsqrt(var + eps); weight * s; normed and residual cast to x's dtype.
 *   - "MoE update" / "Add shared output" pages, MoE.forward excerpt and the equation
 *     delta_ffn = y_routed + y_shared: router weights and indices; every routed (token, slot)
 *     adds expert(x) * weight into a float32 y; the shared expert is added to every token; y is
 *     cast to x's dtype with shape [B, T, d].
 *   - "Gate projection" page: expert = w2((silu(w1 x).float() * (w3 x).float()).type_as(x)),
 *     weights held [out, in] without bias; 1-byte weights carry one float32 scale per 128x128
 *     block, scale shape [ceil(out/128), ceil(in/128)].
 *
 * The router's body is not on the pages.  This library computes scores = sigmoid(xn . Wg_e +
 * bias_e), keeps the top_k experts (on equal scores the lower expert index wins) and normalises
 * their scores to sum 1.  Logits come from a float32 tensor-core GEMM; the winners and every
 * expert within 2e-3 (logit units) of the k-th winner are re-evaluated in float64, so the
 * selection is the exact one and the weights are float64 scores rounded to float32.
 *
 * Conventions for every entry point
 *   - Tensors are device pointers (CUDA global memory of the current device), contiguous and
 *     row-major, 16-byte aligned.  The caller owns all memory; the library allocates none and
 *     keeps no pointer after a call returns.
 *   - bf16 = IEEE bfloat16 bits (uint16); e4m3 = OCP FP8 E4M3 codes (uint8).
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).  Work is
 *     enqueued on it; moe_forward never synchronises the host.
 *   - Argument errors are returned synchronously and enqueue nothing.  Launch failures return
 *     MOE_ERR_CUDA.  Errors found on the device (a bounded wait that gave up) are latched into
 *     the workspace status word; moe_get_status() reads it.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,     /* NULL pointer, bad size, misaligned pointer, k > E, ... */
    MOE_ERR_UNSUPPORTED = 2,     /* valid per the pages but not built (see moe_config_t) */
    MOE_ERR_WORKSPACE = 3,       /* workspace NULL or smaller than moe_workspace_bytes() */
    MOE_ERR_CUDA = 4,            /* a CUDA runtime/driver call or a launch failed */
    MOE_ERR_DEVICE_TIMEOUT = 5,  /* a kernel's bounded wait gave up (latched on the device) */
    MOE_ERR_DEVICE_CHECK = 6     /* a device-side consistency check failed (latched) */
} moe_status_t;

/* Weight storage ("Gate projection" page, Linear excerpt). */
typedef enum {
    MOE_W_BF16 = 0,              /* bf16 [out, in], no scale */
    MOE_W_FP8_E4M3_B128 = 1      /* e4m3 [out, in] + float32 scale [out/128, in/128] */
} moe_wtype_t;

/* Precision of the activations fed to the expert GEMMs (the FP8 GEMM body is not on the
 * pages).  MOE_ACT_FP8_1x128: per token and per 128-column group, sc = amax/448,
 * q = e4m3(v/sc) -- applied to the normed input and to the SwiGLU hidden state h; FP8 tensor-core
 * GEMMs.  MOE_ACT_BF16: bf16 activations -- the only mode for bf16 weights; with FP8 weights, the
 * plain reading of a block-scaled FP8 Linear: bf16 activations times the dequantised weights, each
 * e4m3 weight tile widened to bf16 on chip and the block scales applied to the float32 partials. */
typedef enum {
    MOE_ACT_FP8_1x128 = 0,
    MOE_ACT_BF16 = 1
} moe_amode_t;

typedef struct {
    int32_t num_tokens;    /* T = B * S, >= 1 */
    int32_t dim;           /* d, multiple of 256, at most 8192 */
    int32_t inter_dim;     /* I (moe_inter_dim), multiple of 128 */
    int32_t n_experts;     /* E routed experts, 1..256, multiple of 8 or E <= 8; 0 = a dense block
                              ("MoE update" page, Block excerpt: MLP(dim, inter_dim) in the first
                              n_dense_layers blocks): no router, the MLP given as the shared
                              SwiGLU (shared_inter = its width), out = MLP(ffn_norm(x)) */
    int32_t top_k;         /* k, 1..E; 0 for a dense block */
    int32_t shared_inter;  /* width of the shared SwiGLU (n_shared * per-expert inter; several
                              shared experts are one SwiGLU with concatenated hidden units);
                              multiple of 128; 0 = no shared expert */
    int32_t wtype;         /* moe_wtype_t, same for routed and shared weights */
    int32_t amode;         /* moe_amode_t; bf16 weights need MOE_ACT_BF16 */
    float eps;             /* RMSNorm eps (1e-6 on the pages) */
} moe_config_t;

/* Expert weights, [out, in] row-major.  Routed: w1, w3 [E, I, d]; w2 [E, d, I].
 * Scales (FP8 only, else NULL): s1, s3 [E, I/128, d/128]; s2 [E, d/128, I/128].
 * Shared (NULL when shared_inter == 0): sw1, sw3 [Is, d]; sw2 [d, Is]; ss1, ss3 [Is/128, d/128];
 * ss2 [d/128, Is/128]. */
typedef struct {
    const void *w1, *w3, *w2;
    const float *s1, *s3, *s2;
    const void *sw1, *sw3, *sw2;
    const float *ss1, *ss3, *ss2;
} moe_weights_t;

/* Bytes of device workspace moe_forward needs for this configuration (0 if cfg is invalid).
 * The workspace holds every intermediate (normed and quantised activations, logits, routing,
 * permuted rows, hidden states, expert outputs) and the device status word. */
size_t moe_workspace_bytes(const moe_config_t* cfg);

/* The fused forward pass.
 *   x            [T, d] bf16            input of ffn_norm (the attention output)
 *   residual     [T, d] bf16 or NULL    residual stream; NULL = RMSNorm without the add
 *   norm_w       [d] float32            RMSNorm gain
 *   gate_w       [E, d] bf16            router weight (ignored, may be NULL, for a dense block)
 *   gate_bias    [E] float32 or NULL    per-expert bias added to the logits before the sigmoid
 *   w            expert weights (moe_weights_t); a dense block uses only sw1, sw3, sw2 (and
 *                ss1, ss3, ss2 for FP8), the routed fields may be NULL
 *   out          [T, d] bf16            delta_ffn
 *   residual_out [T, d] bf16            new residual = bf16(x + residual); may equal residual
 *                                       (in place); unused when residual is NULL
 *   workspace    >= moe_workspace_bytes(cfg) bytes of device memory, 256-byte aligned; it must
 *                not be used by another call still running on the device.
 * No other aliasing is allowed. */
moe_status_t moe_forward(const moe_config_t* cfg, const void* x, const void* residual,
                         const float* norm_w, const void* gate_w, const float* gate_bias,
                         const moe_weights_t* w, void* out, void* residual_out,
                         void* workspace, size_t workspace_bytes, void* stream);

/* moe_forward with the next block's attn_norm fused into the combine ("MoE update" page, Block
 * excerpt: residual additions happen inside the next normalisation, `x, residual =
 * self.attn_norm(x, residual)` right after `x = self.ffn(x)`; RMSNorm excerpt for the arithmetic).
 * Runs this layer exactly as moe_forward, then per token
 *   s = fp32(delta) + fp32(bf16(x + residual))     delta = the MoE update (moe_forward's out)
 *   next_residual = bf16(s)
 *   next_xn = bf16(next_norm_w * (s * rsqrt(mean(s^2) + eps)))   (same arithmetic as ffn_norm)
 * without writing delta to memory unless `out` is given.
 *   residual       [T, d] bf16, required (the block's ffn_norm always adds one)
 *   next_norm_w    [d] float32            the next block's attn_norm gain
 *   out            [T, d] bf16 or NULL    delta, as moe_forward would write it
 *   next_xn        [T, d] bf16            the next block's normed input
 *   next_residual  [T, d] bf16            the next block's residual; may equal residual (in place)
 * MOE_ERR_UNSUPPORTED for a dense block (n_experts = 0); other arguments, errors and ownership as
 * moe_forward.  No counterpart call on the pages: it fuses two of their calls. */
moe_status_t moe_forward_next_norm(const moe_config_t* cfg, const void* x, const void* residual,
                                   const float* norm_w, const void* gate_w, const float* gate_bias,
                                   const moe_weights_t* w, const float* next_norm_w, void* out,
                                   void* next_xn, void* next_residual, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* One rank's share of the expert-parallel layer ("MoE update" page, MoE.forward excerpt: a rank
 * runs the experts in [experts_start_idx, experts_end_idx) on the tokens routed to them and adds
 * their weighted outputs into a float32 y, `dist.all_reduce(y)` sums the ranks, the shared
 * expert is added and the result is cast to x's dtype).  Every rank computes the same ffn_norm and
 * routing over all E experts; the GEMMs run only experts [expert_begin, expert_end) (and the
 * shared expert when with_shared != 0, on exactly one rank).
 *   y_partial     [T, d] float32         sum over the token's slots routed to this rank's experts
 *                                        of weight * expert output (+ the shared output), not
 *                                        rounded; the caller sums the ranks' partials and casts
 *                                        once to bf16 (see expert_parallel_forward in the binding)
 *   w             routed weights of this rank's experts must be valid at their places in the
 *                 stacked [E, ...] layout; the others are not read
 *   residual_out  as moe_forward
 * 0 <= expert_begin <= expert_end <= E.  MOE_ERR_UNSUPPORTED for a dense block.  Other arguments,
 * errors and ownership as moe_forward. */
moe_status_t moe_forward_expert_slice(const moe_config_t* cfg, const void* x, const void* residual,
                                      const float* norm_w, const void* gate_w, const float* gate_bias,
                                      const moe_weights_t* w, int32_t expert_begin, int32_t expert_end,
                                      int32_t with_shared, float* y_partial, void* residual_out,
                                      void* workspace, size_t workspace_bytes, void* stream);

/* out[i] = bf16(y[i]) (round to nearest even) for n float32 values, n a multiple of 4; y 16-byte
 * and out 8-byte aligned.  The final cast of the expert-parallel layer after the ranks' partial
 * sums are reduced (the pages' `y.type_as(x)`). */
moe_status_t moe_round_bf16(const float* y, void* out, int64_t n, void* stream);

/* moe_forward that also records caller-created CUDA events (cudaEvent_t passed as void*) on
 * `stream` at the stage boundaries, for timing individual kernels inside a running workload:
 *   events[0] before the first launch      events[4] after the permutation kernels
 *   events[1] after the norm kernel        events[5] after the grouped GEMM up (w1|w3, SwiGLU)
 *   events[2] after the gate GEMM          events[6] after the grouped GEMM down (w2)
 *   events[3] after the top-k kernels      events[7] after the combine kernel
 * n_events may be smaller than 8 (the later boundaries are then not recorded); NULL entries are
 * skipped.  Same arguments, errors and ownership as moe_forward otherwise. */
moe_status_t moe_forward_traced(const moe_config_t* cfg, const void* x, const void* residual,
                                const float* norm_w, const void* gate_w, const float* gate_bias,
                                const moe_weights_t* w, void* out, void* residual_out,
                                void* workspace, size_t workspace_bytes, void* stream,
                                void* const* events, int32_t n_events);

/* Synchronises `stream`, then returns the status latched in the workspace by the last
 * moe_forward on it (MOE_OK, MOE_ERR_DEVICE_TIMEOUT or MOE_ERR_DEVICE_CHECK), or MOE_ERR_CUDA.
 * Undefined for a workspace no moe_forward has run on yet (the call that clears the status word
 * is the first thing moe_forward enqueues). */
moe_status_t moe_get_status(const void* workspace, void* stream);

/* Copies (device to device, enqueued on `stream`) the routing of the last moe_forward that
 * used this workspace: idx [T, k] int32 (slot order = descending score), weights [T, k]
 * float32, counts [E] int32 (tokens per expert), near_tie [T] uint8 (1 = another expert was
 * within the candidate window of the k-th winner and the selection was re-decided in float64).
 * Any output pointer may be NULL.  MOE_ERR_INVALID_ARG for a dense block (it has no routing). */
moe_status_t moe_debug_routing(const moe_config_t* cfg, const void* workspace, int32_t* idx,
                               float* weights, int32_t* counts, uint8_t* near_tie, void* stream);

/* Copies the normed activations of the last moe_forward: xn [T, d] bf16, and in FP8
 * activation mode xq [T, d] e4m3 and xs [d/128, T] float32 (group scales, transposed).
 * Any output pointer may be NULL. */
moe_status_t moe_debug_norm(const moe_config_t* cfg, const void* workspace, void* xn,
                            void* xq, float* xs, void* stream);

/* The expert grouping step alone -- tokens per expert, expert offsets and the permutation by
 * expert -- computed exactly as moe_forward computes it internally, but without any workspace.
 * The pages have no counterpart: this entry point exists for callers that cannot allocate
 * device memory when they call in, e.g. a serving runtime that reserves all device memory up
 * front and hands a layer only the tensors it reads and writes, or code on a latency-critical
 * path where a cudaMalloc would synchronise the device and stall every other stream.
 *   idx        [T, k] int32 device      expert of every (token, slot); values in [0, E)
 *   counts     [E] int32 device         tokens routed to each expert
 *   offsets    [E + 1] int32 device     first permuted row of each expert; each expert's rows
 *                                       start on a multiple of 128; offsets[E] = rows used
 *   row_of     [T, k] int32 device      permuted row of every (token, slot); inside an expert
 *                                       the rows follow token order
 *   row_token  [R] int32 device         token of every permuted row, -1 in padding rows, with
 *                                       R = roundup(T*k + 127*E, 128)
 * Its scratch (per-chunk histograms and tables, 136 KiB) is one file-scope device array that
 * every device loading the library holds until the process exits.  T*k may be at most 262144;
 * larger sizes return MOE_ERR_UNSUPPORTED.  The first call on a device looks up the array's
 * device address with that device current (the caller's current device must own `stream`), so
 * make that first call before any stream capture.  Calls share the array: two calls whose work
 * overlaps on the GPU (different streams, or different host threads) race and give wrong
 * results; calls ordered on one stream are fine.  Nothing left in the array by an earlier call
 * is read.  No allocation of any kind is made.  Errors: MOE_ERR_INVALID_ARG for NULL pointers
 * or sizes out of range, MOE_ERR_CUDA for a failed lookup or launch. */
moe_status_t moe_route_noalloc(const int32_t* idx, int32_t num_tokens, int32_t top_k, int32_t n_experts,
                               int32_t* counts, int32_t* offsets, int32_t* row_of, int32_t* row_token,
                               void* stream);

/* Failure-detection self-test (the pages have no counterpart).  Enqueues one kernel whose only
 * wait is on a barrier that is never signalled, using the same bounded wait as the pipeline
 * kernels with a limit of `limit_cycles` SM clocks (1 .. 2^31).  The wait gives up, the kernel
 * latches MOE_ERR_DEVICE_TIMEOUT into the status word at the start of `workspace` and returns
 * normally; moe_get_status then reports MOE_ERR_DEVICE_TIMEOUT and the context stays usable.
 * The next moe_forward on the workspace clears the status.  workspace_bytes >= 256. */
moe_status_t moe_selftest_wait_timeout(void* workspace, size_t workspace_bytes, int64_t limit_cycles,
                                       void* stream);

/* Number of kernel launches one moe_forward enqueues for this configuration (11; 3 for a dense
 * block: norm and the two SwiGLU GEMMs, the second writing out directly).  For a dense block the
 * traced events 2-4 and 6-7 are recorded back to back (no router, no combine). */
int32_t moe_launches_per_forward(const moe_config_t* cfg);

/* Static description of a status code. */
const char* moe_status_string(moe_status_t s);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
