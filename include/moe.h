/*
 * moe.h - C ABI of libmoe.so, a B200 (sm_100a) mixture-of-experts FFN block.
 *
 * The block (archdiff.com architecture-comparison pages; in the blueprint
 * diagram of qwen3-5-vs-deepseek-v4 a pre-norm RMSNorm feeds the router, which
 * picks the top 6 to 22 of 256 to 896 SwiGLU experts, one or two shared
 * experts run for every token, and a residual add follows):
 *
 *   logits   l = x W_router^T                                   (linear router)
 *   scores   s = softmax(l) | sigmoid(l) | sqrt(softplus(l))
 *   pick     the k largest of c = s (+ expert_bias for sigmoid/sqrt-softplus:
 *            the bias only picks experts), descending, ties to the lower index
 *   weights  w_j = s_{pick_j}; renormalised over the picks if norm_topk;
 *            times route_scale
 *   out      = sum_j w_j SwiGLU_{pick_j}(x) + sum_s SwiGLU_shared_s(x)
 *            SwiGLU(x) = W_down (SiLU(W_gate x) * (W_up x)), no residual.
 *
 * Sources on the pages:
 *   softmax router (softmax over all experts, the k largest kept and
 *     renormalised, no bias in the choice): qwen3-5-vs-deepseek-v4 component
 *     table, Qwen3.5 router cell;
 *   sqrt-softplus router with a bias that only picks experts, the picked
 *     scores renormalised and multiplied by 2.5: same table, DeepSeek-V4-Pro
 *     router cell; sigmoid form: the router node of the DeepSeek-V4-Pro
 *     diagram;
 *   SwiGLU experts at full width: qwen3-5-vs-gemma-4 component table, Qwen3.5
 *     routed-experts cell; shared expert added to the routed sum: same table,
 *     Qwen3.5 shared-expert cell (ungated, DeepSeek-style, by default; the
 *     Qwen3.5 per-token sigmoid gate with W_shared_gate_vec).
 *
 * Beyond the block itself: moe_forward_prenorm (the pre-norm RMSNorm fused in
 * front), moe_forward_fp8 (block-scaled FP8 expert weights),
 * moe_experts_forward (routing supplied by the caller), moe_forward_host
 * (host buffers), the step entry points, and moe_route_noalloc.
 *
 * Conventions for every entry point
 *   - Tensors are dense, row-major, in device memory unless stated otherwise,
 *     and owned by the caller.  bf16 = IEEE bfloat16 bit patterns (uint16).
 *     Weights use the [out, in] layout:
 *        x [T,d]  W_router [E,d]  W_gate, W_up [E,f,d]  W_down [E,d,f]
 *        W_shared_gate, W_shared_up [S,fs,d]  W_shared_down [S,d,fs]
 *   - Every device pointer must be 16-byte aligned; d, f and fs must be
 *     multiples of 64 and at most 65536; 1 <= k <= min(E, 32);
 *     1 <= E <= 2048; 0 <= S <= 8; 1 <= T <= 4,194,304.  Violations return
 *     an error code and enqueue nothing.
 *   - `stream` is a cudaStream_t passed as a plain pointer (NULL = legacy
 *     default stream).  Work is enqueued asynchronously on it; no entry point
 *     except moe_device_status synchronises the host.
 *   - The library allocates no device memory and keeps no per-call state: all
 *     scratch lives in the caller's workspace (size from moe_workspace_bytes),
 *     which must not be used by two calls that overlap on the GPU.  (The one
 *     exception, moe_route_noalloc, uses a scratch array inside the library.)
 *   - Entry points may be called from several host threads at once, each call
 *     with its own workspace.  The only state kept across calls is per device
 *     and filled in once under a lock: the device's properties, the kernels'
 *     shared-memory limits and the tensor-map encoder's address.
 *   - Kernels are launched with programmatic stream serialisation: each waits
 *     for the previous kernel in the stream before touching memory, so stream
 *     order is preserved while launch latency overlaps.
 *   - On an error return nothing has been enqueued and the outputs are
 *     untouched.
 *   - Kernels never trap.  Every device-side wait is bounded; a wait that runs
 *     out sets an error word in the workspace, the kernel returns, and
 *     moe_device_status reports MOE_ERR_DEVICE_TIMEOUT.
 */
#ifndef MOE_H_
#define MOE_H_

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

#define MOE_OK                  0
#define MOE_ERR_INVALID_ARG    -1   /* null pointer, k<1, k>E, T<1, bad enum ... */
#define MOE_ERR_UNSUPPORTED    -2   /* d/f/fs not multiples of 64, misaligned pointer, limits, not sm_100 */
#define MOE_ERR_WORKSPACE      -3   /* workspace missing, misaligned or smaller than moe_workspace_bytes */
#define MOE_ERR_CUDA           -4   /* a CUDA runtime / driver call or a launch failed */
#define MOE_ERR_DEVICE_TIMEOUT -5   /* a bounded device-side wait ran out (reported by moe_device_status) */
#define MOE_ERR_SCRATCH_LIMIT  -6   /* moe_route_noalloc: T * E fp32 logits exceed its built-in 16 MiB scratch */
#define MOE_ERR_NONFINITE      -7   /* a token's router logits, selection keys or combine weights were NaN or
                                       infinite (reported by moe_device_status) */

#define MOE_SCORE_SOFTMAX       0   /* s = softmax(l) over all E experts; expert_bias ignored */
#define MOE_SCORE_SIGMOID       1   /* s = 1/(1+exp(-l)) */
#define MOE_SCORE_SQRT_SOFTPLUS 2   /* s = sqrt(log(1+exp(l))) */

typedef void *moe_stream_t;         /* a cudaStream_t */

typedef struct moe_shape {
    int32_t T;            /* tokens */
    int32_t d_model;      /* d */
    int32_t E;            /* routed experts */
    int32_t k;            /* experts picked per token */
    int32_t d_ff;         /* f: routed expert hidden width */
    int32_t n_shared;     /* S: always-active shared experts (0 allowed) */
    int32_t d_ff_shared;  /* fs: shared expert hidden width (ignored when S == 0) */
} moe_shape;

/* Library version, MAJOR*10000 + MINOR*100 + PATCH. */
MOE_API int moe_version(void);

/* Human-readable name of a status code (static string, never NULL). */
MOE_API const char *moe_status_string(int status);

/* Bytes of workspace that every entry point below needs for this shape
 * (0 if the shape is invalid).  The workspace must be 256-byte aligned.
 * Its contents need no initialisation. */
MOE_API size_t moe_workspace_bytes(const moe_shape *shape);

/* The whole block, steps a1..a7 below in order, on `stream`.
 *   x, weights: inputs as above.  expert_bias: fp32 [E] or NULL (selection
 *   only; ignored for MOE_SCORE_SOFTMAX).  W_shared_*: NULL iff S == 0.
 *   W_shared_gate_vec: bf16 [S,d] or NULL.  NULL: shared experts are added
 *   with weight 1 (DeepSeek-style).  Given: shared expert s is scaled per
 *   token by sigmoid(W_shared_gate_vec[s] . x) before it is added (the
 *   Qwen3.5 shared expert, qwen3-5-vs-gemma-4 component table, shared-expert
 *   cell).  Requires S >= 1.
 *   score_fn: MOE_SCORE_*.  norm_topk: 0/1.  route_scale: multiplies the
 *   combine weights (1.0 = none; DeepSeek-V4-Pro uses 2.5).
 *   out      [T,d] bf16: the block output, residual-free.
 *   topk_idx [T,k] int32: picked experts, descending selection key, ties to
 *            the lower index.
 *   topk_w   [T,k] fp32: the combine weights actually applied.
 * Returns MOE_OK or an error code. */
MOE_API int moe_forward(const moe_shape *shape,
                const void *x, const void *W_router, const float *expert_bias,
                const void *W_gate, const void *W_up, const void *W_down,
                const void *W_shared_gate, const void *W_shared_up, const void *W_shared_down,
                const void *W_shared_gate_vec,
                int score_fn, int norm_topk, float route_scale,
                void *out, int32_t *topk_idx, float *topk_w,
                void *workspace, size_t workspace_bytes, moe_stream_t stream);

/* moe_forward with x and the outputs in HOST memory (page-locked memory lets
 * the copies run asynchronously; pageable memory works but the copies then
 * synchronise with the host).  The library copies x into the workspace,
 * runs the block, and copies out / topk_idx / topk_w back, all on `stream`.
 * Weights and the workspace are device memory.  The host buffers must stay
 * valid until the stream reaches the end of this call. */
MOE_API int moe_forward_host(const moe_shape *shape,
                     const void *x_host, const void *W_router, const float *expert_bias,
                     const void *W_gate, const void *W_up, const void *W_down,
                     const void *W_shared_gate, const void *W_shared_up, const void *W_shared_down,
                     const void *W_shared_gate_vec,
                     int score_fn, int norm_topk, float route_scale,
                     void *out_host, int32_t *topk_idx_host, float *topk_w_host,
                     void *workspace, size_t workspace_bytes, moe_stream_t stream);

/* The block with its pre-norm RMSNorm fused in front (the Qwen3.5 diagram of
 * qwen3-5-vs-deepseek-v4 draws a pre-norm RMSNorm right before the router;
 * the gains are zero-centred: same page, component table, Qwen3.5
 * residual-stream cell).
 *   x         [T,d] bf16: the residual stream (not normalised).
 *   norm_gain [d] bf16: zero-centred gains g; the scale applied is 1 + g.
 *   norm_eps  finite, >= 0 (the pages give no value; Qwen-family models use
 *             1e-6).
 * Runs moe_rmsnorm into the workspace (region MOE_WS_X_STAGE) and then the
 * block on the normalised rows, which are also what the router, the experts
 * and the shared-expert gate see.  Everything else as in moe_forward. */
MOE_API int moe_forward_prenorm(const moe_shape *shape,
                const void *x, const void *norm_gain, float norm_eps,
                const void *W_router, const float *expert_bias,
                const void *W_gate, const void *W_up, const void *W_down,
                const void *W_shared_gate, const void *W_shared_up, const void *W_shared_down,
                const void *W_shared_gate_vec,
                int score_fn, int norm_topk, float route_scale,
                void *out, int32_t *topk_idx, float *topk_w,
                void *workspace, size_t workspace_bytes, moe_stream_t stream);

/* Pre-norm RMSNorm alone:
 *   x_norm[t,i] = bf16( x[t,i] / sqrt(mean_j x[t,j]^2 + eps) * (1 + norm_gain[i]) )
 * computed in double and rounded to bf16 once (nearest, ties to even).
 * Only T and d of the shape are used, but the whole shape must be valid.
 * x, x_norm: bf16 [T,d] device buffers (may not overlap); norm_gain bf16 [d].
 * Returns MOE_ERR_INVALID_ARG for a null pointer or eps < 0 / not finite. */
MOE_API int moe_rmsnorm(const moe_shape *shape, const void *x, const void *norm_gain, float eps,
                void *x_norm, moe_stream_t stream);

/* ---- Block-scaled FP8 expert weights ----
 * The pages mention an FP8 release of the Qwen3.5 weights and block-scaled
 * FP8 in the training blueprint (qwen3-5-vs-gemma-4, component table, Qwen3.5
 * routed-experts cell; qwen3-5-vs-deepseek-v4, blueprint diagram) but give no
 * block size or scale format.  Reading: OCP MX-style blocks of 32 consecutive elements along the
 * input dimension K, one power-of-two scale per block stored as its biased
 * exponent byte (UE8M0).  Element [g, r, c] of the weight is
 *     e4m3(codes[g, r, c]) * 2^(scales[g, c / 32, r] - 127)
 * with codes in the [out, in] layout of the bf16 weight and the scales
 * block-major.  E4M3 is the OCP "E4M3FN" encoding (no infinities, 0x7F/0xFF
 * NaN).  The library widens each tile to bf16 in tensor memory; the widened
 * value is exact whenever it is representable in bf16 (scale bytes 10..246
 * for finite codes), so the block then computes exactly what moe_forward
 * computes on the widened weights, while HBM moves half the weight bytes. */
typedef struct {
  const void *codes;    /* uint8 E4M3 [G, rows, K], 16-byte aligned */
  const void *scales;   /* uint8 UE8M0 [G, K/32, rows], 16-byte aligned */
} moe_fp8_weight;

/* moe_forward with FP8 routed and shared expert weights (W_router stays
 * bf16).  W_gate / W_up: G = E, rows = d_ff, K = d_model; W_down: G = E,
 * rows = d_model, K = d_ff; shared: G = n_shared with d_ff_shared.  The
 * shared pointers are NULL iff n_shared == 0; a moe_fp8_weight with a NULL
 * member is MOE_ERR_INVALID_ARG.  Everything else as in moe_forward. */
MOE_API int moe_forward_fp8(const moe_shape *shape,
                const void *x, const void *W_router, const float *expert_bias,
                const moe_fp8_weight *W_gate, const moe_fp8_weight *W_up, const moe_fp8_weight *W_down,
                const moe_fp8_weight *W_shared_gate, const moe_fp8_weight *W_shared_up,
                const moe_fp8_weight *W_shared_down, const void *W_shared_gate_vec,
                int score_fn, int norm_topk, float route_scale,
                void *out, int32_t *topk_idx, float *topk_w,
                void *workspace, size_t workspace_bytes, moe_stream_t stream);

/* The FP8 forms of the permute and the two expert steps (a3, a4 + a6, a5 + a6),
 * for callers that run the steps one by one: moe_route, moe_permute_fp8,
 * moe_expert_gate_up_fp8, moe_expert_down_fp8, moe_combine.  The FP8 GEMMs
 * take token runs of at most 128 rows and no CTA pairs, so their work lists
 * differ from the bf16 ones; an expert step that meets lists built for the
 * other format does nothing and moe_device_status reports
 * MOE_ERR_INVALID_ARG. */
MOE_API int moe_permute_fp8(const moe_shape *shape, const int32_t *topk_idx, const float *topk_w,
                void *workspace, size_t workspace_bytes, moe_stream_t stream);
MOE_API int moe_expert_gate_up_fp8(const moe_shape *shape, const void *x, const moe_fp8_weight *W_gate,
                const moe_fp8_weight *W_up, const moe_fp8_weight *W_shared_gate,
                const moe_fp8_weight *W_shared_up, void *workspace, size_t workspace_bytes,
                moe_stream_t stream);
MOE_API int moe_expert_down_fp8(const moe_shape *shape, const moe_fp8_weight *W_down,
                const moe_fp8_weight *W_shared_down, void *workspace, size_t workspace_bytes,
                moe_stream_t stream);

/* ---- The steps of moe_forward, callable one by one (same arguments and
 * rules; each step reads what the previous steps left in the workspace, so
 * they must be called in this order with the same shape and workspace). ---- */

/* a1 + a2: router GEMM (fp32 accumulate, tcgen05 tensor cores) into fp32
 * logits in the workspace, then scoring, top-k (bias for selection only) and
 * optional renormalisation -> topk_idx, topk_w.  Also clears the workspace's
 * device error word. */
MOE_API int moe_route(const moe_shape *shape, const void *x, const void *W_router, const float *expert_bias,
              int score_fn, int norm_topk, float route_scale,
              int32_t *topk_idx, float *topk_w,
              void *workspace, size_t workspace_bytes, moe_stream_t stream);

/* a3: per-expert histogram, prefix scan and stable scatter of the (token,
 * slot) pairs into expert-contiguous rows (tokens ascending inside an expert),
 * plus the GEMM work lists, all on the device.  topk_idx / topk_w as written
 * by moe_route (any valid routing may be passed: each row of topk_idx must
 * hold k distinct experts in [0,E)). */
MOE_API int moe_permute(const moe_shape *shape, const int32_t *topk_idx, const float *topk_w,
                void *workspace, size_t workspace_bytes, moe_stream_t stream);

/* a4 + a6 (gate/up half): grouped GEMM over routed rows and the shared
 * experts' rows in one launch; h = SiLU(x W_gate^T) * (x W_up^T) written as
 * bf16 into the workspace (fp32 accumulate and epilogue). */
MOE_API int moe_expert_gate_up(const moe_shape *shape, const void *x,
                       const void *W_gate, const void *W_up,
                       const void *W_shared_gate, const void *W_shared_up,
                       void *workspace, size_t workspace_bytes, moe_stream_t stream);

/* a5 + a6 (down half): grouped GEMM y = w * (h W_down^T) per routed row (w =
 * its combine weight) and y = h W_shared_down^T per shared row, bf16 into the
 * workspace. */
MOE_API int moe_expert_down(const moe_shape *shape, const void *W_down, const void *W_shared_down,
                    void *workspace, size_t workspace_bytes, moe_stream_t stream);

/* a7: out[t] = sum_s g[t,s] y_shared[s,t] + sum_{j<k} y[row(t,j)], summed in
 * fp32 in that fixed order and rounded to bf16 once (bitwise reproducible).
 * g = 1 when W_shared_gate_vec is NULL (x may then be NULL too), else
 * sigmoid(W_shared_gate_vec[s] . x[t]) with x [T,d] the block input. */
MOE_API int moe_combine(const moe_shape *shape, const void *x, const void *W_shared_gate_vec, void *out,
                void *workspace, size_t workspace_bytes, moe_stream_t stream);

/* External-indices mode: steps a3..a7 on a routing the caller supplies
 * (for example experts picked by a fixed token-id hash, as the first MoE
 * layers of DeepSeek-V4-Pro do, or an MTP layer reusing the trunk's routing:
 * qwen3-5-vs-deepseek-v4 router cell; qwen3-5-vs-gemma-4 MTP cell).
 *   topk_idx [T,k] int32: k distinct experts in [0,E) per token (violations
 *   are reported by moe_device_status as MOE_ERR_INVALID_ARG; all indices
 *   are clamped so nothing is read out of bounds).
 *   topk_w [T,k] fp32: combine weights, used as given.
 * Everything else as in moe_forward; clears the device error word. */
MOE_API int moe_experts_forward(const moe_shape *shape, const void *x, const int32_t *topk_idx,
                                const float *topk_w, const void *W_gate, const void *W_up,
                                const void *W_down, const void *W_shared_gate, const void *W_shared_up,
                                const void *W_shared_down, const void *W_shared_gate_vec, void *out,
                                void *workspace, size_t workspace_bytes, moe_stream_t stream);

/* Introspection of the workspace layout, for tests and debugging.  Regions:
 *   MOE_WS_LOGITS   fp32 [P,T,E] router logits (after moe_route) as P partial
 *                                sums over slices of d, added in slice order
 *                                (P > 1 when the plan splits d: to fill the
 *                                SMs with small batches, or where two slices
 *                                load fewer bytes per SM; P <= 16)
 *   MOE_WS_COUNTS   int32 [E]    tokens per expert (after moe_permute)
 *   MOE_WS_OFFSETS  int32 [E+1]  first row of each expert's segment; segments
 *                                are padded to p rows (p = 16, or 32 when the
 *                                expert GEMMs run on CTA pairs: experts of 96+
 *                                rows on average); [E] = total rows
 *   MOE_WS_PERM     int32 [rows] token of each routed row (padding rows: 0)
 *   MOE_WS_ROW_W    fp32 [rows]  combine weight of each routed row (padding: 0)
 *   MOE_WS_INV      int32 [T,k]  row of each (token, slot)
 *   MOE_WS_H        bf16 [rows,f]   routed hidden rows (after moe_expert_gate_up)
 *   MOE_WS_H_SHARED bf16 [S,Tp,fs]  shared hidden rows, Tp = T rounded up to p
 *   MOE_WS_Y        bf16 [rows,d]   weighted routed outputs (after moe_expert_down)
 *   MOE_WS_Y_SHARED bf16 [S,Tp,d]   shared outputs
 *   MOE_WS_X_STAGE  bf16 [T,d]      token rows the library staged: x copied
 *                                   from the host (moe_forward_host) or the
 *                                   normalised x (moe_forward_prenorm)
 *   MOE_WS_WORK_COUNTS  int32 [4]   after moe_permute: gate/up work units U1,
 *                                   down work units U2, routed rows, a tag of
 *                                   the plan that wrote the lists
 *   MOE_WS_WORK_GATE_UP int32 [U1,4] gate/up work units {group, weight block,
 *                                   first row, rows}: groups >= E are the
 *                                   shared experts (first in the list), whose
 *                                   rows index [0, Tp); routed units follow
 *                                   expert by expert, largest, smallest, 2nd
 *                                   largest, 2nd smallest, ... by padded rows
 *   MOE_WS_WORK_DOWN    int32 [U2,4] the same for the down GEMM
 * Writes the region's byte offset in the workspace and its capacity in bytes.
 * Returns MOE_OK, or MOE_ERR_INVALID_ARG for a bad shape, region or pointer. */
#define MOE_WS_LOGITS   0
#define MOE_WS_COUNTS   1
#define MOE_WS_OFFSETS  2
#define MOE_WS_PERM     3
#define MOE_WS_ROW_W    4
#define MOE_WS_INV      5
#define MOE_WS_H        6
#define MOE_WS_H_SHARED 7
#define MOE_WS_Y        8
#define MOE_WS_Y_SHARED 9
#define MOE_WS_X_STAGE  10
#define MOE_WS_WORK_COUNTS  11
#define MOE_WS_WORK_GATE_UP 12
#define MOE_WS_WORK_DOWN    13
MOE_API int moe_workspace_region(const moe_shape *shape, int region, size_t *offset, size_t *bytes);

/* Synchronises `stream`, then returns MOE_ERR_DEVICE_TIMEOUT if a kernel of a
 * call on this workspace (since the last moe_route) gave up a bounded wait,
 * MOE_ERR_INVALID_ARG if routing handed to the permute step was invalid,
 * MOE_ERR_NONFINITE if the routing step met a NaN or infinite logit,
 * selection key or combine weight, MOE_ERR_CUDA if the stream reports an
 * error, else MOE_OK (the first of these that applies).
 *
 * Non-finite inputs never make a kernel read or write out of bounds: a NaN
 * selection key ranks below every other key (with -inf), so each token still
 * gets k distinct experts in [0, E); its weights are whatever the arithmetic
 * gives (NaN for an all-NaN row).  If the router GEMM gives up a bounded wait,
 * the top-k step writes expert -1 and weight 0 for every token instead of
 * routing on incomplete logits. */
MOE_API int moe_device_status(const void *workspace, moe_stream_t stream);

/* Routing (the moe_route step) for callers that cannot allocate device
 * memory, such as an inference-engine plugin whose per-call hook may not
 * allocate, or a process whose device memory is reserved up front by another
 * allocator.  The pages have no counterpart: this is an integration variant,
 * not part of the method.
 *   Same arguments and results as moe_route, without the workspace: the fp32
 *   logits live in a 16 MiB array compiled into this library, which every GPU
 *   that loads the library holds until the process exits.  Shapes with
 *   T * E * 4 bytes > 16 MiB (T * E > 4,194,304) return MOE_ERR_SCRATCH_LIMIT
 *   and enqueue nothing.  x, W_router, expert_bias, topk_idx and topk_w are
 *   the caller's, as for moe_route.  Allocates nothing (no cudaMalloc /
 *   cudaFree) on any call.
 *   The first call on a device looks up the array's device address (a CUDA
 *   runtime query, once per device, with that device current); make that
 *   first call before any stream capture.
 *   Every call uses the same array: two calls that overlap on the GPU (on
 *   different streams, or from different threads without ordering) race and
 *   give undefined results.  The array keeps the last call's contents; the
 *   call clears what must start at zero itself.
 *   A bounded device wait that runs out is recorded only inside that array,
 *   which moe_device_status cannot read; it shows in the outputs instead:
 *   every topk_idx is then -1 and every topk_w 0.  A NaN or infinite logit
 *   is not reported for this entry point (the routing stays in range, as for
 *   moe_route). */
MOE_API int moe_route_noalloc(const moe_shape *shape, const void *x, const void *W_router,
                              const float *expert_bias, int score_fn, int norm_topk, float route_scale,
                              int32_t *topk_idx, float *topk_w, moe_stream_t stream);

/* Self-test of the bounded-wait machinery: launches one block that waits on a
 * shared-memory barrier which nothing ever completes, for at most timeout_ns
 * nanoseconds (clamped to 1 ms .. 1 s), then records the timeout in the
 * workspace's error word and returns.  moe_device_status then reports
 * MOE_ERR_DEVICE_TIMEOUT and the context stays usable. */
MOE_API int moe_debug_wait_timeout(void *workspace, size_t workspace_bytes, uint64_t timeout_ns,
                           moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
