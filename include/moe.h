/*
 * moe.h -- C ABI of libmoe.so: one sparse-MoE layer with GPU-resident expert
 * routing and affine 4-bit experts, on one NVIDIA B200 (sm_100a).
 *
 * The layer is the Qwen3.6-35B-A3B MoE block that the Lily write-ups single
 * out ("Perplexity's Lily: A Breakthrough Local Inference Engine Tailored
 * Exclusively for Apple Silicon", section "The Model: Qwen3.6-35B-A3B in
 * Focus"; "Perplexity Open Sources Apple Chip Inference Engine Lily",
 * paragraphs 3 and 5): a router scores E experts and keeps k of them per
 * token, one always-on shared expert sees every token, and every expert
 * weight is MLX affine 4-bit with one bf16 scale and one bf16 bias per group
 * of 64 weights along the input dimension.  The same write-ups ("How It
 * Works: Prefill and Decode Strategies") keep the routing histogram, prefix
 * scan and scatter on the GPU with no CPU synchronisation, and rebuild the
 * 4-bit weights tile by tile inside the grouped expert GEMM.
 *
 * What one call computes, for tokens t = 0..T-1 (x, out: bf16 [T, H]):
 *   l[t,e]   = x_t . W_r[e] (+ router_bias[e])                    (FP32)
 *   idx[t,:] = the k experts with the largest l[t,e]; equal logits go to
 *              the lower expert index; slot order = (logit desc, index asc)
 *   w[t,j]   = exp(l[t,idx_j] - l[t,idx_0]) / sum_j' exp(...)    (softmax
 *              over all experts renormalised over the k chosen ones)
 *   expert e on row x:  h = bf16(silu(x W_g[e]^T) * (x W_u[e]^T)),
 *                       y = h W_d[e]^T,  silu(z) = z / (1 + exp(-z))
 *   sigma_t  = 1 / (1 + exp(-x_t . w_sg))
 *   out_t    = bf16( sum_{j=0..k-1} w[t,j] * y_{t,idx_j}  +  sigma_t * ys_t )
 *              summed in FP32 in exactly that order (ys = shared expert).
 * Weights are used as w = scale * q + bias per group of 64 (q in 0..15).
 *
 * Storage.
 *   bf16 values are passed as their 16-bit patterns (moe_bf16).
 *   A q-matrix [R, C] is three row-major device arrays:
 *     q      uint32 [R, C/8]  -- code i of a word = element 8w+i, bits 4i..4i+3
 *     scales bf16   [R, C/64]
 *     biases bf16   [R, C/64]
 *   Stacked expert matrices add a leading [E] dimension, contiguous.
 *   All pointers in moe_layer_desc, moe_routing and the x/out/workspace
 *   arguments of moe_route/moe_forward/moe_decode are DEVICE pointers; only
 *   moe_forward_host takes host x/out.
 *
 * Ownership.  The caller owns every buffer (weights, x, out, routing,
 * workspace).  The library allocates no device memory and keeps no state
 * between calls except cached kernel attributes.  Two calls must not share a
 * workspace concurrently.  A workspace must be zero-filled once before its
 * first use (e.g. cudaMemset of the whole buffer).  Its first 256 bytes are a
 * control block (status word, the small-T router's completion counters, the
 * fused decode kernel's exit counter and launch epoch); the library leaves
 * the counters and the status word zero after every call except for a
 * recorded error status, which moe_get_status clears together with the
 * counters.  The fused decode kernel's CTAs exchange values through 64-bit
 * words of the workspace tagged with (launch epoch, layer): a stale word is
 * never taken for a current one, except one last written exactly a multiple
 * of 2^26 launches earlier on the same workspace and not rewritten since.
 *
 * Asynchrony.  moe_route, moe_forward, moe_decode and moe_rmsnorm enqueue
 * work on `stream` (a cudaStream_t; NULL = the legacy default stream) and
 * return without waiting for the device.  Their outputs are valid once the
 * stream reaches that point.  No call reads device data back on the host
 * except moe_get_status and moe_forward_host (moe_forward_host_async does not wait).
 * The prefill kernels and moe_rmsnorm are launched with programmatic
 * dependent launch: a kernel may be scheduled, and set up its own on-chip
 * state, while the preceding work of the stream finishes, but it reads and
 * writes no global memory before that work has completed, so stream order
 * holds for every buffer as with ordinary launches.
 *
 * Errors.  Every entry point returns a moe_status.  Arguments are validated on
 * the host before anything is enqueued: a rejected call enqueues nothing.  A
 * failed kernel launch returns MOE_ERR_CUDA.  Bounded device-side waits that
 * give up record MOE_ERR_DEVICE_TIMEOUT in the workspace's status word, which
 * moe_get_status returns.
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

typedef uint16_t moe_bf16;   /* bf16 bit pattern */
typedef void* moe_stream;    /* a cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1,     /* NULL pointer, T out of range, misaligned pointer */
  MOE_ERR_UNSUPPORTED = -2,     /* layout other than affine 4-bit / group 64, sizes not supported */
  MOE_ERR_WORKSPACE = -3,       /* workspace NULL, too small, or misaligned */
  MOE_ERR_CUDA = -4,            /* a CUDA runtime call or kernel launch failed */
  MOE_ERR_DEVICE_TIMEOUT = -5,  /* a bounded device-side wait gave up */
  MOE_ERR_DEVICE_INDEX = -6     /* a device-side bounds check found an index out of range (attn.h) */
} moe_status;

/* One affine 4-bit matrix (or a stack of E of them); see "Storage" above. */
typedef struct {
  const uint32_t* q;
  const moe_bf16* scales;
  const moe_bf16* biases;
} moe_qmat;

/* One MoE layer.  Accepted layout (anything else is MOE_ERR_UNSUPPORTED, as
 * the Lily loader refuses every layout but the one it was built for --
 * "Perplexity Open Sources Apple Chip Inference Engine Lily", paragraph 3):
 *   bits == 4, group_size == 64, renorm == 1,
 *   1 <= k <= 8, k <= E <= 256,
 *   H a multiple of 128 and <= 8192; I and I_shared multiples of 128 and <= 2048.
 * The layer the write-ups describe ("Perplexity's Lily: ...", section "The
 * Model: Qwen3.6-35B-A3B in Focus": 256 experts, 8 chosen per token) has
 * k = 8, E = 256, H = 2048 and I = I_shared = 512, so these bounds admit it
 * and every size of its family.  They are narrower than "any k <= E, any
 * multiple of the group size" on purpose: every weight tile of the expert
 * GEMMs is 128 rows (one tensor-memory lane per row) and stays full, and each
 * token's k candidates stay in registers through the top-k merges.  A layer
 * outside them is refused on the host before anything is enqueued. */
typedef struct {
  int H;            /* hidden size */
  int I;            /* routed expert intermediate size */
  int I_shared;     /* shared expert intermediate size */
  int E;            /* number of routed experts */
  int k;            /* experts chosen per token */
  int group_size;   /* must be 64 */
  int bits;         /* must be 4 */
  int renorm;       /* must be 1: weights renormalised over the chosen experts */
  const moe_bf16* w_router;       /* [E, H] */
  const float*    router_bias;    /* [E] or NULL; added to the logits before selection */
  moe_qmat gate;                  /* [E, I, H] */
  moe_qmat up;                    /* [E, I, H] */
  moe_qmat down;                  /* [E, H, I] */
  moe_qmat sh_gate;               /* [I_shared, H] */
  moe_qmat sh_up;                 /* [I_shared, H] */
  moe_qmat sh_down;               /* [H, I_shared] */
  const moe_bf16* w_shared_gate;  /* [H]; sigma_t = sigmoid(x_t . w_shared_gate) */
} moe_layer_desc;

/* Routing results (device buffers owned by the caller).
 *   topk_idx[t*k + j], topk_w[t*k + j]: chosen expert and weight of slot j;
 *   counts[e]: rows routed to expert e;  offsets[0..E]: exclusive prefix sum;
 *   perm[pos] = t*k + j, grouped by expert ascending, tokens ascending within
 *   an expert (stable counting sort);  inv_perm[t*k + j] = pos;
 *   sigma[t]: shared-expert gate (may be NULL). */
typedef struct {
  int32_t* topk_idx;   /* [T*k] */
  float*   topk_w;     /* [T*k] */
  int32_t* counts;     /* [E] */
  int32_t* offsets;    /* [E+1] */
  int32_t* perm;       /* [T*k] */
  int32_t* inv_perm;   /* [T*k] */
  float*   sigma;      /* [T] or NULL */
} moe_routing;

/* Bytes of device workspace that moe_route / moe_forward / moe_decode /
 * moe_forward_host / moe_forward_stack need for any T <= T_max.  The
 * workspace holds the routing buffers the GPU builds for itself (histogram,
 * prefix sums, permutation and the tile list of the grouped GEMMs: "Perplexity's
 * Lily: ...", section "How It Works: Prefill and Decode Strategies", which
 * keeps them on the device with no CPU synchronisation) and the experts'
 * intermediate rows.  Returns MOE_ERR_UNSUPPORTED or MOE_ERR_INVALID_ARG for
 * a layer or T_max the other calls would reject. */
MOE_API int moe_workspace_size(const moe_layer_desc* layer, int T_max, size_t* bytes);

/* Router logits, softmax top-k with renormalisation, shared gate, and the
 * on-device expert histogram, prefix sum and permutation ("Perplexity's
 * Lily: ...", section "How It Works: Prefill and Decode Strategies").
 * x: device bf16 [T, H], 16-byte aligned.  r: required.  1 <= T <= 65536. */
MOE_API int moe_route(const moe_layer_desc* layer, const moe_bf16* x, int T, moe_routing* r,
              void* workspace, size_t workspace_bytes, moe_stream stream);

/* The whole layer: routing, fused-dequant gate/up grouped GEMM with the
 * SwiGLU epilogue, down-projection grouped GEMM, shared expert, and the
 * fixed-order gather-combine.  The write-ups ("Perplexity's Lily: ...",
 * sections "The Model: Qwen3.6-35B-A3B in Focus" and "How It Works: Prefill
 * and Decode Strategies") describe this layer: routed experts chosen on the
 * GPU, their 4-bit weights rebuilt tile by tile inside the grouped GEMM with
 * bf16 products and FP32 accumulation, and one always-on shared expert.
 * x, out: device bf16 [T, H], 16-byte aligned, not overlapping.
 * r: optional (NULL = keep routing in the workspace).
 * 1 <= T <= 65536.  Three kernel sets, chosen by T:
 *   T <= 3 (T <= 7 inside moe_forward_stack) with H = 1024 or 2048, I and
 *     I_shared whole groups, 16-byte aligned scale and bias stacks and at
 *     most E + 1 SMs: the single-launch fused decode kernel (see moe_decode);
 *   T <= 128 with H a multiple of 256 and I, I_shared multiples of 128 (the
 *     mid-size decode path): the one-launch small-T router, then gate/up +
 *     SwiGLU and down as GEMVs over the active experts only (warp-level
 *     mma.sync on 8-token tiles, codes streamed from global memory into the
 *     operand registers), then the fixed-order combine;
 *   every other T: the tensor-core (tcgen05) kernels above. */
MOE_API int moe_forward(const moe_layer_desc* layer, const moe_bf16* x, int T, moe_bf16* out,
                moe_routing* r, void* workspace, size_t workspace_bytes, moe_stream stream);

/* The same function for 1 <= T <= 64 (batch decoding streams the active
 * experts' weights: "How It Works: Prefill and Decode Strategies"); it runs
 * what moe_forward runs for T.  T > 64 is MOE_ERR_INVALID_ARG.  Under the
 * fused conditions above the whole layer is ONE cooperative launch of one CTA
 * per SM whose CTAs exchange the router logits, the SwiGLU activations and
 * the outputs through tagged workspace words (no grid-wide barrier);
 * otherwise the mid-size decode path's four launches (routing, gate/up, down,
 * combine), or the tensor-core kernels where that path does not apply. */
MOE_API int moe_decode(const moe_layer_desc* layer, const moe_bf16* x, int T, moe_bf16* out,
               moe_routing* r, void* workspace, size_t workspace_bytes, moe_stream stream);

/* A stack of MoE layers joined by RMSNorm, enqueued on one stream with no
 * host synchronisation between layers ("Perplexity's Lily: ...", section "How
 * It Works: Prefill and Decode Strategies": the layers of a forward pass are
 * recorded into one GPU submission with no CPU round trip), so the whole call
 * can also be captured once as a CUDA graph and replayed:
 *   a_0 = x;  y_l = layer_l(a_l);  a_{l+1} = bf16(y_l / sqrt(mean(y_l^2) + eps))
 * (RMSNorm with weight 1 and no residual, over the bf16 values of y_l);
 * out = y_{n_layers-1}.  Each layer runs what moe_forward runs for T.  On the
 * tensor-core and mid-size paths the RMSNorm is computed inside the layer's
 * combine kernel (the row's sum of squares is formed while its output is
 * written).  On the fused decode path up to 40 layers run in ONE launch,
 * the RMSNorm between them inside it (each CTA publishes the sum of squares of its outputs);
 * longer stacks are cut into launches of 40 layers joined by a small
 * RMSNorm kernel.
 *   layers: host array of n_layers (1..1024) descriptors with equal H, I,
 *           I_shared, E and k.
 *   x, out: device bf16 [T, H], 16-byte aligned, not overlapping.
 *   trace:  NULL, or device bf16 [n_layers][2][T][H] that receives a_l in
 *           trace[l][0] and y_l in trace[l][1] (for debugging and tests).
 *   workspace: as for moe_forward with the same T (moe_workspace_size); the
 *           activations between layers live in it.
 * Validation covers every layer before anything is enqueued. */
MOE_API int moe_forward_stack(const moe_layer_desc* layers, int n_layers, const moe_bf16* x, int T, moe_bf16* out,
                              moe_bf16* trace, float eps, void* workspace, size_t workspace_bytes,
                              moe_stream stream);

/* moe_route for callers that cannot allocate device memory.  The pages have
 * no counterpart to this entry point; it exists for hosts that hand the
 * library only the tensors it reads and writes -- a plug-in inside another
 * runtime that exposes no allocator, or a serving loop with a fixed memory
 * plan where a cudaMalloc (which may also synchronise the device) is not
 * allowed.  It runs the same kernels as moe_route for the same T (T <= 64:
 * the one-launch small-T router; larger T: the tensor-core router and the
 * counting-sort passes), so its outputs are those of moe_route, but it takes
 * no workspace: its scratch (a 256-byte control block with a status word,
 * then for T <= 64 the T x (E+1) logits, otherwise the per-segment expert
 * counts and the chunk list; the active-expert list; and sigma when r->sigma
 * is NULL) lives in one static device array of 512 KiB inside libmoe.so,
 * which every GPU that loads the library holds until the process exits.
 *   Limit: the call needs 256 bytes of control block, plus for T <= 64
 *   T*(E+1)*4 bytes of logits, or for T > 64 ceil(T/128)*E*4 bytes of counts
 *   and (T*k/160 + T/160 + E + 2)*16 + 4 bytes of chunk list, plus
 *   (E+1)*4 + 4 bytes of active list, plus T*4 bytes if r->sigma is NULL,
 *   each piece rounded up to 256 bytes; a call whose need exceeds 512 KiB
 *   returns MOE_ERR_WORKSPACE and enqueues nothing (for E=256, k=8 this
 *   admits T <= 58112 when r->sigma is given, T <= 40099 when it is NULL).
 *   Set-up: the first call on each device looks up the array's device
 *   address with cudaGetSymbolAddress while that device is current, so make
 *   that first call before any stream capture on that device.
 *   Sharing: all calls in the process use the same array.  Its control block
 *   starts at zero (static storage) and every call leaves it zero except for
 *   a recorded error status; nothing else in it needs to start at zero
 *   (every call rewrites what it reads).  Two calls whose GPU work overlaps
 *   (different streams, or host threads) race on it.
 *   Errors: a bounded device-side wait that gives up records
 *   MOE_ERR_DEVICE_TIMEOUT in the array's status word; moe_get_status(NULL,
 *   stream) returns it (and clears the control block).
 * Allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 * Arguments as for moe_route, minus the workspace; r is required. */
MOE_API int moe_route_static(const moe_layer_desc* layer, const moe_bf16* x, int T, moe_routing* r,
                             moe_stream stream);

/* moe_forward with x and out in HOST memory (page-locked for full speed):
 * copies x to the workspace, runs the layer, copies the result back and waits
 * for `stream`.  Weights stay device pointers. */
MOE_API int moe_forward_host(const moe_layer_desc* layer, const moe_bf16* x_host, int T, moe_bf16* out_host,
                     void* workspace, size_t workspace_bytes, moe_stream stream);

/* moe_forward_host without the final wait: enqueues the copy of x to the
 * workspace, the layer and the copy of the result to out_host on `stream` and
 * returns.  out_host is valid once the stream reaches that point; x_host must
 * stay unchanged until then.  With page-locked buffers the copies are
 * asynchronous, so a caller that rotates over a few streams (each with its
 * own workspace and output buffer) overlaps one call's copies with the other
 * calls' kernels: one stream runs its copy in, layer and copy out in order,
 * so with large T three streams are needed to hide both copies. */
MOE_API int moe_forward_host_async(const moe_layer_desc* layer, const moe_bf16* x_host, int T, moe_bf16* out_host,
                                   void* workspace, size_t workspace_bytes, moe_stream stream);

/* y_out[t] = bf16(y[t] / sqrt(mean(y[t]^2) + eps)) over H columns, weight 1,
 * no residual: the input of the next layer in a stack of MoE layers.
 * y, y_out: device bf16 [T, H], 16-byte aligned (may alias). */
MOE_API int moe_rmsnorm(const moe_bf16* y, moe_bf16* y_out, int T, int H, float eps, moe_stream stream);

/* Stage timing (tracing).  Same as moe_forward, but records a CUDA event on
 * `stream` before the first and after every stage, waits for the stream, and
 * writes each stage's device time in milliseconds to stage_ms[0..n-1]:
 *   tensor-core path: router, group (histogram+scan+scatter), gather of the
 *            grouped token rows, gate/up GEMM, down GEMM, combine (6 stages)
 *   mid-size decode path: routing, gate/up, down, combine (4 stages)
 *   fused decode kernel (when moe_forward uses it): one stage
 * stage_ms: host array of at least 6 floats; *n_stages receives the count.
 * The events are created and destroyed inside the call. */
MOE_API int moe_forward_profiled(const moe_layer_desc* layer, const moe_bf16* x, int T, moe_bf16* out,
                                 void* workspace, size_t workspace_bytes, moe_stream stream,
                                 float* stage_ms, int* n_stages);

/* Waits for `stream`, returns the status word kept in `workspace` (MOE_OK or
 * MOE_ERR_DEVICE_TIMEOUT) and, when it is not MOE_OK, clears the control
 * block.  workspace == NULL reads the status word of moe_route_static's
 * static scratch on the current device instead.  MOE_ERR_CUDA if the wait
 * fails; MOE_ERR_WORKSPACE if workspace is not 256-byte aligned. */
MOE_API int moe_get_status(void* workspace, moe_stream stream);

/* Failure detection control: the kernels' bounded device-side waits (on
 * mbarriers and grid barriers) give up after `cycles` SM clock cycles and
 * record MOE_ERR_DEVICE_TIMEOUT (cycles <= 0 restores the default, 2^32 cycles,
 * about 2 s).  Process-wide; it applies to kernels enqueued after the call.
 * Waits that drain copies or tensor-core work a kernel has already issued keep
 * the default, so a kernel that gives up never exits with a copy into its
 * shared memory in flight.  A short limit exists to test the error path: a
 * call whose waits give up leaves its outputs unwritten (kernels that would
 * read unwritten routing indices do nothing while the status word holds an
 * error) and reports the timeout through moe_get_status. */
MOE_API int moe_set_wait_limit(long long cycles);

/* Static description of a status code. */
MOE_API const char* moe_strerror(int status);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H_ */
