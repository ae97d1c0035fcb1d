/*
 * gqe.h — C ABI of the Grouped Query Experts (GQE) attention forward (prefill) library.
 *
 * GQE is a mixture-of-experts layer on grouped-query attention ("GQE: Grouped Query
 * Experts", FrontiersMindAI/GQE README, Algorithm Overview): N query-head experts in G
 * groups, each group with one dense KV head. Per token and per group a router takes a
 * softmax over the group's E = N/G experts and keeps the top k; only the selected query
 * heads plus one always-on shared head are projected and attend over the dense K/V; the
 * outputs are combined ("gqe", "weighted_concat", "hard_concat": README, Ablations and
 * Parameters) and projected by W_o. A Switch-style load-balancing loss is reduced on the
 * side (README, Algorithm Overview; gist.science summary, Training and Loss).
 *
 * Conventions for every entry point
 *   - Tensor pointers are DEVICE pointers owned by the caller, contiguous, row-major,
 *     16-byte aligned, in the handle's dtype (bf16 or fp32) unless stated otherwise.
 *   - Weights use the nn.Linear layout [out, in]; y = x W^T; there are no biases.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *     Work is enqueued on it; no entry point synchronises the device except
 *     gqe_check_device_status.
 *   - Errors are reported by return code only. On an error return nothing has been
 *     launched. No entry point aborts or throws.
 *   - A handle may be used by one stream at a time.
 */
#ifndef GQE_H
#define GQE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct gqe_ctx* gqe_handle;

typedef enum {
    GQE_OK = 0,
    GQE_ERR_INVALID_ARG = 1,  /* null / misaligned pointer, bad size, mismatch with create */
    GQE_ERR_UNSUPPORTED = 2,  /* a shape this build does not implement (see gqe_create)   */
    GQE_ERR_WORKSPACE = 3,    /* B*T larger than the handle's max_tokens                   */
    GQE_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed                          */
    GQE_ERR_TIMEOUT = 5       /* a device-side bounded wait gave up (see status below)      */
} gqe_status;

typedef enum {
    GQE_VARIANT_GQE = 0,             /* routed blocks + renormalised slot + shared block */
    GQE_VARIANT_WEIGHTED_CONCAT = 1, /* routed blocks scaled by raw router p + shared    */
    GQE_VARIANT_HARD_CONCAT = 2      /* routed blocks as computed + shared               */
} gqe_variant;

typedef enum { GQE_BF16 = 0, GQE_F32 = 1 } gqe_dtype;

/* Internal tensors that gqe_get_tensor can copy out (for tests and inspection). */
typedef enum {
    GQE_T_K = 0,      /* [G, M, d_h]       keys, dtype                                      */
    GQE_T_V = 1,      /* [G, M, d_h]       values, dtype                                    */
    GQE_T_Q = 2,      /* [S, M, d_h]       query streams (routed g*k+r, then shared), dtype */
    GQE_T_Z = 3,      /* [M, D_o]          concatenated attention output, dtype             */
    GQE_T_PSEL = 4,   /* [M, G, k] float   router softmax p of each selected expert         */
    GQE_T_W = 5,      /* [M, G, k] float   slot weights (p renormalised over all G*k)       */
    GQE_T_LOGITS = 6  /* [M, N]    float   router logits                                    */
} gqe_tensor;

/*
 * gqe_create — make a handle for one layer shape and allocate its device workspace.
 *
 *   dim         hidden size d ("dim", README Parameters), 16 <= dim, dim % 16 == 0 for bf16.
 *   N           routed query-head experts ("num_query_experts"); N % G == 0 (README
 *               Parameters), N <= 64.
 *   G           GQA groups = dense KV heads ("num_kv_heads").
 *   k           experts kept per group per token ("top_k"), 1 <= k <= min(N/G, 8).
 *   d_h         head dimension ("head_dim"; its default dim/N is applied by the Python
 *               binding, not here). d_h in {16, 32, 48, 64, 80, 96, 112, 128} for
 *               both dtypes (GQE_ERR_UNSUPPORTED otherwise).
 *   dtype       GQE_BF16 (bf16 storage, fp32 accumulation) or GQE_F32.
 *   max_tokens  the largest B*T any gqe_forward on this handle will use.
 *
 * Allocates (cudaMalloc, on the current device) the workspace for K, V, the query streams,
 * Z, the routing tables and a device status word; the handle owns it until gqe_destroy.
 * Returns GQE_ERR_INVALID_ARG / GQE_ERR_UNSUPPORTED for bad shapes and GQE_ERR_CUDA if an
 * allocation fails (*h is then NULL).
 */
gqe_status gqe_create(gqe_handle* h, int dim, int N, int G, int k, int d_h, gqe_dtype dtype,
                      int64_t max_tokens);

/*
 * gqe_forward — one GQE attention forward pass on B sequences of T tokens.
 *
 *   x         [B*T, dim]        input activations (token-major; sequence b owns rows b*T..).
 *   W_r       [N, dim]          router; expert e = g*E + j belongs to group g.
 *   W_q       [N*d_h, dim]      query projections; expert e owns rows e*d_h .. e*d_h+d_h-1.
 *   W_k, W_v  [G*d_h, dim]      dense key / value projections; head g owns rows g*d_h...
 *   W_shared  [d_h, dim]        always-on shared query head (README, Algorithm Overview;
 *                               it reads KV head 0), or NULL for a layer without it.
 *   W_o       [dim, D_o]        output projection, D_o = (G*k + [variant==GQE] +
 *                               [W_shared != NULL]) * d_h. Z's column blocks are: routed
 *                               streams g-major then rank r, then the slot (GQE only), then
 *                               the shared stream.
 *   N, G, k, d_h                must equal the values given to gqe_create.
 *   variant   gqe_variant (gist.science summary, Output Construction; README Ablations).
 *   causal    1: token t attends to positions <= t of its own sequence; 0: to all T.
 *   out       [B*T, dim]        result y = Z W_o^T, written in the handle's dtype.
 *   aux_loss  device float*     the Switch load-balancing loss (without the caller's 0.01
 *                               coefficient, README Usage), or NULL to skip writing it.
 *   stream    cudaStream_t      as void*.
 *
 * Routing per token and group: softmax over the E logits in fp32, top-k on the fp32
 * logits with the lower expert index winning ties, selected experts listed in ascending
 * index. Allocates nothing and does not synchronise. Returns GQE_ERR_WORKSPACE if
 * B*T > max_tokens, GQE_ERR_INVALID_ARG for null required pointers, pointers not 16-byte
 * aligned, B < 1, T < 1, or N/G/k/d_h different from the handle's.
 *
 * CUDA graphs: a call (gqe_forward or gqe_decode) may be captured on `stream` and the graph
 * replayed any number of times, interleaved with eager calls on the same handle in stream
 * order; every per-call state the kernels keep (the routing cursors' two alternating sets
 * and their set flag, the attention's work counter) lives in the handle's device workspace
 * and is advanced by the kernels themselves. The replay reads the pointers and sizes of the
 * captured call. Two captured graphs of one handle must not run concurrently.
 */
gqe_status gqe_forward(gqe_handle h, const void* x, int B, int T, const void* W_r,
                       const void* W_q, const void* W_k, const void* W_v, const void* W_shared,
                       const void* W_o, int N, int G, int k, int d_h, int variant, int causal,
                       void* out, float* aux_loss, void* stream);

/*
 * gqe_decode — one generation step with a KV cache: for each of B sequences, its next token
 * at position lengths[b]. GQE keeps the KV heads dense and unchanged (README, Algorithm
 * Overview), so the cache is GQA's; the new token is routed, its selected query heads and the
 * shared head are projected, and each attends over positions 0 .. lengths[b] of its KV head.
 * The result equals row lengths[b] of gqe_forward (causal) over the whole sequence.
 *
 *   x         [B, dim]               the new tokens.
 *   k_cache,  [G, B, L_max, d_h]     caller-owned caches in the handle's dtype; rows
 *   v_cache                          0 .. lengths[b]-1 of (g, b) hold K / V of those positions.
 *                                    The step writes the new token's K / V at row lengths[b]
 *                                    and reads no row after it; no other row is written.
 *   L_max     rows per (group, sequence) in the caches, >= 1.
 *   lengths   [B] int32, DEVICE      positions of the new tokens, 0 <= lengths[b] < L_max.
 *                                    Not modified: the caller advances them after the step.
 *   W_*, N, G, k, d_h, variant, out [B, dim], aux_loss, stream: as gqe_forward (the aux loss
 *                                    is the Switch loss over the B new tokens).
 *
 * A handle restricted to groups [g0, g1) (gqe_set_group_range) takes the weights as its
 * gqe_forward does and caches of its heads only, [(g1-g0), B, L_max, d_h]; `out` receives its
 * share of the new tokens' y (the layer's is the sum over the ranges).
 *
 * bf16 handles only (GQE_ERR_UNSUPPORTED for fp32, or for B > 65535). Requires
 * B <= max_tokens (GQE_ERR_WORKSPACE). Allocates nothing and does not synchronise; the routing and tensors
 * of the step are available through gqe_get_routing / gqe_get_tensor (M = B). A position
 * outside [0, L_max) cannot be checked on the host: the step then reads and writes nothing
 * for that sequence, leaves its output undefined, and the next gqe_check_device_status
 * returns GQE_ERR_INVALID_ARG. Other errors as gqe_forward.
 */
gqe_status gqe_decode(gqe_handle h, const void* x, int B, void* k_cache, void* v_cache,
                      int L_max, const int32_t* lengths, const void* W_r, const void* W_q,
                      const void* W_k, const void* W_v, const void* W_shared, const void* W_o,
                      int N, int G, int k, int d_h, int variant, void* out, float* aux_loss,
                      void* stream);

/*
 * gqe_enable_backward — prepare the handle for training (README, Usage: the layer is trained
 * with loss.backward()): allocate its backward workspace (cudaMalloc, on the current device;
 * the gradients of dZ, of the stream outputs and of the query, key and value projections
 * for max_tokens tokens, and a cuBLAS handle with its 32 MiB workspace). The
 * handle owns it until gqe_destroy. bf16 handles only (every head dim they accept, 16 to 128;
 * GQE_ERR_UNSUPPORTED for float32 handles); GQE_ERR_CUDA if an allocation fails. Calling it
 * again does nothing.
 */
gqe_status gqe_enable_backward(gqe_handle h);

/*
 * gqe_backward — gradients of one GQE attention layer for training (README, Usage: the
 * task loss plus 0.01 times the aux loss is back-propagated; gist.science summary, Output
 * Construction: the renormalised slot is the router's differentiable path).
 *
 * Returns the gradients of F = <dy, y> + aux_grad * L, where y and L are the output and the
 * aux loss of the handle's LAST call, which must be a gqe_forward with the same x, weights,
 * B, T, variant, causal and presence of W_shared (its K, V, query streams, Z, routing and
 * per-row attention log-sum-exp are reused; GQE_ERR_INVALID_ARG otherwise, or if
 * gqe_enable_backward has not been called). The top-k selection is held constant.
 *
 *   x, W_*, B, T, N, G, k, d_h, variant, causal   as the forward (device, handle dtype).
 *   dy        [B*T, dim]   upstream gradient of y, handle dtype (bf16), device.
 *   aux_grad  host float   coefficient of the aux loss in the loss (0.01 in README, Usage).
 *   dx        [B*T, dim]   float32, device: gradient of x.
 *   dW_r      [N, dim], dW_q [N*d_h, dim], dW_k, dW_v [G*d_h, dim], dW_shared [d_h, dim]
 *             (NULL exactly when W_shared is NULL), dW_o [dim, D_o]: float32, device,
 *             overwritten (not accumulated into).
 *
 * Enqueued on `stream`; allocates nothing and does not synchronise. Hand-written kernels
 * form the combine/router backward and the attention backward (tcgen05); the dense weight
 * and input gradient GEMMs run in cuBLAS. The result is the same from run to run (no
 * atomics). Errors as gqe_forward. A gqe_forward followed by this call may be captured in
 * one CUDA graph and replayed as a training step (cuBLAS runs with the handle's preset
 * workspace, so the capture allocates nothing).
 */
gqe_status gqe_backward(gqe_handle h, const void* x, int B, int T, const void* W_r,
                        const void* W_q, const void* W_k, const void* W_v, const void* W_shared,
                        const void* W_o, int N, int G, int k, int d_h, int variant, int causal,
                        const void* dy, float aux_grad, float* dx, float* dW_r, float* dW_q,
                        float* dW_k, float* dW_v, float* dW_shared, float* dW_o, void* stream);

/*
 * gqe_backward_begin / gqe_backward_finish — the backward pass in two phases, for a handle
 * restricted to a group range (gqe_set_group_range) as well as for a whole layer; gqe_backward
 * is the two in one call on a whole layer.
 *
 * The group-parallel split (one range per GPU, the layer's y the sum of the ranges' shares)
 * keeps the backward local to each range except for one number per token: the gqe slot
 * weights w = p_sel / P_t divide by the selected probabilities of ALL groups (gist.science
 * summary, Output Construction), so the router gradient of every range needs
 * <dslot, slot> = sum over all routed streams of w_s <dslot, O_s>. begin writes this range's
 * share of it, the caller sums the shares over the ranges (an all-reduce of B*T floats, which
 * may overlap begin's attention backward on another stream), and finish takes the sum.
 *
 * begin: the arguments of gqe_backward up to dy, then
 *   slot_dot  [B*T] float32, device, 4-byte aligned: written (zero for the weighted_concat
 *             and hard_concat variants, whose router gradient needs no exchange).
 * finish: the same arguments, aux_grad, slot_dot (the sum over the ranges; for a whole layer
 * begin's own output), then the gradients as gqe_backward, each this range's share, in the
 * shapes of the weights this handle was given: dW_q [(g1-g0)*E*d_h, dim], dW_k, dW_v
 * [(g1-g0)*d_h, dim], dW_shared (the range holding group 0, with W_shared), dW_o [dim, D_o of
 * this range's Z], dW_r [N, dim] (zero outside the range's experts) and dx [B*T, dim]; the
 * layer's gradients are the sums of the shares (dW_o's slot columns are a share of the
 * slot's; every other block belongs to one range).
 *
 * finish must follow a successful begin on the same handle with the same arguments, with no
 * gqe_forward or gqe_decode between them (GQE_ERR_INVALID_ARG otherwise). Both enqueue on
 * `stream`, allocate nothing and do not synchronise. Errors as gqe_backward.
 */
gqe_status gqe_backward_begin(gqe_handle h, const void* x, int B, int T, const void* W_r,
                              const void* W_q, const void* W_k, const void* W_v,
                              const void* W_shared, const void* W_o, int N, int G, int k,
                              int d_h, int variant, int causal, const void* dy, float* slot_dot,
                              void* stream);
gqe_status gqe_backward_finish(gqe_handle h, const void* x, int B, int T, const void* W_r,
                               const void* W_q, const void* W_k, const void* W_v,
                               const void* W_shared, const void* W_o, int N, int G, int k,
                               int d_h, int variant, int causal, const void* dy, float aux_grad,
                               const float* slot_dot, float* dx, float* dW_r, float* dW_q,
                               float* dW_k, float* dW_v, float* dW_shared, float* dW_o,
                               void* stream);

/* gqe_backward_launches — kernels of this library the last gqe_backward (or begin and finish)
 * launched (the cuBLAS GEMMs are not counted). */
int gqe_backward_launches(gqe_handle h);

/*
 * gqe_get_routing — copy the routing of the last gqe_forward on this handle.
 *   sel        [M, G, k] int32   selected expert index j within the group, ascending.
 *   gates      [M, G, k] float   p renormalised within the group (sums to 1 per group).
 *   counts     [N] int32         tokens routed to each expert.
 *   mean_prob  [N] float         mean over tokens of the router softmax p.
 * Any pointer may be NULL (that output is skipped). Device pointers; enqueued on stream.
 */
gqe_status gqe_get_routing(gqe_handle h, int32_t* sel, float* gates, int32_t* counts,
                           float* mean_prob, void* stream);

/*
 * gqe_get_tensor — copy an internal tensor of the last gqe_forward (see gqe_tensor for
 * shapes) into the caller's device buffer dst of `bytes` bytes. Returns
 * GQE_ERR_INVALID_ARG if `bytes` is smaller than the tensor.
 */
gqe_status gqe_get_tensor(gqe_handle h, int which, void* dst, size_t bytes, void* stream);

/*
 * gqe_check_device_status — synchronise `stream`, then read and clear the handle's device
 * status word. Returns GQE_ERR_TIMEOUT if a kernel's bounded wait gave up since the last
 * check (its output is then invalid), GQE_ERR_INVALID_ARG if a gqe_decode met a position
 * outside its cache, GQE_ERR_CUDA if the stream reports an error or the routed projection
 * found its routing cursors out of range (a state no sequence of calls should reach: the
 * bucket reads were clamped and the output is invalid), else GQE_OK.
 */
gqe_status gqe_check_device_status(gqe_handle h, void* stream);

/*
 * gqe_set_group_range — make the handle compute only groups g0 .. g1-1 of the layer, for
 * group-parallel execution over several GPUs (one rank per range): routing is per group
 * (README, Algorithm Overview), so the ranges split the layer with no exchange except the
 * sum of their outputs.
 *
 * After this call gqe_forward still takes the WHOLE router W_r [N, dim] (every rank routes
 * every group, so the slot weights and the aux loss are the whole layer's, bit-identical on
 * every rank), but only the range's rows of the other weights:
 *   W_q       [(g1-g0)*E*d_h, dim]  rows of experts g0*E .. g1*E-1;
 *   W_k, W_v  [(g1-g0)*d_h, dim]    rows of heads g0 .. g1-1;
 *   W_shared  the shared head, on the range with g0 == 0 only (NULL elsewhere;
 *             GQE_ERR_INVALID_ARG otherwise);
 *   W_o       [dim, D_o'] the columns of the range's blocks of Z, in Z's order: its routed
 *             streams, the slot (variant gqe), the shared block (g0 == 0): D_o' =
 *             ((g1-g0)*k + [gqe] + [shared here]) * d_h.
 * `out` then receives this range's share of y; the layer's y is the sum over ranges (one
 * all-reduce or reduce-scatter over the ranks). K, V, the query streams and Z of
 * gqe_get_tensor hold the range's heads only. bf16 handles whose routing runs in the dense
 * projection (N a power of two up to 32) only, else GQE_ERR_UNSUPPORTED. gqe_decode takes
 * the range's caches and gives its share of y; the one-call gqe_backward returns
 * GQE_ERR_UNSUPPORTED unless the range is the whole layer (gqe_set_group_range(h, 0, G)
 * restores it): a range trains with gqe_backward_begin / gqe_backward_finish.
 * GQE_ERR_INVALID_ARG unless 0 <= g0 < g1 <= G.
 */
gqe_status gqe_set_group_range(gqe_handle h, int g0, int g1);

/* gqe_set_spin_limit — iteration cap of the device-side waits (0 = default). For tests
 * of the timeout path: a tiny limit makes the waits give up and report GQE_ERR_TIMEOUT. */
gqe_status gqe_set_spin_limit(gqe_handle h, int64_t limit);

/*
 * gqe_set_stage_events — for measurement: record caller-created CUDA events (cudaEvent_t
 * passed as void*) on the forward's stream around its stages. count = 0 turns recording
 * off; otherwise count must be GQE_NUM_STAGES + 1: events[i] is recorded just before stage
 * i and events[GQE_NUM_STAGES] after the last. The events must outlive the forwards that
 * record them. Stage names: gqe_stage_name.
 */
#define GQE_NUM_STAGES 6
gqe_status gqe_set_stage_events(gqe_handle h, void* const* events, int count);

/* gqe_stage_name — "dense_proj", "route", "qproj", "attention", "combine", "oproj" for
 * i = 0..5; NULL otherwise. */
const char* gqe_stage_name(int i);

/*
 * gqe_route_static — the router's selection and load statistics from precomputed router
 * logits, allocating nothing. The paper has no counterpart: this entry point exists for
 * callers that cannot call cudaMalloc (their device memory belongs to another allocator
 * or a fixed budget, they are plug-in code handed only input and output buffers, or they
 * cannot accept cudaMalloc's device-wide synchronisation), and so cannot create a handle.
 *
 *   logits     [M, N] float (device)  router logits x W_r^T.
 *   sel        [M, G, k] int32        selected expert index j in its group, ascending
 *                                     (top-k of the fp32 logits, lower index wins ties).
 *   gates      [M, G, k] float        softmax probability renormalised within the group.
 *   counts     [N] int32              tokens routed to each expert.
 *   mean_prob  [N] float              mean over tokens of the per-group softmax p.
 *   aux_loss   device float* or NULL  the Switch load-balancing loss (as gqe_forward).
 *
 * Scratch lives in one file-scope device array of 2.5 MiB (+512 B), held by every GPU that
 * loads the library until the process exits. Limits: M <= 131072 and M*G*k <= 262144;
 * larger calls return GQE_ERR_WORKSPACE and launch nothing. N <= 64, k <= 8
 * (GQE_ERR_UNSUPPORTED otherwise). The first call on each device looks up the array's
 * device address (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture. All calls share the one array: calls whose kernels overlap
 * on the GPU (different streams, or different threads without ordering) race and may
 * return wrong results; order them on one stream. Every scratch element a call reads is
 * written earlier in the same call, so nothing needs clearing between calls.
 */
gqe_status gqe_route_static(const float* logits, int M, int N, int G, int k, int32_t* sel,
                            float* gates, int32_t* counts, float* mean_prob, float* aux_loss,
                            void* stream);

/*
 * gqe_exp2_fma — diagnostic: out[i] = 2^in[i] computed the way the attention softmax
 * computes part of its exponentials on the FMA pipe (range reduction to [-1/2, 1/2], a
 * degree-2 polynomial, exponent-field scaling; inputs below -125 give 2^-125). Maximum
 * relative error 1.9e-3 for in[i] in [-125, 9]. in, out: n floats on the device.
 */
gqe_status gqe_exp2_fma(const float* in, float* out, int n, void* stream);

/*
 * gqe_selftest_timeout — diagnostic of the failure-detection path (failure made on purpose,
 * without any GPU fault): launches one warp that waits, with the bounded mbarrier wait the
 * pipeline kernels use and an iteration cap of `spin` (>= 1), on a barrier phase that nothing
 * completes. When the cap runs out the warp writes the timeout code into h's device status
 * word, as a pipeline kernel that gave up would, and returns. The next
 * gqe_check_device_status(h) reports GQE_ERR_TIMEOUT and clears the word; the handle and
 * the CUDA context stay usable. Stream-ordered; GQE_ERR_INVALID_ARG for a null handle or
 * spin < 1.
 */
gqe_status gqe_selftest_timeout(gqe_handle h, int64_t spin, void* stream);

/* gqe_destroy — free the handle and its workspace (synchronises the device first). */
void gqe_destroy(gqe_handle h);

/* gqe_status_str — static text for a status code. */
const char* gqe_status_str(int status);

/* gqe_workspace_bytes — device bytes gqe_create would allocate for this shape, or -1. */
int64_t gqe_workspace_bytes(int dim, int N, int G, int k, int d_h, gqe_dtype dtype,
                            int64_t max_tokens);

/* gqe_kernel_launches — kernels the last gqe_forward or gqe_decode on this handle launched
 * (-1 for a null handle). */
int gqe_kernel_launches(gqe_handle h);

#ifdef __cplusplus
}
#endif
#endif /* GQE_H */
