/*
 * expert_decode.h -- C ABI of the B200 (sm_100a) routed MoE FFN with an
 * expert-parallel band decomposition.
 *
 * The operation.  Every rank runs one copy of the router on the same rows, so
 * all ranks agree on the picked experts; the experts are split into contiguous bands, one band per rank, and
 * each band's SwiGLU experts contribute an [H] partial that is summed in rank
 * order (fak note "GLM-5.2 multi-GPU: expert-parallel sharding + the
 * resident-fit benchmark", section "What landed": ExpertParallelPlan, one
 * AllReduceSum of the per-rank partials; TensorFold issue #214 "GLM-5.3-Flash
 * on CUDA: attention on one GPU, routed experts on the Sparks", "Per MoE
 * layer": rows, top-k ids and weights in, partials out, summed in rank
 * order).  On one GPU the bands are a logical partition only.
 *
 * Conventions shared by every entry point:
 *  - Ownership.  The caller allocates and owns every buffer, including the
 *    workspace; the library allocates no device memory and frees nothing.
 *  - Layout.  Device arrays are dense, row-major, and their base addresses are
 *    16-byte aligned (the workspace 256-byte aligned).  bf16 is IEEE
 *    bfloat16 (the upper 16 bits of a binary32).
 *  - Streams.  `stream` is a cudaStream_t (NULL = the legacy default stream).
 *    Calls are asynchronous on that stream and never synchronise the host,
 *    except ep_check_status().
 *  - Errors.  Arguments are validated on the host before anything is
 *    launched; on any error status nothing is launched and no output is
 *    written.  ep_last_error() gives the reason (per host thread).  Errors
 *    found on the device (an expert id outside [0, E)) never trap and never
 *    read out of bounds: the pick is skipped, a sticky device status word is
 *    set, and ep_check_status() reports it.
 *  - Thread safety.  Every function may be called from several host threads.
 */
#ifndef EXPERT_DECODE_H
#define EXPERT_DECODE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    EP_OK = 0,
    EP_EINVAL = 1,    /* bad size, null or misaligned pointer, bad plan layout */
    EP_EDIM = 2,      /* plan does not match the expert count (plan.Dim != NumExperts) */
    EP_EBADID = 3,    /* device side: an expert id outside [0, E) was skipped */
    EP_ENOMEM = 4,    /* the workspace is smaller than moe_ffn_workspace_size() */
    EP_ECUDA = 5,     /* a CUDA runtime call failed; ep_last_error() has its text */
    EP_ETIMEOUT = 6   /* device side: a bounded wait ran out */
} ep_status;

typedef enum { EP_BF16 = 0, EP_F32 = 1 } ep_dtype;

#define EP_MAX_BANDS 64

/*
 * ExpertParallelPlan(numExperts, ranks): contiguous bands over [0, E), band r
 * = [band_start[r], band_start[r+1]) (fak note "GLM-5.2 multi-GPU", "What
 * landed").  Band sizes follow the shard rule of TensorFold issue #310
 * ("GLM-5.3-Flash on CUDA over three ranks (--tp 3)", MiaAI-Lab's proposal,
 * shares.py): whole experts, as even as they go, the first E % bands bands
 * taking one more (largest remainder; of equal remainders the lower rank wins).
 */
typedef struct {
    int32_t num_experts;
    int32_t bands;
    int32_t band_start[EP_MAX_BANDS + 1];
} ep_plan_t;

/*
 * ep_plan -- build the plan on the host.  Refused with EP_EINVAL (and *out
 * untouched) when num_experts < 1, bands < 1, bands > num_experts (the fak
 * note's fail-closed gate: "ranks > experts") or bands > EP_MAX_BANDS.
 */
ep_status ep_plan(int32_t num_experts, int32_t bands, ep_plan_t *out);

/*
 * moe_route -- the router, one copy of which every rank runs on the same rows
 * so that all ranks agree on the picks (fak note "GLM-5.2 multi-GPU", "What
 * landed").
 *   l[t,e] = sum_h x[t,h] * W_router[e,h] + bias[e]
 *   p = softmax(l); S = the top_k experts by logit, ties to the lower id;
 *   weights[t,j] = p[S_j] / sum_{e in S} p[e]
 * ids[t,:] are written in descending weight order (equal weights: ascending
 * id).  The pick is decided on compensated fp32 logits (Dot2, Ogita, Rump and
 * Oishi 2005): every product is exact in fp32 and the running sum carries its
 * own rounding error, so a logit is within about 1e-9 (relative to
 * sum_h |x_h W_h|) of its exact value.  Up to 32 tokens every logit is formed
 * that way; above, fp32 logits with a proven error bound come first and every
 * expert that could still reach the top_k under that bound is recomputed by
 * Dot2 before the pick.  The selection and its order therefore equal those of
 * exact arithmetic, except between logits closer than the Dot2 bound; the
 * weights carry that error plus one fp32 rounding.
 *
 *   x         device, [T, H], bf16 (EP_BF16) or fp32 (EP_F32)
 *   w_router  device, [E, H] bf16, one row per expert
 *   bias      device, [E] fp32, or NULL for none (added to the logits)
 *   ids       device, [T, top_k] int32 (output)
 *   weights   device, [T, top_k] fp32 (output)
 * Limits: 0 <= T <= 65536 (T = 0 is a no-op), 8 <= H <= 16384 with H % 8 ==
 * 0, 1 <= E <= 1024, 1 <= top_k <= min(E, 16).
 */
ep_status moe_route(const void *x, ep_dtype x_dtype, int64_t T, int64_t H,
                    const void *w_router, const float *bias, int64_t E, int32_t top_k,
                    int32_t *ids, float *weights, void *stream);

/*
 * moe_route_logits -- for inspection: the fp32 logits (with the bias) that
 * moe_route forms above 32 tokens before it refines its candidates, and the
 * bound of each one's error, |logits[t,e] - exact l[t,e]| <= bounds[t,e],
 * on which the selection of those candidates relies.  The router chosen by
 * ep_set_router runs (for any T >= 1); nothing is picked.
 *   logits, bounds  device, [T, E] fp32 (outputs)
 * Other arguments, limits and errors as moe_route.
 */
ep_status moe_route_logits(const void *x, ep_dtype x_dtype, int64_t T, int64_t H,
                           const void *w_router, const float *bias, int64_t E, float *logits,
                           float *bounds, void *stream);

/*
 * moe_route_sigmoid -- the GLM router variant (TensorFold #593, a
 * contributor's comment "What exists now", glm_route.cu), which the page
 * describes only by its parts: a sigmoid score, a bias that takes part in
 * the top-k choice, and weights taken from the unbiased scores.  Read as:
 *   l_e = sum_h x[t,h] W_router[e,h]       (no bias)
 *   s_e = 1 / (1 + exp(-l_e))              the score
 *   S   = top_k experts by s_e + bias[e]   (the bias moves the selection only),
 *         ties to the lower id
 *   weights[t,j] = scale * s_{S_j}, or with normalize = 1
 *   weights[t,j] = scale * s_{S_j} / sum over S of s
 * ids written by descending s + bias.  Arguments, layouts, limits and errors
 * as moe_route, plus normalize (0 or 1) and scale (finite, > 0; else
 * EP_EINVAL).  The logits are the compensated fp32 (Dot2) sums of moe_route,
 * with the same candidate refinement above 32 tokens; the scores and keys
 * are formed from them in fp64.
 */
ep_status moe_route_sigmoid(const void *x, ep_dtype x_dtype, int64_t T, int64_t H,
                            const void *w_router, const float *bias, int64_t E, int32_t top_k,
                            int32_t normalize, float scale, int32_t *ids, float *weights,
                            void *stream);

/*
 * moe_ffn_workspace_size -- bytes of device workspace moe_ffn_forward needs
 * for these sizes (0 when T = 0).  The workspace holds the token grouping,
 * the grouped activations, the SwiGLU activations h (fp32, or bf16 hi/lo rows
 * for the tensor-core down projection of T <= 8) and the per-pick partial
 * outputs; its contents on entry do not matter.
 */
size_t moe_ffn_workspace_size(int64_t T, int64_t H, int64_t E, int32_t top_k, int64_t I,
                              int64_t I_s);

/*
 * moe_ffn_workspace_layout -- where moe_ffn_forward keeps, inside its
 * workspace, the two results that its last step (the fold) reads, so that a
 * caller can check that step on its own.  After a moe_ffn_forward call with
 * these sizes that ran the grouped tensor-core path (T > 8) or the
 * tensor-core streaming kernels (2 <= T <= 8 with bf16 x):
 *   contrib  [T * top_k, H] fp32 at byte offset contrib_offset: row
 *            t * top_k + j holds weights[t,j] * f_e(x[t]) of pick (t, j), as
 *            rounded to fp32 (rows of skipped picks are not written);
 *   shared   [T, H] fp32 at byte offset shared_offset: f_shared(x[t])
 *            (written only when I_s > 0);
 * and y[t] is the left fold of t's valid contrib rows in ascending (expert
 * id, j), then + shared[t].  The CUDA-core streaming kernels (T = 1, or fp32
 * x) fold on chip and write neither.  After a call on the grouped path
 * (T > 8) the workspace also holds the grouping of the picks by expert:
 *   group_offset  [E + 2] int32 at group_offset_offset: the picks of expert
 *            e are rows [group_offset[e], group_offset[e+1]) of the grouped
 *            order; group_offset[E] = the number of valid picks,
 *            group_offset[E+1] = T * top_k;
 *   perm     [T * top_k] int32 at perm_offset: row r of the grouped order is
 *            pick perm[r] = t * top_k + j; inside an expert the picks keep
 *            their (t, j) order (a stable sort by expert id).
 * bytes = moe_ffn_workspace_size.  The sizes are checked as moe_ffn_forward
 * checks them (EP_EINVAL), and T = 0 gives an all-zero layout.
 */
typedef struct {
    size_t bytes;
    size_t contrib_offset;
    size_t shared_offset;
    size_t group_offset_offset;
    size_t perm_offset;
} ep_workspace_layout_t;
ep_status moe_ffn_workspace_layout(int64_t T, int64_t H, int64_t E, int32_t top_k, int64_t I,
                                   int64_t I_s, ep_workspace_layout_t *out);

/*
 * moe_ffn_forward -- the routed MoE FFN with the shared expert.
 * For every token t and pick j (e = ids[t,j], w = weights[t,j]):
 *   f_e(x) = W_down[e] (silu(W_gate[e] x) * (W_up[e] x)),  silu(g) = g/(1+e^-g)
 *   (expertSwiGLU, fak note "GLM-5.2 multi-GPU", "What is not yet" update)
 *   y[t] = fold over the picks in ascending (expert id, j) of w * f_e(x[t]),
 *          then + f_shared(x[t]) when I_s > 0.
 * The fold runs band by band in rank order and hands its running sum from
 * one band to the next, so the order of the additions is the same for every
 * plan (TensorFold #310, maintainer's reply: one sum order that does not
 * depend on how the slices are placed on ranks): y is bit-identical for
 * every plan and from run to run.
 *
 *   x        device, [T, H], bf16 or fp32
 *   ids      device, [T, top_k] int32 expert ids (any order, repeats allowed)
 *   weights  device, [T, top_k] fp32 routing weights
 *   w_gate, w_up  device, [E, I, H] bf16 (row i of expert e = one unit of I)
 *   w_down   device, [E, H, I] bf16 (row r of expert e = one output feature)
 *   ws_gate, ws_up  device, [I_s, H] bf16; ws_down device, [H, I_s] bf16;
 *            all three NULL when I_s = 0 (no shared expert)
 *   plan     host, must satisfy plan->num_experts == E (else EP_EDIM) and be
 *            a valid contiguous partition of [0, E) (else EP_EINVAL)
 *   y        device, [T, H] fp32 (output)
 *   workspace device, >= moe_ffn_workspace_size(T, H, E, top_k, I, I_s) bytes
 *            (else EP_ENOMEM), 256-byte aligned
 * Limits: 0 <= T <= 65536, T * top_k <= 2^20; 8 <= H <= 16384; 1 <= E <= 1024;
 * 1 <= top_k <= min(E, 16); 8 <= I, I_s <= 16384 (I_s may be 0); H, I and
 * I_s multiples of 8.
 * Precision: bf16 products, fp32 accumulation, fp32 routing weight applied
 * to the down projection's fp32 result.  The SwiGLU activations h between the
 * two projections are kept as follows:
 *   - T = 1, or fp32 x, up to 8 rows: fp32 (CUDA-core streaming kernels);
 *   - 2 <= T <= 8 with bf16 x: as the two bf16 parts hi = bf16(h) and
 *     lo = bf16(h - hi), about 16 significant bits (tensor-core streaming
 *     kernels);
 *   - T > 8: rounded to bf16 once (grouped tensor-core GEMMs).
 * x in fp32 is rounded to bf16 on the tensor-core paths.
 */
ep_status moe_ffn_forward(const void *x, ep_dtype x_dtype, int64_t T, int64_t H,
                          const int32_t *ids, const float *weights, int32_t top_k,
                          const void *w_gate, const void *w_up, const void *w_down,
                          int64_t E, int64_t I,
                          const void *ws_gate, const void *ws_up, const void *ws_down,
                          int64_t I_s, const ep_plan_t *plan, float *y,
                          void *workspace, size_t workspace_bytes, void *stream);

/*
 * moe_ffn_forward_noalloc -- moe_ffn_forward without a caller's workspace.
 * The method has no counterpart for this: it is a library convenience.
 * Some callers cannot hand over a workspace: a host runtime that has given
 * all device memory to its own pool, or a latency-bound loop in which an
 * allocation (which may synchronise the device, or fail once memory is
 * committed) is not allowed.  This entry point allocates nothing and calls
 * no allocating routine; instead it uses a scratch area of
 * EP_STATIC_SCRATCH_BYTES that is part of the library's own device memory.
 * Arguments, results, limits and precision are those of moe_ffn_forward,
 * less `workspace` and `workspace_bytes`.
 *   Sizes whose moe_ffn_workspace_size exceeds EP_STATIC_SCRATCH_BYTES
 *   (4 MiB: every T <= 16 at H = 4096, E = 128, top_k = 8, I = I_s = 1536)
 *   return EP_ENOMEM before anything is launched.
 *   The first call on each device looks the scratch's address up (with that
 *   device current) and may make the CUDA runtime load the library's kernels
 *   onto the device; make that first call before any stream capture begins.
 *   Nothing in the scratch needs to start at zero.
 *   There is one scratch per device: calls that can be in flight at the
 *   same time on one device (on different streams, or from different host
 *   threads without ordering) race on it and give wrong results.  Calls
 *   issued in order on one stream are safe.
 */
#define EP_STATIC_SCRATCH_BYTES (4u << 20)
ep_status moe_ffn_forward_noalloc(const void *x, ep_dtype x_dtype, int64_t T, int64_t H,
                                  const int32_t *ids, const float *weights, int32_t top_k,
                                  const void *w_gate, const void *w_up, const void *w_down,
                                  int64_t E, int64_t I,
                                  const void *ws_gate, const void *ws_up, const void *ws_down,
                                  int64_t I_s, const ep_plan_t *plan, float *y, void *stream);

/*
 * NVFP4 expert weights (TensorFold #593, "Checkpoint formats on that
 * family": NVIDIA's NVFP4 checkpoint used as stored, 4-bit weights against
 * 16-bit activations).  The page names the format only; this library takes
 * NVIDIA's public definition: FP4 E2M1 elements (magnitudes 0, 0.5, 1, 1.5,
 * 2, 3, 4, 6), one FP8 E4M3 block scale per 16 consecutive elements of a row
 * along the reduction dimension, one fp32 scale per tensor; a weight is
 * tensor_scale x block scale x element.
 *   codes   device, [mats][rows][cols / 2] bytes, 16-byte aligned: element
 *           2i of a row in the low nibble of byte i, 2i + 1 in the high one
 *   scales  device, [mats][rows][cols / 16] bytes (E4M3), 4-byte aligned
 * mats = E for the routed experts, 1 for the shared expert.
 */
typedef struct {
    const void *codes;
    const void *scales;
    float tensor_scale;
} ep_nvfp4_t;

/*
 * moe_ffn_nvfp4_workspace_size -- device workspace moe_ffn_forward_nvfp4
 * needs (0 when T = 0).
 *
 * moe_ffn_forward_nvfp4 -- moe_ffn_forward for decode batches (1 <= T <= 8)
 * with every expert matrix (routed and shared) in NVFP4: W_gate, W_up
 * [E][I][H], W_down [E][H][I]; Ws_gate, Ws_up [I_s][H], Ws_down [H][I_s].
 * Same operation, same fold order (ascending (expert id, j), then the
 * shared expert), bit-identical for every plan and from run to run.  The
 * weights stream as stored (4.5 bits each) and are dequantised on chip to
 * fp16 (exact); the products run on the tensor cores with fp16 operands and
 * fp32 accumulation: x is rounded to fp16 (exact for bf16 values of
 * magnitude 2^-14 .. 65504) and h passes between the projections as an fp16
 * hi/lo pair (about 22 significant bits).  The tensor scale multiplies the
 * fp32 accumulator.  x must be bf16 (EP_EINVAL otherwise).
 * Limits: 1 <= T <= 8 (0 is a no-op); H, I and I_s (when not 0) multiples of
 * 64 in [64, 16384]; 1 <= E <= 1024; 1 <= top_k <= min(E, 16).  Errors and
 * the other arguments as moe_ffn_forward.
 */
size_t moe_ffn_nvfp4_workspace_size(int64_t T, int64_t H, int64_t E, int32_t top_k, int64_t I,
                                    int64_t I_s);
ep_status moe_ffn_forward_nvfp4(const void *x, int64_t T, int64_t H, const int32_t *ids,
                                const float *weights, int32_t top_k, const ep_nvfp4_t *w_gate,
                                const ep_nvfp4_t *w_up, const ep_nvfp4_t *w_down, int64_t E,
                                int64_t I, const ep_nvfp4_t *ws_gate, const ep_nvfp4_t *ws_up,
                                const ep_nvfp4_t *ws_down, int64_t I_s, const ep_plan_t *plan,
                                float *y, void *workspace, size_t workspace_bytes, void *stream);

/*
 * EP_ID_NONE -- an empty pick slot.  A pick whose id is EP_ID_NONE is skipped
 * by every call that takes ids and is not reported as a bad id (any other id
 * outside [0, E) is skipped and reported).
 */
#define EP_ID_NONE ((int32_t)0x80000000)

/*
 * The expert-parallel form across ranks (fak note "GLM-5.2 multi-GPU", "What
 * landed": contiguous bands of experts, every rank the partial of the picks
 * in its band, the partials summed in rank order; TensorFold #310: one fixed
 * order of that sum).
 *
 * moe_ffn_partial_workspace_size -- bytes of device workspace moe_ffn_partial
 * needs with E_band experts in the band (0 for an empty input).
 *
 * moe_ffn_partial -- rank `rank`'s partial for every token:
 *   partial[t] = fold over t's picks with expert ids in band `rank` of the
 *                plan, in ascending (expert id, slot), starting from the first,
 *                of weights[t,j] * f_e(x[t]);  0 when t has no pick in the band.
 *   No shared expert (it enters after the rank-order sum, in moe_ep_combine).
 *   The weights are band-resident: w_gate, w_up [E_band, I, H], w_down
 *   [E_band, H, I] hold the band's experts only, expert e at index
 *   e - plan->band_start[rank].  ids and weights as moe_ffn_forward, with the
 *   global expert ids of the plan (ids of other bands are simply not this
 *   rank's; ids outside [0, plan->num_experts) are skipped and reported).
 *   partial device [T, H] fp32; workspace 256-byte aligned, at least
 *   moe_ffn_partial_workspace_size(T, H, E_band, top_k, I) bytes.  Limits
 *   and errors as moe_ffn_forward; rank outside [0, plan->bands) -> EP_EINVAL.
 *
 * moe_ep_combine -- y[t] = the partials of the bands that hold at least one of
 *   t's valid picks, left-folded in rank order, + shared[t] (shared device
 *   [T, H] fp32 or NULL).  A token without a valid pick gets shared[t] (or 0).
 *   partials device [plan->bands][T][H] fp32 (rank r's partial at r); ids
 *   device [T, top_k] int32; y device [T, H] fp32.  The result is the fp64
 *   oracle's band form (expertParallelPartials + rank-order sum), which for
 *   more than one band may differ in the last bits from moe_ffn_forward's one
 *   fold with the carry passed along.
 */
size_t moe_ffn_partial_workspace_size(int64_t T, int64_t H, int64_t E_band, int32_t top_k,
                                      int64_t I);
ep_status moe_ffn_partial(const void *x, ep_dtype x_dtype, int64_t T, int64_t H,
                          const int32_t *ids, const float *weights, int32_t top_k,
                          const void *w_gate, const void *w_up, const void *w_down, int64_t I,
                          const ep_plan_t *plan, int32_t rank, float *partial, void *workspace,
                          size_t workspace_bytes, void *stream);
ep_status moe_ep_combine(const float *partials, int64_t T, int64_t H, const int32_t *ids,
                         int32_t top_k, const ep_plan_t *plan, const float *shared, float *y,
                         void *stream);

/*
 * Which moe_ffn_forward path runs.  EP_DISPATCH_AUTO (the default) takes the
 * weight-streaming path for T <= 8 when its on-chip buffers fit, else the
 * tensor-core path; inside the streaming path, the tensor-core kernels from
 * 2 tokens with bf16 x, the CUDA-core kernels otherwise.  Forcing a path that does not fit the sizes makes
 * moe_ffn_forward return EP_EINVAL.  Process-wide; meant for tests and tuning.
 */
typedef enum {
    EP_DISPATCH_AUTO = 0,
    EP_DISPATCH_STREAMING = 1,      /* streaming path, kernels chosen as in AUTO */
    EP_DISPATCH_TENSOR = 2,
    /* streaming path, gate/up and down on the tensor cores (bf16 x), then the
       fold of the picks' contributions (three launches) */
    EP_DISPATCH_STREAMING_TC = 3,
    /* streaming path, gate/up on the CUDA cores and down with the fold (two
       launches) */
    EP_DISPATCH_STREAMING_SIMT = 4
} ep_dispatch;
ep_status ep_set_dispatch(ep_dispatch mode);

/*
 * Which router moe_route and moe_route_sigmoid run for more than 32 tokens
 * (up to 32 tokens every logit is a Dot2 sum on the CUDA cores).
 * EP_ROUTER_AUTO (the default) takes the tensor-core router where it fits
 * (bf16 x, E <= 256, H >= 128), else the CUDA-core one.  Both form fp32
 * logits with an error bound and refine every expert that could reach the
 * top_k by Dot2, so they give the same ids and the same weights.  Forcing
 * EP_ROUTER_TENSOR where it does not fit makes those calls return EP_EINVAL.
 * Process-wide; meant for tests and tuning.
 */
typedef enum {
    EP_ROUTER_AUTO = 0,
    EP_ROUTER_TILED = 1,   /* register-tiled fp32 logits on the CUDA cores */
    EP_ROUTER_TENSOR = 2   /* fp32 logits on the tensor cores (tcgen05) */
} ep_router_mode;
ep_status ep_set_router(ep_router_mode mode);

/*
 * Launch mode.  Kernels are launched with programmatic dependent launch: a
 * kernel may start while the previous kernel on the stream is still running
 * and reads that kernel's outputs only after griddepcontrol.wait.  Setting
 * the environment variable EXPERT_DECODE_NO_PDL=1 before the first call of a
 * process launches every kernel without it (the value is read once).
 */

/*
 * ep_check_status -- synchronise `stream`, then return and clear the sticky
 * device status of the current device: EP_OK, EP_EBADID or EP_ETIMEOUT
 * (EP_ECUDA if the synchronisation itself failed).
 */
ep_status ep_check_status(void *stream);

/* Text of the last error on the calling host thread ("" if none). */
const char *ep_last_error(void);

/* Number of kernels the last successful call on this host thread launched. */
int32_t ep_last_launch_count(void);

/*
 * ep_profile_events -- per-kernel timing aid.  While `events` is not NULL,
 * every kernel that a later moe_route / moe_ffn_forward call on this host
 * thread launches is bracketed on the call's stream by
 * cudaEventRecord(events[2j]) and cudaEventRecord(events[2j+1]), j counting
 * the kernels of that one call (kernels past n_events / 2 are not bracketed;
 * on the tensor-core path the two kernels of the grouping plan share one
 * bracket, j = 0, so its brackets are plan, gather, gate/up, down, combine).
 * `events` are cudaEvent_t handles the caller created and owns; the array is
 * read at each call, so the caller may change its contents between calls.
 * Pass NULL (or n_events = 0) to stop.  EP_EINVAL for n_events < 0.
 */
ep_status ep_profile_events(void *const *events, int32_t n_events);

#ifdef __cplusplus
}
#endif

#endif /* EXPERT_DECODE_H */
