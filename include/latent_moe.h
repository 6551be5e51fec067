/*
 * latent_moe.h -- C ABI of the B200 (sm_100a) LatentMoE forward library.
 *
 * The library computes the forward pass of the LatentMoE feed-forward layer of
 * the K3 notes (sec-07, "SiTU-GLU 与 Stable LatentMoE", compute flow in five
 * steps; kda/layers/latent_moe.py in the K3 compare view 584f7e9..main):
 *
 *   z = W_down x                                   (latent compression, l = d/2)
 *   s = sigmoid(W_r x), T = TopK(s + b, k),
 *   p_i = s_i / max(sum_{j in T} s_j, 1e-9)        (K3 eq.13; b selects only)
 *   u = sum_{i in T} p_i E_i(z)                    (routed SiTU-GLU experts in l)
 *   s_sh = sum_j E^sh_j(x)                         (shared SiTU-GLU experts in d)
 *   y = s_sh + W_up RMSNorm(u)
 *   E(v) = W_o [beta1 tanh(W_g v / beta1) sigmoid(W_g v) * beta2 tanh(W_u v / beta2)]
 *
 * Conventions shared by every entry point:
 *   - Every tensor pointer is a DEVICE pointer owned by the caller, except
 *     where a function says "host".  The library never allocates, frees or
 *     keeps device memory; scratch lives in a caller-provided workspace.
 *   - Row-major, contiguous, 16-byte-aligned buffers.  Weights follow
 *     nn.Linear: [out, in], the reduction dimension contiguous.
 *   - Activations and weights have the dtype in lmoe_dims.dtype (bf16 or
 *     fp32); accumulation is always fp32.  expert_bias, rms_weight and probs
 *     are always fp32; ids and permutation arrays are int32.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *     default stream) unless stated.  Argument errors are returned before any
 *     launch; launch failures return LMOE_ECUDA.  Anomalies found on the device
 *     (a capped wait that ran out, a failed consistency check) are recorded in
 *     the workspace status word, read by lmoe_get_device_status.
 *   - Calls that share one workspace must not overlap on the device.
 *   - Requires an sm_100a device (B200).  Otherwise LMOE_EUNSUPPORTED.
 */
#ifndef LATENT_MOE_H
#define LATENT_MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LMOE_API __attribute__((visibility("default")))
#else
#define LMOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LMOE_OK = 0,
  LMOE_EINVAL = 1,       /* bad dims, null or misaligned pointer              */
  LMOE_EUNSUPPORTED = 2, /* not an sm_100a device, or a size out of range     */
  LMOE_EWORKSPACE = 3,   /* workspace too small                               */
  LMOE_ECUDA = 4,        /* a CUDA runtime/driver call or a launch failed     */
  LMOE_EDEVICE = 5,      /* the device status word holds a failed check       */
  LMOE_ETIMEOUT = 6      /* a capped device-side wait ran out                 */
} lmoe_status;

typedef enum { LMOE_F32 = 0, LMOE_BF16 = 1 } lmoe_dtype;

typedef void* lmoe_stream; /* cudaStream_t */

/* Layer sizes (the pages' LatentMoE(hidden_size, latent_size, n_routed, top_k,
 * n_shared, d_ff, beta1, beta2) with B*T flattened to n_tokens and separate
 * routed/shared hidden widths).  Limits: 1 <= top_k <= n_routed <= 4096;
 * d, latent, ff_routed, ff_shared multiples of 8 (ragged 64-wide K blocks
 * and output tiles are zero-filled / masked on the tensor-core path);
 * 0 <= n_shared <= 7; n_tokens * top_k < 2^31. */
typedef struct {
  int64_t n_tokens; /* N                                    */
  int32_t d;        /* model width                          */
  int32_t latent;   /* l (d/2 in the pages)                 */
  int32_t n_routed; /* R                                    */
  int32_t top_k;    /* k                                    */
  int32_t n_shared; /* S                                    */
  int32_t ff_routed;/* F, routed expert hidden width        */
  int32_t ff_shared;/* G, shared expert hidden width        */
  float beta1;      /* SiTU gate cap (pages: 4)             */
  float beta2;      /* SiTU up cap (pages: 25)              */
  float rms_eps;    /* RMSNorm epsilon (1e-6)               */
  int32_t dtype;    /* lmoe_dtype                           */
  int32_t router;   /* lmoe_router: which routing rule      */
} lmoe_dims;

/* Routing rules.  LMOE_ROUTER_K3 is the layer's (sec-07 K3 eq.13):
 * s = sigmoid(l), T = TopK(s + b, k), p = s_T / max(sum s_T, 1e-9).
 * LMOE_ROUTER_SOFTMAX_TOPK is the router that latent_moe.py had before it
 * (the lines the compare view removes from LatentMoE.forward): T = TopK(l, k)
 * on the raw logits, expert_bias unused, p = softmax over the k selected
 * logits.  Either way the slots are in descending key order, a tie going to
 * the lower expert index. */
typedef enum { LMOE_ROUTER_K3 = 0, LMOE_ROUTER_SOFTMAX_TOPK = 1 } lmoe_router;

/* Layer weights, device pointers in nn.Linear layout. */
typedef struct {
  const void* w_down;       /* [l, d]      W_down                               */
  const void* w_router;     /* [R, d]      W_r                                  */
  const void* w_up;         /* [d, l]      W_up                                 */
  const float* rms_weight;  /* [l] fp32    RMSNorm weight                       */
  const float* expert_bias; /* [R] fp32    selection bias b; NULL means b = 0   */
  const void* w_g;          /* [R, F, l]   routed gate projections              */
  const void* w_u;          /* [R, F, l]   routed up projections                */
  const void* w_o;          /* [R, l, F]   routed output projections            */
  const void* ws_g;         /* [S, G, d]   shared gate projections (S > 0)      */
  const void* ws_u;         /* [S, G, d]   shared up projections                */
  const void* ws_o;         /* [S, d, G]   shared output projections            */
} lmoe_weights;

/* Bytes of device workspace that every entry point below accepts for these
 * dims (one size serves all of them).  0 on invalid dims. */
LMOE_API size_t lmoe_workspace_size(const lmoe_dims* dims);

/* Router (sec-07 compute flow step 2, K3 eq.13; latent_moe.py LatentMoE._route):
 * l = W_r x (fp32 accumulation), s = sigmoid(l), T = TopK(s + b, k) with the
 * slots in descending s + b (a tie goes to the lower expert index),
 * p_i = s_i / max(sum_T s, 1e-9).  dims->router selects the rule (lmoe_router).
 *   x        [N, d]      input rows
 *   w_router [R, d]
 *   expert_bias [R] fp32 or NULL
 *   ids      [N, k] int32 out;  probs [N, k] fp32 out.
 * Workspace: lmoe_workspace_size(dims) bytes; the logits l are left in it (see
 * moe_router_losses). */
LMOE_API lmoe_status moe_route(const lmoe_dims* dims, const void* x, const void* w_router,
                      const float* expert_bias, int32_t* ids, float* probs, void* ws,
                      size_t ws_bytes, lmoe_stream stream);

/* Pair permutation (latent_moe.py LatentMoE._routed_u; sec-07 sparse dispatch,
 * step 1): the N*k (token, expert) pairs, flattened token-major, stably sorted
 * by expert id.  Bit-exact and deterministic.
 *   ids        [N, k] int32 in, each row k distinct ids in [0, R)
 *   counts     [R]    int32 out: pairs per expert (bincount)
 *   offsets    [R+1]  int32 out: exclusive prefix sum, offsets[R] = N*k
 *   perm_token [N*k]  int32 out: token of each sorted pair (expert-major,
 *                     tokens ascending inside an expert)
 *   inv_pair   [N, k] int32 out: sorted position of pair (t, slot)
 * An out-of-range id sets LMOE_EDEVICE in the status word; its pair is
 * dropped (counted nowhere, no sorted slot) and its inv_pair entry is -1. */
LMOE_API lmoe_status moe_dispatch(const lmoe_dims* dims, const int32_t* ids, int32_t* counts,
                         int32_t* offsets, int32_t* perm_token, int32_t* inv_pair, void* ws,
                         size_t ws_bytes, lmoe_stream stream);

/* Consistency check of a permutation (what moe_dispatch promises, verified on
 * the device; the pages' stable argsort + bincount + cumsum define it):
 * every id in [0, R); counts summing to N*k; offsets[0] = 0 and offsets[e+1] -
 * offsets[e] = counts[e]; inv_pair a bijection onto the N*k sorted slots
 * (every slot taken exactly once); perm_token[inv_pair[t, i]] = t; the slot of
 * (t, i) inside its expert's range; tokens ascending inside an expert.  A
 * violation sets LMOE_EDEVICE in the workspace status word (read it with
 * lmoe_get_device_status); nothing is written otherwise.  Workspace:
 * lmoe_workspace_size(dims) bytes. */
LMOE_API lmoe_status lmoe_check_dispatch(const lmoe_dims* dims, const int32_t* ids,
                                         const int32_t* counts, const int32_t* offsets,
                                         const int32_t* perm_token, const int32_t* inv_pair,
                                         void* ws, size_t ws_bytes, lmoe_stream stream);

/* Routed experts on the sorted pairs (sec-07 compute flow step 3 and the
 * sparse-dispatch subsection; latent_moe.py _routed_u, without padding to
 * the capacity C): for each expert e and sorted row r in
 * [offsets[e], offsets[e+1]):
 *   expert_out[r] = W_o,e [beta1 tanh(a/beta1) sigmoid(a) * beta2 tanh(c/beta2)],
 *   a = W_g,e z[perm_token[r]],  c = W_u,e z[perm_token[r]].
 *   z          [N, l]
 *   perm_token [N*k], offsets [R+1]   from moe_dispatch
 *   w_g, w_u   [R, F, l];  w_o [R, l, F]
 *   expert_out [N*k, l]   out, in sorted-pair order (not yet weighted by p). */
LMOE_API lmoe_status moe_expert_ffn(const lmoe_dims* dims, const void* z, const int32_t* perm_token,
                           const int32_t* offsets, const void* w_g, const void* w_u,
                           const void* w_o, void* expert_out, void* ws, size_t ws_bytes,
                           lmoe_stream stream);

/* Weighted combine + RMSNorm (latent_moe.py index_add and self.norm; sec-07
 * step 3 sum and step 5 RMSNorm): for each token t, in slot order,
 *   u_t = sum_i probs[t, i] * expert_out[inv_pair[t, i]]   (fp32, no atomics)
 *   u_normed_t = u_t / sqrt(mean(u_t^2) + eps) * rms_weight
 *   u_normed [N, l] out.
 * Slots whose inv_pair entry is negative (pairs the dispatch dropped) add
 * nothing to u_t. */
LMOE_API lmoe_status moe_combine(const lmoe_dims* dims, const void* expert_out, const int32_t* inv_pair,
                        const float* probs, const float* rms_weight, void* u_normed,
                        lmoe_stream stream);

/* Router balancing losses (latent_moe.py LatentMoE._balancing_losses; the
 * pages' test_moe_aux_loss_penalizes_collapse), before their coefficients:
 *   frac_e      = (pairs routed to e) / max(N*k, 1)
 *   prob_mean_e = mean_t sigmoid(l_te)
 *   aux         = R * sum_e frac_e * prob_mean_e
 *   z           = mean_t (logsumexp_e l_te)^2
 * The pages multiply them by aux_loss_coef and z_loss_coef.
 *   logits [N, ld] fp32, or NULL for the logits that the last moe_route or
 *          latent_moe_forward on this workspace left in it (ld is then ignored)
 *   ids    [N, k] int32: the routing whose histogram gives frac
 *   out    [2 + 2R] fp32 device memory out: aux, z, frac[R], prob_mean[R]
 * Deterministic (fixed-order fp32 sums, integer histograms).  Workspace:
 * lmoe_workspace_size(dims) bytes. */
LMOE_API lmoe_status moe_router_losses(const lmoe_dims* dims, const float* logits, int64_t ld,
                                       const int32_t* ids, float* out, void* ws, size_t ws_bytes,
                                       lmoe_stream stream);

/* The whole layer: y [N, d] = s_sh + W_up RMSNorm(u).  Optional outputs (NULL
 * to skip): ids_out [N, k], probs_out [N, k], counts_out [R].  All work is on
 * `stream`; no host synchronisation.  The router logits stay in the
 * workspace for moe_router_losses.  Results are bitwise repeatable for given
 * dims on a given GPU.  When whole output tiles would fill the SMs' last wave
 * below 90%, the x-pass and the final GEMM (bf16) split the K loop of some
 * tiles between CTA pairs (stream-K) and add the fp32 partials in a fixed
 * order; the environment variable LMOE_STREAM_K=0 turns that off, =1 uses it
 * whenever its scratch fits. */
LMOE_API lmoe_status latent_moe_forward(const lmoe_dims* dims, const lmoe_weights* weights, const void* x,
                               void* y, int32_t* ids_out, float* probs_out, int32_t* counts_out,
                               void* ws, size_t ws_bytes, lmoe_stream stream);

/* Gradients of the layer (fp32 device buffers, caller-owned, every one
 * fully overwritten; shapes as the weights). */
typedef struct {
  float* dx;          /* [N, d]                                          */
  float* dw_down;     /* [l, d]                                          */
  float* dw_router;   /* [R, d]                                          */
  float* dw_up;       /* [d, l]                                          */
  float* drms_weight; /* [l]                                             */
  float* dw_g;        /* [R, F, l]                                       */
  float* dw_u;        /* [R, F, l]                                       */
  float* dw_o;        /* [R, l, F]                                       */
  float* dws_g;       /* [S, G, d]   (unused when S = 0)                 */
  float* dws_u;       /* [S, G, d]                                       */
  float* dws_o;       /* [S, d, G]                                       */
} lmoe_grads;

/* Backward of the layer: the gradients of <dy, y> with respect to x and every
 * weight, y = latent_moe_forward(x) (the pages train the layer; its tests check
 * the gradients: unselected experts get exactly 0).  The routing ids are not
 * differentiable and expert_bias only selects, so it gets no gradient; W_r gets
 * its gradient through the routing weights p only.  The forward's internals
 * are recomputed in fp32 from x (routing with the same kernels as the forward),
 * so no forward state is needed; every sum runs in a fixed order
 * (deterministic).  dy [N, d] in the activation dtype.  Workspace:
 * lmoe_backward_workspace_size(dims) bytes, 256-byte aligned (its own layout,
 * not the forward's). */
LMOE_API size_t lmoe_backward_workspace_size(const lmoe_dims* dims);
LMOE_API lmoe_status latent_moe_backward(const lmoe_dims* dims, const lmoe_weights* weights,
                                         const void* x, const void* dy, const lmoe_grads* grads,
                                         void* ws, size_t ws_bytes, lmoe_stream stream);

/* The whole layer from HOST memory: copies x_host [N, d] (pinned or pageable)
 * to the device, runs latent_moe_forward, copies y back to y_host [N, d] and
 * waits for the stream.  Weights and workspace are device memory.  The
 * workspace must be lmoe_workspace_size_host(dims) bytes (it also holds the
 * device copies of x and y).
 * The tokens may be processed in up to 8 chunks (tokens are independent; y
 * equals one latent_moe_forward over all N to within the final GEMM's fp32
 * summation order, which may split K differently per chunk size, and is
 * bit-identical when one chunk is used): x chunks are copied
 * in on a library-owned stream, each chunk's forward runs on `stream` once its
 * x has landed, and its y is copied out on a second library-owned stream while
 * the next chunk computes.  The chunk count comes from a cost model of copy
 * time against forward time (one chunk when streaming the expert weights
 * dominates; the environment variable LMOE_HOST_CHUNKS=1..8 overrides it).
 * The copy streams and their events are created on the first
 * call on each device and kept until the process exits; the copies wait for
 * work queued on `stream` before the call, and the call returns after all of
 * it has finished.  Pinned host buffers are needed for the copies to overlap. */
LMOE_API size_t lmoe_workspace_size_host(const lmoe_dims* dims);
LMOE_API lmoe_status latent_moe_forward_host(const lmoe_dims* dims, const lmoe_weights* weights,
                                    const void* x_host, void* y_host, void* ws, size_t ws_bytes,
                                    lmoe_stream stream);

/* The launch plan latent_moe_forward takes for these dims (host only,
 * nothing is launched), as LMOE_PLAN_* bits in *flags:
 *   COMBINE_FUSED     the combine + RMSNorm runs in the final GEMM's epilogue;
 *   XPASS_WIDE        x-pass on 256 x 512 tiles (not taken by the current
 *                     rule: 256 x 256 tiles measured faster at every shape);
 *   GEMM1_PAIRS / GEMM2_PAIRS  routed GEMM1 / GEMM2 on CTA pairs (256-row tiles);
 *   GEMM1_WIDE        routed GEMM1 on 256 x 512 tiles;
 *   ROWS_IN_SCATTER   the dispatch's scatter writes the sorted copy of z
 *                     (at most 16 MiB and at least 4096 pairs; else a gather
 *                     kernel does);
 *   COUNTS_IN_XPASS   the x-pass's routing epilogue (bf16, R <= 32) also
 *                     counts each 32 tokens' pairs per expert and the
 *                     dispatch starts from those counts, with no histogram
 *                     kernel (each chunk of pairs the counting sort takes is
 *                     whole 32-token rows, always so for k = 1, 2, 4, 8, and
 *                     ceil(N / 32) * R <= 8192; the environment variable
 *                     LMOE_XPASS_COUNTS=0 turns it off).  The permutation is
 *                     the same either way.
 * The final GEMM's stream-K choice is made at launch and not reported here.
 * EINVAL on bad dims or flags == NULL. */
enum {
  LMOE_PLAN_COMBINE_FUSED = 1,
  LMOE_PLAN_XPASS_WIDE = 2,
  LMOE_PLAN_GEMM1_PAIRS = 4,
  LMOE_PLAN_GEMM2_PAIRS = 8,
  LMOE_PLAN_GEMM1_WIDE = 16,
  LMOE_PLAN_ROWS_IN_SCATTER = 32,
  LMOE_PLAN_COUNTS_IN_XPASS = 64
};
LMOE_API lmoe_status lmoe_forward_plan(const lmoe_dims* dims, int32_t* flags);

/* Byte offsets of the forward's intermediates inside the workspace, for
 * inspection after latent_moe_forward: offsets[0..6] = z [N,l], router logits
 * [N, ld] fp32, shared hidden units [N, S*G], RMSNorm(u) [N,l], routed expert
 * outputs [N*k, l], routed hidden units [N*k, F], sorted z rows [N*k, l]
 * (these two hold the final GEMM's stream-K scratch instead when it splits
 * K, see latent_moe_forward); offsets[7] = ld, the row stride (elements) of
 * the logits.  With n >= 11
 * also offsets[8..10] = the permutation the forward built: expert offsets
 * [R+1], perm_token [N*k] and inv_pair [N,k], all int32.  n < 8 is EINVAL. */
LMOE_API lmoe_status lmoe_workspace_layout(const lmoe_dims* dims, size_t* offsets, int32_t n);

/* moe_dispatch without a workspace: the same permutation, bit for bit, for
 * callers that cannot provide device scratch memory -- for example a plugin
 * host that gives a kernel only its tensors, a memory pool that is capped and
 * full, or a thread that must not enter the device allocator.  The pages have
 * no counterpart; it exists for such callers.
 *   The sort's scratch (per-block histograms, routed tile list, status word)
 *   is one fixed 1 MiB array in device memory, defined by the library; every
 *   GPU that loads the library holds it until the process exits.  The call
 *   allocates nothing.  Sizes whose scratch exceeds the array --
 *   4 * (64 + C * R rounded up to a multiple of 4 + 4 * (N*k/128 + R + 1))
 *   bytes > 1 MiB, C <= 128 the number of chunks the sort splits the pairs
 *   into -- return LMOE_EUNSUPPORTED with a message, before any launch.
 *   The first call on a device looks the array's address up (make it before
 *   any stream capture).  All calls share the array and it keeps the last
 *   call's contents, so calls that overlap on the GPU race: serialise them.
 *   Out-of-range ids are dropped as in moe_dispatch (inv_pair -1 for their
 *   pairs) but not reported: the status word is private to this call.
 * Arguments and outputs as in moe_dispatch. */
LMOE_API lmoe_status moe_dispatch_noalloc(const lmoe_dims* dims, const int32_t* ids,
                                          int32_t* counts, int32_t* offsets, int32_t* perm_token,
                                          int32_t* inv_pair, lmoe_stream stream);

/* Zeroes the workspace header (status word and scheduling counters) and the
 * synchronisation area that follows it (the final GEMM's per-tile row counts
 * for its fused combine, which every launch leaves zeroed).  Call once on a
 * new workspace before its first use, and again after a call reported
 * LMOE_ETIMEOUT (an aborted launch can leave counts behind). */
LMOE_API lmoe_status lmoe_workspace_init(void* ws, size_t ws_bytes, lmoe_stream stream);

/* Waits for `stream`, then reads and clears the workspace status word.
 * Returns LMOE_OK, LMOE_EDEVICE or LMOE_ETIMEOUT (or LMOE_ECUDA). */
LMOE_API lmoe_status lmoe_get_device_status(void* ws, lmoe_stream stream);

/* Launches one kernel that waits on a device flag nothing sets, with a cap of
 * about `cap_ms` milliseconds, then records LMOE_ETIMEOUT in the status word and
 * returns.  Exists to test the capped-wait path; the GPU stays usable. */
LMOE_API lmoe_status lmoe_selftest_capped_wait(void* ws, size_t ws_bytes, int32_t cap_ms,
                                      lmoe_stream stream);

/* Human-readable name of a status code. */
LMOE_API const char* lmoe_status_string(lmoe_status status);

/* Last error message of this thread (empty string if none). */
LMOE_API const char* lmoe_last_error(void);

/* Brackets every launch of the kernels named in `tags` (a comma-separated
 * list, "*" for all, NULL or "" to turn it off) with CUDA events, per thread.
 * Each event is recorded on a library-owned side stream forked from the
 * launching stream right before / after the launch (so it never sits between
 * two kernels and cuts their programmatic overlap); the public call joins
 * the side stream back into its own stream before it returns, so a stream
 * capture of the call stays closed.  Tags: "xpass", "route", "dispatch",
 * "gather", "expert_gemm1", "expert_gemm2", "combine", "final",
 * "router_losses". */
LMOE_API lmoe_status lmoe_profile_enable(const char* tags);
/* Waits for the recorded events of kernel `tag` (NULL: every tag); returns the
 * summed device time (ms) and the number of bracketed launches since the last
 * read of that tag, and clears them. */
LMOE_API lmoe_status lmoe_profile_read_tag(const char* tag, double* total_ms, int64_t* launches);
LMOE_API lmoe_status lmoe_profile_read(double* total_ms, int64_t* launches);
/* Like lmoe_profile_read_tag but keeps the event pairs: for launches captured
 * in a CUDA graph, whose events are recorded again on every replay. */
LMOE_API lmoe_status lmoe_profile_peek_tag(const char* tag, double* total_ms, int64_t* launches);

/* Number of kernel launches the library issued on this thread since the last
 * reset (instrumentation for benchmarks). */
LMOE_API uint64_t lmoe_launch_count(int32_t reset);

#ifdef __cplusplus
}
#endif

#endif /* LATENT_MOE_H */
