/*
 * moe.h -- C ABI of the B200 (sm_100a) Grok-1 mixture-of-experts feed-forward layer.
 *
 * The layer (as described in "Grok-1 Admin & Architecture Guide", section 3
 * "The Model", "Mixture of Experts (MoELayer + Router)" and "Quantized weights"):
 *
 *   1. routing logits L = x . router_w in fp32, softmax over the E experts;
 *   2. the top-2 experts of each token (ties go to the lower expert index);
 *   3. each chosen expert e computes  y_e = linear_1( gelu(linear(x)) * linear_v(x) )
 *      with 8-bit weights dequantised as  int8 value * per-output-channel bf16 scale;
 *   4. out = p[e0] * y_e0 + p[e1] * y_e1, where p is the softmax probability
 *      (the gates are not renormalised over the two picks).
 * FFN width: "llm-architectures-explained: Grok-1", table "Every architecture
 * field", row ffns.moe.d_expert (32768 at d_model 6144).
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers unless the name ends in _host; the
 *     caller owns all of them.  Every pointer must be 16-byte aligned and every
 *     tensor dense and row-major with the layout stated below.
 *   - bf16 tensors are passed as void* (IEEE bfloat16, 2 bytes per element).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls only enqueue work on it.  The host waits only in moe_sync_status,
 *     moe_get_kernel_times and moe_destroy, and in a forward call that has to
 *     grow the handle's workspace or that follows a call of the same handle on
 *     another stream (it then first synchronises that earlier stream).
 *   - Every call returns MOE_OK (0) or a negative MOE_E* code; no exception or
 *     abort crosses the ABI.  Arguments are checked on the host before any CUDA
 *     call, so an invalid call has no effect on the device.
 *   - A handle is bound to the CUDA device that is current at its first
 *     forward call.  Calls on one handle must not run concurrently from several
 *     host threads (the handle's workspace is shared).
 *
 * Layout of one layer's parameters (E experts, model width d, FFN width F):
 *   router_w  fp32 [d, E]      routing weight (x . router_w)
 *   w_lin     int8 [E, d, F]   linear   (x @ W orientation), s_lin bf16 [E, F]
 *   w_v       int8 [E, d, F]   linear_v,                     s_v   bf16 [E, F]
 *   w_1       int8 [E, F, d]   linear_1,                     s_1   bf16 [E, d]
 * Scales are per output channel:  W_deq[e, i, o] = w[e, i, o] * s[e, o].
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

/* ---- status codes ---------------------------------------------------------- */
#define MOE_OK            0
#define MOE_EINVAL       -1   /* invalid argument (null/misaligned pointer, bad size)      */
#define MOE_EUNSUPPORTED -2   /* valid request this library does not implement           */
#define MOE_ENOMEM       -3   /* device or host allocation failed                         */
#define MOE_ECUDA        -4   /* a CUDA runtime call or kernel launch failed               */
#define MOE_ETIMEOUT     -5   /* a bounded device-side wait ran out (see moe_sync_status)  */
#define MOE_ENODEV       -6   /* no CUDA device, or not an sm_100 device                   */
#define MOE_ERANGE       -7   /* a weight value the requested layout cannot hold (-128 in  */
                              /* MOE_LAYOUT_PACKED; see moe_pack_weight)                   */

/* Largest token count one call accepts. */
#define MOE_MAX_TOKENS   262144

/* Weight layouts (moe_set_weight_layout). */
#define MOE_LAYOUT_IN_OUT 0   /* w_lin, w_v [E, d, F]; w_1 [E, F, d]  (x @ W orientation, default) */
#define MOE_LAYOUT_PACKED 1   /* w_lin, w_v [E, F, d]; w_1 [E, d, F]  (input dim contiguous)      */

typedef struct moe_ctx *moe_handle;

/* Human-readable text for a status code.  Never NULL; the string is static. */
MOE_API const char *moe_strerror(int code);

/* Library version, major * 10000 + minor * 100 + patch. */
MOE_API int moe_version(void);

/*
 * Create a layer handle for model width d, FFN width ffn, E experts and k picks
 * per token ("Configuration objects" of the admin guide: emb_size, the FFN
 * width from widening_factor, num_experts, num_selected_experts).
 * Supported: E == 8, k == 2, d % 128 == 0, ffn % 128 == 0, 128 <= d, ffn <= 65536.
 * Returns MOE_EINVAL for non-positive sizes or k > E, MOE_EUNSUPPORTED for
 * other shapes.  Allocates host memory only.  Device memory (the workspace) is
 * taken with cudaMalloc on the first forward call and grows with the largest T
 * seen: a forward call that has to grow it first synchronises the stream of the
 * handle's previous call and frees the smaller buffers, so that call blocks the
 * host until the earlier work is done.  Forwards that fit the workspace allocate
 * nothing and do not block.  On success *out owns the handle; release it with
 * moe_destroy.
 */
MOE_API int moe_create(int d, int ffn, int E, int k, moe_handle *out);

/*
 * Release the handle and its device workspace.  Waits for the handle's last
 * enqueued work to finish first.  NULL is accepted and ignored.
 */
MOE_API int moe_destroy(moe_handle h);

/*
 * Add a fixed fp32 bias to every token's routing logits (after the fp32 dot
 * product, before the softmax).  bias: device fp32 [E], or NULL to remove it.
 * The pointer is kept, not copied: it must stay valid while forwards that use
 * it run.  This is a test hook (the skewed-routing workload); the model itself
 * has no router bias.
 */
MOE_API int moe_set_router_bias(moe_handle h, const float *bias);

/*
 * Padding mask of the MoE call: the grok-field-guide source-code map, fourth stop,
 * passes one to the layer (moe(rms_norm(h), padding_mask)).  mask: device uint8
 * [T] (one byte per token: nonzero = a real token, 0 = padding), or NULL for "every
 * token real".  A padding token is routed nowhere: moe_get_routing reports experts
 * -1 and gates 0 for it, the dispatch skips its routes, its output row of
 * moe_forward / moe_forward_host is 0 and moe_block_forward leaves its residual
 * row unchanged.  The pointer is kept, not copied: it must hold at least T bytes
 * for every later forward on this handle and stay valid while they run.
 * Errors: MOE_EINVAL for a NULL handle.
 */
MOE_API int moe_set_padding_mask(moe_handle h, const uint8_t *mask);

/*
 * Scale format of the int8 weights: "Grok-1 Admin & Architecture Guide", section 3
 * "Quantized weights", stores each weight as int8 values with per-block dequant
 * scales (w.weight * w.scales).  kb = 0 (the default): one bf16 scale per output
 * channel, s_lin, s_v [E, ffn] and s_1 [E, d].  kb = 128: one bf16 scale per output
 * channel and block of 128 consecutive input rows, s_lin, s_v [E, d/128, ffn] and
 * s_1 [E, ffn/128, d]; the weight at input row i uses scale row i / 128.  With
 * block scales each weight is dequantised to bf16(w * s) (one rounding) before the
 * MMA; per-channel scales are applied to the fp32 sums instead.  Applies to later
 * forwards; block scales need MOE_LAYOUT_PACKED (forwards otherwise return
 * MOE_EUNSUPPORTED).  Errors: MOE_EINVAL for a NULL handle or d / ffn not
 * multiples of kb; MOE_EUNSUPPORTED for any other kb.
 */
MOE_API int moe_set_scale_block(moe_handle h, int kb);

/*
 * The MoE layer on T tokens ("Mixture of Experts (MoELayer + Router)", steps 1-4).
 *   x    bf16 [T, d]   input tokens
 *   out  bf16 [T, d]   output; must not overlap x or the weights
 * Weights and scales as in the layout block above.  T == 0 is a no-op.
 * Enqueues the routing (router, dispatch, gather; one launch for T <= 32),
 * up-projection, down-projection and combine kernels on `stream` and returns.  Deterministic: the same inputs give
 * bit-identical outputs.  Device-side wait timeouts are reported later by
 * moe_sync_status.  Returns MOE_EINVAL on a bad argument, MOE_ENOMEM if the
 * workspace could not grow, MOE_ECUDA if a launch failed.
 */
MOE_API int moe_forward(moe_handle h, int T, const void *x, const float *router_w,
                        const int8_t *w_lin, const void *s_lin, const int8_t *w_v,
                        const void *s_v, const int8_t *w_1, const void *s_1, void *out,
                        void *stream);

/*
 * moe_forward with the tokens and the result in HOST memory: copies x_host
 * (bf16 [T, d]) to the device, runs the layer, copies the result into out_host
 * (bf16 [T, d]), all enqueued on `stream`.  The weights are device pointers.
 * Pinned host buffers make the copies asynchronous; the caller must
 * synchronise (moe_sync_status) before reading out_host.  With host overlap on
 * (moe_set_host_overlap) the output copy runs on a stream of the handle.
 */
MOE_API int moe_forward_host(moe_handle h, int T, const void *x_host, const float *router_w,
                             const int8_t *w_lin, const void *s_lin, const int8_t *w_v,
                             const void *s_v, const int8_t *w_1, const void *s_1,
                             void *out_host, void *stream);

/*
 * Host overlap for moe_forward_host (on = 1; 0, the default, turns it off).  With
 * it on, successive host-buffer forwards of this handle alternate between two
 * device staging slots; each call copies x_host in on one copy stream of the
 * handle and the result out to out_host on another, so both copies overlap the
 * neighbouring calls' layers, which stay on `stream`.  The input copy waits for
 * its slot's previous call and, where x_host overlaps the host output of the call
 * before, for that output (layers chained through host memory), but not for other
 * work enqueued earlier on `stream`: x_host must hold its values when the call is
 * made.  The output copy follows the call's layer but `stream` does not wait for
 * it: out_host holds the result after moe_sync_status (which also waits for the
 * handle's copy streams) or once `stream` has passed moe_host_wait.  Results are
 * identical with overlap on or off.  Costs a second pair of [T, d] staging
 * buffers.  Returns MOE_EINVAL for a NULL handle or another value.
 */
MOE_API int moe_set_host_overlap(moe_handle h, int on);

/*
 * Make `stream` wait (on the device, without blocking the host) until every host
 * copy of the handle's host-overlap forwards issued so far has completed, so that
 * work or an event enqueued on `stream` afterwards follows the results' arrival in
 * host memory.  MOE_EINVAL for a NULL handle.
 */
MOE_API int moe_host_wait(moe_handle h, void *stream);

/*
 * One residual MoE block ("Transformer stack and language model head": pre/post
 * RMSNorm around the MoE, h += h_dense), in place on the residual stream:
 *   u = bf16( RMSNorm(h; g_pre) ),   h <- bf16( h + RMSNorm( MoE(u); g_post ) )
 * with RMSNorm(z; g) = z / sqrt(mean(z^2) + eps) * g evaluated in fp32.  The
 * routing kernels form u as they read h (no separate normalisation pass) and the
 * post-norm and residual add run inside the combine; u stays in the handle's
 * workspace until the next forward (moe_get_block_input).
 *   h_io          bf16 [T, d]  residual stream, read and overwritten
 *   g_pre, g_post bf16 [d]     RMSNorm gains
 * Other arguments as in moe_forward.
 */
MOE_API int moe_block_forward(moe_handle h, int T, void *h_io, const void *g_pre,
                              const void *g_post, float eps, const float *router_w,
                              const int8_t *w_lin, const void *s_lin, const int8_t *w_v,
                              const void *s_v, const int8_t *w_1, const void *s_1, void *stream);

/*
 * Copy the routing of the handle's last forward (device to device, on `stream`):
 *   idx     int32 [T, 2]  chosen experts, slot 0 = larger probability
 *   gate    fp32  [T, 2]  their softmax probabilities
 *   offsets int32 [E+1]   first row of each expert in the grouped order
 *   perm    int32 [2T]    route id (2*t + slot) of each grouped row
 * Any pointer may be NULL.  Returns MOE_EINVAL if no forward ran yet.
 */
MOE_API int moe_get_routing(moe_handle h, int32_t *idx, float *gate, int32_t *offsets,
                            int32_t *perm, void *stream);

/*
 * Copy the bf16 MoE input u = bf16(RMSNorm(h; g_pre)) of the handle's last forward
 * (device to device, on `stream`) into u: bf16 [T, d], 16-byte aligned.  This is
 * the row the layer routed and multiplied, so a test can check the routing and the
 * expert outputs on the very values the kernels used.  Returns MOE_EINVAL if the
 * last forward was not moe_block_forward (or none ran), MOE_ECUDA if the copy
 * could not be enqueued.
 */
MOE_API int moe_get_block_input(moe_handle h, void *u, void *stream);

/*
 * Synchronise `stream`, then report the device status of the handle's kernels:
 * MOE_OK, MOE_ETIMEOUT if a bounded wait inside a pipelined kernel ran out (the
 * kernel then stopped early and its output is invalid), or MOE_ECUDA if the
 * stream reported an error.  Reading the status clears it.
 */
MOE_API int moe_sync_status(moe_handle h, void *stream);

/*
 * Limit, in nanoseconds, of every bounded wait inside the pipelined GEMM
 * kernels (default 2e9).  A wait that runs out records MOE_ETIMEOUT and the
 * kernel returns early with its async copies drained.  0 makes any wait that
 * does not succeed at once give up: a test hook for the timeout path.
 */
MOE_API int moe_set_timeout(moe_handle h, long long ns);

/*
 * Per-kernel timing with CUDA events recorded on the launch stream.
 * moe_set_profiling(h, 1) starts recording around each kernel of every forward;
 * moe_get_kernel_times synchronises on those events and returns, per kernel id
 * (0 router, 1 dispatch, 2 gather, 3 up-projection, 4 down-projection,
 * 5 combine, 6 unused (the residual block's pre-norm runs inside the routing
 * kernels), 7 small-batch routing: router and dispatch in one
 * launch, used instead of 0-2 when T <= 32; in MOE_LAYOUT_PACKED the
 * up-projection then loads the routed rows itself, in MOE_LAYOUT_IN_OUT that
 * launch also gathers them), the total milliseconds and the
 * launch count since the previous call, then resets them.  n = capacity of
 * ms/launches (8 suffices).
 */
MOE_API int moe_set_profiling(moe_handle h, int on);
MOE_API int moe_get_kernel_times(moe_handle h, float *ms, int *launches, int n);

/*
 * Select how the forward calls of this handle read w_lin, w_v and w_1:
 *   MOE_LAYOUT_IN_OUT (default)  [E, in, out]: the layout block above;
 *   MOE_LAYOUT_PACKED            [E, out, in]: each output feature's input
 *                                elements contiguous (w_lin, w_v [E, F, d];
 *                                w_1 [E, d, F]), one byte per value, each value
 *                                as a sign and a 7-bit magnitude (layout below);
 *                                written by moe_pack_weight.
 * Both give the same result up to fp32 summation order.  With MOE_LAYOUT_PACKED
 * the GEMMs keep the dequantised bf16 weights in tensor memory instead of shared
 * memory: the fast path.  There a weight w enters the tensor cores as the bf16
 * w * 2^-133 (zero exponent field, |w| as the mantissa: three instructions per four
 * weights), the routed rows and H at 2^64 times their values, and the
 * epilogues take the products back by exact powers of two; so the packed path
 * holds weights in [-127, 127] (symmetric int8 quantisation), scales below 2^59
 * and routed rows and H (gelu(x W) * (x V)) below 2^64 in magnitude.  The layout change is a one-time cost at weight-load
 * time.  Scales are the same in both layouts.  Returns MOE_EINVAL for an unknown
 * layout.
 */
MOE_API int moe_set_weight_layout(moe_handle h, int layout);

/*
 * The grouped GEMMs on CTA pairs (MOE_LAYOUT_PACKED, d and ffn multiples of 256): one tcgen05
 * MMA of 256 output features spans the two SMs of a two-CTA cluster, each SM converting its
 * 128 features' weights and holding half of the tile's routes' activations.  For large
 * batches that halves the activation traffic through each SM's shared memory (the
 * up-projection takes tiles of 128 routes, the down-projection of 256); for small batches each
 * MMA, of few columns, covers twice the features (tiles of 32 routes).
 *   mode 0  one CTA per tile everywhere;
 *   mode 1  pairs for the down-projection of plans of 128-route tiles (T > 64), the default:
 *           on a B200 it ran 12% faster than one CTA per tile at T = 8192;
 *   mode 2  pairs for both GEMMs of those plans (the up-projection measured slower on pairs:
 *           its two-stage TMEM operand ring leaves the cross-SM signals too little slack);
 *   mode 3  pairs also for both GEMMs of T <= 32 (32-route tiles; there the int8 -> bf16
 *           conversion, which pairs do not shorten, limits both paths).
 * Pairs run only where the device can hold a full wave of them.  Both paths add the same
 * products in the same order along the reduction, except where the tiles of a last, partial
 * wave are cut into K pieces added afterwards (each path cuts its own last wave); elsewhere
 * the results are bit-identical.  The mode applies to later forwards (it also sets the tile
 * width moe_plan reports: 32 from T = 1 with mode 3).  Returns MOE_EINVAL for a NULL handle or
 * another mode.
 */
MOE_API int moe_set_cta_pairs(moe_handle h, int mode);

/*
 * Rewrite one int8 weight tensor from MOE_LAYOUT_IN_OUT to MOE_LAYOUT_PACKED: a
 * per-expert transpose; every four consecutive input elements w0..w3 of an output
 * feature become the bytes  s2|m0, s0|m2, s3|m1, s1|m3  (mi = |wi|, si = 0x80 if wi < 0),
 * the signs crossed over so that a mask, and a byte swap and a mask, give bf16 pairs.
 *   which = 0: w is linear or linear_v, [E, d, F] -> w_packed [E, F, d]
 *   which = 1: w is linear_1,           [E, F, d] -> w_packed [E, d, F]
 * w and w_packed are device buffers of E*d*F bytes that must not overlap.  The
 * call synchronises `stream` (a load-time step) and returns MOE_ERANGE if w holds
 * -128, which has no packed form (w_packed is then not usable; such weights run
 * in MOE_LAYOUT_IN_OUT, which holds every int8 value).
 */
MOE_API int moe_pack_weight(moe_handle h, const int8_t *w, int8_t *w_packed, int which, void *stream);

/*
 * moe_pack_weight for a tensor of n_experts experts (1 <= n_experts <= E): [n, d, F] ->
 * [n, F, d] (which = 0) or [n, F, d] -> [n, d, F] (which = 1).  An expert-parallel rank
 * packs its own E / W experts with it.  Buffers of n_experts * d * F bytes; MOE_EINVAL for
 * an n_experts outside that range.
 */
MOE_API int moe_pack_weight_n(moe_handle h, const int8_t *w, int8_t *w_packed, int which, int n_experts,
                              void *stream);

/*
 * The tile shape and split chosen for T tokens (for tests and benchmarks):
 * *bn = routes per GEMM tile, *splits = K-splits of the down-projection.
 */
MOE_API int moe_plan(moe_handle h, int T, int *bn, int *splits);

/*
 * Expert parallelism: the experts spread over W ranks, as the pages' own layout spreads
 * them over the `model` mesh axis ("Grok-1 Admin & Architecture Guide", section 6
 * "Sharding & Parallelism Deep Dive", the MoE matmuls under shard_map).  Rank r of W
 * holds E_local = E / W consecutive experts, [r * E_local, (r + 1) * E_local), and its
 * own tokens.  One layer is three device steps on each rank, with two exchanges between
 * ranks that the caller makes (all-to-all; the Python package does it with
 * torch.distributed over NCCL):
 *
 *   moe_ep_dispatch   route the rank's T tokens; routed rows grouped by expert (hence by
 *                     destination rank) into send_rows, per-expert row counts;
 *   exchange          counts, then rows: rank j receives, from every source s in rank
 *                     order, s's rows for j's experts (in s's order);
 *   moe_ep_experts    the rank's experts on the rows it received -> y rows, same order;
 *   exchange          y rows back to their sources (the reverse of the row exchange);
 *   moe_ep_combine    out[t] = gate0 * y(t, slot 0) + gate1 * y(t, slot 1).
 *
 * The result is the layer of moe_forward on the rank's tokens.  The handle keeps the
 * dispatch's routing until moe_ep_combine; a moe_forward / moe_block_forward on the same
 * handle in between discards it.
 */

/*
 * Step 1: routing ("Mixture of Experts (MoELayer + Router)", steps 1-2, with the handle's
 * router bias and padding mask) and grouping of this rank's T tokens.
 *   x            bf16 [T, d]   this rank's tokens
 *   router_w     fp32 [d, E]   the full router (every rank routes over all E experts)
 *   send_rows    bf16 [2T, d]  out: row i = x[perm[i] / 2] for the n = sum(send_counts)
 *                              routed rows, grouped by expert, ascending token order within one
 *   send_counts  int32 [E]     out (device): routed rows per expert
 * moe_get_routing then reports this routing (perm = the order of send_rows).  Returns
 * MOE_EINVAL on a bad argument, MOE_ECUDA if a launch failed.  T == 0 only sets the
 * counts to 0 (x and send_rows may then be NULL).
 */
MOE_API int moe_ep_dispatch(moe_handle h, int T, const void *x, const float *router_w, void *send_rows,
                            int32_t *send_counts, void *stream);

/*
 * Step 3: the rank's E_local experts (step 3 of the MoE section: linear_1(gelu(linear(x)) *
 * linear_v(x)), 8-bit weights) on the rows it received.
 *   recv_counts  int32 [n_src, E_local]  HOST array: rows received from source rank s for
 *                                       local expert k (what the count exchange delivered)
 *   recv_rows    bf16 [R, d]   the received rows, R = sum(recv_counts): source after source,
 *                              each source's rows grouped by local expert
 *   weights      the E_local experts' w_lin, s_lin, w_v, s_v, w_1, s_1 in the handle's
 *                weight layout and scale format ([E_local, ...] in place of [E, ...])
 *   y_rows       fp32 [R, d]   out: row i = s_1 * (H_i . W_1) of received row i's expert
 *                              (not gate-weighted: the source applies the gates)
 * Returns MOE_EUNSUPPORTED if n_src * E_local > 64, MOE_EINVAL on a bad argument or
 * R > 2 * MOE_MAX_TOKENS.  R == 0 is a no-op.
 */
MOE_API int moe_ep_experts(moe_handle h, int n_src, int E_local, const int32_t *recv_counts, const void *recv_rows,
                           const int8_t *w_lin, const void *s_lin, const int8_t *w_v, const void *s_v,
                           const int8_t *w_1, const void *s_1, float *y_rows, void *stream);

/*
 * Step 5: the gate-weighted combine of step 4 of the MoE section, in slot order.
 *   y_back  fp32 [n, d]   the y rows of this rank's sent rows, back in send_rows order
 *   out     bf16 [T, d]   out[t] = bf16(gate[t,0] * y(t,0) + gate[t,1] * y(t,1)); 0 for a
 *                         padding token
 * T must be the T of the handle's last moe_ep_dispatch (else MOE_EINVAL).
 */
MOE_API int moe_ep_combine(moe_handle h, int T, const float *y_back, void *out, void *stream);

/* Largest token count moe_route_noalloc accepts (its static scratch is sized for it). */
#define MOE_NOALLOC_MAX_TOKENS 65536

/*
 * Routing only -- router (fp32 logits, softmax, top-2) and dispatch (grouping by
 * expert) -- without allocating any device memory.  The pages have no counterpart:
 * this entry point exists for callers that cannot call cudaMalloc, such as code
 * running inside a device-memory arena that is sized once up front, or code inside
 * a framework that owns the allocator.  It needs no handle.
 *   x         bf16 [T, d] input tokens (d a multiple of 8)
 *   router_w  fp32 [d, 8]
 *   bias      fp32 [8] added to the logits, or NULL
 *   idx       int32 [T, 2], gate fp32 [T, 2], offsets int32 [9], perm int32 [2T]:
 *             outputs with the meaning of moe_get_routing (E = 8 experts)
 * All pointers are device pointers, 16-byte aligned, owned by the caller.
 * Scratch: dispatch's working arrays live in one file-scope device array of about
 * 1 MB (MOE_NOALLOC_MAX_TOKENS tokens), which every GPU that loads the library holds
 * until the process exits.  The first call on a device looks up that array's device
 * address (cudaGetSymbolAddress, with the device current) and keeps it while the same
 * CUDA context stays current (a new context, e.g. after cudaDeviceReset, looks it up
 * again); make that first call before any stream capture.  Every call shares the array and it keeps the last
 * call's contents; each call writes every word it later reads, so nothing needs
 * clearing, but calls whose kernels overlap on the GPU (different streams, or
 * concurrent host threads) race on it: serialise them.
 * Returns MOE_EINVAL for T > MOE_NOALLOC_MAX_TOKENS, a bad d, or a null or
 * misaligned pointer; MOE_ENODEV without a device; MOE_ECUDA if a launch failed.
 * Calls no allocating routine.  T == 0 is a no-op.
 */
MOE_API int moe_route_noalloc(int T, int d, const void *x, const float *router_w, const float *bias,
                              int32_t *idx, float *gate, int32_t *offsets, int32_t *perm, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
