/*
 * adafuse.h -- C ABI of the AdaFuse adapter switch for NVIDIA B200 (sm_100a).
 *
 * What the library computes (page title "AdaFuse: Accelerating Dynamic
 * Adapter Inference via Token-Level Pre-Gating and Fused Kernel
 * Optimization"):
 *
 *   adafuse_pregate   token-level pre-gating: ONE top-2 routing decision per
 *                     token, made from the hidden state entering the first
 *                     layer, and applied to every adapter layer
 *                     (gist.science technical summary, section 2-ga, items
 *                     1-3; shd-paper.top summary, English abstract).
 *   adafuse_switch    the fused adapter switch: in ONE kernel launch, for
 *                     every layer and every LoRA-targeted weight, remove the
 *                     previous token's gated experts and merge the current
 *                     token's, in place:
 *                       W <- W - s*sum_{e in prev} g_e B_e A_e
 *                              + s*sum_{e in cur}  g_e B_e A_e
 *                     (gist.science technical summary, section 2-na: the SGMM
 *                     "segmented gather matrix multiplication" kernel,
 *                     concatenated adapter matrices, in-place update,
 *                     prefetch buffer).
 *   adafuse_switch_batch_layers   the same switch restricted to a contiguous
 *                     range of layers (for pipelining against the forward).
 *
 * Numerics: W is bf16; each W element is updated as
 *   W <- bf16_round_nearest_even(float(W) + dW)
 * with dW = sum_e c_e * (B_e A_e), the products accumulated in fp32 and the
 * per-expert coefficients c_e = s*(g_cur(e) - g_prev(e)) applied in fp32
 * (the folded kernel instead carries c_e * A_e as three bf16 terms that
 * reproduce it to about 2^-24 of its size, one fp32 rounding's worth).
 * One rounding per element per switch.  s = alpha / rank.
 *
 * Layouts (all row-major, all device memory unless stated):
 *   W  [out, in]        bf16   the backbone weight, updated in place
 *   A  [E, rank, in]    bf16   LoRA down-projections of the E experts
 *   B  [E, out, rank]   bf16   LoRA up-projections of the E experts
 *   h  [T, d]           fp32   hidden states entering the first layer
 *   Wr [d, E]           fp32   router weight
 *   route [T]           adafuse_route (16 bytes each)
 *
 * Ownership: the caller owns every buffer named above, keeps it alive and
 * in place for the life of the context, and must not write W while a switch
 * on it is in flight.  The library owns the context, its device-side
 * segment table and its device status word.  The library keeps no copy of W.
 * For ranks below 8 it keeps a zero-padded copy of every B (see
 * adafuse_refresh_adapters); for ranks up to 8, once the folded kernel is
 * first used, a buffer that kernel rewrites from A on every switch (see
 * adafuse_set_switch_kernel).
 *
 * Errors: every call returns ADAFUSE_OK (0) or a negative code.  Calls that
 * take a stream are asynchronous with respect to the host; host-side
 * argument errors are reported before anything is launched.  Problems only
 * the device can see (an expert index outside [-1, E), a non-finite gate in
 * a route) make the switch write NOTHING and raise a bit in the context's
 * device status word (read it with adafuse_get_device_status).  No C++
 * exception crosses this boundary.  A context may be used from one host
 * thread and one stream at a time.
 */
#ifndef ADAFUSE_H_
#define ADAFUSE_H_

#include <stdint.h>

#if defined(__GNUC__)
#define ADAFUSE_API __attribute__((visibility("default")))
#else
#define ADAFUSE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- return codes ------------------------------------------------------- */
#define ADAFUSE_OK                     0
#define ADAFUSE_ERR_INVALID_ARG       -1  /* NULL pointer, bad count, misaligned pointer */
#define ADAFUSE_ERR_UNSUPPORTED_SHAPE -2  /* dims not multiples of 8, rank outside [1,64], E outside [1,64] */
#define ADAFUSE_ERR_CUDA              -3  /* a CUDA runtime call failed (see adafuse_last_error) */
#define ADAFUSE_ERR_DEVICE_FAULT      -4  /* the device status word is non-zero */
#define ADAFUSE_ERR_UNSUPPORTED_DEVICE -5 /* not a compute-capability 10.0 (B200-class) GPU */
#define ADAFUSE_ERR_OUT_OF_MEMORY     -6  /* host or device allocation failed */

/* ---- device status word bits (adafuse_get_device_status) ---------------- */
#define ADAFUSE_STATUS_BAD_EXPERT   0x1   /* a route held an index outside [-1, E) */
#define ADAFUSE_STATUS_BAD_GATE     0x2   /* a route held a non-finite gate on a used slot */
#define ADAFUSE_STATUS_TIMEOUT      0x4   /* a bounded wait inside a kernel gave up (1 s); the
                                             launch is incomplete (see "State of W after a
                                             timeout" below) */

/* ---- switch kernel variants (adafuse_set_switch_kernel) ------------------ */
#define ADAFUSE_KERNEL_AUTO      0  /* rank <= 8: TCGEN05; other multiples of 8: TCGEN05_PAIR;
                                       any other rank: MMA_SYNC */
#define ADAFUSE_KERNEL_MMA_SYNC  1  /* register-streaming kernel, any rank in [1, 64] */
#define ADAFUSE_KERNEL_TCGEN05   2  /* TMA + tcgen05/TMEM kernel, rank <= 8 or a multiple of 8 */
#define ADAFUSE_KERNEL_TCGEN05_PAIR 3 /* the same on CTA pairs (tcgen05 cta_group::2, 256 x 128
                                         W blocks), rank a multiple of 8 */
#define ADAFUSE_KERNEL_TCGEN05_FOLD 4 /* rank <= 8: the coefficients folded into the adapter
                                         operand (c*A as three bf16 terms, written by a fold
                                         launch before each switch launch), one TMEM
                                         accumulator per tile; needs |c * A| within the
                                         bf16 range */

/* ---- tile schedules (adafuse_set_tile_schedule) ------------------------- */
#define ADAFUSE_SCHEDULE_STATIC  0
#define ADAFUSE_SCHEDULE_DYNAMIC 1
#define ADAFUSE_SCHEDULE_AUTO    2  /* default: dynamic for ADAFUSE_KERNEL_TCGEN05, static
                                       for ADAFUSE_KERNEL_TCGEN05_PAIR */

/* ---- TMA tensor-map layouts (adafuse_get_tensor_map_layout) ------------- */
#define ADAFUSE_MAPS_NONE    0  /* no tensor maps: only the mma.sync kernel runs */
#define ADAFUSE_MAPS_PLAIN   1  /* some weight's in is not a multiple of 64: a 128 x 128
                                   W tile moves as two 64-column TMA operations */
#define ADAFUSE_MAPS_BLOCKED 2  /* every in a multiple of 64: W viewed as 64-column
                                   blocks, one TMA operation per W tile load or store
                                   and per expert's A columns */

/* One token's routing decision: the two chosen experts and their gates.
 * idx[j] == -1 marks an empty slot (its gate is ignored).  adafuse_pregate
 * writes gate[0] >= gate[1], gate[0] + gate[1] == 1 (up to rounding). */
typedef struct adafuse_route {
    int32_t idx[2];
    float gate[2];
} adafuse_route;

/* A top-k routing decision, k in [1, ADAFUSE_MAX_TOP_K] (32 bytes): the k
 * chosen experts in order and their gates; slots past k, or past the number
 * of experts, hold idx -1 (their gate is ignored).  adafuse_pregate_topk
 * writes non-increasing gates that sum to 1 up to rounding.  The pages'
 * router is top-2 (gist.science technical summary, section 2-ga); top-k is
 * the same router widened to k picks. */
#define ADAFUSE_MAX_TOP_K 4
typedef struct adafuse_route4 {
    int32_t idx[4];
    float gate[4];
} adafuse_route4;

/* One LoRA-targeted weight of one layer (for example q_proj of layer 7).
 *   out, in  W's shape; both multiples of 8.
 *   W        device pointer, [out, in] bf16, 16-byte aligned, updated in place.
 *   A        device pointer, [E, rank, in] bf16, 16-byte aligned.
 *   B        device pointer, [E, out, rank] bf16, 16-byte aligned.
 *   name     optional label (may be NULL); not copied, not used by kernels. */
typedef struct adafuse_target {
    const char* name;
    int64_t out;
    int64_t in;
    void* W;
    const void* A;
    const void* B;
} adafuse_target;

/* The adapter-carrying model.  targets has n_layers * n_targets entries,
 * layer-major: targets[l * n_targets + k] is target k of layer l.
 * 1 <= n_experts <= 64, 1 <= rank <= 64, alpha finite; s = alpha / rank. */
typedef struct adafuse_desc {
    int32_t n_layers;
    int32_t n_targets;
    int32_t n_experts;
    int32_t rank;
    float alpha;
    const adafuse_target* targets;
} adafuse_desc;

typedef struct adafuse_ctx adafuse_ctx;

/* Validate the model, build the device-side segment table (the list of
 * disjoint 128x128 W tiles of every (layer, target), layer-major) and the
 * per-weight descriptors, and copy them to `device`.  Not on the hot path.
 * Returns INVALID_ARG / UNSUPPORTED_SHAPE / UNSUPPORTED_DEVICE / CUDA /
 * OUT_OF_MEMORY without creating anything.  *out receives the context. */
ADAFUSE_API int adafuse_create(adafuse_ctx** out, const adafuse_desc* desc, int device);

/* Free the context and its device memory.  The caller must make sure no
 * call using it is still in flight.  NULL is accepted (no-op). */
ADAFUSE_API int adafuse_destroy(adafuse_ctx* ctx);

/* Token-level pre-gating (section 2-ga): for each of T tokens,
 *   z_e = sum_i h[t,i] * Wr[i,e]  (fp32; every column reduced in the same
 *         order, so equal columns give bitwise-equal logits),
 *   the two experts first under (z descending, index ascending),
 *   gates = softmax over all E renormalised over the two picks, computed
 *         in the equal closed form g0 = 1/(1+x), g1 = x/(1+x),
 *         x = exp(z1 - z0),
 * written to route[t].  E comes from the context.  With E == 1 the route is
 * {0, -1} with gates {1, 0}.  h, Wr, route are device pointers; h and route
 * 16-byte aligned, Wr 4-byte aligned, d a multiple of 4 and d >= 1; T == 0
 * is a no-op.
 * Non-finite h gives an unspecified route (the switch rejects non-finite
 * gates).  One kernel launch on `stream` (a cudaStream_t, NULL = legacy
 * default stream).  Batches of 64+ tokens with E == 8 and a 16-byte-aligned
 * Wr bring Wr into each CTA by TMA tile loads behind a bounded wait: if
 * those loads do not land within 1 s, the launch sets ADAFUSE_STATUS_TIMEOUT
 * in the context's status word (adafuse_get_device_status) and writes no
 * route. */
ADAFUSE_API int adafuse_pregate(adafuse_ctx* ctx, const float* h, int64_t T, int64_t d,
                    const float* Wr, adafuse_route* route, void* stream);

/* The fused adapter switch (section 2-na) over ALL layers and targets, one
 * kernel launch on `stream`.  prev / cur are 16-byte aligned device
 * pointers to ONE route each, or NULL for "no experts" (prev == NULL: first
 * token, or a static
 * pre-merge; cur == NULL: full unmerge).  Per expert e in prev U cur the
 * coefficient is c_e = s*(g_cur(e) - g_prev(e)) (an absent side counts 0);
 * experts with c_e == 0 are dropped, so prev == cur (same indices, bitwise
 * equal gates) launches work that writes nothing and leaves W bit-identical.
 * The route records are read on the device: no host synchronisation. */
ADAFUSE_API int adafuse_switch(adafuse_ctx* ctx, const adafuse_route* prev,
                   const adafuse_route* cur, void* stream);

/* As adafuse_switch, restricted to layers [layer_begin, layer_begin +
 * n_layers).  n_layers == 0 is a no-op; a range outside [0, L) is
 * INVALID_ARG.  Running it over a partition of [0, L) equals one
 * adafuse_switch. */
ADAFUSE_API int adafuse_switch_batch_layers(adafuse_ctx* ctx, int32_t layer_begin,
                                int32_t n_layers, const adafuse_route* prev,
                                const adafuse_route* cur, void* stream);

/* Choose the kernel adafuse_switch launches for this context (default
 * ADAFUSE_KERNEL_AUTO).  All compute the same update to within the
 * documented rounding; ADAFUSE_KERNEL_TCGEN05 needs rank <= 8 or a multiple
 * of 8, ADAFUSE_KERNEL_TCGEN05_PAIR a multiple of 8 above 8 and
 * ADAFUSE_KERNEL_TCGEN05_FOLD rank <= 8; each returns UNSUPPORTED_SHAPE
 * otherwise.  With ADAFUSE_KERNEL_TCGEN05_FOLD every switch, re-base or layer
 * range is two launches on the stream: the fold of c_e * A_e for the route's
 * experts into a context-owned buffer, then the switch.  That buffer holds at
 * most 4 pairs of experts x 12 KB per 128 columns of every weight (48 KB per
 * 128 columns; 437 MB at the Llama-2-7B shape) and is allocated on first use:
 * by this call when it selects ADAFUSE_KERNEL_TCGEN05_FOLD, or by the first
 * in-place top-k switch that ADAFUSE_KERNEL_AUTO gives to the folded kernel.
 * That first use synchronises the device and must not be captured into a
 * CUDA graph (INVALID_ARG, nothing enqueued).  If the allocation fails it
 * returns OUT_OF_MEMORY and the folded kernel is off for the context (AUTO
 * then takes ADAFUSE_KERNEL_TCGEN05 for top-k switches).  Selecting any other
 * kernel is host-only, with no device work. */
ADAFUSE_API int adafuse_set_switch_kernel(adafuse_ctx* ctx, int kernel);

/* The kernel adafuse_switch_topk and adafuse_switch_topk_layers launch: the
 * context's choice, except that ADAFUSE_KERNEL_AUTO takes
 * ADAFUSE_KERNEL_TCGEN05_FOLD for ranks <= 8 (an in-place top-k switch can
 * touch 8 experts, which the folded kernel sums in one TMEM accumulator).
 * Re-base calls follow adafuse_get_switch_kernel.  Host-only. */
ADAFUSE_API int adafuse_get_topk_switch_kernel(adafuse_ctx* ctx);

/* Tile schedule of ADAFUSE_KERNEL_TCGEN05 and ADAFUSE_KERNEL_TCGEN05_PAIR
 * (the other kernels always use the static one).  ADAFUSE_SCHEDULE_STATIC:
 * CTA b (CTA pair b) of the persistent grid takes tiles (256 x 128 blocks)
 * b, b + grid, b + 2*grid, ... of its table.  ADAFUSE_SCHEDULE_DYNAMIC: each
 * CTA (the even CTA of each pair, for both) takes its next tile from a
 * context-owned ticket counter in table order, so the tiles in flight on the
 * GPU stay a compact window of the table (neighbouring W rows) however far the
 * CTAs' speeds drift apart; the launch leaves the counter at zero.
 * ADAFUSE_SCHEDULE_AUTO (default): dynamic for the single-CTA kernel, static
 * for the pair kernel (the faster of the two for each on B200 at the 13B and
 * Llama-3-8B shapes).  The schedule decides only which CTA takes a tile,
 * never how a tile is computed: W is bit for bit the same.  INVALID_ARG for
 * any other value.  Host-only, no device work. */
ADAFUSE_API int adafuse_set_tile_schedule(adafuse_ctx* ctx, int schedule);

/* Cap the persistent grid of this context's switch and re-base launches at
 * max_ctas CTAs (0 = no cap: one CTA per SM, two for the mma.sync kernel;
 * the pair kernel rounds the cap down to whole CTA pairs, at least one).  A
 * launch fills every SM it is given, so work on other streams cannot start
 * beside it; a caller that pipelines the switch against its forward pass
 * (adafuse_switch_batch_layers on a second stream) leaves SMs to the forward
 * this way.  The grid only decides which CTA takes a tile, never how a tile
 * is computed: W is bit for bit the same.  INVALID_ARG for max_ctas < 0.
 * Host-only, no device work. */
ADAFUSE_API int adafuse_set_max_ctas(adafuse_ctx* ctx, int32_t max_ctas);

/* The kernel adafuse_switch will launch (ADAFUSE_KERNEL_MMA_SYNC,
 * ADAFUSE_KERNEL_TCGEN05, ADAFUSE_KERNEL_TCGEN05_PAIR or
 * ADAFUSE_KERNEL_TCGEN05_FOLD), or a negative code. */
ADAFUSE_API int adafuse_get_switch_kernel(adafuse_ctx* ctx);

/* The tensor-map layout adafuse_create chose for this context
 * (ADAFUSE_MAPS_NONE, _PLAIN or _BLOCKED), or a negative code.  The layout
 * changes how many TMA operations move a tile, never a result: the same
 * elements are read and written either way, so W is bit for bit the same. */
ADAFUSE_API int adafuse_get_tensor_map_layout(const adafuse_ctx* ctx);

/* ---- re-base switch ------------------------------------------------------
 * A variant of the switch that the AdaFuse pages do not describe (they merge
 * in place, section 2-na): the caller keeps a pristine copy W0 of every
 * targeted weight, and each call writes W <- bf16_rne(W0 + s*sum_{e in cur}
 * g_e B_e A_e).  It moves the same bytes as the in-place switch (W0 read, W
 * written), needs no previous route, cannot drift, and costs a second copy
 * of the targeted weights in device memory. */

/* Register the pristine weights: W0 is a host array of n_layers*n_targets
 * device pointers, one per (layer, target) in the same order as the
 * context's targets, each [out, in] bf16, 16-byte aligned, distinct from W.
 * The caller owns W0 and must not modify it while re-base calls may run.
 * Builds device-side descriptors (allocates; not for the hot path) and
 * synchronises the device.  Calling it again replaces the base. */
ADAFUSE_API int adafuse_set_base(adafuse_ctx* ctx, const void* const* W0);

/* W <- bf16_rne(W0 + s*sum_{e in cur} g_e B_e A_e) for every layer and
 * target, one kernel launch on `stream`.  cur: 16-byte aligned device route
 * or NULL (then W <- W0).  INVALID_ARG without a registered base.  Bad
 * routes behave as in adafuse_switch (status bit, nothing written). */
ADAFUSE_API int adafuse_rebase(adafuse_ctx* ctx, const adafuse_route* cur, void* stream);

/* As adafuse_rebase, restricted to layers [layer_begin, layer_begin + n_layers). */
ADAFUSE_API int adafuse_rebase_layers(adafuse_ctx* ctx, int32_t layer_begin, int32_t n_layers,
                                      const adafuse_route* cur, void* stream);

/* ---- top-k routing --------------------------------------------------------
 * The router and the switches above with k in [1, 4] experts per token.  An
 * in-place switch then touches up to 2k experts (k leaving, k arriving). */

/* Top-k pre-gating: as adafuse_pregate, with route[t] the k experts first
 * under (logit descending, index ascending) and gates g_j = the softmax over
 * all experts renormalised over the k picks.  k outside [1, 4] is
 * INVALID_ARG.  route: device array of T adafuse_route4, 16-byte aligned.
 * For k = 2 the experts and gates equal adafuse_pregate's bit for bit.  A
 * token's route does not depend on the batch it is gated in. */
ADAFUSE_API int adafuse_pregate_topk(adafuse_ctx* ctx, const float* h, int64_t T, int64_t d,
                                     const float* Wr, int32_t k, adafuse_route4* route,
                                     void* stream);

/* ---- batch decode ---------------------------------------------------------
 * The pages make one routing decision per token (gist.science technical
 * summary, section 2-ga).  A decode batch of T sequences that shares one
 * merged weight can carry only one expert set, so these calls make ONE
 * decision for the batch (a reading beyond the pages): the token rule applied
 * to the mean of the batch's router logits,
 *   zbar_e = (sum_t z_t,e) / T,  z_t,e as adafuse_pregate computes them,
 * summed in token order in fp32; then the experts first under (zbar
 * descending, index ascending) and gates = the softmax over all E of zbar
 * renormalised over the picks.  With T = 1 the record equals the token's
 * adafuse_pregate / adafuse_pregate_topk record bit for bit.  The result is
 * one route record; pass it to adafuse_switch / adafuse_switch_topk like a
 * token's route.
 * Arguments as for adafuse_pregate; 1 <= T <= ADAFUSE_MAX_BATCH_TOKENS
 * (INVALID_ARG above it; T == 0 is a no-op).  Two launches on `stream`: the
 * tokens' logits into a context-owned scratch of ADAFUSE_MAX_BATCH_TOKENS x E
 * fp32 (allocated at create), then the mean and the decision.  The scratch
 * is shared by the context's calls; calls on one stream are ordered.  If the
 * first launch raises ADAFUSE_STATUS_TIMEOUT (see adafuse_pregate), the
 * decision is taken from stale logits and must be discarded. */
#define ADAFUSE_MAX_BATCH_TOKENS 4096
ADAFUSE_API int adafuse_pregate_batch(adafuse_ctx* ctx, const float* h, int64_t T, int64_t d,
                                      const float* Wr, adafuse_route* route, void* stream);

/* As adafuse_pregate_batch with k in [1, 4] picks into one adafuse_route4. */
ADAFUSE_API int adafuse_pregate_batch_topk(adafuse_ctx* ctx, const float* h, int64_t T,
                                           int64_t d, const float* Wr, int32_t k,
                                           adafuse_route4* route, void* stream);

/* As adafuse_switch with top-k routes: per expert e in prev U cur the
 * coefficient is c_e = s*(g_cur(e) - g_prev(e)), experts with c_e == 0 are
 * dropped, and W <- bf16_rne(W + sum_e c_e B_e A_e) with fp32 accumulation
 * (up to 8 experts in one launch).  prev / cur: 16-byte aligned device
 * routes or NULL.  Bad routes set the status word and write nothing. */
ADAFUSE_API int adafuse_switch_topk(adafuse_ctx* ctx, const adafuse_route4* prev,
                                    const adafuse_route4* cur, void* stream);

/* As adafuse_switch_topk, restricted to layers [layer_begin, layer_begin + n_layers). */
ADAFUSE_API int adafuse_switch_topk_layers(adafuse_ctx* ctx, int32_t layer_begin,
                                           int32_t n_layers, const adafuse_route4* prev,
                                           const adafuse_route4* cur, void* stream);

/* As adafuse_rebase with a top-k route: W <- bf16_rne(W0 + s*sum_{e in cur}
 * g_e B_e A_e).  INVALID_ARG without a registered base. */
ADAFUSE_API int adafuse_rebase_topk(adafuse_ctx* ctx, const adafuse_route4* cur, void* stream);

/* Ranks below 8 only (a no-op otherwise): the tensor-core path reads B
 * through a copy whose rows are zero-padded to 8 (B rows of 2*rank bytes are
 * not a legal TMA stride).  adafuse_create takes that copy; after changing
 * the contents of any B of the context, call this before the next switch.
 * It enqueues the copies on `stream`.  The copy costs 8/rank times the bytes
 * of the B tensors in device memory. */
ADAFUSE_API int adafuse_refresh_adapters(adafuse_ctx* ctx, void* stream);

/* State of W after a timeout.  The tensor-core kernels bound every wait;
 * when one runs out the launch raises ADAFUSE_STATUS_TIMEOUT and its CTAs stop
 * where they are.  Each 128 x 128 tile of the segment table is updated in
 * shared memory as a whole and written back by one store, after its whole
 * update, so after the stop every tile is in one of two states: switched
 * (its new values were stored before the stop) or untouched (it keeps its
 * values from before the launch).  No tile is partly switched, but which
 * tiles were reached is not recorded.  An in-place switch is not idempotent:
 * running the same switch again would apply it twice to the switched tiles.
 * Recovery: with a pristine copy registered (adafuse_set_base),
 * adafuse_rebase(ctx, cur) rewrites every tile as bf16_rne(W0 + s * sum_{e in
 * cur} g_e B_e A_e), a consistent state for the route `cur`; without one, the
 * caller restores W from its own copy of the weights.  A re-base that timed
 * out is recovered by running it again.  The mma.sync kernel has no waits
 * and never times out. */

/* Test hook for the timeout path (no counterpart on the pages).  The next
 * switch or re-base launched with a tensor-core kernel announces 16 bytes of
 * operand transfers that never arrive on the first operand stage of the
 * `tile`-th tile (1-based) that each CTA -- each CTA pair for
 * ADAFUSE_KERNEL_TCGEN05_PAIR -- takes, so the MMA warp's bounded wait (1 s)
 * runs out: the launch raises ADAFUSE_STATUS_TIMEOUT, every warp leaves
 * through its bounded waits and TMEM is freed; the context stays usable.  A
 * CTA's tiles before that one are switched and stored, that tile and later
 * ones are untouched (the state described above); with tile == 1 nothing is
 * written.  INVALID_ARG when tile < 1; UNSUPPORTED_SHAPE when the context's
 * kernel is ADAFUSE_KERNEL_MMA_SYNC (it has no waits).  Host-only; consumed
 * by the next launch. */
ADAFUSE_API int adafuse_debug_stall_next_switch_at(adafuse_ctx* ctx, int32_t tile);

/* adafuse_debug_stall_next_switch_at(ctx, 1): the next launch stalls on each
 * CTA's first tile and writes no W. */
ADAFUSE_API int adafuse_debug_stall_next_switch(adafuse_ctx* ctx);

/* Synchronise `stream`, read the device status word into *status, then
 * clear it.  Returns ADAFUSE_ERR_DEVICE_FAULT when the word was non-zero,
 * ADAFUSE_OK otherwise. */
ADAFUSE_API int adafuse_get_device_status(adafuse_ctx* ctx, void* stream, int32_t* status);

/* Host-only introspection (no device work): the segment table the context
 * would build for `desc`, as n entries of 4 int32 {layer, target, row0,
 * col0}, tile size 128x128.  With entries == NULL only *count is written.
 * capacity counts entries.  Returns INVALID_ARG if capacity is too small. */
ADAFUSE_API int adafuse_segment_table(const adafuse_desc* desc, int32_t* entries,
                          int64_t capacity, int64_t* count);

/* ---- allocation-free switch -------------------------------------------- */
#define ADAFUSE_NOALLOC_SCRATCH_BYTES 65536  /* static device scratch per GPU */
#define ADAFUSE_NOALLOC_MAX_WEIGHTS   1638   /* (layer, target) weights it can hold */

/* The fused switch for callers that cannot allocate device memory.  The
 * AdaFuse pages have no counterpart to this entry point: it exists for
 * deployment, not for the method.
 *
 * adafuse_create calls cudaMalloc for its tile table, weight descriptors and
 * status word.  Some callers cannot: a serving engine that has handed all
 * free HBM to its own memory pool (a later cudaMalloc fails or fragments the
 * pool), or a decode loop that must not stall on cudaMalloc's implicit
 * device synchronisation.  This call needs no context and allocates nothing
 * -- no cudaMalloc, no cudaFree, no allocating library routine.  It performs
 * the same switch as adafuse_switch over every (layer, target) of `desc`, on
 * the current device, with the mma.sync kernel, and gives the same result to
 * within the documented rounding.
 *
 * Scratch: one file-scope static device array of
 * ADAFUSE_NOALLOC_SCRATCH_BYTES (64 KiB), which every GPU that loads this
 * library holds until the process exits.  Each call rewrites it with the
 * weight table of `desc`, written on the device by small launches that carry
 * the table entries as kernel arguments (no host buffer is read after the
 * call returns), so ALL calls share it: two calls whose work overlaps on the
 * GPU (different streams, or threads without ordering) race and may switch
 * the wrong weights.  Calls on one stream are ordered and safe.  The first
 * call on each device also looks up the array's device address
 * (cudaGetSymbolAddress, once per device, under a host mutex that guards
 * only that lookup).
 *
 * Arguments: desc as for adafuse_create (host memory, read during the call
 * only; its device pointers must stay valid until the switch completes);
 * prev / cur as for adafuse_switch; status: optional 4-byte-aligned device
 * int32 that the call first sets to 0 and the kernel then ORs
 * ADAFUSE_STATUS_* bits into (a bad route writes no W); stream: cudaStream_t.
 * Returns ADAFUSE_ERR_UNSUPPORTED_SHAPE when desc has more than
 * ADAFUSE_NOALLOC_MAX_WEIGHTS weights (or a shape adafuse_create rejects),
 * INVALID_ARG / UNSUPPORTED_DEVICE / CUDA otherwise as adafuse_create and
 * adafuse_switch do; every argument is checked before anything is enqueued.
 * Asynchronous like adafuse_switch: it enqueues ceil(weights / 96) table
 * launches, the status reset and the switch launch on `stream`. */
ADAFUSE_API int adafuse_switch_noalloc(const adafuse_desc* desc, const adafuse_route* prev,
                                       const adafuse_route* cur, int32_t* status, void* stream);

/* Tile edge of the segment table (128). */
ADAFUSE_API int adafuse_tile_size(void);

/* Human-readable text for a return code (static storage). */
ADAFUSE_API const char* adafuse_strerror(int code);

/* Text of the last CUDA error this host thread saw in the library (static
 * thread-local storage, "" when none). */
ADAFUSE_API const char* adafuse_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* ADAFUSE_H_ */
