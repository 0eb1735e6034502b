/*
 * moe_cache.h -- C ABI of libmoe: the sparse Mixture-of-Experts FFN step of batch-1
 * decode with a bounded GPU expert cache, for NVIDIA B200 (sm_100a).
 *
 * The method is Luce Spark as described on theneuralfeed.com ("Luce Spark runs 35B MoE
 * models on 16GB GPU without speed loss", key-components paragraph): an A3B MoE routes
 * each token to about 8 of 256 experts; (1) calibrated placement accumulates per-expert
 * routing frequencies and pins the most-used set on the GPU; (2) a bounded asynchronous
 * cache with a fixed ring of spare GPU slots copies a cold expert from pinned host
 * memory into a spare slot while evicting the least recently used entry; (3) the whole
 * token runs as one graph instead of one per layer; at full residency the output is
 * bit-identical to all-GPU.  The baguaai.com summary ("Luce Spark: Shattering the VRAM
 * Ceiling ...", event core) adds that the long tail lives in system RAM and is swapped
 * in on demand.
 *
 * The MoE layer these calls compute (the pages do not spell it out; the library takes
 * the plainest reading): router z = W_r x + b (W_r bf16, fp32 accumulation), softmax,
 * top-k, renormalise; expert i: a = silu(G_i x) * (U_i x), o_i = D_i a with Q4_0 weights
 * (GGUF block: fp16 scale d, 16 bytes of nibbles, weight = (q - 8) d); y = sum_i w_i o_i
 * + o_shared; stacks are pre-norm residual: h <- h + MoE(RMSNorm(h)).  Routing
 * decisions, routing histograms and the cache event log are exact; outputs are fp32.
 *
 * Conventions for every call:
 *   - Return value: MOE_OK (0) or a negative MOE_ERR_* code.  No exception and no
 *     abort crosses the ABI.  Calls on a NULL context return MOE_ERR_INVALID.
 *   - Host pointers are read during the call only; the library copies what it keeps.
 *   - Device pointers (suffix _dev) are CUDA device addresses on cfg.device, owned by
 *     the caller, stream-ordered on the stream passed (a cudaStream_t, NULL = legacy).
 *   - One context is not thread-safe: serialise calls on it.  Distinct contexts are
 *     independent.
 */
#ifndef MOE_CACHE_H
#define MOE_CACHE_H

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

#define MOE_OK 0
#define MOE_ERR_INVALID (-1)     /* bad argument or configuration */
#define MOE_ERR_NOMEM (-2)       /* device or pinned-host allocation failed */
#define MOE_ERR_CUDA (-3)        /* a CUDA runtime/driver call failed */
#define MOE_ERR_TIMEOUT (-4)     /* a bounded device-side wait ran out (see moe_sync) */
#define MOE_ERR_STATE (-5)       /* call out of order (e.g. decode before residency) */
#define MOE_ERR_UNSUPPORTED (-6) /* shape or feature outside the library's limits */
#define MOE_ERR_DEVICE (-7)      /* the kernel flagged a bad route or slot (see moe_sync) */

/* Cache event kinds (key-components item 2 of the Luce Spark write-up). */
#define MOE_PIN_HIT 0  /* expert is in the calibrated pinned set */
#define MOE_RING_HIT 1 /* expert is resident in the layer's ring; recency refreshed */
#define MOE_MISS 2     /* expert copied from pinned host memory into a ring slot */

/* Placement policies for moe_set_residency. */
#define MOE_PLACE_CALIBRATED 0 /* top-P experts by routing count, ties -> lower index */
#define MOE_PLACE_UNIFORM 1    /* experts 0..P-1 (the write-up's naive offload) */

typedef struct moe_ctx moe_ctx; /* opaque; owned by the library */

typedef struct {
  int32_t n_layers;       /* L >= 1 */
  int32_t hidden;         /* H, multiple of 32, <= 4096 */
  int32_t n_experts;      /* E, top_k <= E <= 1024 */
  int32_t top_k;          /* k, 1..32 */
  int32_t inter;          /* expert SwiGLU width I, multiple of 32 */
  int32_t shared_inter;   /* shared expert width, multiple of 32; 0 = no shared expert */
  int32_t ring_slots;     /* R spare slots per layer, 0..32 (0 only with full residency) */
  int32_t use_rmsnorm;    /* 1: pre-norm residual stack h += MoE(RMSNorm(h)); 0: h = MoE(h) */
  float rms_eps;          /* RMSNorm epsilon (1e-6 for the pages' A3B shape) */
  int32_t device;         /* CUDA device ordinal */
  int32_t log_steps;      /* event-log capacity in decode steps; 0 -> 4096 */
  uint32_t wait_timeout_ms; /* bound on every device-side wait; 0 -> 2000 */
} moe_config;

/* Weights, canonical layouts (caller-owned, read during the call):
 *   expert_q4_0[l*E + e]: gate [I x H] | up [I x H] | down [H x I], each row-major with
 *     K = the column count contiguous, as GGUF Q4_0 blocks (18 bytes per 32 weights);
 *   shared_q4_0[l]: the same for the shared expert with width shared_inter (NULL if 0);
 *   router_bf16: [L][E][H] bf16 bit patterns; router_bias: [L][E] fp32 or NULL (zero);
 *   rms_gain: [L][H] fp32 or NULL (ones). */
typedef struct {
  const uint8_t *const *expert_q4_0;
  const uint8_t *const *shared_q4_0;
  const uint16_t *router_bf16;
  const float *router_bias;
  const float *rms_gain;
} moe_weights;

/* One cache event.  step counts decode steps since moe_create; rank is the position
 * in the token's top-k (descending logit); slot numbers pinned experts 0..P-1 in
 * ascending expert order and ring slot r as P + r; evicted is the expert a miss
 * displaced, or -1. */
typedef struct {
  int32_t step, layer, rank, expert, kind, slot, evicted;
} moe_event;

typedef struct {
  uint64_t steps;        /* decode steps completed since create */
  uint64_t accesses;     /* expert selections (steps * L * k) since the last reset */
  uint64_t pin_hits, ring_hits, misses, evictions;
  uint64_t bytes_copied; /* host-to-device bytes moved by misses since the last reset */
  uint64_t staged_misses; /* misses whose ring slot was still read in the same layer */
  uint64_t log_dropped;  /* events lost because the log wrapped before being read */
  int32_t device_error;  /* 0, or the kernel's error word (MOE_DEVERR_*) */
  int32_t n_pinned;      /* P of the current residency */
  float residency;       /* fraction passed to the last moe_set_residency */
  int32_t placement;     /* policy of the last moe_set_residency */
  uint64_t repins;       /* moe_recalibrate calls since the last moe_set_residency or create */
  uint64_t repin_copies; /* experts copied host-to-device by those re-pins */
  uint64_t miss_requests; /* miss requests the kernel has issued since create */
  uint64_t miss_served;   /* miss requests the proxy has taken from the mailbox since create */
  int32_t proxy_error;    /* 0; 1 the proxy met a malformed request, 2 a copy could not be
                             enqueued, 3 its completion signal could not be enqueued (each
                             left unsignalled: the step ends with MOE_ERR_TIMEOUT) */
  int32_t miss_path;      /* MOE_MISS_COPY_ENGINE or MOE_MISS_SM_PULL */
  uint64_t pulled_misses; /* misses served by the kernel's own reads of host memory since the last reset */
  uint64_t copies_timed;  /* proxy copies whose duration was measured (CUDA events on the side
                             stream around each copy) since the last reset */
  uint64_t copy_ns_timed; /* their summed device durations, ns: copies_timed * slot bytes /
                             copy_ns_timed is the host-to-device rate of the miss path itself */
} moe_stats_t;

#define MOE_DEVERR_BARRIER 1 /* grid barrier wait ran out */
#define MOE_DEVERR_MISS 2    /* wait for a miss copy ran out */
#define MOE_DEVERR_TMA 3     /* wait for a bulk shared-memory load ran out */
#define MOE_DEVERR_ROUTE 4   /* a logit was NaN: no valid top-k */
#define MOE_DEVERR_SLOT 5    /* an expert had no slot (cold with an empty ring) */
#define MOE_DEVERR_RANGE 6   /* a unit's share of a layer output was not finite or |v| >= 2^26 */

/* Miss-path variants for moe_set_miss_path. */
#define MOE_MISS_COPY_ENGINE 0 /* host proxy thread + cudaMemcpyAsync on a side stream (default) */
#define MOE_MISS_SM_PULL 1     /* the kernel's CTAs read the expert from mapped pinned host memory */

/* Create a context on cfg->device: allocates the pinned host tier that holds every
 * expert (the write-up's long tail "in system RAM", baguaai.com event core; "pinned host
 * memory", theneuralfeed.com key components item 2), the device tables, and the proxy
 * thread that serves miss copies.  weights may be NULL (then load layers with
 * moe_load_layer).  *out is set only on MOE_OK.  MOE_ERR_UNSUPPORTED when the decode
 * kernel's shared-memory plan for the shape does not fit the device. */
MOE_API int moe_create(const moe_config *cfg, const moe_weights *weights, moe_ctx **out);

/* Load (or replace) one layer's weights.  Experts go to the pinned host tier in the
 * library's slot layout; the shared expert, router, bias and gain go to the device.
 * Invalidates the residency: call moe_set_residency before decoding. */
MOE_API int moe_load_layer(moe_ctx *ctx, int32_t layer, const uint8_t *const *expert_q4_0,
                   const uint8_t *shared_q4_0, const uint16_t *router_bf16,
                   const float *router_bias, const float *rms_gain);

/* Choose the resident set (Luce Spark key components (1) and (2)).  fraction in [0, 1]
 * gives P = round(fraction * E) pinned experts per layer, chosen by placement from
 * hist ([L][E] counts; NULL = the library's own accumulated histogram); every layer
 * also gets ring_slots spare slots, emptied here.  Copies the pinned experts to the
 * device and synchronises the device.  fraction < 1 needs ring_slots >= 1. */
MOE_API int moe_set_residency(moe_ctx *ctx, float fraction, const uint32_t *hist, int32_t placement);

/* Online recalibration (the write-up's "self-tunes over time"; key components item 1,
 * routing frequencies accumulated from real requests).  Off the token graph: call it
 * between steps, e.g. every 64 tokens.  For every layer and expert, the routing counts
 * since the previous (re)calibration w (from the library's histogram) update the score
 * score <- floor(score / 2) + w, the score being seeded by the histogram the current
 * placement came from; the pinned set becomes the top-P experts by score (ties -> lower
 * index), P unchanged.  Only experts entering the set are copied (host tier -> the slot
 * an expert leaving the set frees); every ring is emptied.  Synchronises the device. */
MOE_API int moe_recalibrate(moe_ctx *ctx);

/* Replace one layer's router bias ([E] fp32 host array; NULL = zero), e.g. to follow
 * traffic whose popularity has drifted.  Synchronises the device. */
MOE_API int moe_set_router_bias(moe_ctx *ctx, int32_t layer, const float *bias);

/* One decode step (one token through all L layers) as one graph launch on stream (the
 * write-up's fused token, theneuralfeed.com key components item 3: one graph instead of
 * 40 per-layer graphs; the cache of items 1 and 2 decides where each expert is read):
 * reads x_dev [H] fp32, writes y_dev [H] fp32 (h_L of the stack, or MoE(x) when
 * use_rmsnorm = 0).  Routing, the histogram, the cache and the event log advance.
 * Asynchronous: device-side failures surface at moe_sync / moe_stats.
 * A step that misses waits inside the kernel for the library's proxy thread to issue
 * the copy; while such a step is in flight, no other host thread should make a CUDA call
 * that blocks on the device while holding the driver (a synchronous copy to pageable host
 * memory is one): the proxy's copy would queue behind it and the step would end with
 * MOE_ERR_TIMEOUT after wait_timeout_ms.  Synchronise (moe_sync, cudaStreamSynchronize)
 * before such calls. */
MOE_API int moe_decode_step(moe_ctx *ctx, const float *x_dev, float *y_dev, void *stream);

/* The same step on host buffers, synchronously: x_host [H] fp32 is staged to the
 * device, the step runs, y_host [H] receives the result.  Returns the step's status. */
MOE_API int moe_decode_step_host(moe_ctx *ctx, const float *x_host, float *y_host);

/* Batched prefill: n_tokens tokens through the whole stack at once, x_dev [T][H] ->
 * y_dev [T][H] (fp32, device, caller-owned, may not overlap), enqueued on stream.
 * The pages describe decode only; this is the same layer computed for a batch of tokens
 * (a 2048-token prompt through the 40-layer stack is the workload it is sized for), the
 * one place where the expert FFNs are dense contractions: per layer,
 * each token's top-k is the one the canonical fp32 logits give, as in decode (found
 * from tensor-core approximate logits, certified against exact canonical logits of the
 * candidates), so it agrees with a decode of the same hidden state; the routing
 * histogram accumulates as in decode), tokens grouped by expert, the expert SwiGLU FFNs
 * as grouped tensor-core GEMMs (Q4_0 weights dequantised to fp16, activations carried
 * as fp16 hi + lo pairs, fp32 accumulation), and the weighted combine plus shared
 * expert.  Needs every expert resident (moe_set_residency(1.0)): else MOE_ERR_STATE.
 * Shapes need experts % 16 == 0, hidden % 256 == 0 and inter, shared_inter % 256 == 0:
 * else MOE_ERR_UNSUPPORTED.  Scratch for the largest n_tokens seen so far is kept by
 * the context (about T * ((k + 1) * (8 * hidden + 4 * max(inter, shared_inter)) +
 * 18 * hidden + 32 * experts) bytes: 430 MB for 2048 tokens of the 2048-hidden,
 * 256-expert, top-8 shape); a larger n_tokens reallocates it, synchronising the device.
 * The cache's rings, counters and event log are not touched.  Errors of the kernels'
 * bounded waits surface at moe_sync as MOE_ERR_TIMEOUT.  Prefill calls on one context
 * share its scratch: calls that overlap on the GPU (different streams, no ordering)
 * race on it. */
MOE_API int moe_prefill(moe_ctx *ctx, const float *x_dev, int32_t n_tokens, float *y_dev, void *stream);

/* Prefill tracing: when non-NULL, moe_prefill writes its input and every layer's output
 * to h_trace_dev ([(L+1)][T][H] fp32) and each layer's top-k choices in rank order to
 * sel_trace_dev ([L][T][k] int32), T being the call's n_tokens.  Device pointers owned
 * by the caller; pass NULLs to stop. */
MOE_API int moe_set_prefill_trace(moe_ctx *ctx, float *h_trace_dev, int32_t *sel_trace_dev);

/* Wait for all work of the context and report a device-side failure as an error code
 * (MOE_ERR_TIMEOUT for a wait that ran out, MOE_ERR_DEVICE otherwise). */
MOE_API int moe_sync(moe_ctx *ctx);

/* Clear a device-side failure so decoding can resume: empties every ring (its state
 * may be torn), resynchronises the miss queue and the grid barrier. */
MOE_API int moe_clear_error(moe_ctx *ctx);

/* Counters, histogram and event log: the routing-frequency histogram that calibrated
 * placement accumulates (theneuralfeed.com key components item 1) and the hit / miss /
 * eviction record behind the write-up's cold-hit rate (items 1 and 2, the 36% -> 7%
 * figure).  Synchronises the device.  hist_out: [L][E] or
 * NULL.  log_out: room for log_cap events or NULL; receives the events of the steps
 * not yet read, oldest first, and *log_n their count.  reset != 0 zeroes the counters
 * and the histogram after reading. */
MOE_API int moe_stats(moe_ctx *ctx, moe_stats_t *out, uint32_t *hist_out, moe_event *log_out,
              size_t log_cap, size_t *log_n, int32_t reset);

/* Tracing: when h_trace_dev is non-NULL, every decode step writes its input and each
 * layer's output ([(L+1)][H] fp32) there; w_trace_dev ([L][k] fp32, or NULL) receives
 * the routing weights.  Pass NULLs to stop.  Device pointers owned by the caller. */
MOE_API int moe_set_trace(moe_ctx *ctx, float *h_trace_dev, float *w_trace_dev);

/* Phase timing: when stamps_dev is non-NULL, every decode step writes timing marks
 * there.  The buffer holds n_words uint64 and must hold at least
 * (L + 1) * 32 + L * n_sm * 4 words (n_sm = the device's SM count, one CTA per SM):
 * else MOE_ERR_INVALID and nothing changes.  Layout: first [(L+1)][32] marks of CTA 0 in
 * SM clock cycles (clock64); per layer l: [l][0] layer start, [1] the previous layer's
 * output complete, [2] h updated, [3] own logits published and input quantised, [4] all
 * logits read, [5] routing and cache decided, [6] unit loads issued, [7] gate/up
 * computed, [8] units done, [9] arrival posted, [10..19] finer marks (norm, own logit,
 * input quantised, top-k (with this CTA's unit loads issued inside it when its expert
 * is pinned), cache, warp 0's pinned-slot lookup, SwiGLU, down part landed, down adds
 * issued, fence); [L][0] kernel start and [L][2] kernel end in cycles, [L][4]
 * and [L][5] the same two instants on the global timer (ns), which converts cycles to
 * ns; [L][1] prologue done (cycles).  Then [L][n_sm][4] global-timer marks (ns) of every
 * CTA: [0] routing decided, [1] units done, [2] arrival posted, [3] own logits
 * published.  While a buffer is set, steps run the kernel instance that carries these
 * marks (a few percent slower than the default one).  NULL stops it (n_words ignored). */
MOE_API int moe_set_phase_trace(moe_ctx *ctx, uint64_t *stamps_dev, size_t n_words);

/* Miss path (how a cold expert crosses PCIe; theneuralfeed.com, key components item 2): with
 * MOE_MISS_COPY_ENGINE (the default) the kernel posts a cold expert to a host-mapped
 * mailbox, the library's proxy thread copies it pinned host -> ring slot with
 * cudaMemcpyAsync on a side stream and signals the kernel through a stream memory write;
 * with MOE_MISS_SM_PULL the CTAs that compute the expert read it themselves from the
 * mapped pinned host tier and write the ring slot, with no host thread involved.  Both
 * give the same routing, event log and outputs.  Other values: MOE_ERR_INVALID. */
MOE_API int moe_set_miss_path(moe_ctx *ctx, int32_t mode);

/* Speculative loads while a layer's routing is computed (the HBM would otherwise idle):
 * the layer's pinned experts ordered by the placement histogram (decayed by
 * recalibration), most frequently routed first.  The units of the first n_preload are
 * loaded straight into the shared memory of the CTAs that will compute them if they are
 * routed (n_preload x inter/32 CTAs, one unit each); after routing, every CTA derives
 * the same assignment: a preloaded unit whose expert was routed is computed at once,
 * and the CTAs that guessed wrong take the units of the other routed experts.  The next
 * n_l2 experts are prefetched into L2 only.  Changes no result, only where and when bytes
 * are read; wrong guesses cost HBM bandwidth that routing leaves idle.  n_preload <=
 * min(top_k, 16) and n_preload + n_l2 <= 32, else MOE_ERR_INVALID; (0, 0), the default,
 * turns it off.  n_preload is taken as 0 when the device has fewer SMs than a layer has
 * units.  Synchronises the device. */
MOE_API int moe_set_prefetch(moe_ctx *ctx, int32_t n_preload, int32_t n_l2);

/* Host-to-device rate of the miss path's own copy: n_copies expert slots copied back to
 * back from the library's pinned host tier into device slots with cudaMemcpyAsync on the
 * side stream the proxy uses (after one untimed pass), timed with CUDA events.  *gbs =
 * n_copies * slot bytes / elapsed, in GB/s (1e9 B/s).  Needs a residency; synchronises
 * the device; do not call it while a decode step is in flight. */
MOE_API int moe_measure_h2d(moe_ctx *ctx, int32_t n_copies, double *gbs);

/* Fault injection for tests: the miss proxy issues the next n copies but never
 * signals them, so the kernel's bounded wait runs out (no GPU fault involved).  The
 * completion word is monotonic, so a later signal also completes earlier copies; drop
 * every signal of a step to make it time out.  moe_clear_error cancels the count. */
MOE_API int moe_debug_drop_signals(moe_ctx *ctx, int32_t n);

/* Weights for moe_decode_step_noalloc: device memory owned by the caller, every expert
 * resident, in the library's own layouts (a byte regrouping of the canonical Q4_0
 * blocks, values unchanged):
 *   experts_dev: [L][E] routed experts, one slot each, slots slot_bytes(I) apart, where
 *     slot_bytes(W) = (W / 32) * 54 * H rounded up to a multiple of 256.  A slot is W/32
 *     units of 54 H bytes; unit rb holds, in order: four gate/up tiles (gate rows
 *     32rb..+15, gate rows 32rb+16..+31, up rows 32rb..+15, up rows 32rb+16..+31), each
 *     [16 rows x H/32 blocks x 16 nibble bytes] then [16 rows x H/32 fp16 scales]; then
 *     the nibble bytes of Q4_0 block rb of every down row j = 0..H-1 ([H x 16] bytes);
 *     then the fp16 scales of those blocks ([H] x 2 bytes).
 *   shared_dev: [L] shared experts in the same layout with W = shared_inter, slots
 *     slot_bytes(shared_inter) apart; NULL when shared_inter = 0.
 *   router_dev: [L][E][H] bf16 bit patterns (the canonical router rows).
 *   bias_dev: [L][E] fp32 or NULL; gain_dev: [L][H] fp32 or NULL. */
typedef struct {
  const uint8_t *experts_dev;
  const uint8_t *shared_dev;
  const uint16_t *router_dev;
  const float *bias_dev;
  const float *gain_dev;
} moe_noalloc_weights;

/* The decode step of moe_decode_step for callers that cannot allocate device memory:
 * code that runs under a fixed memory budget or its own allocator, code inside a
 * stream-capture region where cudaMalloc is not allowed, or a real-time path that must
 * not take the implicit synchronisation an allocation can bring.  No paper passage
 * corresponds to it; it is a deployment variant of the same kernel and arithmetic.
 *
 * It allocates nothing: no context, no graph, no cudaMalloc / cudaFree.  Its scratch
 * (control block with the arrival counter and error word, output accumulators,
 * published logits, slot tables, histogram, one step of event log) lives in a static
 * 2 MiB device array that every GPU which loads the library holds until the process
 * exits; the call rejects shapes whose scratch would not fit (MOE_ERR_UNSUPPORTED).  All
 * experts must be resident (no cache, no miss path); cfg's ring_slots and log_steps are
 * ignored.  Reads x_dev [H], writes y_dev [H] on stream (the current device must be
 * cfg->device).  The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) and sets the kernel's shared-memory limit: make that first call
 * before any stream capture.  Each call resets the parts of the array a step depends on
 * (control block, accumulators, logit words, slot tables) and leaves the rest (histogram
 * and event log) as the kernel writes it; every call shares the array, so calls that
 * overlap on the GPU, on any stream, race.  Asynchronous; returns the launch status.  A
 * step that fails on the device (a bounded wait that ran out, an out-of-range value)
 * writes NaN to every element of y_dev, since this entry point has no moe_sync. */
MOE_API int moe_decode_step_noalloc(const moe_config *cfg, const moe_noalloc_weights *w,
                                    const float *x_dev, float *y_dev, void *stream);

/* Free everything.  NULL is a no-op. */
MOE_API void moe_destroy(moe_ctx *ctx);

/* Static description of a status code. */
MOE_API const char *moe_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_CACHE_H */
