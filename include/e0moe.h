/*
 * e0moe.h -- C ABI of the B200 (sm_100a) streaming int4 MoE block with a prerouter.
 *
 * What the calls compute (sources are named by page title and section; no page prints
 * code):
 *   [G] "The Other Half of the Memory Wall: Serving 35B MoEs from SSD with Trained
 *       Routing Prediction" (reading guide): "Temel fikirler", "Yöntem / Ön
 *       Yönlendirici Başlık Mimarisi", "Yöntem / Birleştirilmemiş Adaptör Yürütme",
 *       "Yöntem / Üç Aşamalı Eğitim", "Temel terimler", "Sorular".
 *   [A] "Edge0 serve un MoE da 35B a 20 token al secondo in 3 GiB" (ai.info), section
 *       "La versione da 35B usa 256 esperti distribuiti su 40 livelli".
 *
 * Conventions for every call:
 *   - Every function returns an int status (E0_OK or a negative E0_ERR_*); the message
 *     of the last failure on the calling host thread is e0_last_error().  Nothing here
 *     aborts, traps or prints.
 *   - The caller owns every device buffer and the pinned host expert store; pointers are
 *     plain device (or pinned host) addresses and are only read during the enqueued work.
 *     The library owns only the opaque e0_ctx (its workspaces, routing tables, slot table,
 *     side stream and events), created by e0_create and released by e0_destroy.
 *   - Work is enqueued on the caller's CUDA stream (passed as void*, a cudaStream_t) and
 *     is asynchronous.  Errors found on the device (an expert index out of range, a
 *     duplicated index, a slot-table tag that does not match the expert a kernel expects)
 *     are latched in a device error word; e0_sync_status() synchronises and reports it.
 *   - Layouts are row-major and contiguous.  bf16 is IEEE bfloat16.  One expert is one
 *     contiguous blob (the int4 affine group-64 format of [G] "Temel fikirler" and [A]):
 *         gate.codes [I, d/2] u8 | gate.scale [I, d/64] bf16 | gate.min [I, d/64] bf16 |
 *         up.codes   [I, d/2]    | up.scale   [I, d/64]      | up.min   [I, d/64]      |
 *         down.codes [d, I/2]    | down.scale [d, I/64]      | down.min [d, I/64]
 *     code element 2i is the low nibble of byte i, w = scale * q + min, q = 0..15; groups
 *     of 64 run along K (the input dimension).  1,769,472 bytes at d=2048, I=512.
 *   - Supported sizes: d % 256 == 0 (d <= 4096), I % 128 == 0 (I <= 4096), 1 <= k <= 8,
 *     k <= E <= 256, r <= 32, group == 64, head_hidden % 8 == 0, E % 4 == 0 when
 *     head_onehot = 1.  Weight matrices, blobs and the host store are 16-byte aligned.
 */
#ifndef E0MOE_H
#define E0MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  E0_OK = 0,
  E0_ERR_INVALID_ARG = -1,   /* rejected before anything was enqueued */
  E0_ERR_CUDA = -2,          /* a CUDA runtime call failed (message names it) */
  E0_ERR_OOM = -3,           /* a workspace allocation failed */
  E0_ERR_STAGING = -4,       /* an expert copy into the HBM pool could not be issued */
  E0_ERR_SLOT_MISMATCH = -5, /* a kernel found a pool slot holding another expert */
  E0_ERR_TIMEOUT = -6,       /* a bounded device-side wait gave up */
  E0_ERR_DEVICE = -7         /* a kernel rejected its data (index out of range, duplicate,
                                an activation beyond the one-launch decode's fp16 operand range) */
};

typedef struct e0_ctx e0_ctx;

/* Model geometry.  head_hidden = 0 selects the linear head l(u); > 0 adds
 * fc2(gelu_erf(fc1 u + b1)) + b2 ([G] "Ön Yönlendirici Başlık Mimarisi").
 * head_onehot = 1 makes the head input u = [x; onehot_k(cur); onehot_k(prev)] (width
 * d + 2E); 0 makes u = x.  lora_scale is alpha / r of [G] "Birleştirilmemiş Adaptör
 * Yürütme".  rms_eps is the RMSNorm epsilon. */
typedef struct {
  int d_model, n_experts, d_ff, top_k, group, lora_rank, head_hidden, head_onehot;
  float rms_eps, lora_scale;
} e0_dims;

/* One layer's weights (device pointers, all owned by the caller).
 * experts  [E][blob]  routed experts; may be NULL for a layer served only from the
 *                     streaming pool (e0_stream_register).
 * shared   [blob]     the always-on shared expert ([A]).
 * lora_*   bf16: Ag, Au [r, d]; Bg, Bu [I, r]; Ad [r, I]; Bd [d, r]  (NULL: no LoRA).  The
 *          delta is unmerged: g += c Bg (Ag x), u += c Bu (Au x), y_s += c Bd (Ad a_s)
 *          ([G] "Birleştirilmemiş Adaptör Yürütme"; on the shared expert only, as
 *          "Üç Aşamalı Eğitim" places it).
 * router_w bf16 [E, d];  norm_w bf16 [d] (RMSNorm gamma). */
typedef struct {
  const void *experts;
  const void *shared;
  const void *lora_Ag, *lora_Bg, *lora_Au, *lora_Bu, *lora_Ad, *lora_Bd;
  const void *router_w;
  const void *norm_w;
} e0_layer;

/* One layer's prerouter head (device pointers; w_lin NULL = the layer has no head).
 * w_lin bf16 [E, d (+2E)]; fc1_w bf16 [H, d (+2E)], fc1_b [H], fc2_w [E, H], fc2_b [E]
 * (fc* only when head_hidden > 0). */
typedef struct {
  const void *w_lin, *fc1_w, *fc1_b, *fc2_w, *fc2_b;
} e0_head;

/* Counters of the streaming tier and the decode loop (host-side accounting). */
typedef struct {
  uint64_t steps;              /* e0_moe_stack_decode calls */
  uint64_t staged_experts;     /* expert blobs copied into the pool */
  uint64_t staged_bytes;       /* host-link bytes issued by the staging copies */
  uint64_t prefetched_experts; /* of which issued from a prediction (one token ahead) */
  uint64_t ondemand_experts;   /* of which issued after the layer's own router ran */
  uint64_t dropped;            /* routed experts that were not staged (always 0) */
  double   stage_ms;           /* sum of copy durations (side-stream event pairs) */
  double   exposed_wait_ms;    /* compute-stream time spent waiting on staging */
  uint64_t kernel_launches;    /* kernels this context has launched */
  uint64_t gemm_timed;         /* expert-GEMM launches timed (see e0_debug_time_gemm) */
  double   gemm_ms;            /* their summed durations (event pairs on the launch stream) */
  uint64_t hit_experts;        /* staging requests served by an expert already in its slot
                                  (persistent per-layer sets; no copy) */
} e0_stats;

/* Create a context on the current CUDA device.  n_layers >= 1; max_tokens bounds T of
 * every call (and B of decode).  Allocates the workspaces.  Errors: INVALID_ARG (sizes
 * outside the supported set), OOM, CUDA. */
int e0_create(const e0_dims *dims, int n_layers, int max_tokens, e0_ctx **out);

/* Release the context and everything it allocated (synchronises its streams). */
int e0_destroy(e0_ctx *ctx);

/* Record the weights of all layers.  layers[n_layers]; heads[n_layers] or NULL (no
 * heads).  Only the pointers are stored; the buffers must stay valid while the context
 * uses them.  Heads on layer N predict layer N+1 ([G] "Ön Yönlendirici Başlık
 * Mimarisi"; 33 heads on 40 layers per [A]). */
int e0_register_model(e0_ctx *ctx, const e0_layer *layers, const e0_head *heads);

/* One MoE block on T tokens of `layer` ([G] "Temel fikirler"; [A]):
 *   x = bf16(RMSNorm(h)), logits = W_r x (fp32), S = top-k(logits) (descending, ties to
 *   the lower index) or route_idx, w = softmax(logits[S]) over the selection,
 *   y = sum_j w_j E_{S_j}(x) + E_shared(x) with the shared expert's unmerged LoRA.
 * h        [T, d] bf16 device.
 * route_idx NULL, or [T, k] int32 device: the routing to use ("prediction as routing");
 *          a row whose first entry is -1 uses the layer's own router.
 * y_bf16   [T, d] bf16 device (required);  y_f32 [T, d] fp32 or NULL.
 * idx_out  [T, k] int32 or NULL;  gate_out [T, k] fp32 or NULL.
 * Errors: INVALID_ARG (layer, T, NULL h/y), DEVICE (latched: route index out of range or
 * duplicated within a token). */
int e0_moe_layer_forward(e0_ctx *ctx, int layer, const void *h, int T, const int32_t *route_idx,
                         void *y_bf16, float *y_f32, int32_t *idx_out, float *gate_out,
                         void *stream);

/* The prerouter head of `layer` on normed inputs ([G] "Ön Yönlendirici Başlık
 * Mimarisi"): z = l(u) (+ fc2(gelu_erf(fc1 u + b1)) + b2), u = [x; onehot(cur);
 * onehot(prev)]; pred = top-k(z) is layer+1's routing at the next token.
 * x [T, d] bf16 device; cur_idx, prev_idx [T, k] int32 device or NULL (zero one-hot);
 * pred_idx [T, k] int32 device (required); logits_out [T, E] fp32 or NULL.
 * Errors: INVALID_ARG (no head on `layer`, sizes). */
int e0_prerouter_predict(e0_ctx *ctx, int layer, const void *x, int T, const int32_t *cur_idx,
                         const int32_t *prev_idx, int32_t *pred_idx, float *logits_out,
                         void *stream);

/* Streaming tier ([G] "Temel fikirler": weights stay off the GPU, only the working set
 * is resident; "Temel terimler": staged decode with a fixed-slot double buffer and a
 * GPU slot table, and the incremental sticky-slot stack).  host_blob: pinned host memory
 * [L][E][expert_bytes] (caller-owned, must stay valid).  Allocates the HBM pool of
 * pool_layers x slots_per_layer blobs; slots_per_layer must be >= k and >= the number of
 * distinct experts a layer routes to in one step.
 *   2 <= pool_layers < n_layers: shared slot sets (layer l uses set l % pool_layers), the
 *     double buffer of staged decode: every staging rewrites its set.
 *   pool_layers == n_layers: one persistent set per layer, kept across steps (sticky
 *     slots): an expert already in the set is not copied again; a missing one replaces
 *     the least recently needed slot not needed now (empty first, ties to the lower
 *     slot).  With slots_per_layer = k at one stream this rewrites only the slots whose
 *     expert changed; with more slots it is a least-recently-used expert cache in HBM.
 * Errors: INVALID_ARG, OOM. */
int e0_stream_register(e0_ctx *ctx, const void *host_blob, size_t expert_bytes, int pool_layers,
                       int slots_per_layer);

/* Stage the experts host_idx[0..n) of `layer` into the layer's pool slot set: waits (on
 * the side stream) until the previous user of that slot set has finished on
 * compute_stream, issues one cudaMemcpyAsync per expert blob, writes the slot table and
 * records the "ready" event that the consuming layer waits on.  host_idx is host memory.
 * Errors: INVALID_ARG, STAGING (a copy could not be issued). */
int e0_stage_experts(e0_ctx *ctx, int layer, const int32_t *host_idx, int n, void *compute_stream);

/* One decode step of B streams through all layers.
 * h_in [L, B, d] bf16 device (each layer's generated MoE input); y_out [L, B, d] bf16;
 * y_f32 [L, B, d] fp32 or NULL.  Routing of layer N at step t: the head prediction of
 * layer N-1 made at step t-1 when layer N-1 has a head and t > 0, else the layer's own
 * router ([G] "Temel fikirler", "Sorular").  Every head runs and writes step t+1's
 * routing into the context.  step == 0 starts a new sequence.  streaming = 1 serves the
 * routed experts from the pool (e0_stream_register), 0 from the resident weights.
 * chained = 1 feeds bf16(h_N + y_{N-1}) to layer N (a dependency check); 0 feeds h_N.
 * Errors: INVALID_ARG, STAGING, CUDA; DEVICE/SLOT_MISMATCH are latched.  The one-launch
 * kernel (B = 1, resident experts) holds activations as fp16 tensor-core operands: a
 * finite activation at or beyond 65520 in magnitude latches DEVICE and the step's
 * outputs are not valid (e0_debug_force_general takes such models through the per-layer
 * kernels). */
int e0_moe_stack_decode(e0_ctx *ctx, const void *h_in, int B, int step, void *y_out, float *y_f32,
                        int streaming, int chained, void *stream);

/* e0_moe_stack_decode with the step's input and outputs in host memory: h_host [L, B, d]
 * bf16, y_host [L, B, d] bf16, y_f32_host [L, B, d] fp32 or NULL, all caller-owned and
 * page-locked for the copies to be asynchronous (pageable memory works, but its copies
 * block the calling thread).  The library copies them through two alternating device
 * staging buffers that it owns, on a copy stream of its own, ordered with the step on
 * `stream` by events, so that the input copy of the next call and the output copy of this
 * one overlap the steps' kernels.  The outputs are in host memory once the call's copies
 * have completed: after e0_host_io_wait(ctx, stream) and a synchronisation of `stream`.
 * The input buffer must not change, and the output buffers must not be read, before then.
 * Same routing, streaming, step rules and errors as e0_moe_stack_decode; OOM if the
 * staging buffers (2 x L x max_tokens x d bf16, twice more with fp32 outputs) cannot be
 * allocated. */
int e0_moe_stack_decode_host(e0_ctx *ctx, const void *h_host, int B, int step, void *y_host, float *y_f32_host,
                             int streaming, int chained, void *stream);
/* Make `stream` wait for every copy issued so far by e0_moe_stack_decode_host and
 * e0_moe_prefill_stack_host (no-op if there was none).  Errors: INVALID_ARG (NULL
 * context), CUDA. */
int e0_host_io_wait(e0_ctx *ctx, void *stream);

/* Streaming decode mode ([G] "Sonuçlar": prerouter prefetch against fully reactive
 * on-demand loading).  reactive = 0 (default): a layer preceded by a head is routed by
 * that head's prediction made one token earlier and its experts are copied while the
 * previous layer computes; other layers stage on demand.  reactive = 1: every layer
 * routes with its own router and its experts are copied only after that router ran; no
 * head runs (e0_get_routing reports -1 predictions).  Changing the mode starts a new
 * sequence (the next decode call must be step 0).  Errors: INVALID_ARG. */
int e0_stream_mode(e0_ctx *ctx, int reactive);

/* One prefill chunk of T tokens through all layers ([G] "Temel fikirler", "Sorular":
 * prediction as routing, one token ahead).  h_in [L, T, d] bf16 (each layer's generated
 * MoE input), y_out [L, T, d] bf16, y_f32 [L, T, d] or NULL, idx_out [L, T, k] int32 or
 * NULL (the routing each layer used).  Layer N+1 routes token t by the head of layer N
 * on token t-1; token 0, and every layer not preceded by a head, use their own router.
 * From 64 tokens the experts run as tcgen05 grouped GEMMs (fp16 operands from the int4
 * weights, fp32 accumulation).  Linear heads without one-hot inputs only.
 * Errors: INVALID_ARG, CUDA. */
int e0_moe_prefill_stack(e0_ctx *ctx, const void *h_in, int T, void *y_out, float *y_f32, int32_t *idx_out,
                         void *stream);

/* Combine order of the tensor-core prefill path (e0_moe_layer_forward and the prefill
 * stacks from 64 tokens).  0 (default): the down GEMM adds each expert's gate-weighted
 * rows into the fp32 output with vector reductions in completion order, so the last bits
 * of y can differ between runs.  1: each (expert slot, token) contribution is stored once
 * in its own plane ([k + 1, max_tokens, d] fp32 of device memory, allocated on the first
 * call with on = 1 and kept until e0_destroy) and the planes are summed in slot order
 * (routed slots 0..k-1, then the shared expert), so y is bit-reproducible; it reads and
 * writes (k + 1) * T * d * 4 more bytes per layer.  Errors: INVALID_ARG, OOM. */
int e0_prefill_fixed_order(e0_ctx *ctx, int on);

/* e0_moe_prefill_stack with the input and outputs in host memory (pinned, so that the
 * copies are asynchronous): h_host [L, T, d] bf16, y_host [L, T, d] bf16, y_f32_host
 * [L, T, d] or NULL; idx_out [L, T, k] int32 device memory or NULL.  Layer l's input is
 * copied in while layer l-1 computes and its outputs copied out while layer l+1 computes
 * (two copy streams of the context, two alternating device staging buffers of max_tokens
 * x d, allocated on the first call).  The outputs are complete after
 * e0_host_io_wait(ctx, stream) and a synchronisation of `stream`; the host buffers must
 * stay valid until then.  Errors: as e0_moe_prefill_stack, and OOM. */
int e0_moe_prefill_stack_host(e0_ctx *ctx, const void *h_host, int T, void *y_host, float *y_f32_host,
                              int32_t *idx_out, void *stream);

/* Routing the last e0_moe_stack_decode used and predicted, copied to host memory:
 * idx [L, B, k] (routing used at that step), pred [L, B, k] (next step's routing; -1 for
 * layers without a head).  Synchronises the context's last stream. */
int e0_get_routing(e0_ctx *ctx, int B, int32_t *idx_host, int32_t *pred_host);

int e0_get_stats(e0_ctx *ctx, e0_stats *out);

/* Synchronise the last stream used and return E0_OK or the latched device error
 * (DEVICE, SLOT_MISMATCH, TIMEOUT); the error word is cleared. */
int e0_sync_status(e0_ctx *ctx);

/* One MoE block, like e0_moe_layer_forward, for callers that cannot allocate device memory:
 * a serving runtime that fixes its memory plan at start-up and forbids allocation later,
 * code that runs while another component owns the device allocator, or code that must not
 * risk the device synchronisation an allocation can cause.  No context is needed and
 * nothing is allocated (no cudaMalloc, cudaFree or allocating library call).  The pages
 * have no counterpart of this call.
 * dims, layer   host structs as for e0_create / e0_register_model (layer->experts required).
 * h, T, route_idx, y_bf16, y_f32, idx_out, gate_out   as for e0_moe_layer_forward.
 * dev_status    device int or NULL: the kernels OR their error bits into it (1 = index out
 *               of range, 2 = duplicated index); the caller zeroes it.  With NULL, device
 *               errors are not reported.
 * Scratch: one fixed 4 MiB device array inside the library (every GPU that loads the
 * library holds it until the process exits).  A call whose intermediates do not fit is
 * rejected with E0_ERR_INVALID_ARG and a message naming the bytes needed (at d = 2048,
 * E = 256, I = 512, k = 4, r = 16 the limit is about T = 200 tokens).  The array's device
 * address belongs to the CUDA context the call runs in (a device reset or a second context
 * on the same device has its own copy): the first call in each context looks it up
 * (cudaGetSymbolAddress, under a lock, so concurrent first calls from several host threads
 * are safe); make that first call outside any stream capture.  All calls share the one array and each overwrites it:
 * calls on one device whose work overlaps on the GPU (for example on two streams)
 * race and give wrong results, so serialise them.
 * Errors: INVALID_ARG (arguments, sizes beyond the maximum), CUDA. */
int e0_moe_layer_forward_noalloc(const e0_dims *dims, const e0_layer *layer, const void *h, int T,
                                 const int32_t *route_idx, void *y_bf16, float *y_f32, int32_t *idx_out,
                                 float *gate_out, int *dev_status, void *stream);

/* Host-side fault injection for tests (no GPU fault is involved):
 * e0_debug_fail_staging_after(ctx, n): the (n+1)-th next staging copy is refused, so the
 *   staging call returns E0_ERR_STAGING.
 * e0_debug_set_slot_tag(ctx, set, slot, expert): the next slot-table write of pool set
 *   `set` tags `slot` with `expert`; the expert kernels must then latch SLOT_MISMATCH. */
int e0_debug_fail_staging_after(e0_ctx *ctx, int n);
int e0_debug_set_slot_tag(e0_ctx *ctx, int pool_set, int slot, int expert);
/* Streaming test hooks:
 * e0_debug_stream_log(ctx, log): from the next streamed layer on, copy the slot tags of the
 *   layer's pool set, as its expert kernels read them, into log[layer * slots + s] (int32
 *   device buffer [L][slots_per_layer], caller-owned; one device-to-device copy on the
 *   compute stream per layer); NULL stops it.
 * e0_debug_pool_slot(ctx, set, slot, &ptr): the device address of one pool slot's blob. */
int e0_debug_stream_log(e0_ctx *ctx, int32_t *log);
int e0_debug_pool_slot(e0_ctx *ctx, int pool_set, int slot, void **out);

/* Test hooks of the one-launch decode path (B = 1, resident experts, linear heads):
 * e0_debug_decode_stall(ctx, cta, timeout_ns): in the next decode step CTA `cta` waits for
 *   a word that nothing writes, and every device wait of that launch gives up after
 *   timeout_ns; the step must end with E0_ERR_TIMEOUT from e0_sync_status (the context
 *   stays usable).  timeout_ns = 0 restores the default budget (2 s).
 * e0_debug_force_general(ctx, on): 1 sends every decode step through the per-layer
 *   kernels instead of the one-launch kernel (for comparisons); 0 restores the default. */
int e0_debug_decode_stall(e0_ctx *ctx, int cta, unsigned long long timeout_ns);
/* Expert path of e0_moe_layer_forward: 0 = tensor cores (tcgen05) from 64 tokens per call,
 * CUDA cores below (default); 1 = CUDA cores always; 2 = tensor cores whenever the context
 * was created with max_tokens >= 64.  For comparisons between the two paths. */
int e0_debug_prefill_path(e0_ctx *ctx, int mode);
/* Decode implementation of e0_moe_stack_decode (resident experts): 0 = default (the
 * one-launch kernel at B = 1 where it applies, the phased kernels for unchained steps of
 * up to 8 streams, per-layer kernels otherwise), 1 = one-launch kernel, 2 = graph replay
 * of the per-layer kernels, 3 = per-layer kernels launched one by one, 4 = phased kernels
 * (six kernels per step over every layer, programmatic dependent launch; unchained steps,
 * B <= 8, head_hidden <= 512; other steps fall back to the default). */
int e0_debug_decode_mode(e0_ctx *ctx, int mode);
/* Profiling: the following one-launch decode steps write %globaltimer stamps (uint64,
 * [grid][L][16], caller-owned device buffer; NULL stops it).  Returns the grid size. */
int e0_debug_decode_trace(e0_ctx *ctx, unsigned long long *buf);
/* Profiling of the phased decode kernels: e0_debug_phase_timing(ctx, 1) makes the
 * following phased steps launch their six kernels one after another (no programmatic
 * overlap) with a CUDA event before each and after the last; e0_debug_phase_times adds the
 * elapsed times up per kernel (ms6[0..5]: norm, bf16 rows, routing, gate/up, sums and t_d,
 * down), synchronising on the events, and reports how many steps were timed since the
 * context was created.  Results are unchanged. */
int e0_debug_phase_timing(e0_ctx *ctx, int on);
int e0_debug_phase_times(e0_ctx *ctx, double *ms6, unsigned long long *steps);
int e0_debug_force_general(e0_ctx *ctx, int on);
/* Schedule of the one-launch decode kernel on unchained steps (every layer's input
 * given, none read from another layer's output): 1 (default) = flat — each phase's work
 * (reactive routers, x rows, gate/up, down) over all layers is one list cut into
 * contiguous cost-balanced shares across the CTAs, so that a CTA streams long runs of one
 * or two layers and waits on other CTAs only between phases; 0 = layers in order, every
 * CTA on a share of each layer.  Chained steps always run in order.  Results are
 * bit-identical under both.  E0_ERR_INVALID_ARG unless 0 or 1. */
int e0_debug_decode_flat(e0_ctx *ctx, int on);
/* Profiling: on = 1 brackets every tensor-core expert-GEMM launch (prefill) with a CUDA
 * event pair on its stream; e0_get_stats then reports their count and summed duration
 * (gemm_timed, gemm_ms; it synchronises on the events).  on = 0 stops it.  The pages
 * have no counterpart; for the benchmark's per-kernel roofline. */
int e0_debug_time_gemm(e0_ctx *ctx, int on);
/* The work-item list of one CTA of the one-launch decode kernel, built by the same host
 * function the context uses (host only: no context, no device call).  For a model of
 * n_layers layers of shape `dims` whose layer l carries a prerouter head where
 * has_head[l] != 0 and the shared expert's LoRA where has_lora[l] != 0, on a grid of
 * n_ctas CTAs, under the flat (flat = 1) or in-order (0) schedule, for a sequence's first
 * step (step0 = 1: every layer routes with its own router) or a later one, fills
 * items_out[0, *n_out) with CTA `cta`'s list in execution order.  Item word: bits 0-3
 * kind (0 router rows of a reactive layer, 1 its top-k, 2 x rows, 3 gate/up units,
 * 4 down rows), bit 4 set on the first item of its kind group (x items: R, XR, GU) for its
 * layer in this list, bits 8-15 layer, bits 16-39 first unit, bits 40-63 unit count.
 * Units of a layer: router rows 0..E-1; x rows = the head's E rows, then 2r LoRA A rows
 * (A_g, A_u), then the k router rows of a predicted layer's experts; gate/up = (slot,
 * index) slot-major over k+1 slots of d_ff; down = d_model output rows.  The caller owns
 * items_out (cap entries).  E0_ERR_INVALID_ARG on NULL pointers, n_layers outside 1..64,
 * n_ctas < 1, cta outside [0, n_ctas), dims the kernel cannot take, or a longer list
 * than cap. */
int e0_decode_items(const e0_dims *dims, int n_layers, const uint8_t *has_head, const uint8_t *has_lora, int n_ctas,
                    int flat, int step0, int cta, uint64_t *items_out, int cap, int *n_out);

/* Message of the last failing call on this host thread ("" if none). */
const char *e0_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* E0MOE_H */
