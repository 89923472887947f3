/*
 * kie.h -- C ABI of the persistent batch-1 decode library (libkie.so).
 *
 * What it computes.  One single-request decode path of a pre-norm decoder,
 * run as ONE persistent kernel: every layer of every step back to back, with
 * no kernel launch between layers or tokens, the sampled token fed straight
 * back on the device ("monokernel" bullet of the Kog Inference Engine
 * write-ups: the entire decode path as one persistent kernel with no launches
 * between layers; "Software versus silicon" section: prefill, decode and
 * LM-head sampling in one go, with grid synchronisations and per-launch
 * overhead removed).  Per step: embedding gather, RMSNorm, fused QKV GEMV,
 * rotate-half RoPE, KV-cache append, grouped-query attention over the cache,
 * O GEMV + residual, RMSNorm, gate/up GEMV + SwiGLU, down GEMV + residual,
 * final RMSNorm, LM-head GEMV, greedy argmax (lowest index on ties).  Lane
 * models (lane-structured transformer bullet: 8 parallel lanes; Delayed Tensor
 * Parallelism bullet: each cross-lane sum delayed by delta layers) run every
 * sublayer per lane slice and add  M_i u_i  to the residual at the start of
 * layer i + delta (pending sums are added before the final norm).
 *
 * Precision: weights and KV cache in the storage dtype (FP16 per the pages'
 * results table, or bfloat16); activations, accumulators and logits fp32.
 *
 * Conventions for every call:
 *   - returns KIE_OK (0) or a negative kie_status; kie_strerror() names it;
 *   - calls are synchronous: they return after the work queued on the
 *     context's stream has finished;
 *   - after KIE_ERR_DEVICE_TIMEOUT, KIE_ERR_NONFINITE or KIE_ERR_CUDA the
 *     context is poisoned: every later kie_prefill and kie_decode* call
 *     returns KIE_ERR_POISONED.  kie_destroy and the calls that only read
 *     state back (kie_get_stats, kie_copy_kv, kie_get_profile,
 *     kie_get_trace) still work, so a failed launch can be inspected; the
 *     settings calls still take effect but nothing runs again.
 *   - a context is not thread-safe; use one per host thread.
 */
#ifndef KIE_H
#define KIE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KIE_OK = 0,
  KIE_ERR_INVALID = -1,        /* bad descriptor, null pointer or argument */
  KIE_ERR_OOM = -2,            /* device allocation failed */
  KIE_ERR_CUDA = -3,           /* a CUDA call failed (message via kie_strerror) */
  KIE_ERR_CAPACITY = -4,       /* pos + n would exceed max_seq */
  KIE_ERR_NOT_RESIDENT = -5,   /* the persistent grid cannot be co-resident */
  KIE_ERR_DEVICE_TIMEOUT = -6, /* a bounded in-kernel wait ran out (watchdog) */
  KIE_ERR_POISONED = -7,       /* an earlier device error poisoned this context */
  KIE_ERR_NONFINITE = -8       /* a NaN logit, or a token id outside [0, vocab), met
                                  on the device; the kernel stops before using it */
} kie_status;

typedef enum { KIE_F16 = 0, KIE_BF16 = 1 } kie_dtype;

/* Model shape.  Dense models: n_lanes = 1 and n_heads * head_dim == d_model.
 * Lane models: every per-lane size is the total divided by n_lanes
 * (lane width d_model/n_lanes, n_heads/n_lanes query heads, n_kv_heads/n_lanes
 * KV heads, ffn_dim/n_lanes hidden units), lane_delay >= 2.
 * Requirements: n_heads % n_kv_heads == 0 with at most 4 query heads per KV
 * head; head_dim in {64, 128}; d_model <= 4096; lane width and d_model
 * 128 times a power of two (so n_lanes is a power of two); ffn_dim per lane
 * a multiple of 8.  kie_create returns KIE_ERR_INVALID
 * (reason via kie_strerror) for any other shape. */
typedef struct {
  int32_t n_layers, d_model, n_heads, n_kv_heads, head_dim, ffn_dim, vocab;
  float rms_eps, rope_theta;
  int32_t dtype;      /* kie_dtype: weights and KV cache */
  int32_t n_lanes;    /* 1 = dense */
  int32_t lane_delay; /* delta, layers; used when n_lanes > 1 */
  int32_t max_seq;    /* KV capacity in positions (prompt + decode) */
} kie_model_desc;

typedef struct kie_ctx kie_ctx;

/* Build a context on the current CUDA device.
 * Passage: "Startup Perancis Ini Kata Perisian Sahaja Cukup..." page, stack
 * bullets -- the monokernel bullet (the whole decode path as one persistent
 * kernel, nothing launched between layers) and the assembly-level bullet
 * (aim at every cycle of memory bandwidth).  What this call prepares for that
 * kernel: the weights re-laid out once into one contiguous stream per SM in
 * the order the SM consumes them, the KV cache, and the scratch of one call.
 *   weights: DEVICE pointer to all weights in the canonical layout (storage
 *     dtype, row-major [out, in], concatenated, no padding):
 *       embed[V,d];
 *       per layer, per lane: attn_norm[dl], wq[Hql*dh,dl], wk[Hkvl*dh,dl],
 *         wv[Hkvl*dh,dl], wo[dl,Hql*dh], ffn_norm[dl], w_gate[Fl,dl],
 *         w_up[Fl,dl], w_down[dl,Fl];  lane models then mix[d,d];
 *       final_norm[d], lm_head[V,d].
 *     The buffer must hold kie_weights_bytes(desc) bytes; the library reads
 *     exactly those and cannot check a raw pointer's extent itself.
 *     Borrowed for this call only: the library copies the weights into its
 *     own per-SM streaming layout, so the caller may free them on return.
 *   stream: cudaStream_t to run on (NULL = legacy default stream).
 *   out: receives the context (owner: caller, release with kie_destroy). */
int kie_create(const kie_model_desc *desc, const void *weights, void *stream, kie_ctx **out);

/* Size in bytes of the canonical weights of `desc` (what kie_create reads).
 * Host-only, no device work; KIE_ERR_INVALID (reason via kie_strerror) for a
 * descriptor kie_create would refuse, or a null out. */
int kie_weights_bytes(const kie_model_desc *desc, int64_t *out);

/* Process a prompt from position 0 (the KV cache is reset and its unused
 * slots filled with NaN) and return the greedy next token, the argmax of the
 * logits at position n-1.
 * Passage: "Startup Kog dosahuje 3 000 tokenu/s..." page, section "Software
 * versus kremik": the persistent program covers prefill as well as decode
 * and LM-head sampling.  Here the prompt is run through that same persistent
 * kernel, one position per step, with the LM head evaluated only at the last
 * position.
 *   tokens: HOST array of n ids in [0, vocab); next_token: HOST out.
 *   n < 1 or an id outside [0, vocab) returns KIE_ERR_INVALID and n > max_seq
 *   KIE_ERR_CAPACITY, before any device work (the cache and position are left
 *   as they were).  The prompt runs through the decode path one position per
 *   step, in the same persistent kernel. */
int kie_prefill(kie_ctx *ctx, const int32_t *tokens, int32_t n, int32_t *next_token);

/* kie_prefill that also returns the logits of the last prompt position:
 *   logits_out: DEVICE fp32 array [vocab], or NULL. */
int kie_prefill_ex(kie_ctx *ctx, const int32_t *tokens, int32_t n, int32_t *next_token,
                   float *logits_out);

/* How kie_prefill / kie_prefill_ex process a prompt (applies to later calls):
 *   KIE_PREFILL_GEMM (default for dense fp16 models): the prompt pass on the
 *     tensor cores.  Per layer, for all prompt rows at once: RMSNorm, the
 *     q/k/v, O, gate/up and down projections as tcgen05 GEMMs (operands
 *     staged by tensor-map bulk copies, fp32 accumulation in tensor memory;
 *     the fp32 activations enter as a sum of two fp16 or three bf16 parts, so
 *     the products keep fp32-level precision), RoPE and the K/V cache write,
 *     causal attention on the CUDA cores; then the final norm, LM head and
 *     greedy token of the last row.  Needs a second, canonical copy of the
 *     weights in device memory, made by kie_create when there is room.
 *   KIE_PREFILL_STEPS: the prompt runs through the persistent decode kernel
 *     one position per step (the only mode for lane models, and the default
 *     for bf16 models: bf16's 8-bit significand turns the fp32-level
 *     differences of the tensor-core accumulation into one-ulp differences of
 *     cached K/V, which the decode path's own arithmetic avoids).
 * Both leave the same state: the KV cache of positions 0..n-1 and the greedy
 * next token.  KIE_ERR_INVALID for another mode, or for KIE_PREFILL_GEMM
 * when the prompt pass is not available for this context (lane model, or no
 * room for its weight copy; kie_strerror says which).
 * Passage: "Startup Kog dosahuje 3 000 tokenu/s..." page, section "Software
 * versus kremik": prefill as part of the same engine's decode cycle. */
enum { KIE_PREFILL_STEPS = 0, KIE_PREFILL_GEMM = 1 };
int kie_set_prefill_mode(kie_ctx *ctx, int32_t mode);

/* Greedy decode: step k feeds the pending token at position pos+k, appends
 * its K/V, and the argmax of its logits becomes out_tokens[k] and the next
 * pending token.  The first pending token is kie_prefill's next_token.
 * Passages: the monokernel bullet of the "Startup Perancis Ini Kata Perisian
 * Sahaja Cukup..." page (every layer of the decode path inside one persistent
 * kernel), the "Software versus kremik" section of the "Startup Kog dosahuje
 * 3 000 tokenu/s..." page (no per-token launch cost, grid synchronisations
 * removed, the sampled token produced inside the kernel), and the results
 * table of the first page ("Laneformer 2B: Keputusan yang Ditunjukkan":
 * FP16, batch 1, greedy).  One call is one launch of that kernel for all
 * n_steps tokens; the sampled token is fed back on the device.
 *   out_tokens: HOST array of n_steps.
 *   n_steps < 1, or no pending token (no kie_prefill yet), returns
 *   KIE_ERR_INVALID, and pos + n_steps > max_seq KIE_ERR_CAPACITY, before any
 *   device work.  All steps run in one kernel launch, or in several back to
 *   back beyond the per-launch limit (kie_set_max_steps_per_launch). */
int kie_decode(kie_ctx *ctx, int32_t n_steps, int32_t *out_tokens);

/* kie_decode with options (same passages as kie_decode; the two options
 * expose the decode path for checking it: teacher forcing fixes the fed
 * tokens, and logits_out keeps the LM-head output the greedy sampling reads):
 *   forced_tokens: HOST array of n_steps ids, or NULL.  When given, step k
 *     feeds forced_tokens[k] instead of the pending token (teacher forcing);
 *     out_tokens still receives each step's argmax.
 *   logits_out: DEVICE fp32 array [n_steps, vocab], or NULL. */
int kie_decode_ex(kie_ctx *ctx, int32_t n_steps, const int32_t *forced_tokens,
                  int32_t *out_tokens, float *logits_out);

/* Sampling beyond greedy at the LM head, inside the same persistent kernel.
 * Passage: the "Software versus kremik" section of the "Startup Kog dosahuje
 * 3 000 tokenu/s..." page names LM-head sampling among the work done in one
 * go on the device; the pages report greedy decoding only and define no
 * sampler, so the plain one is taken, in this order:
 *   1. temperature T > 0 scales the logits, y = z / T;
 *   2. top_k > 0 keeps the top_k largest logits (equal logits: the lower id
 *      first, as the argmax); top_k == 0 keeps every token;
 *   3. top_p keeps, of those and most probable first, the smallest leading
 *      set whose softmax(y) probability within the top-k set reaches top_p;
 *   4. the token is drawn by inverse CDF: walking the kept tokens in
 *      increasing id, the first whose cumulative probability, renormalised
 *      over the kept set, exceeds that step's uniform.
 * The random numbers are inputs: uniforms[k], in [0, 1), is step k's.  The
 * arithmetic is fp32 (expf, sequential sums); every SM draws the same token
 * from the same data, so the token is fed back with no extra exchange. */
#define KIE_MAX_TOP_K 64
typedef struct {
  float temperature;  /* 0: greedy (the uniforms are then unused); else > 0 and finite */
  int32_t top_k;      /* 0 .. KIE_MAX_TOP_K; 0 = no top-k cut */
  float top_p;        /* (0, 1]; must be 1 when top_k is 0 */
} kie_sampling;

/* kie_decode_ex with the token of each step drawn per kie_sampling instead
 * of the argmax.
 *   params: HOST, not NULL.  temperature 0 makes this call kie_decode_ex.
 *   uniforms: HOST array of n_steps floats in [0, 1) (not read when greedy).
 *   forced_tokens, out_tokens, logits_out: as for kie_decode_ex; out_tokens
 *     receives the sampled tokens, and the last becomes the pending token.
 * KIE_ERR_INVALID, before any device work: a parameter outside the ranges
 * above, a uniform outside [0, 1) or NaN, or a top-k cut on a model whose
 * LM-head slice per SM exceeds 2048 rows (vocab above about 300,000 on 148
 * SMs).  The prompt's own next token (kie_prefill) stays greedy. */
int kie_decode_sample(kie_ctx *ctx, int32_t n_steps, const kie_sampling *params,
                      const float *uniforms, const int32_t *forced_tokens, int32_t *out_tokens,
                      float *logits_out);

/* kie_decode_ex without any allocation.  The pages have no counterpart to
 * this call; it exists for callers that may not allocate device memory at the
 * time they decode (for example a serving thread under a fixed device-memory
 * budget that reserved everything at start-up, or one that must never enter
 * the CUDA allocator because an allocation can block behind device-wide work).
 * Same arguments, semantics and context state as kie_decode_ex; the kernel's
 * per-launch scratch (activation vectors, attention partials, epoch counters,
 * argmax keys, token staging) comes from one fixed 1 MiB array in the
 * library's device image instead of the context's buffers.
 *   - every GPU that loads the library holds that 1 MiB until the process exits;
 *   - the array's device address is looked up (cudaGetSymbolAddress) on the
 *     first call on each device, with that device current; make that first
 *     call before any stream capture;
 *   - calls whose scratch would not fit (large models or very long n_steps)
 *     return KIE_ERR_CAPACITY, and kie_strerror gives the sizes;
 *   - every call on a GPU shares the one array, which keeps the last call's
 *     contents (the counters and keys are cleared at the start of each call):
 *     calls that overlap on that GPU, from any context or stream, race. */
int kie_decode_ex_static(kie_ctx *ctx, int32_t n_steps, const int32_t *forced_tokens,
                         int32_t *out_tokens, float *logits_out);

/* Release every resource of the context (valid on a poisoned context). */
int kie_destroy(kie_ctx *ctx);

/* Static text for a kie_status; for KIE_ERR_CUDA and KIE_ERR_DEVICE_TIMEOUT
 * it includes the detail of the most recent error in this process. */
const char *kie_strerror(int status);

/* Facts about a context, for measurement. */
typedef struct {
  int32_t n_ctas;             /* persistent CTAs (one per SM) */
  int32_t threads_per_cta;
  int32_t ring_slots;         /* shared-memory weight ring depth */
  int32_t slot_bytes;
  int32_t smem_bytes;         /* dynamic shared memory per CTA */
  int32_t pos;                /* next position to be written */
  int64_t weight_bytes_per_step; /* weights one decode step streams (incl. LM head) */
  int64_t kv_bytes_per_position; /* K+V bytes per cached position, all layers */
  float last_kernel_ms;       /* device time of the most recent call's launches, from the
                                 first one's start to the last one's end (CUDA events) */
  int32_t last_launch_steps;  /* steps run by that call */
  int32_t pending_token;
  float last_prefill_ms;      /* device time of the most recent prompt (either mode) */
  int32_t prefill_mode;       /* KIE_PREFILL_GEMM or KIE_PREFILL_STEPS */
} kie_stats;

int kie_get_stats(const kie_ctx *ctx, kie_stats *out);

/* Copy n cached positions [pos0, pos0 + n) of one layer and KV head to the
 * host, as raw storage words: k_out and v_out are HOST arrays of n*head_dim
 * uint16 (either may be NULL).  Positions never written hold NaN words. */
int kie_copy_kv(const kie_ctx *ctx, int32_t layer, int32_t kv_head, int32_t pos0, int32_t n,
                uint16_t *k_out, uint16_t *v_out);

/* Per-SM activity counters of the most recent launch, in SM clock cycles:
 * out[cta * 32 + slot] for slots 0 total, 1 waiting on other SMs, 2 GEMV
 * stages, 3 waiting for weight tiles, 4 attention, 5 input staging and norm,
 * 6 end-of-stage barrier, 7 LM head, 8 producer blocked on a full ring,
 * 9 producer total, 10 tiles issued, 11 dependency waits, 12..17 GEMV time
 * per stage (QKV, O, gate/up, down, mix, LM head), 18..23 waiting time per
 * dependency counter (after O, after down, lane-mix flush, token, q/k/v of
 * the KV group, attention partials of the group), 24..26 waiting for weight
 * tiles per consumer warp (mean, max, min over the 16 warps).  Only the
 * profiling build (libkie_prof.so, compiled with
 * KIE_PROFILE) records them; the normal build returns KIE_ERR_INVALID.
 * n_words must be >= 32 * n_ctas. */
int kie_get_profile(const kie_ctx *ctx, uint64_t *out, int32_t n_words);

/* Event trace of one SM over one decode step of later launches (profiling
 * build only; the normal build returns KIE_ERR_INVALID): step = index of the
 * step inside a launch, -1 to stop tracing.  The SM's thread 0 records
 * 64-bit events (SM clock << 8) | (type << 4) | argument: 0 layer start
 * (argument layer & 15, 15 = LM head), 1/2 wait for other SMs begins/ends
 * (argument: counter kind as in kie_get_profile), 3/4 end-of-stage barrier,
 * 5/6 RMSNorm staging, 7/8 weight stage (argument: QKV 0, O 1, gate/up 2,
 * down 3, mix 4, LM 5), 9/10 waiting for a weight tile, 11 tile released,
 * 12 attention (0 begin, 1 positions folded, 2 partials written, 3 merged).
 * kie_get_trace copies out[0] = number of events, out[1..] the events;
 * n_words <= 65537 are copied. */
int kie_trace_request(kie_ctx *ctx, int32_t cta, int32_t step);
int kie_get_trace(const kie_ctx *ctx, uint64_t *out, int32_t n_words);

/* Test hooks for the device watchdog (no effect unless called).
 *   watchdog_ms: limit of every in-kernel wait (default 2000, env KIE_WATCHDOG_MS).
 *   skip_signal_cta: if >= 0, that CTA never signals the first stage of the
 *     next launch, so the other CTAs' waits must run out and the call must
 *     return KIE_ERR_DEVICE_TIMEOUT.  Reset to -1 after one launch. */
int kie_debug_set(kie_ctx *ctx, int32_t watchdog_ms, int32_t skip_signal_cta);

/* How the persistent kernel's SMs wait for one another (applies to later
 * launches of this context; results are the same in both modes).
 *   KIE_SYNC_DEPENDENCY (default): each wait is for exactly the SMs whose
 *     output it reads -- the KV-head group for q/k/v and attention partials,
 *     every SM only for the two residual updates of a layer.
 *   KIE_SYNC_GRID: every wait is a grid-wide barrier across all SMs, the
 *     scheme the monokernel page reports as a third of per-token time on
 *     conventional stacks; kept as a measured ablation.
 * Returns KIE_ERR_INVALID for any other mode. */
enum { KIE_SYNC_DEPENDENCY = 0, KIE_SYNC_GRID = 1 };
int kie_set_sync_mode(kie_ctx *ctx, int32_t mode);

/* How the persistent kernel adds up the O and down projections, whose
 * outputs every SM contributes to (applies to later launches of this context):
 *   KIE_SUM_FP32_ATOMIC (default): fp32 vector atomics.  The order in which
 *     SMs add differs from run to run, so the last bits of the residual
 *     stream, and of the logits, can differ between two identical calls.
 *   KIE_SUM_EXACT: each contribution v is split into hi (v rounded to a
 *     multiple of 2^-8) and lo (the rest, rounded to a multiple of 2^-25),
 *     added with fp32 vector atomics into two accumulators whose partial sums
 *     are then always exactly representable, so no addition rounds and the
 *     sums do not depend on the order.  Two identical calls give
 *     bit-identical logits and tokens as long as every contribution to an O
 *     or down output is below 256 in magnitude (fewer than 256 SMs); larger
 *     contributions are still added, without that guarantee.  The rounding of
 *     lo costs at most 2^-26 absolute per contribution, and every O and down
 *     output takes two vector atomics instead of one.
 * Returns KIE_ERR_INVALID for any other mode. */
enum { KIE_SUM_FP32_ATOMIC = 0, KIE_SUM_EXACT = 1 };
int kie_set_sum_mode(kie_ctx *ctx, int32_t mode);

/* Most decode steps one kernel launch runs (applies to later calls of this
 * context).  A call with more steps runs as several launches back to back,
 * each starting at the position and token where the previous one stopped;
 * the results are those of one launch.  The kernel's epoch counters are
 * 32-bit, so a launch never runs more than (2^31 - 1) / ((4 n_layers + 2) *
 * SMs) steps whatever is set here (about 105,000 steps for 34 layers on 148
 * SMs).  n = 0 restores that limit; n > 0 lowers it (to bound how long one
 * launch holds the GPU).  Returns KIE_ERR_INVALID for n < 0. */
int kie_set_max_steps_per_launch(kie_ctx *ctx, int32_t n);

#ifdef __cplusplus
}
#endif
#endif /* KIE_H */
