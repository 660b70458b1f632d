/*
 * dg.h — C ABI of the block discrete-diffusion denoising step (sm_100a).
 *
 * The method is the one described for "DiffusionGemma Technical Report":
 *   - codemajin.net "DiffusionGemma architecture", section 3.2 (causal encoder
 *     writes a KV cache; a weight-shared bidirectional decoder denoises the
 *     256-token block while attending to it; finished blocks are appended to
 *     the cache and never rewritten);
 *   - same page, sections 3.1 and 3.3, and aibars.net "Uniform State
 *     Diffusion" (confident tokens are kept, the rest are reset to uniformly
 *     random vocabulary tokens);
 *   - aiboss88.com "hybrid attention architecture" (prefill: causal attention
 *     that writes the KV cache; denoising: bidirectional attention).
 *
 * Conventions common to every call
 *   - All tensors are row-major.  "bf16" buffers hold IEEE bfloat16 bit
 *     patterns (uint16_t).  Pointers named *_dev are CUDA device pointers,
 *     *_host are host pointers.
 *   - Weights are owned by the caller and must stay valid and unchanged until
 *     dg_destroy.  The context owns the KV cache and every workspace buffer.
 *   - Every call is asynchronous on the stream given to dg_create, except
 *     dg_create, dg_destroy, dg_sync and dg_denoise_step_host, which
 *     synchronise.  Device inputs must be ready in that stream's order (made
 *     on it, or the stream made to wait for the one that made them), and
 *     device outputs are ready in that order too.  Arguments and capacities are checked on the host before
 *     anything is launched; a rejected call returns an error and changes no
 *     state.  Errors raised on the device (a bounded wait that ran out) are
 *     reported by the next dg_sync as DG_ERR_DEVICE_TIMEOUT.
 *   - dg_last_error() returns a message for the last failed call on ctx
 *     (or, for ctx == NULL, for this thread's last failed dg_create).
 *   - A context holds host-side state (its captured step graphs, the cached
 *     length, error text): calls on one ctx must not overlap in time (one
 *     host thread at a time, or the caller's own lock).  Distinct contexts
 *     share nothing but the two process-wide device buffers described below
 *     (the timeline records of the tracing build, and the scratch of
 *     dg_lmhead_argmax_static).
 */
#ifndef DG_H
#define DG_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct dg_ctx dg_ctx;

typedef enum dg_status {
  DG_OK = 0,
  DG_ERR_INVALID_ARG = 1,    /* a pointer, size or configuration value is out of range   */
  DG_ERR_OOM = 2,            /* device allocation failed                                  */
  DG_ERR_CAPACITY = 3,       /* batch or sequence length beyond what dg_create reserved   */
  DG_ERR_CUDA = 4,           /* a CUDA runtime call failed (message in dg_last_error)     */
  DG_ERR_DEVICE_TIMEOUT = 5, /* a kernel's bounded wait ran out; outputs are invalid      */
  DG_ERR_STATE = 6,          /* call out of order (e.g. a step before any prefill)        */
  DG_ERR_UNSUPPORTED = 7     /* shape the kernels do not support (see dg_config)          */
} dg_status;

/* Model shape and capacities.
 * Supported shapes: d_model, expert_hidden and shared_hidden multiples of 64;
 * head_dim in {64, 128, 176}; n_q_heads a multiple of n_kv_heads, and the
 * group size n_q_heads / n_kv_heads a divisor of 128 (one attention tile
 * holds whole groups); vocab a multiple of 128; top_k <= 16 and <= n_experts
 * <= 256, n_experts a multiple of 4; d_model a multiple of 128 and <= 4096;
 * canvas a multiple of 16 and <= 256.  The three output projections of a layer are the only places
 * where a layer writes the residual stream. */
typedef struct dg_config {
  int32_t n_layers;
  int32_t d_model;
  int32_t n_q_heads;
  int32_t n_kv_heads;
  int32_t head_dim;
  int32_t n_experts;       /* routed experts                                 */
  int32_t top_k;           /* routed experts per token                       */
  int32_t expert_hidden;   /* SwiGLU hidden width of a routed expert         */
  int32_t shared_hidden;   /* SwiGLU hidden width of the shared expert       */
  int32_t vocab;
  float rope_base;         /* RoPE base (rotate-half pairs j, j + head_dim/2) */
  float rms_eps;           /* RMSNorm epsilon                                */
  float temperature;       /* logits are divided by this before the softmax  */
  int32_t canvas;          /* tokens per block (256)                         */
  int32_t max_batch;       /* sequences per call                             */
  int32_t max_seq;         /* KV-cache capacity per sequence (tokens)        */
  int32_t prefill_rows;    /* rows per causal chunk in dg_prefill (0: 2048)  */
} dg_config;

/* One layer's weights, bf16 device pointers, stored [out, in] (row = output).
 *   attn_norm [d]              RMSNorm gain before attention
 *   wqkv      [(Hq+2Hkv)*D, d] rows: Hq query heads, then Hkv key heads, then
 *                              Hkv value heads, head-major, D rows per head
 *   wo        [d, Hq*D]
 *   ffn_norm  [d]
 *   w_router  [E, d]
 *   w_gate    [E, F, d], w_up [E, F, d], w_down [E, d, F]   routed experts
 *   ws_gate   [Fs, d],   ws_up [Fs, d],   ws_down [d, Fs]   shared expert   */
typedef struct dg_layer_weights {
  const void* attn_norm;
  const void* wqkv;
  const void* wo;
  const void* ffn_norm;
  const void* w_router;
  const void* w_gate;
  const void* w_up;
  const void* w_down;
  const void* ws_gate;
  const void* ws_up;
  const void* ws_down;
} dg_layer_weights;

/* Model weights.  embed [V, d] bf16 is also the (tied) LM head.  router_bias
 * [E] fp32 device pointer or NULL is added to every layer's router logits
 * before top-k.  layers points to a HOST array of n_layers entries that is
 * read during dg_create only.  sc_gate, sc_up [F, d] and sc_down [d, F] bf16
 * (F = expert_hidden) are the feed-forward layer of the self-conditioning
 * signal (dg_set_self_conditioning), or all NULL. */
typedef struct dg_weights {
  const void* embed;
  const void* final_norm;
  const float* router_bias;
  const dg_layer_weights* layers;
  const void* sc_gate;
  const void* sc_up;
  const void* sc_down;
} dg_weights;

/* Create a context: validates cfg, allocates the KV cache
 * ([n_layers][max_batch][n_kv_heads][max_seq][head_dim] bf16 for K and for V)
 * and all workspaces, builds the RoPE table (angles in double precision) and
 * the TMA descriptors of every weight.  cuda_stream is a cudaStream_t (NULL:
 * legacy default stream).  On success *out receives the context. */
dg_status dg_create(const dg_config* cfg, const dg_weights* weights, void* cuda_stream,
                    dg_ctx** out);

/* Release every resource of ctx (synchronises its stream first). */
dg_status dg_destroy(dg_ctx* ctx);

/* Causal encoder (aiboss88.com "hybrid attention architecture"; codemajin.net
 * section 3.2): reset the cache and encode tokens_dev [batch, prefix_len]
 * int32, every row attending to itself and the rows before it; keys/values of
 * all layers are written to cache positions [0, prefix_len).
 * Needs batch <= max_batch and prefix_len + canvas <= max_seq. */
dg_status dg_prefill(dg_ctx* ctx, const int32_t* tokens_dev, int32_t batch, int32_t prefix_len);

/* One denoising step over the canvas (codemajin.net sections 3.1-3.3):
 * canvas_in_dev [batch, canvas] int32 tokens at positions [P, P+canvas) are
 * run through every layer with bidirectional attention over cache[0,P) plus
 * the whole canvas; the tied LM head gives, per position, the argmax token a
 * and the confidence conf = max softmax probability (logits never leave the
 * chip); the sampler then writes canvas_out = (conf >= tau) ? a : uniform
 * token, the uniform token drawn by Philox4x32-10 with counter (P+i, step,
 * sequence, 0) and key (seed low 32 bits, seed high 32 bits).
 *   conf_dev        [batch, canvas] fp32 (written)
 *   all_settled_dev [batch] int32 or NULL: 1 where every conf >= tau, else 0.
 * The committed cache is not modified.  canvas_out_dev may equal
 * canvas_in_dev; other outputs must not alias inputs.  batch is the batch of
 * the last dg_prefill. */
dg_status dg_denoise_step(dg_ctx* ctx, const int32_t* canvas_in_dev, int32_t step, uint64_t seed,
                          float tau, int32_t* canvas_out_dev, float* conf_dev,
                          int32_t* all_settled_dev);

/* Entropy-constrained sampler of one step (codemajin.net "DiffusionGemma
 * architecture", section 3.3).
 *   temperature   this step's temperature (the page anneals it linearly from
 *                 0.8 to 0.4 over at most 48 steps; the caller picks it)
 *   gamma         entropy budget (nats): positions are accepted in ascending
 *                 (entropy, position) order while the float32 running sum of
 *                 their entropies stays <= gamma; the first is always accepted
 *   stop_entropy  adaptive stop (nats): when a previous argmax is given, the
 *                 canvas's mean entropy (float32 sum in position order / C)
 *                 is < stop_entropy and every argmax equals the previous
 *                 one, every position takes its argmax and the sequence is
 *                 reported stopped */
typedef struct dg_entropy_args {
  float temperature;
  float gamma;
  float stop_entropy;
} dg_entropy_args;

/* One denoising step like dg_denoise_step, ended by the entropy-constrained
 * sampler instead of the confidence threshold.  Accepted positions take
 * their argmax, the others the same Philox uniform draw as dg_denoise_step.
 *   prev_argmax_dev [batch, canvas] int32: the previous step's argmax, or
 *                   NULL at the first step of a block (no stop possible)
 *   argmax_out_dev  [batch, canvas] int32 or NULL: this step's argmax (may
 *                   equal prev_argmax_dev, for the next call)
 *   canvas_out_dev  [batch, canvas] int32 (may equal canvas_in_dev)
 *   entropy_dev     [batch, canvas] fp32 or NULL: softmax entropy (nats)
 *   stopped_dev     [batch] int32 or NULL: 1 where the adaptive stop fired
 * The committed cache is not modified.  The logits never leave the chip: the
 * entropy comes from one more running sum in the LM-head reduction. */
dg_status dg_denoise_step_entropy(dg_ctx* ctx, const int32_t* canvas_in_dev, int32_t step, uint64_t seed,
                                  const dg_entropy_args* args, const int32_t* prev_argmax_dev,
                                  int32_t* argmax_out_dev, int32_t* canvas_out_dev, float* entropy_dev,
                                  int32_t* stopped_dev);

/* Same step with HOST buffers: copies canvas_in_host to the device, runs the
 * step, copies canvas_out/conf/all_settled back and synchronises.  Any of
 * conf_host and all_settled_host may be NULL. */
dg_status dg_denoise_step_host(dg_ctx* ctx, const int32_t* canvas_in_host, int32_t step,
                               uint64_t seed, float tau, int32_t* canvas_out_host,
                               float* conf_host, int32_t* all_settled_host);

/* Self-conditioning (codemajin.net "DiffusionGemma architecture", section
 * 3.2): with enable = 1 every denoising step (either sampler) also computes,
 * from its LM head, the predicted clean-token distribution p = softmax(z E^T
 * / T), passes it through the embedding matrix (p E) and the SwiGLU layer of
 * sc_gate / sc_up / sc_down, and the next step adds the result to its input
 * embeddings.  The first step after dg_prefill, dg_commit_block or this call
 * has no signal to add.  The step then also writes p as bf16 to a context
 * buffer ([batch*canvas, vocab]; the one place probabilities reach memory).
 * DG_ERR_UNSUPPORTED when the context was created without those weights. */
dg_status dg_set_self_conditioning(dg_ctx* ctx, int32_t enable);

/* Block commit (codemajin.net section 3.2 block-AR; section 5.1 counts it as
 * one extra forward per block): one causal forward of block_dev
 * [batch, canvas] int32 at positions [P, P+canvas), appending its keys/values
 * to the cache; then P += canvas.  Needs P + 2*canvas <= max_seq. */
dg_status dg_commit_block(dg_ctx* ctx, const int32_t* block_dev);

/* Wait for all work of ctx and report device-side errors. */
dg_status dg_sync(dg_ctx* ctx);

/* Committed cache length P (tokens per sequence). */
int32_t dg_cached_len(const dg_ctx* ctx);

/* Message for the last failed call on ctx (never NULL).  With ctx == NULL:
 * the calling thread's last dg_create failure (a failed create returns no
 * context), or "null context" if it has none; a successful dg_create clears it. */
const char* dg_last_error(const dg_ctx* ctx);

/* ---------------------------------------------------------------------------
 * Test hooks.  Exported for the parity tests; not part of the stable API.
 * ------------------------------------------------------------------------- */

/* Record, during the following denoising steps, the residual stream after
 * every layer and the experts chosen in every layer (enable = 1), or stop
 * recording and free the buffers (enable = 0). */
dg_status dg_debug_capture(dg_ctx* ctx, int32_t enable);

/* Residual stream of the last recorded step: layer 0 is the embedding, layer
 * l > 0 the stream after layer l.  out_dev [batch*canvas, d] fp32. */
dg_status dg_debug_hidden(dg_ctx* ctx, int32_t layer, float* out_dev);

/* Experts of the last recorded step in layer l: out_dev [batch*canvas, top_k]
 * int32, ordered by (logit desc, index asc). */
dg_status dg_debug_experts(dg_ctx* ctx, int32_t layer, int32_t* out_dev);

/* bf16 rows [batch*canvas, d] of the last recorded step, exactly as the
 * kernels consumed them: for 0 <= layer < n_layers the rows fed to that
 * layer's router and experts (RMSNorm of the residual after attention), for
 * layer == n_layers the rows fed to the LM head (the final RMSNorm).  Lets a
 * test give the oracle the very operands of a decision (expert choice,
 * argmax) the kernels took. */
dg_status dg_debug_norm_rows(dg_ctx* ctx, int32_t layer, void* out_dev);

/* LM-head reduction of the last step: per position the argmax (lowest index
 * of the maximum), log-sum-exp, confidence and top-1 minus top-2
 * probability.  Each pointer [batch*canvas] or NULL. */
dg_status dg_debug_lmhead(dg_ctx* ctx, int32_t* argmax_dev, float* lse_dev, float* conf_dev,
                          float* margin_dev);

/* Router decision alone on given fp32 logits [n_rows, n_experts] (router bias
 * NOT added): idx_dev [n_rows, top_k] int32, gates_dev [n_rows, top_k] fp32. */
dg_status dg_debug_router(dg_ctx* ctx, const float* logits_dev, int32_t n_rows, int32_t* idx_dev,
                          float* gates_dev);

/* Sampler decision alone on given argmax/conf [batch*canvas] (positions
 * P + i of the current cache length). */
dg_status dg_debug_sample(dg_ctx* ctx, const int32_t* argmax_dev, const float* conf_dev,
                          int32_t batch, int32_t step, uint64_t seed, float tau, int32_t* out_dev);

/* Entropy sampler decision alone on given argmax / entropy [batch*canvas]
 * (positions P + i of the current cache length), prev_argmax or NULL:
 * out_dev [batch*canvas] int32, stopped_dev [batch] int32 or NULL. */
dg_status dg_debug_entropy_sample(dg_ctx* ctx, const int32_t* argmax_dev, const float* entropy_dev,
                                  const int32_t* prev_argmax_dev, int32_t batch, int32_t step, uint64_t seed,
                                  float gamma, float stop_entropy, int32_t* out_dev, int32_t* stopped_dev);

/* Self-conditioning signal computed by the last step, [batch*canvas, d] fp32. */
dg_status dg_debug_self_cond(dg_ctx* ctx, float* out_dev);

/* Softmax entropy (nats) per position of the last step [batch*canvas]. */
dg_status dg_debug_entropy(dg_ctx* ctx, float* out_dev);

/* Launch a kernel that waits on a barrier nothing ever signals, with a wait
 * limit of limit_ns nanoseconds; the following dg_sync must report
 * DG_ERR_DEVICE_TIMEOUT and clear it.  Exercises the failure path of the
 * bounded waits without faulting the device. */
dg_status dg_debug_wait_timeout(dg_ctx* ctx, uint64_t limit_ns);

/* One weight-streaming GEMM through the tcgen05 kernel alone:
 * out_dev [splits, T, M] fp32 holds, for each split s of the K range, the
 * partial sums of x_dev [T, K] bf16 times w_dev [M, K] bf16 transposed (the
 * caller adds the splits).  K a multiple of 64, M a multiple of 4,
 * 1 <= splits <= K/64. */
dg_status dg_debug_gemm(dg_ctx* ctx, const void* w_dev, int32_t M, int32_t K, const void* x_dev, int32_t T,
                        int32_t splits, float* out_dev);

/* Kernel classes timed by the profiling hooks. */
enum {
  DG_PROF_EXPERTS = 0,       /* fused routed + shared expert GEMM: gate/up (SwiGLU) and down   */
  DG_PROF_ROUTING = 1,       /* router top-k, expert row claim and row gather (one kernel)    */
  DG_PROF_LMHEAD = 2,        /* LM-head GEMM with the argmax / log-sum-exp epilogue            */
  DG_PROF_ATTENTION = 3,     /* attention kernel and the merge of its key chunks              */
  DG_PROF_DENSE = 4,         /* QKV, output and router projections                            */
  DG_PROF_OTHER = 5,         /* norms, RoPE, combine, LM-head merge + sampler                 */
  DG_PROF_CLASSES = 6
};

/* Start (enable = class mask, bit c for class c) or stop (0) recording a CUDA
 * event pair on the context stream around every launch of the selected
 * classes; starting clears the totals. */
dg_status dg_debug_profile(dg_ctx* ctx, int32_t class_mask);

/* Synchronise and return, for one class, the summed device time (ms) and the
 * number of launches recorded since dg_debug_profile. */
dg_status dg_debug_profile_read(dg_ctx* ctx, int32_t cls, double* total_ms, int64_t* launches);

/* Number of this library's kernel launches issued by ctx so far. */
int64_t dg_debug_launch_count(const dg_ctx* ctx);

/* ---------------------------------------------------------------------------
 * Timeline (tracing).  libdg_timeline.so is this library compiled with
 * -DDG_TIMELINE: thread 0 of every CTA of every kernel appends one record
 * {start ns, end ns (%globaltimer, taken when thread 0 leaves the kernel),
 * kernel id, CTA index} to a device buffer of 262144 records shared by all
 * contexts of the process (records past its end are dropped).  Launches run one after another on the context's
 * stream, so sorting the records by start time and grouping consecutive
 * records of one kernel id recovers the launch sequence of a graph replay
 * with every launch's span and the gaps between launches.  In libdg.so both
 * calls return DG_ERR_UNSUPPORTED.
 *
 * Kernel ids: DG_K_GEMM_DENSE 10, DG_K_GEMM_MOE 11, DG_K_GEMM_LMHEAD 13,
 * DG_K_ATTENTION 20, DG_K_ATTN_MERGE 21, DG_K_ROUTE_DISPATCH 30, DG_K_COMBINE_NORM 31,
 * DG_K_EMBED_NORM 32, DG_K_RESIDUAL_NORM 33, DG_K_REDUCE_SPLITS 34,
 * DG_K_SWIGLU_SPLITS 35, DG_K_ROPE_QKV 36, DG_K_LMHEAD_MERGE_SAMPLE 37,
 * DG_K_ENTROPY_SAMPLE 38, DG_K_ROUTER_TOPK 39, DG_K_SAMPLE_ONLY 40,
 * DG_K_OTHER 50.
 * ------------------------------------------------------------------------- */
enum {
  DG_K_GEMM_DENSE = 10, DG_K_GEMM_MOE = 11, DG_K_GEMM_LMHEAD = 13, DG_K_ATTENTION = 20, DG_K_ATTN_MERGE = 21,
  DG_K_ROUTE_DISPATCH = 30, DG_K_COMBINE_NORM = 31, DG_K_EMBED_NORM = 32, DG_K_RESIDUAL_NORM = 33,
  DG_K_REDUCE_SPLITS = 34, DG_K_SWIGLU_SPLITS = 35, DG_K_ROPE_QKV = 36, DG_K_LMHEAD_MERGE_SAMPLE = 37,
  DG_K_ENTROPY_SAMPLE = 38, DG_K_ROUTER_TOPK = 39, DG_K_SAMPLE_ONLY = 40, DG_K_OTHER = 50
};

typedef struct {
  uint64_t t0_ns;  /* CTA start */
  uint64_t t1_ns;  /* CTA end (thread 0) */
  int32_t kernel;  /* DG_K_* */
  int32_t cta;     /* linear CTA index in its grid */
} dg_timeline_record;

/* Synchronise ctx's stream and empty the record buffer. */
dg_status dg_debug_timeline_reset(dg_ctx* ctx);

/* Synchronise ctx's stream and copy up to `capacity` records (in the order
 * they were appended) to host_records (caller-owned host memory); *n_records
 * receives the number appended since the last reset, which may exceed
 * capacity (and 262144, when records were dropped). */
dg_status dg_debug_timeline(dg_ctx* ctx, dg_timeline_record* host_records, int32_t capacity,
                            int64_t* n_records);

/* ---------------------------------------------------------------------------
 * LM-head reduction without any device allocation.
 *
 * The pages describe nothing like this; it is a deployment convenience.  It
 * serves callers that cannot allocate device memory when they need the
 * reduction: code running while another framework records a CUDA graph
 * (allocation is forbidden inside the capture), processes whose caching
 * allocator already holds the whole device, or embedded deployments that fix
 * all device memory at start-up.
 *
 * Computes, for each of the n_rows rows of z_dev [n_rows, d_model] bf16, the
 * logits z . embed^T / temperature over embed_dev [vocab, d_model] bf16 (the
 * tied LM head) without writing them, and returns argmax_dev [n_rows] int32
 * (lowest index of the maximum), lse_dev [n_rows] fp32 (log-sum-exp) and
 * conf_dev [n_rows] fp32 (maximum softmax probability); any of the three may
 * be NULL but not all.  It runs the same tcgen05 LM-head kernel as
 * dg_denoise_step, asynchronously on cuda_stream (a cudaStream_t, NULL = the
 * legacy default stream), with its partials in a fixed 8 MiB array inside the
 * library (n_rows * vocab / 128 <= 524288, e.g. 256 rows of a 262144-token
 * vocabulary).  Nothing is allocated and no context is needed.
 *   - Larger problems are rejected with DG_ERR_CAPACITY before any launch;
 *     malformed arguments (d_model not a multiple of 64, vocab not a multiple
 *     of 128, unaligned pointers) with DG_ERR_INVALID_ARG.
 *   - The first call on a device looks up the array's device address and sets
 *     the kernel attributes for that device (the device current at the call);
 *     make that first call before any stream capture.  That set-up runs under
 *     a lock, so first calls may come from any thread.
 *   - Only the two launches' own status is checked: a CUDA error the caller
 *     left pending from earlier work is neither reported nor cleared.
 *   - Every call on a device shares the one array, whose contents persist
 *     between calls: each call writes every partial it later reads and clears
 *     its own error flag first, but calls that overlap on the GPU (different
 *     streams, or several host threads) race on the array and must be
 *     serialised by the caller.
 *   - If a bounded wait inside the kernel ran out, the rows come back with
 *     argmax -1 and NaN statistics.  */
dg_status dg_lmhead_argmax_static(const void* z_dev, int32_t n_rows, int32_t d_model, const void* embed_dev,
                                  int32_t vocab, float temperature, int32_t* argmax_dev, float* lse_dev,
                                  float* conf_dev, void* cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* DG_H */
