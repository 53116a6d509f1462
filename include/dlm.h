/*
 * dlm.h -- C ABI of the masked block-diffusion denoise-step library
 * (NVIDIA B200, sm_100a).
 *
 * One denoising step of masked block-diffusion decoding over a fixed canvas of
 * C positions per sequence:
 *   1. bidirectional attention of every canvas position over the cached
 *      prefix K/V plus all canvas positions (Nemotron Labs Diffusion guide,
 *      section 6: the whole block is denoised with a bidirectional mask;
 *      course "Diffusion LLMs", section 14: the current block reads the
 *      finished prefix and all of its own positions);
 *   2. the LM-head projection to vocabulary logits (same guide, section 7:
 *      an untied diffusion head over a 131072-token vocabulary), whose
 *      per-position softmax maximum, argmax, normaliser and entropy are
 *      reduced inside the GEMM, so full logits never reach HBM (same guide,
 *      section 5.3: non-materialised chunked scoring);
 *   3. per-position confidence = probability of the candidate and entropy
 *      (course section 12 and section 9);
 *   4. the sampler: commit every uncommitted position whose confidence is at
 *      least the threshold, at least a uniform per-step quota of the most
 *      confident, and everything left on the last step of the budget; keep
 *      the mask id or re-noise the rest with uniform random ids; or, with an
 *      entropy bound, commit the lowest-entropy positions whose summed
 *      entropy stays under the bound (diffusers DiffusionGemma page,
 *      BlockRefinementScheduler and EntropyBoundScheduler; Nemotron guide,
 *      sections 3.2 and 6).
 *
 * Conventions for every call:
 *   - Pointers named *_dev / documented "device" are CUDA device pointers
 *     owned by the caller; pointers documented "host" are host memory.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL is the legacy default stream).  The int result reports argument
 *     and launch errors synchronously; it is DLM_OK (0) or a negative code.
 *   - Device-detected errors (a bounded wait that ran out) set an error word
 *     in the context; dlm_check() synchronises `stream` and returns it.
 *   - A context is not thread-safe: one host thread drives it at a time.
 *   - On any error, dlm_last_error() describes the first one.
 */
#ifndef DLM_H_
#define DLM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* status codes */
enum {
  DLM_OK = 0,
  DLM_EINVAL = -1,    /* an argument is out of range or inconsistent          */
  DLM_ENOMEM = -2,    /* device or host allocation failed                     */
  DLM_ECUDA = -3,     /* a CUDA runtime call failed                           */
  DLM_ECAP = -4,      /* KV capacity (max_prefix) would be exceeded           */
  DLM_ETIMEOUT = -5,  /* a device-side bounded wait ran out                   */
  DLM_EBOUNDS = -6,   /* a device-side index check failed                     */
  DLM_ESTATE = -7     /* the call does not fit the context's current state    */
};

enum { DLM_F32 = 0, DLM_BF16 = 1 };          /* model / weight element type  */
enum { DLM_MASK = 0, DLM_UNIFORM = 1 };      /* corruption of uncommitted slots */
enum { DLM_LM_MODEL = 0, DLM_LM_E4M3 = 1, DLM_LM_NVFP4 = 2 };   /* LM-head format  */

typedef struct dlm_ctx dlm_ctx;

/* Shape of the single-attention-layer denoiser.  Weights are row-major,
 * out-features x in-features.  mask_id 100 and eos_id 11 are the Nemotron
 * ids (guide, section 7); rope_theta 1e6 likewise; rope_theta <= 0 turns RoPE
 * off.  eos_id < 0 disables EOS handling.  head_dim must be 64 or 128 for
 * DLM_BF16 (128 only for bf16 attention) and <= 128 for DLM_F32. */
typedef struct {
  int d_model, n_heads, n_kv_heads, head_dim, vocab, dtype;
  float rope_theta;
  int mask_id, eos_id;
  int max_batch;    /* sequences (canvases) per call                       */
  int max_prefix;   /* KV capacity per sequence for the finished prefix    */
  int max_canvas;   /* largest canvas length, <= 1024                       */
  /* Element format of the LM head (NLD tutorial, section 8.6: online FP8
   * weight quantisation; course "Diffusion LLMs", section 15: low-bit
   * weights, NVFP4 on Blackwell).  The tensor cores take both operands in
   * the low-bit format, so every step quantises the head's input rows y the
   * same way as the weights, which dlm_create quantises once per vocabulary
   * row into a context-owned copy (W_lm is not read afterwards).
   *   DLM_LM_MODEL  the model's element type.
   *   DLM_LM_E4M3   (bf16 models, d_model % 16 == 0) scale s_v = max|W_v| /
   *                 448 (1 for a zero row), q = e4m3(W / s_v), round to nearest
   *                 even, saturating; the logits are (sum_k qy_rk qW_vk) *
   *                 (a_r * s_v), the factor rounded to float32.
   *   DLM_LM_NVFP4  (bf16 models, d_model % 256 == 0) a float32 row scale
   *                 s = max|row| / (448 * 6) (1 for a zero row), an e4m3 scale
   *                 per 16 elements e4m3(max|block| / (6 s)), elements
   *                 e2m1(x / (block scale * s)) (0 in a block whose scale is
   *                 0), every division and product in float32, round to
   *                 nearest even, saturating; the logits are the block-scaled
   *                 sums times the two row scales' product rounded to float32. */
  int lm_quant;
} dlm_model_desc;

/* Device pointers, caller-owned, valid for the life of the context; element
 * type per dlm_model_desc.dtype (bf16 bit patterns or float32).
 *   emb [vocab][d], w_q [H*Dh][d], w_k, w_v [Hkv*Dh][d], w_o [d][H*Dh],
 *   w_lm [vocab][d].  w_q/w_k/w_v are copied into one fused matrix at
 *   dlm_create; emb, w_o and w_lm are read in place. */
typedef struct { const void *emb, *w_q, *w_k, *w_v, *w_o, *w_lm; } dlm_weights;

/* Sampler parameters (DiffusionGemma page, __call__ and scheduler config;
 * Nemotron guide, sections 3.2 and 5.5).
 *   canvas      canvas length C, 1 <= C <= max_canvas
 *   steps       step budget S >= 1; the step with index S-1 commits all
 *   threshold   confidence threshold (>= is a hit); 0 commits everything
 *   quota       minimum commits per step; <= 0 means ceil(C / S)
 *   corruption  DLM_MASK: uncommitted slots hold mask_id (which is excluded
 *               from the argmax, softmax and entropy); DLM_UNIFORM: they are
 *               re-noised with uniform random ids after every step
 *   editing     0: committed tokens are final; 1: token editing (see
 *               editing_threshold below)
 *   entropy_bound  >= 0 selects the entropy-bound rule (temperature annealed
 *               linearly from t_max at step 0 to t_min at step S-1, Gumbel
 *               sampling); < 0 selects threshold + quota
 *   temperature 0: greedy argmax; > 0: Gumbel sampling at this temperature
 *               (threshold + quota rule only)
 *   seed        key of the counter-based generator (Philox4x32-10)        */
typedef struct {
  int canvas, steps;
  float threshold;
  int quota;
  int corruption;
  int editing;
  float entropy_bound;
  float temperature, t_max, t_min;
  unsigned long long seed;
  /* adaptive stopping (DiffusionGemma page, "adaptive stopping" and the
   * stability_threshold / confidence_threshold arguments): a canvas is
   * frozen -- every uncommitted position commits its current candidate and
   * the canvas is done -- once its argmax over all positions has been the
   * same for `stability_steps` consecutive steps and the mean entropy of its
   * positions is below `stop_entropy` (nats).  stop_entropy <= 0 turns it
   * off (then prev_cand / stable in dlm_canvas may be NULL). */
  int stability_steps;
  float stop_entropy;
  /* token editing (DiffusionGemma page, editing_threshold: committed tokens
   * may be re-edited; course "Diffusion LLMs", section 14: LLaDA2.1
   * token-to-token editing).  With editing = 1, at the start of every step a
   * position committed earlier and lying before the first committed EOS
   * takes the step's candidate when the candidate differs from its token
   * and its confidence is >= editing_threshold; it stays committed.  A
   * canvas is done once every position is committed, as without editing. */
  float editing_threshold;
} dlm_sampler_params;

/* Canvas state of `batch` sequences, device, caller-owned, updated in place:
 *   tokens [B][C] int32, committed [B][C] uint8 (0/1), step [B] int32 (steps
 *   taken), done [B] uint8, eos_pos [B] int32 (first committed EOS or -1),
 *   and for adaptive stopping prev_cand / stable (may be NULL when it is
 *   off; dlm_canvas_init sets prev_cand to -1 and stable to 0).
 * Canvas b attends to KV sequence b. */
typedef struct {
  int32_t *tokens;
  uint8_t *committed;
  int32_t *step;
  uint8_t *done;
  int32_t *eos_pos;
  int32_t *prev_cand;   /* [B][C] last step's candidates (adaptive stopping)     */
  int32_t *stable;      /* [B] consecutive steps with unchanged candidates       */
} dlm_canvas;

/* Per-canvas counters, device, caller-owned and caller-zeroed; every step
 * adds to them.  committed_by_sampler counts positions the selection chose
 * (forced ones included); forced_at_budget those committed only because the
 * budget ran out; eos_autofill the uncommitted positions filled with EOS
 * after the first committed EOS; frozen those committed when adaptive
 * stopping froze the canvas (not counted in committed_by_sampler); edited
 * the committed tokens replaced by token editing. */
typedef struct {
  int32_t steps_used;
  int32_t committed_by_sampler;
  int32_t forced_at_budget;
  int32_t eos_autofill;
  int32_t frozen;       /* positions committed by adaptive stopping */
  int32_t edited;       /* committed tokens replaced by token editing */
} dlm_canvas_stats;

/* Create a context: validates the descriptor, allocates the KV cache
 * [max_batch][Hkv][max_prefix + max_canvas][Dh] (K and V), the activations
 * and scratch, the fused QKV weight and the RoPE table on the current device.
 * Returns DLM_EINVAL / DLM_ENOMEM / DLM_ECUDA; *out is NULL on failure. */
int dlm_create(const dlm_model_desc *desc, const dlm_weights *weights, dlm_ctx **out);

/* Free everything the context owns (synchronises the device first). */
void dlm_destroy(dlm_ctx *ctx);

/* Append n finished tokens to KV sequence `seq` (course section 14: the
 * finished prefix is cached; the clean pass over a finished block supplies
 * its states).  Either `tokens` (device int32[n]) is given and K = RoPE(E[t]
 * W_k^T), V = E[t] W_v^T are computed at absolute positions len..len+n-1,
 * or tokens == NULL and `k`, `v` (device, [Hkv][n][Dh], already rotated, in
 * the model's element type) are copied in.  DLM_ECAP if len + n >
 * max_prefix; the length is tracked on the host and on the device. */
int dlm_kv_append(dlm_ctx *ctx, int seq, int n, const int32_t *tokens, const void *k,
                  const void *v, void *stream);

/* Set the length of KV sequence `seq` to 0 (no device work). */
int dlm_reset_kv(dlm_ctx *ctx, int seq);

/* Current length of KV sequence `seq`, or a negative code. */
int dlm_kv_length(const dlm_ctx *ctx, int seq);

/* Initialise `batch` canvases: all mask_id (DLM_MASK) or uniform random ids
 * from Philox counter (b, 0, i, 0xFFFFFFFF) (DLM_UNIFORM); committed = 0,
 * step = 0, done = 0, eos_pos = -1. */
int dlm_canvas_init(dlm_ctx *ctx, const dlm_canvas *canvas, int batch,
                    const dlm_sampler_params *params, void *stream);

/* One denoising step over the canvases that are not done: embed, QKV+RoPE,
 * attention, output projection, fused LM-head reduction, cross-tile reduce,
 * commit/re-noise, one kernel launch each.  Canvas K/V of
 * the step occupy cache slots len..len+C-1 of each sequence (not appended).
 * `stats` (device, [batch]) may be NULL. */
int dlm_denoise_step(dlm_ctx *ctx, const dlm_canvas *canvas, int batch,
                     const dlm_sampler_params *params, dlm_canvas_stats *stats, void *stream);

/* `params->steps` denoising steps (the whole block; steps of canvases that
 * are already done do no work), captured once per configuration into a CUDA
 * graph and replayed on `stream`.  Same arguments as dlm_denoise_step. */
int dlm_decode_block(dlm_ctx *ctx, const dlm_canvas *canvas, int batch,
                     const dlm_sampler_params *params, dlm_canvas_stats *stats, void *stream);

/* The first n_steps (1 <= n_steps <= params->steps) denoising steps of
 * dlm_decode_block as one CUDA graph, captured once per configuration and
 * step count and replayed on `stream`.  Every step reads the canvas's own
 * step counters on the device, so n_steps steps from any canvas state do
 * what n_steps dlm_denoise_step calls would; dlm_decode_block is this call
 * with n_steps = params->steps.  Same arguments otherwise; DLM_EINVAL for
 * n_steps out of range. */
int dlm_decode_steps(dlm_ctx *ctx, const dlm_canvas *canvas, int batch,
                     const dlm_sampler_params *params, int n_steps, dlm_canvas_stats *stats,
                     void *stream);

/* The split plan of the canvas attention that dlm_denoise_step runs for
 * `batch` canvases of `canvas` positions over the context's current prefix
 * lengths (bf16 contexts): *nsplit key splits of *chunk keys (a multiple of
 * 128) per (sequence, KV head, row tile); *cluster = nsplit when the splits
 * combine inside one thread-block cluster, else 1 (partials and a combine
 * kernel when nsplit > 1); *rows_per_cta query rows per CTA.  Host-only, no
 * device work.  DLM_EINVAL for an fp32 context or sizes out of range. */
int dlm_attention_plan(dlm_ctx *ctx, int batch, int canvas, int *nsplit, int *chunk,
                       int *cluster, int *rows_per_cta);

/* dlm_decode_block with HOST buffers: copies the canvas state in (host
 * arrays shaped as in dlm_canvas), runs the block, copies the canvas state
 * and `stats` (host, may be NULL) back, and synchronises `stream`.  The
 * device copies live in the context. */
int dlm_decode_block_host(dlm_ctx *ctx, int32_t *tokens, uint8_t *committed, int32_t *step,
                          uint8_t *done, int32_t *eos_pos, int batch,
                          const dlm_sampler_params *params, dlm_canvas_stats *stats,
                          void *stream);

/* Multi-block generation (Nemotron guide, section 6: blocks follow one
 * another until gen_length or EOS; DiffusionGemma page: the outer loop over
 * canvases, each finished canvas joins the cache, eos_early_stop; course
 * "Diffusion LLMs", section 14: the finished block is cached through a clean
 * pass).  For block k = 0, 1, ..., n_blocks-1: initialise the canvases with
 * seed + k, decode the block (the steps of dlm_decode_block, launched
 * directly on `stream` rather than through a graph), copy its tokens to
 * out_tokens[b][k*C .. k*C+C-1], then append it to every sequence's KV cache:
 * K/V recomputed from the block's final tokens at absolute positions
 * len_b .. len_b+C-1 (the lengths grow by C).  With eos_early_stop != 0 the
 * loop ends after a block in which every sequence has a committed EOS.
 * out_tokens: device int32 [batch][n_blocks*C]; blocks not generated are
 * left as they were.  *blocks_done (host, may be NULL) receives the number
 * of blocks run.  With eos_early_stop the call synchronises `stream` after
 * every block to read the EOS positions; without it, it returns with the
 * work queued.  Canvas stats accumulate over the blocks.
 * DLM_ECAP before any work if a prefix plus n_blocks*C exceeds max_prefix. */
int dlm_generate(dlm_ctx *ctx, const dlm_canvas *canvas, int batch,
                 const dlm_sampler_params *params, int n_blocks, int eos_early_stop,
                 int32_t *out_tokens, dlm_canvas_stats *stats, int *blocks_done, void *stream);

/* Kernel (c) alone: the sampler update of dlm_denoise_step applied to given
 * per-position candidates (device int32 [B][C]), confidences and entropies
 * (device float32 [B][C]).  Used to check the selection bit for bit. */
int dlm_commit(dlm_ctx *ctx, const dlm_canvas *canvas, int batch,
               const dlm_sampler_params *params, const int32_t *cand, const float *conf,
               const float *entropy, dlm_canvas_stats *stats, void *stream);

/* Read-only views of the context's buffers after a step, for inspection.
 * which: DLM_BUF_X [M][d], DLM_BUF_Q [M][H][Dh], DLM_BUF_O [M][H*Dh],
 * DLM_BUF_Y [M][d] (model element type; M = batch * C, row b*C + i),
 * DLM_BUF_CAND int32 [M], DLM_BUF_CONF float [M], DLM_BUF_ENTROPY float [M],
 * DLM_BUF_K_CACHE / DLM_BUF_V_CACHE [max_batch][Hkv][max_prefix+max_canvas][Dh];
 * with a low-bit LM head also DLM_BUF_LM_Q (the quantised weights: e4m3
 * bytes [vocab][d], or NVFP4 e2m1 pairs [vocab][d/2] with element 2i in the
 * low nibble), DLM_BUF_LM_SCALE float row scales [vocab rounded up to 256]
 * (zero padding), DLM_BUF_Y_Q / DLM_BUF_Y_SCALE the last step's quantised
 * rows and their scales ([M][d] or [M][d/2]; [M]); with the NVFP4 head
 * DLM_BUF_LM_SF / DLM_BUF_Y_SF the e4m3 block scales in the layout the
 * block-scaled tensor cores read: per 128-row block and 64-element k group a
 * 512-byte chunk, byte (m % 32) * 16 + (m / 32) * 4 + s for row m of the
 * block and its s-th 16-element block ([ceil(rows/128)][d/64][512]).
 * DLM_EINVAL for a buffer the context does not have.
 * *ptr receives a device pointer owned by the context, *bytes its size. */
enum { DLM_BUF_X = 0, DLM_BUF_Q = 1, DLM_BUF_O = 2, DLM_BUF_Y = 3, DLM_BUF_CAND = 4,
       DLM_BUF_CONF = 5, DLM_BUF_ENTROPY = 6, DLM_BUF_K_CACHE = 7, DLM_BUF_V_CACHE = 8,
       DLM_BUF_LM_Q = 9, DLM_BUF_LM_SCALE = 10, DLM_BUF_Y_Q = 11, DLM_BUF_Y_SCALE = 12,
       DLM_BUF_LM_SF = 13, DLM_BUF_Y_SF = 14 };
int dlm_debug_buffer(dlm_ctx *ctx, int which, void **ptr, size_t *bytes);

/* Full float32 logits of the rows in DLM_BUF_Y: `logits` (device float
 * [batch*canvas][vocab]) receives y W_lm^T from the same GEMM main loop as
 * the fused reduction (the store epilogue instead of the reduction); with a
 * low-bit head the logits of the last step's quantised rows (DLM_BUF_Y_Q)
 * with the same scales as the step. */
int dlm_debug_logits(dlm_ctx *ctx, int batch, int canvas, float *logits, void *stream);

/* Stages of a step, for dlm_set_stage_events.  DLM_STAGE_COMMIT is the one
 * launch that combines the LM head's partials and commits / re-noises. */
enum { DLM_STAGE_EMBED = 0, DLM_STAGE_QKV = 1, DLM_STAGE_ATTENTION = 2, DLM_STAGE_WO = 3,
       DLM_STAGE_LM_HEAD = 4, DLM_STAGE_COMMIT = 5, DLM_NUM_STAGES = 6 };

/* Measurement hook: record caller-created CUDA events (cudaEvent_t passed as
 * void*, created with timing enabled, owned by the caller) on the launch
 * stream immediately before and after `stage` of the steps issued from now
 * on: step s of a dlm_decode_block (or the s-th dlm_denoise_step call since
 * this call) uses events[2*(s % n_pairs)] and events[2*(s % n_pairs) + 1].
 * Inside a CUDA graph the records are graph nodes, so after a replay each
 * pair brackets that stage of one step.  n_pairs = 0 (events may be NULL)
 * turns the hook off.  The array is copied; the events must outlive their
 * use.  DLM_EINVAL for a bad stage or n_pairs < 0. */
int dlm_set_stage_events(dlm_ctx *ctx, int stage, void *const *events, int n_pairs);

/* Canvas attention that allocates nothing.  The pages have no counterpart to
 * this call: it exists for callers that cannot allocate device memory, such
 * as a serving engine that reserves all device memory for its own pool at
 * start-up, or code issued while a stream is being captured into a CUDA graph
 * (where cudaMalloc would synchronise the device or is not allowed).  It runs
 * the same split-KV attention kernels as dlm_denoise_step, but the split
 * partials live in a fixed array compiled into the library (8 MiB of
 * partial outputs plus 128 KiB of (max, sum) pairs: 16384 row slots, each
 * GPU that loads the library holds it until the process exits).
 *   q        device bf16 [batch*canvas][n_heads][head_dim], row b*canvas + i
 *   k_cache, v_cache  device bf16 [kv_batch][n_kv_heads][kv_capacity][head_dim];
 *            sequence b's keys are slots [0, lens[b] + canvas) (prefix
 *            followed by the canvas's own K/V)
 *   lens     device int32 [batch]; max_len (host) must be >= every lens[b]
 *   o        device bf16 [batch*canvas][n_heads*head_dim], written
 * head_dim must be 128, n_heads a multiple of n_kv_heads, batch <= kv_batch,
 * max_len + canvas <= kv_capacity (else DLM_EINVAL, nothing launched).  The
 * split plan is dlm_denoise_step's, restricted to plans whose partials fit
 * the 16384 slots (batch * n_kv_heads * splits * query-rows-per-KV-head);
 * one split needs none, so every valid size runs.
 * The first call on a device looks up the array's device address; make that
 * first call before any stream capture.  Every call shares the array, so
 * calls that overlap on the GPU (different streams, or other threads) race;
 * serialise them.  Launch errors are returned.  A device-side wait that gives
 * up (DLM_ETIMEOUT) or a failed index check (DLM_EBOUNDS, index-checking
 * build) is recorded in a device error word of the library, first error
 * kept, until dlm_attention_noalloc_check reads and clears it. */
int dlm_attention_noalloc(const void *q, const void *k_cache, const void *v_cache,
                          const int32_t *lens, int max_len, void *o, int batch, int canvas,
                          int n_heads, int n_kv_heads, int head_dim, int kv_batch,
                          int kv_capacity, void *stream);

/* Synchronise `stream`, then read and clear the device error word of
 * dlm_attention_noalloc on the current device: DLM_OK, or DLM_ETIMEOUT /
 * DLM_EBOUNDS recorded by a kernel of an earlier call (the text is in
 * dlm_last_error(NULL)); DLM_ECUDA if the runtime fails.  Like the array, the
 * word is shared by every caller on the device. */
int dlm_attention_noalloc_check(void *stream);

/* Synchronise `stream` and return the device error word (DLM_OK, or
 * DLM_ETIMEOUT / DLM_EBOUNDS set by a kernel); clears it. */
int dlm_check(dlm_ctx *ctx, void *stream);

/* ---- device timeline (tracing) ------------------------------------------
 * A library built with `python -m masked_block_diffusion_denoise_b200.build
 * --trace` (libdlm_trace.so, compiled with DLM_TRACE) stamps the GPU's
 * global timer (%globaltimer, ns) per CTA in every kernel of the step: slot
 * 0 the CTA's entry, 1 its exit (last warp out), 2 the programmatic-launch
 * wait returned, 3.. kernel phases (GEMM: first / last ring stage full,
 * first accumulator ready, last epilogue done; attention: query and first
 * K/V tile loaded, O complete, cluster barrier, peers' rows received,
 * combined; commit: rows reduced, keys sorted, done).  The table keeps the
 * last launch of each kind; 0 = not reached.  Kinds: 0 embed, 1 QKV GEMM,
 * 2 QKV epilogue, 3 attention, 4 attention combine, 5 Wo GEMM, 6 Wo
 * epilogue, 7 row quantisation, 8 LM head, 9 commit.  The default build
 * exports the same calls; they return DLM_ESTATE. */

/* Table dimensions: kinds x ctas (linear CTA index) x slots. */
int dlm_trace_layout(int *kinds, int *ctas, int *slots);
/* Synchronise the device and copy the table (uint64, kinds*ctas*slots
 * words, row-major) to host memory `table`; `words` is its capacity. */
int dlm_trace_read(unsigned long long *table, size_t words);
/* Zero the table (synchronises the device). */
int dlm_trace_clear(void);

/* Failure-detection test hook (bf16 contexts).  The next n_launches
 * tensor-core GEMM launches this context issues withhold their TMA loads:
 * the MMA warp's bounded wait for the first ring stage then runs out (after
 * 20 ms instead of the normal 2 s), the CTA stops issuing work, lets
 * nothing in flight outlive it, frees its tensor memory and records
 * DLM_ETIMEOUT in the context's error word (dlm_check returns it).  The
 * rest of the step runs on the stale activations, so its results are
 * meaningless; the context stays usable.  No device fault is involved.
 * DLM_EINVAL for n_launches < 0 or an fp32 context. */
int dlm_test_withhold_loads(dlm_ctx *ctx, int n_launches);

/* Test hook for the attention kernels' polynomial exponential (part of
 * every key tile's exponentials are computed on the FMA pipe instead of the
 * exponential unit): out[i] = 2^x[i] by Cody-Waite range reduction and a
 * cubic on [-1/2, 1/2] (maximum relative error 7.5e-5 for -125 <= x <= 8; 0
 * below -125).  x, out: device float [n].  DLM_EINVAL for NULL or n < 0. */
int dlm_test_exp2(const float *x, float *out, int n, void *stream);

/* Number of kernel launches one dlm_denoise_step made for this batch and
 * configuration (the last one issued), for launch accounting. */
int dlm_launches_per_step(const dlm_ctx *ctx);

/* Text of the first error since the last successful call, or "". */
const char *dlm_last_error(const dlm_ctx *ctx);

#ifdef __cplusplus
}
#endif
#endif /* DLM_H_ */
