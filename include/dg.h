/*
 * dg.h — C-ABI of the masked (absorbing) discrete-diffusion denoise path.
 *
 * The operations follow the problem statement of "DiffusionGemma 技术报告"
 * (full translation page):
 *   - §3.1 "块自回归生成", KV-cache initialisation: the context is encoded once
 *     by a causal pass, H = Encoder(h), and its keys/values are kept
 *     (dg_prefill);
 *   - §3.1 / §3.2 "推理时的去噪框架": a 256-token canvas is denoised by a decoder
 *     that attends bidirectionally inside the canvas and to the KV cache, and
 *     produces logits per canvas position (dg_denoise_step, without ever writing
 *     the logits);
 *   - §3.3 "DiffusionGemma 采样器", entropy-bounded refinement: positions are
 *     accepted in ascending order of entropy (dg_eb_sample, also run inside
 *     dg_denoise_step);
 *   - §3.1: one canvas is denoised to completion before it is committed
 *     (dg_generate_block).
 * Architecture numbers (30 layers, sliding window 1024, 256-token canvas, 262K
 * vocabulary, 128 experts top-8 plus a shared expert, timestep embedding) come
 * from the explainer page "DiffusionGemma 深度解析", list "核心架构参数".
 *
 * Conventions
 *   - Every data pointer is a DEVICE pointer owned by the caller unless stated.
 *     Handles (dg_model, dg_kv) are owned by the library and released with their
 *     destroy call.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls enqueue work and return without synchronising, except where noted.
 *   - Every call returns a dg_status; nothing is thrown across the ABI and
 *     nothing aborts.  Arguments are validated before any launch.  Errors of
 *     kernels already enqueued surface on a later call or on dg_sync_status.
 *   - Row-major layouts; [a, b] means a rows of b contiguous elements.
 *   - Model dimensions: d = d_model, Hq / Hkv query / key-value heads of size h,
 *     E experts with top_k routing and intermediate I, shared expert
 *     intermediate Is, vocabulary V (the [MASK] id is V), canvas C, window Wn.
 *     For a prefilled prompt of length P the cached window is W = min(P, Wn).
 */
#ifndef DG_H
#define DG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum dg_status {
  DG_OK = 0,
  DG_ERR_INVALID_ARG = 1, /* a null pointer, a size out of range, a bad value */
  DG_ERR_UNSUPPORTED = 2, /* a valid request this build does not implement    */
  DG_ERR_OOM = 3,         /* device allocation failed                          */
  DG_ERR_CUDA = 4,        /* a CUDA runtime/driver error (message kept)         */
  DG_ERR_TIMEOUT = 5,     /* a bounded device-side wait gave up                 */
  DG_ERR_INTERNAL = 6
} dg_status;

typedef enum dg_dtype {
  DG_F32 = 0,        /* fp32 weights; the SIMT path carries activations in fp64 */
  DG_BF16 = 1,       /* bf16 weights and activations, fp32 accumulation          */
  DG_BF16_FP8EXP = 2, /* as DG_BF16 but routed-expert weights in FP8 E4M3        */
  DG_BF16_FP4EXP = 3  /* as DG_BF16 but routed-expert weights in NVFP4            */
} dg_dtype;

typedef struct dg_config {
  int32_t n_layers, d_model, n_q_heads, n_kv_heads, head_dim;
  int32_t n_experts, top_k, expert_inter, shared_inter;
  int32_t vocab;       /* V; the [MASK] token id is V                       */
  int32_t window;      /* sliding window Wn of the causal prompt pass        */
  int32_t canvas;      /* C                                                   */
  float rope_base;     /* rotary base (pairs (i, i + h/2), angle p*base^(-2i/h)) */
  float rms_eps;
  float logit_scale;   /* logits = logit_scale * RMSNorm(x) W_lm^T          */
  int32_t dtype;       /* dg_dtype                                            */
  int32_t max_batch;   /* largest B any call on this model will pass          */
  int32_t max_prompt;  /* largest P any dg_prefill on this model will pass    */
  int32_t sc_inter;    /* inner size of the self-conditioning FFW; 0: none    */
} dg_config;

/* Weights of one layer (device pointers, borrowed for the model's lifetime).
 * Element type: fp32 for DG_F32, bf16 otherwise; for DG_BF16_FP8EXP the three
 * routed-expert tensors are FP8 E4M3 bytes with fp32 scales, one per
 * (row, 128 consecutive input columns): w = q * scale.  For DG_BF16_FP4EXP
 * ("NVFP4", the agentlenshq page on DiffusionGemma: NVFP4 kernels for Blackwell)
 * they are E2M1 codes packed two per byte ([E, I, d/2] and [E, d, I/2] bytes,
 * element 2i in the low nibble), one E4M3 block scale byte per (row, 16 consecutive
 * input columns) in the *_scale fields and one fp32 tensor scale per tensor in the
 * *_tscale fields: w = e2m1(code) * block scale * tensor scale.  The kernel widens
 * the codes to bf16 in shared memory, so a weight must be exact in fp32: the
 * tensor scale must be a positive power of two (read at model creation;
 * DG_ERR_INVALID_ARG otherwise). */
typedef struct dg_layer_weights {
  const void* wqkv;   /* [(Hq + 2 Hkv) h, d]: query heads, key heads, value heads */
  const void* wo;     /* [d, Hq h]                                                */
  const void* router; /* [E, d]                                                   */
  const void* gate;   /* [E, I, d]                                                */
  const void* up;     /* [E, I, d]                                                */
  const void* down;   /* [E, d, I]                                                */
  const void* gate_scale;  /* FP8: fp32 [E, I, d/128]; NVFP4: E4M3 [E, I, d/16]; else NULL */
  const void* up_scale;    /* FP8: fp32 [E, I, d/128]; NVFP4: E4M3 [E, I, d/16]           */
  const void* down_scale;  /* FP8: fp32 [E, d, I/128]; NVFP4: E4M3 [E, d, I/16]           */
  const void* sgate;  /* [Is, d]                                                  */
  const void* sup;    /* [Is, d]                                                  */
  const void* sdown;  /* [d, Is]                                                  */
  const float* gate_tscale; /* NVFP4 only: fp32 [1] tensor scale, else NULL       */
  const float* up_tscale;   /* NVFP4 only: fp32 [1]                               */
  const float* down_tscale; /* NVFP4 only: fp32 [1]                               */
} dg_layer_weights;

typedef struct dg_weights {
  const void* tok_emb;            /* [V + 1, d]; row V embeds [MASK]           */
  const void* lm_head;            /* [V, d] (untied)                           */
  const dg_layer_weights* layers; /* HOST array of n_layers entries, copied    */
  /* The self-conditioning FFW (sc_inter > 0; else ignored): z = sc_down (silu(sc_gate y)
   * * (sc_up y)) for y = p0 E ("DiffusionGemma 技术报告", §3.2 "去噪迭代").        */
  const void* sc_gate;            /* [sc_inter, d]                              */
  const void* sc_up;              /* [sc_inter, d]                              */
  const void* sc_down;            /* [d, sc_inter]                              */
} dg_weights;

typedef struct dg_model dg_model;
typedef struct dg_kv dg_kv;

/* Human-readable name of a status code (static storage). */
const char* dg_status_str(dg_status s);

/* Detail of the last error raised on the calling thread ("" if none). */
const char* dg_last_error(void);

/* Validates the configuration and weight pointers, plans the kernels and
 * allocates the library's device workspace for max_batch canvases and prompts
 * up to max_prompt tokens, on the current CUDA device.  Synchronous.  With
 * sc_inter > 0 it also builds the transposed embedding [d, V] the self-conditioning
 * product reads and the workspace for p0 [max_batch C, V] (bf16 on the bf16 paths).
 * Errors: DG_ERR_INVALID_ARG (null, non-positive or inconsistent sizes, d_model not a
 * multiple of 8, C > 1024,
 * Hq not a multiple of Hkv, h odd; with sc_inter > 0: a null FFW pointer, V not a
 * multiple of 2 (fp32) or 8 (bf16), sc_inter not a multiple of 64 (bf16)),
 * DG_ERR_UNSUPPORTED (a shape the tensor-core
 * kernels do not tile: bf16 and FP8 need d % 256, I % 128, Is % 64, (Hq + 2 Hkv) h % 64
 * and Hq h % 64; FP8 experts also d, I <= 4096), DG_ERR_OOM, DG_ERR_CUDA. */
dg_status dg_model_create(const dg_config* cfg, const dg_weights* w, dg_model** out);

/* Synchronises the device and frees the model's workspace. NULL is a no-op. */
dg_status dg_model_destroy(dg_model* m);

/* Waits for the model's queued work and reports asynchronous failures: a CUDA
 * error (DG_ERR_CUDA) or a device-side bounded wait that gave up
 * (DG_ERR_TIMEOUT; the flag is cleared by this call). */
dg_status dg_sync_status(dg_model* m, void* stream);

/* Causal encoder pass over B prompts of P tokens (prompt: [B, P] int32 ids in
 * [0, V)).  Rows attend to keys j with i - Wn < j <= i; no timestep embedding.
 * The post-RoPE keys and the values of the last W = min(P, Wn) positions of every
 * layer are kept in a new library-owned handle *out:
 *   K, V: [n_layers, B, Hkv, W, h] (bf16; fp64 for DG_F32).
 * Requires 1 <= B <= max_batch, 1 <= P <= max_prompt.  Ids are checked on the
 * device; an id outside [0, V) yields DG_ERR_INVALID_ARG on the next status read. */
dg_status dg_prefill(dg_model* m, const int32_t* prompt, int32_t B, int32_t P,
                     dg_kv** out, void* stream);

/* The same causal pass into an existing handle made by dg_prefill for this model
 * with the same B (any 1 <= P <= max_prompt; a handle grown by dg_append_block returns
 * to a prompt of P tokens): its buffers are overwritten in place (no allocation), so a
 * serving loop can keep one handle per slot.  Block graphs are captured per (handle,
 * context length), so a graph captured for the same P is replayed.  The caller orders
 * this call after every earlier use of the handle (same stream, or synchronised).
 * DG_ERR_INVALID_ARG if the handle belongs to another model or B differs. */
dg_status dg_prefill_into(dg_model* m, const int32_t* prompt, int32_t B, int32_t P,
                          dg_kv* kv, void* stream);

/* Frees a KV handle (after synchronising its stream). NULL is a no-op. */
dg_status dg_kv_destroy(dg_kv* kv);

/* Batch size, prompt length and window of a KV handle (host values). */
dg_status dg_kv_info(const dg_kv* kv, int32_t* B, int32_t* P, int32_t* W);

/* One denoise forward plus one Entropy-Bound sampler step on B = kv's batch
 * canvases (canvas: [B, C] int32 ids in [0, V], V = [MASK]; mask: [B, C] uint8,
 * 1 = still masked; both updated in place).
 * The forward embeds the canvas, adds the sinusoidal embedding of
 * tau = steps_left / T, runs the layers (queries at absolute positions P..P+C-1,
 * keys = the cached window followed by all C canvas rows, one softmax) and the
 * LM head, and writes per position the softmax entropy in nats (entropy: [B, C]
 * fp32, clamped at 0) and the argmax id (argmax: [B, C] int32, lowest id on
 * ties).  The logits are never stored.  The sampler then commits, per canvas, the
 * n = min(m, max(k_gamma, ceil(m / steps_left))) masked positions of lowest
 * (entropy, position), where m is the number masked and k_gamma the longest
 * prefix whose entropies sum to <= gamma (sums in 2^-48 fixed point); committed
 * positions take their argmax and are unmasked.  n_committed: [B] int32.
 * A canvas with m = 0 is left unchanged (n = 0).
 * Requires 1 <= steps_left <= T, gamma >= 0 (not NaN). */
dg_status dg_denoise_step(dg_model* m, const dg_kv* kv, int32_t* canvas, uint8_t* mask,
                          int32_t steps_left, int32_t T, float gamma,
                          float* entropy, int32_t* argmax, int32_t* n_committed,
                          void* stream);

/* Denoises B = kv's batch canvases from all [MASK] with at most T forwards
 * (steps_left = T, T-1, ..., 1), without synchronising the host between steps;
 * the loop stops on the device as soon as no canvas has a masked position left.
 * canvas_out: [B, C] int32 (no [MASK] remains); n_forwards: [B] int32, the
 * number of forwards after which that canvas had no [MASK] left (nullable);
 * router_load: [n_layers, E] int32 counts of (token, expert) routings summed
 * over the block (nullable).  Requires T >= 1, gamma >= 0. */
dg_status dg_generate_block(dg_model* m, const dg_kv* kv, int32_t T, float gamma,
                            int32_t* canvas_out, int32_t* n_forwards,
                            int32_t* router_load, void* stream);

/* Block-autoregressive continuation ("DiffusionGemma 技术报告", §3.1: each finished
 * block joins the context through the causal encoder pass before the next block is
 * denoised; §3.4, the K - 1 extra forwards of K blocks in the tokens-per-forward
 * count).  tokens: [B, C] int32 ids in [0, V), the finished canvases of kv's batch.
 * The block's rows run the causal pass at positions P .. P + C - 1 (keys: the cached
 * window and the block's own rows within the sliding window, no timestep embedding);
 * then every layer's cache keeps the last min(W + C, window) positions and kv's P grows
 * by C.  (Block graphs are captured per context length, so none is invalidated.)
 * Requires P + C <= max_prompt (the context a model is created for bounds the whole
 * sequence, prompt and appended blocks) and no [MASK] in tokens (checked on the
 * device: DG_ERR_INVALID_ARG on the next status read). */
dg_status dg_append_block(dg_model* m, dg_kv* kv, const int32_t* tokens, void* stream);

/* n_blocks blocks one after the other: dg_generate_block, then (except after the
 * last) dg_append_block of the finished canvases.  out: [B, n_blocks C] int32, block k
 * of canvas b in columns k C .. k C + C - 1; n_forwards: [n_blocks, B] int32 forwards
 * per block and canvas (nullable).  kv ends extended by n_blocks - 1 blocks.
 * Requires n_blocks >= 1 and P + (n_blocks - 1) C <= max_prompt. */
dg_status dg_generate_blocks(dg_model* m, dg_kv* kv, int32_t n_blocks, int32_t T, float gamma,
                             int32_t* out, int32_t* n_forwards, void* stream);

/* The sampler step alone, on caller-provided statistics: entropy [B, C] fp32,
 * argmax [B, C] int32, canvas/mask [B, C] updated in place, n_committed [B].
 * Same rule as in dg_denoise_step (a NaN entropy sorts as +inf, a negative one
 * as 0).  Requires 1 <= C <= 1024, 1 <= steps_left, gamma >= 0. */
dg_status dg_eb_sample(const float* entropy, const int32_t* argmax, int32_t* canvas,
                       uint8_t* mask, int32_t B, int32_t C, int32_t steps_left,
                       float gamma, int32_t* n_committed, void* stream);

/* ---- the Report's default sampler ("DiffusionGemma 技术报告", §3.2 "画布初始化",
 * "多项式扩散", §3.3 "熵有界的 token 精炼", "温度退火", "自适应停止启发式") ----------
 * A canvas starts from uniformly drawn tokens and is refined for at most N steps:
 * step k (0-based) runs the forward at t = (N - k) / N (timestep input t), tempers the
 * logits by tau = tau_min + (tau_max - tau_min) t, draws a token at every position
 * from softmax(l / tau) (Gumbel-max), and accepts, in ascending order of the tempered
 * entropy (ties: lower position), the longest prefix whose entropies satisfy
 * sum - max <= b (the mutual-information bound; at least one position); every other
 * position is re-noised to a uniform token.  After a step the canvas stops when the
 * mean tempered entropy is below e_stop (sum of 2^-48 fixed-point entropies
 * < C floor(e_stop 2^48)) and the argmax sequence equals the previous step's; then,
 * or after step N - 1, the canvas becomes that step's argmax sequence.
 * Random draws: SplitMix64 used counter-wise, one seed per canvas (seeds: [B] uint64,
 * device); stream keys mix64(seed + j G), j = 1 initial tokens, 2 Gumbel noise,
 * 3 re-noising (the exact counters are stated in k_anneal.cuh and oracle/anneal.py). */
typedef struct dg_anneal_params {
  int32_t N;      /* maximum denoising steps, 1 .. 65536 (the Report: 48) */
  float b;        /* mutual-information tolerance, >= 0, not NaN (0.1) */
  float tau_max;  /* temperature at t = 1, finite > 0 (0.8) */
  float tau_min;  /* temperature at t = 0, finite > 0 (0.4) */
  float e_stop;   /* mean-entropy threshold of the adaptive stop, 0 .. 16 (0.005) */
} dg_anneal_params;

/* The whole annealed block for B = kv's batch canvases without host synchronisation
 * (a device-controlled loop that ends once every canvas has stopped).
 * params: host pointer; seeds: [B] uint64 device; canvas_out: [B, C] int32 in [0, V);
 * n_forwards: [B] int32, the forward count at which each canvas stopped (nullable).
 * Requires V <= 2^24. */
dg_status dg_generate_block_annealed(dg_model* m, const dg_kv* kv,
                                     const dg_anneal_params* params, const uint64_t* seeds,
                                     int32_t* canvas_out, int32_t* n_forwards, void* stream);

/* Step k's forward alone: canvas [B, C] int32 ids in [0, V); writes the tempered
 * entropy [B, C] fp32, the argmax [B, C] int32 and the Gumbel-max draw sampled
 * [B, C] int32.  Self-conditioning (nullable, as in dg_selfcond_forward): z_in [B, C, d]
 * added to the canvas rows' input, z_out [B, C, d] the next forward's z (p0 at
 * temperature 1; requires sc_inter > 0).  Requires 0 <= k < N. */
dg_status dg_anneal_forward(dg_model* m, const dg_kv* kv, const int32_t* canvas, int32_t k,
                            const dg_anneal_params* params, const uint64_t* seeds,
                            float* entropy, int32_t* argmax, int32_t* sampled,
                            const void* z_in, void* z_out, void* stream);

/* Step k's refinement alone, on caller-provided statistics (entropy, argmax, sampled:
 * [B, C]).  canvas [B, C] is rewritten; prev_argmax [B, C] holds the previous step's
 * argmax sequence (read at k > 0) and receives this one; state [B] int32 is 0 while a
 * canvas runs and becomes k + 1 when it stops (a canvas whose state is not 0 is left
 * untouched); n_accepted [B] int32 (nullable).  The initial canvas of dg_anneal_init
 * and state 0 start a block.  Requires 1 <= C <= 1024, 1 <= V <= 2^24, 0 <= k < N. */
dg_status dg_anneal_sample(const float* entropy, const int32_t* argmax, const int32_t* sampled,
                           int32_t* canvas, int32_t* prev_argmax, int32_t* state,
                           int32_t* n_accepted, int32_t B, int32_t C, int32_t V, int32_t k,
                           const dg_anneal_params* params, const uint64_t* seeds,
                           void* stream);

/* x_1 of every canvas: canvas [B, C] int32 uniform tokens in [0, V) from stream 1 of
 * seeds [B]; prev_argmax [B, C] set to -1 and state [B] to 0 (both nullable). */
dg_status dg_anneal_init(int32_t* canvas, int32_t* prev_argmax, int32_t* state, int32_t B,
                         int32_t C, int32_t V, const uint64_t* seeds, void* stream);

/* ---- self-conditioning ("DiffusionGemma 技术报告", §3.2 "解码器前向传播", "去噪迭代";
 * models created with sc_inter > 0) -------------------------------------------------
 * After a forward the decoder's clean-token probabilities p0 = softmax(l) (temperature
 * 1, the V real tokens) are mixed with the embedding rows, y = p0 E, and
 * z = sc_down (silu(sc_gate y) * (sc_up y)) is added to the canvas rows' input of the
 * next forward.  The block calls (dg_generate_block, dg_generate_blocks,
 * dg_generate_block_annealed) carry z from forward to forward, 0 at a block's first, as
 * long as it is switched on (the default for such models); dg_denoise_step,
 * dg_debug_forward and dg_anneal_forward run without it (z = 0). */

/* Switches the block calls' self-conditioning on (on != 0; needs sc_inter > 0) or off. */
dg_status dg_set_selfcond(dg_model* m, int32_t on);

/* One Entropy-Bound forward with self-conditioning: z_in [B, C, d] is added to the
 * canvas rows' input (NULL: none), entropy/argmax as in dg_denoise_step, and the next
 * forward's z written to z_out [B, C, d] (may equal z_in).  z is in the accumulate type:
 * fp64 for DG_F32 models, fp32 otherwise.  Requires sc_inter > 0. */
dg_status dg_selfcond_forward(dg_model* m, const dg_kv* kv, const int32_t* canvas,
                              int32_t steps_left, int32_t T, const void* z_in, float* entropy,
                              int32_t* argmax, void* z_out, void* stream);

/* Test hook: the forward of dg_denoise_step without the sampler.  Writes
 * entropy/argmax as above and, when non-NULL, the logits [B*C, V] fp32 and the
 * final residual stream [B*C, d] fp32 (before the final norm). */
dg_status dg_debug_forward(dg_model* m, const dg_kv* kv, const int32_t* canvas,
                           int32_t steps_left, int32_t T, float* entropy,
                           int32_t* argmax, float* logits, float* hidden, void* stream);

/* Copies a KV handle's cached keys and values into caller buffers
 * (k, v: [n_layers, B, Hkv, W, h] of the cache's element type). */
dg_status dg_kv_read(const dg_kv* kv, void* k, void* v, void* stream);

/* ---- measurement hooks (no counterpart on the pages) -------------------------
 * Kernel groups whose device time can be recorded while the path runs. */
typedef enum dg_kernel_kind {
  DG_KIND_EXPERTS = 0,   /* routed-expert FFN: gate/up (SwiGLU) and down launches   */
  DG_KIND_LMHEAD = 1,    /* LM-head GEMM + online entropy statistics (+ merge)     */
  DG_KIND_ATTENTION = 2, /* canvas / prompt attention                             */
  DG_KIND_DENSE = 3,     /* QKV and O projections (main stream)                   */
  DG_KIND_SHARED = 4,    /* shared-expert projections (a concurrent graph branch) */
  DG_KIND_ROUTING = 5,   /* RMSNorm, router, top-k and permutation launches       */
  DG_KIND_GLUE = 6,      /* embedding, combine + RMSNorm, sampler                 */
  DG_KIND_COUNT = 7
} dg_kernel_kind;

/* Starts recording a pair of CUDA events around every launch group of each
 * kind, on the stream the launches use.  Costs one event record per launch.
 * While recording, dg_generate_block runs an unrolled block of at most
 * max_forwards forwards (0: T) instead of its device-controlled loop; given the
 * number of forwards the loop ran (n_forwards), it replays the same forwards on the
 * same canvases. */
dg_status dg_profile_start(dg_model* m, int32_t max_forwards);

/* Synchronises the device, writes the summed device milliseconds
 * (ms[DG_KIND_COUNT]) and the number of recorded launch groups
 * (groups[DG_KIND_COUNT]) since dg_profile_start, and stops recording. */
dg_status dg_profile_stop(dg_model* m, float* ms, int64_t* groups);

/* Number of (MoE layer pass, expert) pairs in which the expert received at least
 * one row — i.e. expert weight tiles streamed — since dg_profile_start (or model
 * creation).  Synchronises the device. */
dg_status dg_expert_units(dg_model* m, int64_t* units);

/* Kernels launched per loop iteration (one forward + sampler step + loop control) by
 * the last dg_generate_block replay; its device-controlled loop runs as many
 * iterations as forwards were needed (at most T), which n_forwards reports. */
dg_status dg_block_loop_launches(const dg_model* m, int64_t* per_forward);

/* Number of kernels this model has launched since it was created (host count). */
dg_status dg_launch_count(const dg_model* m, int64_t* out);

/* ---- allocation-free entry point (no counterpart on the pages) --------------
 * The LM-head entropy step of the forward (final RMSNorm, logits = logit_scale *
 * xn W_lm^T, per-row softmax entropy and argmax; the logits are never stored),
 * for callers that cannot allocate device memory: code whose allocator belongs
 * to another runtime, real-time or embedded callers whose device memory is fixed
 * up front, or callers that must not touch the allocator between steps.  It
 * needs no model handle and calls no cudaMalloc, cudaFree or allocating library
 * routine.  Its scratch is a file-scope device array of 6 MiB (256 rows x 4096
 * columns of bf16, plus the per-tile statistics for up to 262,144 classes) that
 * every GPU loading the library holds until the process exits.
 *   hidden:  [M, d] fp32 residual rows (device);  lm_head: [V, d] bf16 (device,
 *            16-byte aligned);  entropy: [M] fp32 out;  argmax: [M] int32 out.
 *   Limits:  1 <= M <= 256, 1 <= V <= 262144, d a multiple of 64 in [64, 4096];
 *            larger sizes return DG_ERR_INVALID_ARG before any launch.
 * The first call on a device (with that device current) looks up the scratch
 * array's device address, so make that first call before any stream capture.
 * All calls on a device share the scratch: calls whose kernels may overlap on
 * the GPU (other streams, other host threads) race and must be serialised.  A
 * device-side wait that gives up marks the outputs (entropy NaN, argmax -1). */
dg_status dg_lmhead_entropy_noalloc(const float* hidden, const void* lm_head, int32_t M,
                                    int32_t V, int32_t d, float rms_eps, float logit_scale,
                                    float* entropy, int32_t* argmax, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* DG_H */
