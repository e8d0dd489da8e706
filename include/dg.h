/*
 * dg.h -- C ABI of the B200 (sm_100a) canvas denoising step library (libdg.so).
 *
 * The operation: a canvas of canvas_len token slots (256 on the pages) that
 * starts as all [MASK] is refined by repeated passes through a stack of
 * decoder blocks; each pass ends by locking in the most confident
 * still-masked slots.  Sources (page title, section):
 *   "Hands-On with Diffusion Gemma: Another Gemma with a Diffusion Mechanism",
 *     "How Is This Different from Previous Models?" (canvas of 256 masked
 *     slots, repeated decoding passes) and "Detailed Specs" (30 blocks as
 *     (5 local + 1 global) x 5, hidden 2816, MoE, sliding-window local
 *     attention, GQA global attention, RoPE / p-RoPE, tied embed_tokens and
 *     lm_head, input / post-attention / pre-feedforward / final norms,
 *     router, encoder KV cache shared with the decoder);
 *   "DiffusionGemma: The Diffusion Era Begins with 4x Faster Text Generation",
 *     "What is Diffusion ..." (locked tokens become context) and
 *     "DiffusionGemma's Technical Architecture" (128 experts, 8 active + 1
 *     shared, canvas 256, window 1024, vocab 262K, bidirectional attention
 *     over the canvas plus cross-attention into the prompt's cached KV);
 *   "DiffusionGemma: Google's Experimental Diffusion LLM", "How Text
 *     Diffusion Actually Works" (a small fixed number of passes per block).
 * Readings where the pages are silent (one joint softmax over prompt window
 * and canvas, RMSNorm with unit scales, p = 0.25 for p-RoPE, top-k by logit
 * with lowest-index ties, k = ceil(remaining / steps_left) commits per pass,
 * confidence = largest softmax probability with the mask id excluded) are the
 * library's defined behaviour; each is stated at the call it affects.
 *
 * Conventions for every call:
 *  - Return value: DG_OK (0) or a negative DG_ERR_* code.  No C++ exception
 *    crosses this interface.  dg_last_error() gives a text for the last error
 *    of a context.
 *  - Argument errors are detected before any work is queued and leave every
 *    output untouched.
 *  - All work is queued on the CUDA stream given to dg_create() and is
 *    asynchronous unless stated otherwise.  A context is not thread-safe.
 *  - Errors raised inside kernels (a bounded wait that gave up, an index out
 *    of range) are recorded in a device error word and reported by dg_sync()
 *    (and by the calls that end with a synchronisation).
 *  - "dev" pointers are CUDA device pointers, "host" pointers ordinary host
 *    memory.  The library never frees a caller's pointer.
 *  - Matrices are row-major.  bf16 is IEEE bfloat16 stored as uint16_t.
 */
#ifndef DG_H
#define DG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  DG_OK = 0,
  DG_ERR_INVALID_ARG = -1,   /* a null pointer, a size out of range, a bad config */
  DG_ERR_BAD_STATE = -2,     /* call out of order (e.g. a step before the prompt KV is set) */
  DG_ERR_OOM = -3,           /* a device allocation failed or would pass alloc_limit_bytes */
  DG_ERR_CUDA = -4,          /* a CUDA runtime call failed (no device, launch failure) */
  DG_ERR_TIMEOUT = -5,       /* a bounded in-kernel wait gave up; results are invalid */
  DG_ERR_DEVICE_FAULT = -6,  /* a kernel flagged an out-of-range index; results are invalid */
  DG_ERR_UNSUPPORTED = -7    /* a shape outside what the kernels implement */
};

typedef struct dg_ctx dg_ctx;

/*
 * Model and capacity description.  Shape limits checked by dg_create():
 *   d_model a multiple of 64 in [128, 4096]; d_ff a multiple of 64;
 *   head_dim in {64, 128, 256};
 *   n_q_heads a multiple of n_kv_heads; 1 <= top_k <= min(n_experts, 32);
 *   n_experts a multiple of 4 in [4, 256]; (n_q_heads + 2 n_kv_heads) * head_dim <= 16384;
 *   n_shared in {0, 1}; 1 <= canvas_len <= 256; max_batch * canvas_len <= 4096;
 *   0 <= mask_id < vocab; window >= 1; global_every >= 1;
 *   2 * n_experts * ceil(max_batch * canvas_len / 32) + 2 * n_experts + 1 <= 51200
 *   (the router groups a pass's rows in one CTA's 200 KB of shared memory).
 * Layer l (0-based) is global iff (l + 1) % global_every == 0: it attends to
 * all prompt keys and rotates the first ceil(prope_fraction * head_dim / 2)
 * RoPE pairs.  Other layers attend to the last min(window, n_prompt) prompt
 * keys and rotate every pair.  rope_enabled = 0 turns all rotation off.
 * weight_std is the standard deviation of the seeded weights (0.02).
 */
typedef struct dg_config {
  int n_layers, d_model, n_q_heads, n_kv_heads, head_dim;
  int n_experts, top_k, n_shared, d_ff;
  int vocab, canvas_len, window, global_every;
  int mask_id, max_batch, max_prompt;
  float rms_eps, rope_theta, prope_fraction;
  int rope_enabled;
  double weight_std;         /* the generator's scale is float32(weight_std * sqrt(3) / 65536) */
  size_t alloc_limit_bytes;  /* 0 = no limit; otherwise dg_create fails with DG_ERR_OOM
                                instead of allocating more than this many device bytes */
  int expert_dtype;          /* DG_DTYPE_BF16, or DG_DTYPE_FP8_E4M3: the expert FFN weights
                                (routed and shared) are used as FP8 E4M3 codes q with one
                                fp32 scale s per weight row, w = q * s, where
                                s = max|w_bf16| / 448 and q = E4M3(w_bf16 / s) (fp32
                                division, round to nearest even); activations stay bf16 */
  int max_context;           /* capacity, in positions per sequence, of the library's own KV
                                cache (dg_encode, dg_generate); 0 = none is allocated.  It
                                takes max_batch * n_kv_heads * max_context * head_dim * 2
                                bf16 values per layer */
} dg_config;

enum { DG_DTYPE_BF16 = 0, DG_DTYPE_FP8_E4M3 = 1 };

/* Pages: "Hands-On with Diffusion Gemma", Detailed Specs (the block structure
 * and sizes a config describes).
 * Creates a context on the current CUDA device: checks the config, allocates
 * the weights (bf16) and the workspace, and records `cuda_stream`
 * (a cudaStream_t, NULL = legacy default stream).  Weights are not yet drawn.
 * *out is set only on success.  Synchronous. */
int dg_create(const dg_config* cfg, void* cuda_stream, dg_ctx** out);

/* Pages: "Hands-On with Diffusion Gemma", Detailed Specs (the tensors: tied
 * embed_tokens / lm_head, q/k/v/o, router, experts, shared expert, norms); the
 * pages give no weight values, so they are seeded and synthetic.
 * Draws every weight on the device from `seed` (the tied embedding, and per
 * layer the q/k/v/o projections, router, routed experts' gate/up/down and the
 * shared expert's gate/up/down), N(0, weight_std) by the SplitMix64 counter
 * generator with a four-term Irwin-Hall normal, rounded to bf16; norm scales
 * are set to 1.  The value of each logical element depends only on
 * (seed, tensor, element index), never on the physical layout. */
int dg_init_weights(dg_ctx* ctx, uint64_t seed);

/* Pages: "Hands-On with Diffusion Gemma", Detailed Specs (the tensor names).
 * Replace one weight tensor with the caller's values, after dg_init_weights
 * (which sets every tensor).  src: bf16 row-major of the logical shape below
 * (fp32 for the norm weights), host or device memory, read during the call;
 * bytes must equal the tensor's size exactly.  Names:
 *   "embed" [vocab][d_model] (tied with the head), "ln_final" fp32 [d_model];
 *   per layer l (the name carries ":l", e.g. "wq:3"):
 *   "wq" [n_q_heads*head_dim][d_model], "wk" / "wv" [n_kv_heads*head_dim][d_model],
 *   "wo" [d_model][n_q_heads*head_dim], "wr" [n_experts][d_model],
 *   "wg" / "wu" [n_experts][d_ff][d_model] (routed gate / up), "wd" [n_experts][d_model][d_ff],
 *   "sg" / "su" [d_ff][d_model], "sd" [d_model][d_ff] (the shared expert),
 *   "ln_in" / "ln_post" / "ln_ff" fp32 [d_model].
 * The values are copied into the library's own layout (q/k/v rows fused, gate
 * and up rows interleaved).  Captured passes stay valid.  Returns DG_OK,
 * DG_ERR_INVALID_ARG (unknown name, layer out of range, wrong size),
 * DG_ERR_BAD_STATE (weights not initialised) or DG_ERR_CUDA. */
int dg_load_weights(dg_ctx* ctx, const char* name, const void* src, size_t bytes);

/* Pages: "Hands-On with Diffusion Gemma", Detailed Specs (the encoder's KV cache
 * is shared with the decoder); "DiffusionGemma: The Diffusion Era Begins ...",
 * DiffusionGemma's Technical Architecture (cross-attention into the prompt's
 * cached KV).
 * Borrows the prompt's cached keys and values for one layer (the encoder's KV
 * cache the decoder cross-attends to).  k, v: dev bf16 [batch][n_kv_heads]
 * [n_prompt][head_dim], keys already rotated.  No copy is made: the buffers
 * must stay valid and unchanged until this layer's next dg_set_prompt_kv or
 * dg_destroy.  Every layer must be given the same batch and n_prompt before a
 * step; canvas row i then sits at position n_prompt + i.
 * 1 <= batch <= max_batch, 1 <= n_prompt <= max_prompt. */
int dg_set_prompt_kv(dg_ctx* ctx, int layer, const void* k, const void* v,
                     int batch, int n_prompt);

/* The pages have no counterpart: a workload control (skewed expert popularity).
 * Adds a fixed bias (dev fp32 [n_experts]) to the router logits of every
 * layer, or removes it when bias == NULL.  The bias is copied. */
int dg_set_router_bias(dg_ctx* ctx, const float* bias);

/* Pages: "Hands-On with Diffusion Gemma", How Is This Different from Previous
 * Models? (a canvas of masked slots refined by repeated passes; the probability
 * distribution judges which tokens are final) and "DiffusionGemma: The
 * Diffusion Era Begins ...", What is Diffusion ... (locked-in tokens become
 * context for the rest).
 * One denoising pass over `batch` canvases, then the commit.
 * canvas: dev int32 [batch][canvas_len], updated in place: with r the number
 * of slots equal to mask_id in a canvas, the k = ceil(r / steps_left) masked
 * slots of highest confidence (ties toward the lower slot) receive their
 * argmax token; all other slots are unchanged.  steps_left >= 1.
 * conf_out (dev fp32 [batch][canvas_len]) receives every slot's confidence,
 * the largest softmax probability of its logits with the mask id excluded;
 * committed_out (dev uint8 [batch][canvas_len]) receives 1 for the slots
 * committed by this pass.  Both may be NULL.
 * The pass is enqueued on the context's stream and the call returns without
 * waiting (dg_sync waits and reports device errors).  On a context created
 * with its own (non-default) stream and with profiling off, the second call
 * for a given batch records the pass into a CUDA graph that later calls
 * replay; dg_set_prompt_kv with other buffers or shapes, and
 * dg_set_router_bias, drop the recorded graphs.  Kernels are chained with
 * programmatic dependent launch.  Setting DG_NO_GRAPH=1 or DG_NO_PDL=1 in the
 * environment turns either off. */
int dg_canvas_step(dg_ctx* ctx, int32_t* canvas, int batch, int steps_left,
                   float* conf_out, uint8_t* committed_out);

/* Pages: as dg_canvas_step.
 * dg_canvas_step on HOST buffers: copies the canvas to the device, runs the
 * pass, copies canvas (and conf / committed when not NULL) back, and returns
 * after the results are in host memory (synchronous). */
int dg_canvas_step_host(dg_ctx* ctx, int32_t* canvas_host, int batch, int steps_left,
                        float* conf_host, uint8_t* committed_host);

/* Pages: "DiffusionGemma: Google's Experimental Diffusion LLM", How Text
 * Diffusion Actually Works (a small, fixed number of passes per block).
 * n_steps passes with steps_left = n_steps, n_steps - 1, ..., 1: every masked
 * slot is committed at the end.  canvas: dev int32 [batch][canvas_len], in
 * place.  Ends with a synchronisation and reports device errors. */
int dg_denoise_block(dg_ctx* ctx, int32_t* canvas, int batch, int n_steps);

/* Pages: "Hands-On with Diffusion Gemma", How Is This Different from Previous
 * Models? (the causal part ingests the input once and builds the state the
 * canvas reads; after 256 tokens the model returns to causal context building)
 * and Detailed Specs (Encoder and Decoder: unidirectional causal attention,
 * KV cache relayed to the decoder; weight sharing); "DiffusionGemma: The
 * Diffusion Era Begins ...", DiffusionGemma's Technical Architecture (the
 * autoregressive encoder creates the prompt's KV cache).
 * The causal encoder: runs n tokens per sequence (tokens: host or dev int32
 * [batch][n], read during the call) through every block with the decoder's
 * weights and causal attention (position p sees positions <= p; a local layer
 * only the last `window` of them), after the positions already encoded, and
 * appends each layer's rotated keys and values to the library's own KV cache.
 * Then every layer's prompt K/V is that cache (replacing dg_set_prompt_kv's),
 * so a following dg_canvas_step / dg_denoise_block cross-attends to all encoded
 * positions with canvas row i at position (length + i).  Needs max_context > 0;
 * the batch must equal the encoded context's; length + n <= max_context.
 * DG_ERR_BAD_STATE without weights or without an own cache.  Synchronous at
 * the end (device errors reported). */
int dg_encode(dg_ctx* ctx, const int32_t* tokens, int batch, int n);

/* Pages: as dg_encode.  Empties the library's own KV cache (length 0); the
 * next dg_encode starts at position 0 and may use another batch. */
int dg_reset_context(dg_ctx* ctx);

/* Pages: as dg_encode.  *n_out = positions per sequence in the own KV cache. */
int dg_context_length(dg_ctx* ctx, int* n_out);

/* Pages: as dg_encode.  Copies one layer's own cache, the positions encoded so
 * far: k_out, v_out (host or dev) bf16 [batch][n_kv_heads][length][head_dim],
 * keys rotated.  Synchronous.  DG_ERR_BAD_STATE when nothing is encoded. */
int dg_context_kv(dg_ctx* ctx, int layer, void* k_out, void* v_out);

/* Pages: "Hands-On with Diffusion Gemma", How Is This Different from Previous
 * Models? (causal context building, then non-causal refinement of a 256-token
 * canvas, repeated until the text is complete); "DiffusionGemma: Google's
 * Experimental Diffusion LLM", How Text Diffusion Actually Works (a fixed
 * number of passes per block).
 * Block-autoregressive generation: empties the own cache, encodes the prompt
 * (host or dev int32 [batch][n_prompt]), then n_blocks times: an all-mask
 * canvas gets n_steps fixed passes (dg_denoise_block) against the cache, is
 * written to out[:, blk * canvas_len ...] (host or dev int32
 * [batch][n_blocks * canvas_len]) and is encoded onto the cache.  Needs
 * n_prompt + n_blocks * canvas_len <= max_context.  Synchronous. */
int dg_generate(dg_ctx* ctx, const int32_t* prompt, int batch, int n_prompt, int n_blocks,
                int n_steps, int32_t* out);

/* Pages: "DiffusionGemma: The Diffusion Era Begins with 4x Faster Text
 * Generation", Recommended Inference Settings (an entropy-bound sampler, at most
 * 48 passes, temperature falling linearly from 0.8 to 0.4, entropy bound 0.1, a
 * stop once the mean canvas entropy is below 0.005 with the high-probability
 * tokens stable) and "DiffusionGemma: Exploring the Paradigm Shift in
 * Non-Autoregressive Language Modeling", Serving in Production (the 0.005 halt
 * once two consecutive passes agree).
 * One entropy-bounded pass, pass `step` (0-based) of at most n_max, over `batch`
 * canvases (dev int32 [batch][canvas_len], in place).  Its temperature is
 * temp = 0.8 + (0.4 - 0.8) * step / (n_max - 1) (0.8 when n_max == 1).  Per row,
 * the head gives the entropy H (nats) of softmax(logits / temp) over the
 * vocabulary without the mask id, and the argmax token.  Per canvas:
 *  - it stops when the mean of H over all its slots (summed in slot order in
 *    double precision) is below 0.005 and every argmax equals the previous
 *    pass's (pass 0 never stops);
 *  - at a stop, or at the last pass (step == n_max - 1), every masked slot
 *    takes its argmax token;
 *  - otherwise the masked slots in order of (H, slot) are committed while
 *    their running double-precision sum of H stays <= 0.1 (at least one), each
 *    with a token drawn by inverse CDF: the first vocab index whose cumulative
 *    probability (in vocab order) exceeds the slot's uniform.
 * u: dev or host fp32 [batch][canvas_len] uniforms in [0, 1), one per slot.
 * Pass 0 starts a block: it forgets the previous argmax and the canvases that
 * ended.  A canvas that has stopped, filled up or passed its last pass is left
 * unchanged by later passes of the block.  entropy_out (dev fp32
 * [batch][canvas_len]), committed_out (dev uint8 [batch][canvas_len]) and
 * stopped_out (dev uint8 [batch]) may be NULL.  Asynchronous like
 * dg_canvas_step (graph recorded on the second call for a batch size). */
int dg_eb_step(dg_ctx* ctx, int32_t* canvas, int batch, int step, int n_max, const float* u,
               float* entropy_out, uint8_t* committed_out, uint8_t* stopped_out);

/* Pages: as dg_eb_step.
 * Entropy-bounded denoising of one block: dg_eb_step for step = 0, 1, ... until
 * every canvas has stopped or filled up, or n_max passes ran.  u: dev fp32
 * [n_max][batch][canvas_len] (pass s reads u + s * batch * canvas_len).
 * passes_out (host int [batch], may be NULL) receives the passes each canvas
 * took part in.  Reads the per-canvas state after every pass (one
 * synchronisation per pass) and reports device errors at the end. */
int dg_eb_denoise_block(dg_ctx* ctx, int32_t* canvas, int batch, int n_max, const float* u,
                        int* passes_out);

/* Pages: as dg_eb_step (the decisions of a pass).
 * Test hook: the stop test and the commit of dg_eb_step on given per-slot
 * entropies, argmax tokens and drawn tokens (all dev [batch][canvas_len]:
 * fp32, int32, int32), with prev_argmax (dev int32, or NULL: no previous pass)
 * and `last` (nonzero: the last allowed pass).  canvas in place;
 * committed_out (dev uint8 [batch][canvas_len]) and stopped_out (dev uint8
 * [batch]) may be NULL. */
int dg_eb_commit(dg_ctx* ctx, const float* entropy, const int32_t* argmax, const int32_t* drawn,
                 const int32_t* prev_argmax, int32_t* canvas, int batch, int last,
                 uint8_t* committed_out, uint8_t* stopped_out);

/* Pages: "Hands-On with Diffusion Gemma", Detailed Specs (input, post-attention
 * and pre-feedforward norms, attention, MoE) and "DiffusionGemma: The Diffusion
 * Era Begins ...", DiffusionGemma's Technical Architecture (bidirectional
 * attention over the canvas, cross-attention into the prompt KV, 8 of 128
 * experts + 1 shared).
 * One decoder block on given hidden states (no embedding, head or commit):
 * x_out = block(x_in) with x_in, x_out dev bf16 [n_rows][d_model],
 * n_rows = batch * canvas_len for the batch given to dg_set_prompt_kv.
 * x_in and x_out may be the same buffer. */
int dg_layer_forward(dg_ctx* ctx, int layer, const void* x_in, void* x_out, int n_rows);

/* Pages: "DiffusionGemma: The Diffusion Era Begins ...", DiffusionGemma's
 * Technical Architecture (8 of 128 experts active) and "Hands-On with Diffusion
 * Gemma", Detailed Specs (the router).
 * Router test hook: top_k selection and grouping from given logits.
 * logits: dev fp32 [n_rows][n_experts] (used as given; the router bias is not
 * added).  Outputs (dev): idx int32 [n_rows][top_k], experts by decreasing
 * logit, equal logits toward the lower index; w fp32 [n_rows][top_k], the
 * softmax over the chosen logits; offsets int32 [n_experts + 1]; perm int32
 * [n_rows * top_k] with perm[offsets[e] + r] = t * top_k + j for the r-th
 * assignment (t, j) to expert e in increasing t.  n_rows <= max_batch *
 * canvas_len.  logits must be 16-byte aligned. */
int dg_router_topk(dg_ctx* ctx, const float* logits, int n_rows, int32_t* idx, float* w,
                   int32_t* offsets, int32_t* perm);

/* dg_router_topk for callers that cannot allocate device memory.  The pages
 * have no counterpart: this entry point exists for programs whose device
 * memory is owned entirely by their own pool or arena, or that run under a
 * rule forbidding allocation after start-up, and so cannot create a context
 * (dg_create allocates weights and workspace) or let the library call
 * cudaMalloc.  It takes no context and allocates nothing: the caller passes
 * the inputs and outputs, exactly as for dg_router_topk (logits dev fp32
 * [n_rows][n_experts], 16-byte aligned; idx, w, offsets, perm dev, same
 * layouts), plus the expert count, top_k and a cudaStream_t (NULL = legacy
 * default stream).  The scratch it needs (membership bitmap, last-block
 * counter, inverse permutation: 131,328 bytes) is one fixed array in the
 * library's device data, held by every GPU that loads the library until the
 * process exits.  Limits: 1 <= n_rows <= 2048, n_experts a multiple of 4 in
 * [4, 256], 1 <= top_k <= min(8, n_experts); larger sizes return
 * DG_ERR_INVALID_ARG without touching the GPU.  The first call on a device
 * looks up the array's device address (a runtime query, no allocation), so
 * make that first call before any stream capture.  The scratch is cleared on
 * the stream at the start of each call; calls share it, so calls that may
 * overlap on the GPU (other streams, other host threads) race and must be
 * serialised by the caller.  Returns DG_OK, DG_ERR_INVALID_ARG or
 * DG_ERR_CUDA; the results are ready when the stream reaches them.  The call
 * does not wait for the GPU, so it reports no device-side error: the kernel's
 * own checks (an expert index out of range, a total other than n_rows * top_k)
 * cannot fire for inputs that pass the limits above, and if they did, the
 * scratch error word they set would not be read back. */
int dg_router_topk_static(const float* logits, int n_rows, int n_experts, int top_k,
                          int32_t* idx, float* w, int32_t* offsets, int32_t* perm,
                          void* cuda_stream);

/* The pages have no counterpart: failure detection.
 * Self-test of the bounded waits that every kernel of the library uses (the
 * device half of the failure detection): runs one CTA on cuda_stream (NULL =
 * legacy default stream) that waits on an mbarrier nothing arrives on.  The
 * wait gives up after its limit (2 s), records DG_ERR_TIMEOUT and the kernel
 * returns, so the device and any context stay usable.  Returns DG_ERR_TIMEOUT
 * when the wait ran out as designed, DG_OK if it did not run out, DG_ERR_OOM /
 * DG_ERR_CUDA if the test itself could not run.  Synchronises the stream;
 * allocates (and frees) one int of device memory. */
int dg_selftest_bounded_wait(void* cuda_stream);

/* Pages: as dg_canvas_step (the locking of confident tokens).
 * Commit test hook: the commit rule of dg_canvas_step on given confidences.
 * conf: dev fp32 [batch][canvas_len]; cand_tok: dev int32 [batch][canvas_len]
 * (the token each slot would receive); canvas: dev int32, in place;
 * committed_out: dev uint8 or NULL. */
int dg_commit(dg_ctx* ctx, const float* conf, int32_t* canvas, int batch, int steps_left,
              const int32_t* cand_tok, uint8_t* committed_out);

/* The pages have no counterpart (inspection for tests).
 * Debug hook: copies an internal tensor of the most recent pass (or layer
 * call) into dst (dev or host, `bytes` long; cudaMemcpyDefault), synchronously.
 * *bytes_needed (may be NULL) receives the tensor's size; with dst == NULL
 * only the size is reported.  Names and contents:
 *   "x"        bf16 [T][d]        after dg_layer_forward: the block output; after a
 *                                 pass: the final-normed states fed to the vocab head
 *   "hn"       the same buffer as "x"
 *   "q"        bf16 [B][Hq][Tc][dh]   rotated queries; "kc", "vc" likewise [B][Hkv][Tc][dh]
 *                                 (rotated canvas keys, canvas values) of the last layer run
 *   "attn_o"   bf16 [T][Hq*dh]    attention output before the output projection
 *   "x2"       bf16 [T][d]        pre-feedforward-normed hidden states
 *   "router_logits" fp32 [T][E]   (bias included)
 *   "idx" int32 [T][k]; "w" fp32 [T][k]; "offsets" int32 [E+1]; "perm" int32 [T*k]
 *                                 (the routing of the last layer run, as dg_router_topk)
 *   "h"        fp32 [T][d]        residual stream after the last layer run
 *   "tok"      int32 [T]          argmax token per row (after a pass)
 *   "conf"     fp32 [T]           confidence per row (after a pass)
 *   "head_max" fp32 [T]           largest logit per row, mask id excluded (after a pass)
 *   "entropy"  fp32 [T]           entropy per row (after an entropy-bounded pass)
 *   "eb_drawn" int32 [T]          drawn token of each slot committed by the bound
 *                                 (after an entropy-bounded pass; other rows stale)
 * and the weights (bf16, physical layouts):
 *   "embed"    [vocab][d]
 *   "wqkv:L"   [(Hq+2Hkv)*dh][d]  rows: q heads, then k heads, then v heads
 *   "wo:L"     [d][Hq*dh];  "wr:L" [E][d]
 *   "wgu:L"    [E+1][2*d_ff][d]   group 0 = shared expert, group g = expert g-1;
 *                                 row 2f = gate row f, row 2f+1 = up row f
 *   "wd:L"     [E+1][d][d_ff]     group 0 = shared expert, group g = expert g-1
 * with expert_dtype = DG_DTYPE_FP8_E4M3 also the codes and scales:
 *   "wgu8:L"   uint8 [E+1][2*d_ff][d] (the rows of "wgu:L"), "sgu:L" fp32 [E+1][2*d_ff];
 *   "wd8:L"    uint8 [E+1][d][d_ff],                          "sd8:L" fp32 [E+1][d]
 * with T = batch * canvas_len rows of the last call. */
int dg_debug_tensor(dg_ctx* ctx, const char* name, void* dst, size_t bytes,
                    size_t* bytes_needed);

/* The pages have no counterpart (measurement).
 * Instrumentation: with on != 0, every kernel launched by the following
 * passes is bracketed by CUDA events recorded on the context's stream (this
 * adds two event records per launch); on == 0 stops recording.  Either call
 * synchronises the stream and clears earlier records. */
int dg_profile_enable(dg_ctx* ctx, int on);

/* Sum of the device durations (ms) and the number of launches recorded for
 * one kernel since dg_profile_enable(ctx, 1).  Synchronises.  Kernel names
 * are those returned by dg_kernel_name(0 ..): "embed_norm", "rope_table",
 * "gemm_qkv", "qkv_rope", "attention", "attn_merge", "gemm_o", "post_attn",
 * "gemm_router", "router", "moe_gather", "gemm_gateup",
 * "gemm_down", "moe_combine", "gemm_head", "head_merge", "commit". */
int dg_profile_read(dg_ctx* ctx, const char* kernel, double* total_ms, int* launches);

/* Name of kernel kind i (0-based), or NULL past the last one. */
const char* dg_kernel_name(int i);

/* Waits for the context's stream and reports (then clears) the device error
 * word: DG_ERR_TIMEOUT or DG_ERR_DEVICE_FAULT if a kernel raised one. */
int dg_sync(dg_ctx* ctx);

/* Text of the context's last error ("" if none).  With ctx == NULL, the text
 * of the last error of a dg_create that returned no context.  The pointer
 * stays valid until the next call on the same context. */
const char* dg_last_error(const dg_ctx* ctx);

/* Device bytes held by the context (weights + workspace). */
size_t dg_device_bytes(const dg_ctx* ctx);

/* Kernel launches queued by the most recent dg_canvas_step /
 * dg_layer_forward (for launch accounting). */
int dg_last_launch_count(const dg_ctx* ctx);

/* Frees everything the context owns (not the borrowed prompt K/V).
 * Synchronises the stream first.  NULL is ignored. */
void dg_destroy(dg_ctx* ctx);

#ifdef __cplusplus
}
#endif

#endif /* DG_H */
