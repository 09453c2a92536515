/*
 * dg.h -- C ABI of libdg, a single-GPU (sm_100a) implementation of the
 * denoising step of a block-autoregressive text-diffusion MoE decoder.
 *
 * The method (DiffusionGemma pages):
 *   - output is produced as fixed 256-token canvases; a canvas starts as random
 *     tokens and is denoised by repeated bidirectional decoder passes over all of
 *     its positions, which attend to the committed KV cache and to the whole
 *     canvas ("DiffusionGemma hits ~1,500 TPS on one H100", section "What
 *     DiffusionGemma is"; "Google open-sources DiffusionGemma: H100 reaches 1000
 *     TPS", section "26B MoE Architecture, but Only 3.8B Activated");
 *   - each pass routes every canvas token to the top 8 of 128 experts plus one
 *     shared expert ("DiffusionGemma Hits 1,000 Tokens per Second", section "The
 *     speed numbers and the hardware they require");
 *   - after each pass confident positions are accepted and frozen and the rest
 *     re-randomised; a converged canvas is committed to the KV cache and the next
 *     canvas opens ("DiffusionGemma hits ~1,500 TPS", section "How the sampler
 *     actually works").
 * Sampler rule (default, DG_SAMPLER_THRESHOLD): a position not yet accepted is accepted when its
 * entropy is <= entropy_thresh nats, or when it is among the min_accept most
 * confident (highest log max-probability, ties to the lower position) of the
 * positions not yet accepted; at step max_steps every remaining position is
 * accepted.  Rejected positions get tok(seed, block, step, position) from
 * Philox-4x32-10 (key = seed, counter = (position, step, block, request)).
 * The pages' entropy-budget rule is available as DG_SAMPLER_ENTROPY_BUDGET.
 *
 * Conventions for every entry point:
 *   - All device pointers are caller-owned and must stay valid while the handle
 *     uses them.  libdg never allocates device memory: the KV cache, activations
 *     and scratch live in the caller's workspace (see dg_workspace_size).
 *   - Work is enqueued asynchronously on the stream given to dg_init; only the
 *     calls that return host data (dg_generate, dg_sync, dg_read_remaining)
 *     synchronise that stream.
 *   - Return value: DG_OK (0) or a negative DG_E_* code; dg_strerror() names it.
 *     Arguments are validated before any work is enqueued; on error nothing is
 *     enqueued and the handle state is unchanged.
 *   - A handle is not thread-safe; use one handle per stream.
 */
#ifndef DG_H_
#define DG_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DG_OK 0
#define DG_E_ARG (-1)         /* invalid argument or unsupported shape */
#define DG_E_STATE (-2)       /* call not valid in the request's current state */
#define DG_E_CAPACITY (-3)    /* KV capacity or workspace too small */
#define DG_E_CUDA (-4)        /* a CUDA runtime call failed */
#define DG_E_DEVICE (-5)      /* a kernel set the device error word */
#define DG_E_UNSUPPORTED (-6) /* no sm_100 device */

#define DG_MAX_REQUESTS 8

/* Model shape and sampler knobs.  Supported shapes: d_model, ffn_expert and
 * ffn_shared multiples of 64 (d_model also of 128 and 256, at most 4096); head_dim 64, 128
 * or 256; (n_q_heads+2*n_kv_heads)*head_dim a multiple of 256; n_q_heads a
 * multiple of n_kv_heads; n_experts a multiple of 16 up to 128 (the router
 * is one tensor-core tile wide); top_k <= 8; vocab a multiple of
 * 256; canvas <= 256. */
typedef struct dg_config {
  int n_layers, d_model, n_q_heads, n_kv_heads, head_dim;
  int n_experts, top_k, ffn_expert, ffn_shared, vocab;
  int canvas;          /* canvas length (256) */
  int max_steps;       /* step cap per canvas (12) */
  int min_accept;      /* accept at least this many per step (22) */
  float entropy_thresh;/* nats (1.0) */
  float rope_theta;    /* 10000 */
  float norm_eps;      /* 1e-6 */
  int sampler;         /* DG_SAMPLER_THRESHOLD (the rule above) or DG_SAMPLER_ENTROPY_BUDGET */
  float entropy_budget;/* budget rule: nats of entropy accepted per step (0.1) */
  float stop_entropy;  /* budget rule: converged below this mean entropy (0.005) */
  float temperature;   /* 0: candidates are the argmax; > 0: drawn from softmax(logits / temperature) */
  int ffn_selfcond;    /* self-conditioning gated-MLP width, a multiple of 64 (0: no self-conditioning) */
  int selfcond_topk;   /* softmax entries per position fed back, 1..8 (8) */
  int expert_fp8;      /* 1: routed-expert weights are E4M3 codes with per-row scales (W8A8 GEMMs); 0: bf16 */
} dg_config;

/* FP8 routed experts (expert_fp8 = 1; the pages name FP8 and NVFP4
 * checkpoints of the model without giving the scheme; this W8A8 reading is
 * the library's).  w_gate, w_up and w_down hold E4M3 codes (one byte each, same
 * shapes as the bf16 form) whose rows are scaled by w_gate_scale [E, fe],
 * w_up_scale [E, fe] and w_down_scale [E, d] (fp32): W = decode(q) * scale.
 * The token rows entering gate|up and the SwiGLU rows entering down are
 * quantised per row: codes = E4M3(x * (448 / amax)) (round to nearest even,
 * saturating), scale = amax / 448, amax = max |x| (fp32; a zero row gives
 * zeros).  The tensor cores multiply the codes (kind::f8f6f4, fp32
 * accumulation) and the epilogues apply both scales.  Everything else stays
 * bf16. */

/* Self-conditioning (pages: "DiffusionGemma hits ~1,500 TPS", "How the sampler
 * actually works": the previous step's softmax is fed back through a small
 * gated MLP; its shape is not published, so this reading is the library's).
 * At every denoising step after the first of a canvas, each canvas position
 * adds to its token embedding
 *   sc = sc_down (silu(sc_gate e) * (sc_up e)),  e = sum_k p_k E[id_k],
 * where (p_k, id_k) are the selfcond_topk largest entries (ties to the lower
 * id) of the softmax of that position's logits at the request's previous
 * denoising step (not renormalised) and E is the tied embedding.  The first
 * step of a canvas (after dg_open_canvas), prefill and commit passes have no
 * such term.  dg_set_canvas keeps the request's previous-step state. */

/* Sampler rules.  DG_SAMPLER_ENTROPY_BUDGET follows the pages' default sampler
 * ("DiffusionGemma hits ~1,500 TPS", "How the sampler actually works"): the
 * positions not yet accepted are taken from most to least confident while the
 * running sum of their entropies (fp64, in that order) stays within
 * entropy_budget, and at least the most confident one; when every such
 * position keeps the argmax it had at the previous step and their mean
 * entropy is below stop_entropy, all of them are accepted (the canvas has
 * converged); at step max_steps all are accepted.
 *
 * Candidates (both rules).  With temperature 0 the token accepted at a
 * position is its argmax.  With temperature tau > 0 it is drawn from
 * softmax(z / tau) of the position's logits z (the pages' "sample a candidate
 * token at every position", same section), in two levels over tiles of 256
 * consecutive vocabulary ids: a tile by the inverse CDF of the tile masses
 * sum exp(z_v / tau) with u_row, then an id inside it by the inverse CDF of
 * exp(z_v / tau) with u_tile; both levels in float32.  u = (2 (w >> 9) + 1) / 2^24
 * of a Philox-4x32-10 word w (key = seed): u_row is word 1 of counter
 * (position, step, block, request) (word 0 is the re-noise token), u_tile of
 * tile j is word 0 of counter (position, step, block, request + 256 (j + 1)).
 * Entropy and confidence stay those of softmax(z): the temperature shapes the
 * draw only.  The draw adds two passes over each LM-head tile in its epilogue. */
#define DG_SAMPLER_THRESHOLD 0
#define DG_SAMPLER_ENTROPY_BUDGET 1

/* Device pointers to one layer's weights.  bf16 tensors are row-major
 * "out x in"; gains are fp32.
 *   attn_norm [d] f32, w_qkv [(Hq+2Hkv)*D, d] (q heads, then k, then v),
 *   w_o [d, Hq*D], ffn_norm [d] f32, w_router [E, d], w_gate [E, fe, d],
 *   w_up [E, fe, d], w_down [E, d, fe], ws_gate [fs, d], ws_up [fs, d],
 *   ws_down [d, fs].  Every pointer 16-byte aligned. */
typedef struct dg_layer_weights {
  const void *attn_norm, *w_qkv, *w_o, *ffn_norm, *w_router;
  const void *w_gate, *w_up, *w_down, *ws_gate, *ws_up, *ws_down;
  const void *w_gate_scale, *w_up_scale, *w_down_scale; /* fp32 row scales (expert_fp8 only, else NULL) */
} dg_layer_weights;

/* embed [vocab, d] bf16 (tied with the LM head), final_norm [d] f32,
 * layers: HOST array of n_layers entries (copied by dg_init). */
typedef struct dg_weights {
  const void* embed;
  const void* final_norm;
  const dg_layer_weights* layers;
  /* self-conditioning MLP (NULL unless ffn_selfcond > 0): sc_gate, sc_up
   * [ffn_selfcond, d], sc_down [d, ffn_selfcond], bf16, 16-byte aligned */
  const void *sc_gate, *sc_up, *sc_down;
} dg_weights;

typedef struct dg_handle dg_handle;

/* (No counterpart in the pages: workspace sizing is the library's own, so that
 * the caller owns every device buffer.)
 * Bytes of device workspace dg_init needs for up to `max_requests` requests
 * denoised together, each with a KV cache of `kv_capacity` positions
 * (prompt + committed canvases + one open canvas).  0 on invalid input. */
size_t dg_workspace_size(const dg_config* cfg, int max_requests, int64_t kv_capacity);

/* (No counterpart in the pages: handle set-up.)
 * Create a handle.  `workspace` is a device buffer of at least
 * dg_workspace_size(...) bytes, 1024-byte aligned, owned by the caller (it
 * holds the KV cache); `stream` is a cudaStream_t (NULL = legacy default).
 * Builds the TMA descriptors for every weight and activation buffer.
 * Requests start empty (KV length 0, no open canvas). */
int dg_init(const dg_config* cfg, const dg_weights* weights, int max_requests, int64_t kv_capacity,
            void* workspace, size_t workspace_bytes, void* stream, dg_handle** out);

/* (No counterpart in the pages.)  Release the handle (host state only; the
 * caller frees its device buffers); NULL is ignored. */
void dg_destroy(dg_handle* h);
/* (No counterpart in the pages.)  Static name of a DG_* return code. */
const char* dg_strerror(int code);

/* Defined by: "DiffusionGemma Hits 1,000 Tokens per Second--But Its Benchmarks Reveal the Real Tradeoff",
 * section "How diffusion text generation changes the bottleneck" (committed
 * blocks live in the key-value cache and condition the next canvas), and
 * section "The speed numbers and the hardware they require" of the same page
 * (the serving example prefills the prompt in chunks).  Reading: the prompt is cached
 * by the same segment pass as a committed canvas.
 * Append `n` prompt tokens (device int32 array) to request `req`'s KV cache:
 * the decoder runs over segments of `canvas` tokens counted from the first
 * token; each segment attends to all earlier positions and bidirectionally to
 * itself.  Up to eight full segments share one decoder pass (block-causal
 * slots), with a result bit-identical to one segment per call.  Fails with
 * DG_E_STATE while a canvas is open, DG_E_CAPACITY if the cache would
 * overflow. */
int dg_prefill(dg_handle* h, int req, const int32_t* d_tokens, int n);

/* (No counterpart in the pages: KV inspection and synthetic prefixes.)
 * Write synthetic committed K/V: positions [pos0, pos0+n) of layer `layer`
 * from device arrays k, v of shape [n_kv_heads, n, head_dim] bf16 (post-RoPE
 * keys).  Does not change the KV length.  Like dg_get_kv, dg_set_kv_len,
 * dg_prefill and dg_debug_forward, it first runs a deferred commit pass of
 * the request (see dg_commit_block). */
int dg_set_kv(dg_handle* h, int req, int layer, int64_t pos0, int64_t n, const void* d_k, const void* d_v);
/* Read back K/V of positions [pos0, pos0+n) into [n_kv_heads, n, head_dim] bf16. */
int dg_get_kv(dg_handle* h, int req, int layer, int64_t pos0, int64_t n, void* d_k, void* d_v);
/* Set the committed KV length (after dg_set_kv).  DG_E_STATE while a canvas is open. */
int dg_set_kv_len(dg_handle* h, int req, int64_t len);
int64_t dg_kv_len(const dg_handle* h, int req);

/* Defined by: "DiffusionGemma hits ~1,500 TPS on one H100: when a diffusion LLM beats autoregressive serving",
 * section "What DiffusionGemma is" (each canvas starts as a scratch pad of
 * random tokens).
 * Open canvas number `block` of request `req`: every position gets
 * tok(seed, block, 0, position), nothing accepted.  DG_E_CAPACITY if the canvas
 * does not fit after the committed positions. */
int dg_open_canvas(dg_handle* h, int req, uint64_t seed, int block);

/* Defined by: "DiffusionGemma hits ~1,500 TPS on one H100: when a diffusion LLM beats autoregressive serving",
 * sections "What DiffusionGemma is" (a bidirectional decoder pass over all 256
 * positions, accept the confident tokens, re-randomise the rest) and "How
 * the sampler actually works" (the per-step procedure and the stop rule);
 * the pass's MoE routing: "DiffusionGemma Hits 1,000 Tokens per Second--But Its Benchmarks Reveal the Real Tradeoff",
 * section "The speed numbers and the hardware they require" (128 experts,
 * eight active plus one shared).
 * One denoising step for `n_req` requests (host array `reqs`), denoised
 * together: one bidirectional pass over their canvases (tokens routed
 * together), LM-head statistics, then the accept / re-noise rule.  Each canvas
 * writes its own K/V into cache slots [L, L+canvas) as scratch; L is unchanged.
 * The number of positions still not accepted is written to d_remaining[i]
 * (device int32, may be NULL) and is readable with dg_read_remaining. */
int dg_denoise_step(dg_handle* h, int n_req, const int* reqs, int32_t* d_remaining);

/* (No counterpart in the pages.)  Synchronising read of a request's remaining
 * count (host). */
int dg_read_remaining(dg_handle* h, int req, int32_t* remaining);

/* Defined by: "DiffusionGemma Hits 1,000 Tokens per Second--But Its Benchmarks Reveal the Real Tradeoff",
 * section "How diffusion text generation changes the bottleneck" (a completed
 * block is committed to the key-value cache before the next canvas opens),
 * and "DiffusionGemma hits ~1,500 TPS on one H100: when a diffusion LLM beats autoregressive serving", section "What DiffusionGemma
 * is" (finished blocks are committed to the KV cache).
 * Commit request `req`'s converged canvas: the decoder runs over the final
 * canvas tokens at [L, L+canvas), writing their K/V, and L advances by canvas
 * (dg_kv_len reports the new length at once).  The pass itself is deferred:
 * it joins the request's next dg_denoise_step as an extra block-causal slot
 * (one weight stream for both, bit-identical results), or runs on its own
 * when a call that needs the cache comes first (dg_get_kv, dg_set_kv,
 * dg_set_kv_len, dg_prefill, dg_debug_forward, the end of dg_generate).
 * DG_E_STATE if no canvas is open.  The caller decides convergence (remaining
 * == 0); committing earlier commits the current tokens as they are. */
int dg_commit_block(dg_handle* h, int req);

/* Defined by: "DiffusionGemma hits ~1,500 TPS on one H100: when a diffusion LLM beats autoregressive serving",
 * sections "What DiffusionGemma is" (canvas after canvas until the output is
 * complete) and "The specs that matter for serving" (the measured setup: 4096
 * input and 1024 output tokens at batch 1).
 * Whole generation with HOST buffers: copy `n_prompt` prompt ids from host,
 * prefill, then n_out/canvas canvases (each denoised until nothing remains,
 * at most max_steps steps, then committed), copying the output ids to host
 * `h_out` [n_out].  steps_taken (host, may be NULL) receives the step count of
 * each canvas.  Request `req` must be empty (KV length 0). */
int dg_generate(dg_handle* h, int req, const int32_t* h_prompt, int n_prompt, int n_out, uint64_t seed,
                int32_t* h_out, int* steps_taken);

/* Defined by: "DiffusionGemma hits ~1,500 TPS on one H100: when a diffusion LLM beats autoregressive serving",
 * section "How the sampler actually works" (the canvas, which positions are
 * accepted, and the per-position entropy and confidence the rule reads).
 * Copy the open canvas of `req`: tokens [canvas] int32, accepted mask [canvas]
 * u8 (1 = frozen), and the last step's statistics for its positions:
 * d_stats [canvas][4] f32 = (entropy nats, log max-probability, max logit,
 * log-partition), d_argmax [canvas] int32.  Any output pointer may be NULL.
 * The statistics are kept for the latest LM-head pass of the handle only: if
 * another denoising step, an LM-head operation or a full debug pass ran after
 * this request's last step, d_stats is filled with NaN and d_argmax with -1. */
int dg_get_canvas(dg_handle* h, int req, int32_t* d_tokens, uint8_t* d_mask, float* d_stats, int32_t* d_argmax);

/* (No counterpart in the pages: teacher forcing for tests.)
 * Replace the open canvas of `req` (tokens, accepted mask) and its step counter. */
int dg_set_canvas(dg_handle* h, int req, const int32_t* d_tokens, const uint8_t* d_mask, int step);

/* (No counterpart in the pages.)
 * Wait for all enqueued work; DG_E_DEVICE if a kernel flagged an error (the
 * error word is then cleared), DG_E_CUDA on a CUDA error. */
int dg_sync(dg_handle* h);

#ifdef __cplusplus
}
#endif
#endif /* DG_H_ */
