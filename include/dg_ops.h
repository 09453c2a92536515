/*
 * dg_ops.h -- operation-level entry points of libdg, used to check each step
 * of the denoising pass on its own.  Same conventions as dg.h (caller-owned
 * device pointers, asynchronous on the handle's stream unless stated, DG_OK or
 * a negative DG_E_* code).
 */
#ifndef DG_OPS_H_
#define DG_OPS_H_

#include "dg.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Philox-4x32-10 re-noise draw (Salmon et al., SC'11, "Parallel Random Numbers:
 * As Easy as 1, 2, 3"): d_out[i] = floor(x0 * vocab / 2^32) where x0 is the
 * first output word for key (seed mod 2^32, seed >> 32) and counter
 * (pos0 + i, step, block, request).  Standalone (no handle); stream may be NULL. */
int dg_op_philox_tokens(uint64_t seed, int block, int step, int request, int64_t pos0, int64_t n, int vocab,
                        int32_t* d_out, void* stream);

/* Router selection from given fp32 logits [T, E] (device): top_k experts per
 * token in descending logit order (ties to the lower expert id) and the
 * softmax of the selected logits (the full softmax renormalised over the k
 * picks).  d_idx [T, k] int32, d_w [T, k] f32.  Standalone; stream may be NULL. */
int dg_op_route_topk(const float* d_logits, int T, int E, int k, int32_t* d_idx, float* d_w, void* stream);

/* Grouping of (token, slot) pairs by expert, with the handle's workspace as
 * scratch: from d_idx [T, k] computes counts [E], exclusive offsets [E+1] and
 * d_perm [T*k] = t*k + j in expert order, tokens ascending inside an expert.
 * T <= max_requests * canvas. */
int dg_op_route_group(dg_handle* h, const int32_t* d_idx, const float* d_w, int T, int32_t* d_counts,
                      int32_t* d_offsets, int32_t* d_perm);

/* The accept / re-noise rule for request `req` from given per-position
 * statistics (device, [canvas] each): entropy (nats), logconf (log max-prob)
 * and argmax.  Uses the request's open canvas, mask, seed and block; `step` is
 * the step number (1-based).  Updates canvas, mask, remaining. */
int dg_op_sample(dg_handle* h, int req, const float* d_entropy, const float* d_logconf, const int32_t* d_argmax,
                 int step);

/* Final RMSNorm + tied LM head + fused statistics on given fp32 hidden rows
 * d_x [T, d]: per row argmax, max logit, log-partition, entropy, logconf into
 * d_stats [T][4] = (entropy, logconf, max, logZ) and d_argmax [T].  If d_logits
 * is not NULL the fp32 logits [T, vocab] are written too. */
int dg_op_lm_head(dg_handle* h, const float* d_x, int T, float* d_stats, int32_t* d_argmax, float* d_logits);

/* dg_op_lm_head plus the candidate draw of dg.h ("Candidates"): rows 0..T-1
 * (T <= canvas) are positions 0..T-1 of request `request` at (seed, block,
 * step); `temperature` > 0 overrides the configuration's.  d_cand [T] int32
 * receives the drawn ids; d_stats and d_argmax (may be NULL) as in
 * dg_op_lm_head.  Does not touch the request's canvas. */
int dg_op_lm_sample(dg_handle* h, const float* d_x, int T, float temperature, uint64_t seed, int block, int step,
                    int request, float* d_stats, int32_t* d_argmax, int32_t* d_cand);

/* The self-conditioning term of dg.h from given fp32 hidden rows d_x [T, d]
 * (T <= canvas) of a previous step: final RMSNorm + tied LM head, the
 * selfcond_topk largest softmax entries per row, the soft embeddings and the
 * gated MLP.  d_sc [T, d] f32 receives the term; d_top (may be NULL) receives
 * [T][8] pairs of 32-bit words (p as f32, id as int32), entries k >=
 * selfcond_topk undefined.  Uses and overwrites request `request`'s
 * self-conditioning state.  DG_E_ARG without self-conditioning. */
int dg_op_selfcond(dg_handle* h, int request, const float* d_x, int T, float* d_sc, void* d_top);

/* Run the decoder over `T` tokens (device ids) of request `req` at positions
 * [L, L+T) without advancing L, stopping after `n_layers` layers (the K/V of
 * those layers are written to the cache slots).  The intermediates of the last
 * layer run stay in the workspace; dg_debug_buffer locates them. */
int dg_debug_forward(dg_handle* h, int req, const int32_t* d_tokens, int T, int n_layers);

/* dg_debug_forward starting inside the stack: the residual stream entering
 * layer `layer0` is d_x [T, d_model] f32 (device) instead of the embeddings of
 * d_tokens (which still fix nothing but the pass's shape), and layers layer0 ..
 * layer0 + n_layers - 1 run (their K/V written to the cache slots [L, L+T));
 * the LM head runs when the last layer of the stack is among them.  Lets a
 * test give one deep layer the oracle's own input. */
int dg_debug_forward_hidden(dg_handle* h, int req, const int32_t* d_tokens, const float* d_x, int T, int layer0,
                            int n_layers);

/* Byte offset and size, inside the workspace, of a named internal buffer:
 * "x" f32 [T, d] residual stream; "hn" bf16 [T, d] normed input of the last
 * projection; "q" bf16 [Hq, Tcap, D]; "o" bf16 [T, Hq*D]; "u" bf16 [T, d];
 * "router_logits" f32 [T, E] (written by the dg_debug_forward passes only);
 * "idx" i32 [T, k]; "w" f32 [T, k];
 * "counts" i32 [E]; "offsets" i32 [E+1];
 * "pair_row" i32 [T*k]; "row_pair" i32 [T*k]; "hp" bf16 [T*k, fe];
 * "yp" bf16 [T*k, d]; "hs" bf16 [T, fs]; "stats" f32 [Tcap][4];
 * "argmax" i32 [Tcap]; "cand" i32 [max_req * canvas] drawn candidates;
 * "sc_top" f32/i32 pairs [max_req][canvas][8] self-conditioning state;
 * "canvas" i32 [max_req, canvas]; "mask" u8 [...];
 * "remaining" i32 [max_req]; "route_stats" u64 [2] = (sum over router launches
 * of the number of experts that received a token, number of launches).
 * Returns DG_E_ARG for an unknown name. */
int dg_debug_buffer(const dg_handle* h, const char* name, size_t* offset, size_t* bytes);

/* Per-kernel-class timing: enable=1 records a CUDA event pair on the handle's
 * stream around every launch of the pass, enable=0 stops, enable=-1 clears the
 * totals.  dg_profile_read (synchronising) returns the summed elapsed ms and
 * launch count of one class: "embed", "rmsnorm", "qkv", "attention", "oproj",
 * "group", "experts" (the bf16 routed experts: gate|up, SwiGLU and down in one
 * launch), "experts_gate_up" and "experts_down" (the two launches of the FP8
 * experts), "shared_gate_up" (with the router), "shared_down", "lm_head",
 * "lm_combine", "sample", "selfcond", "other". */
int dg_profile(dg_handle* h, int enable);
int dg_profile_read(dg_handle* h, const char* kernel, double* total_ms, int64_t* launches);

/* Kernels launched by this handle so far (always counted). */
int64_t dg_launch_count(const dg_handle* h);

/* LM-head statistics for callers that cannot allocate device memory.  (No
 * counterpart in the pages: this is a deployment variant of dg_op_lm_head.)
 * Some callers have no workspace to give and must not call cudaMalloc: a
 * serving runtime whose caching allocator already owns all free HBM, or a
 * latency-critical loop where cudaMalloc's implicit device synchronisation is
 * not acceptable.  This entry point needs no handle and allocates nothing: it
 * runs the same final RMSNorm + tied LM head + fused statistics kernels as
 * dg_op_lm_head with their scratch (normalised bf16 rows and per-CTA partial
 * statistics) in a fixed 3 MiB array inside the library, which every GPU that
 * loads the library holds until the process exits.
 *   d_x [T, d_model] f32 hidden rows, d_final_norm [d_model] f32 gain,
 *   d_embed [vocab, d_model] bf16 (the tied embedding), all 16-byte aligned;
 *   outputs d_stats [T][4] = (entropy, logconf, max logit, log-partition) and
 *   d_argmax [T]; d_err (may be NULL) receives the device error word
 *   (0 = ok; cleared by each call).  Asynchronous on `stream`.
 * Limits: 1 <= T <= DG_NOALLOC_MAX_TOKENS, 64 <= d_model <=
 * DG_NOALLOC_MAX_DMODEL with d_model % 64 == 0, vocab % 256 == 0; anything
 * else returns DG_E_ARG before any work is enqueued.  The first call on a
 * device resolves the array's address on that device and must come before any
 * stream capture.  All calls share the array and it keeps the last call's
 * contents (nothing in it needs to start at zero); calls that overlap on the
 * GPU race on it, so the caller must serialise them. */
#define DG_NOALLOC_MAX_TOKENS 256
#define DG_NOALLOC_MAX_DMODEL 4096
int dg_op_lm_head_noalloc(const float* d_x, const float* d_final_norm, const void* d_embed, int T, int d_model,
                          int vocab, float norm_eps, float* d_stats, int32_t* d_argmax, int32_t* d_err,
                          void* stream);

#ifdef __cplusplus
}
#endif
#endif /* DG_OPS_H_ */
