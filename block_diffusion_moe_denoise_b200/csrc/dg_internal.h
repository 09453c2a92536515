// Internal declarations shared by the libdg translation units.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "../../include/dg.h"
#include "../../include/dg_ops.h"

namespace dg {

using bf16 = __nv_bfloat16;

// Launch with programmatic stream serialization (see pdl_trigger / pdl_wait).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// The same launch as thread-block clusters of the given shape.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                      dim3 cluster, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster.x;
  attr[1].val.clusterDim.y = cluster.y;
  attr[1].val.clusterDim.z = cluster.z;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// ---- arguments of the tcgen05 GEMM launchers (gemm_ops.cu) ----
struct QkvArgs {
  const CUtensorMap* tm_x;  // normed tokens [Tcap, d]
  const CUtensorMap* tm_w;  // w_qkv
  int T, d, rows, D, Hq, Hkv, q_T, kv_cap, num_sms;
  long long kv_req_stride;
  const int* tok_pos;
  const int* tok_req;
  const float2* rope;  // [T][D/2] (cos, sin)
  bf16* q;
  bf16* kv;
  int* err;
  int pair = 0;  // 1: M = 256 tiles over CTA pairs (P_QKV2)
};
constexpr int kMaxPartSplits = 8;
constexpr int kExpertRows = 64;       // token rows per FP8 routed-expert GEMM tile
constexpr int kExpertTileRows = 128;  // token rows per bf16 routed-expert tile (and shared-down tile)
constexpr int kExpertBoxRows = 64;    // rows per TMA box of the bf16 grouped rows (measured slower on
                                      // B200: 16-row boxes throughout, and 32/16-row boxes for the rows
                                      // past a tile's last full 64, though both move fewer bytes)
struct WpartArgs {
  const CUtensorMap* tm_w;  // weights [d, K], 128-row boxes
  const CUtensorMap* tm_x;  // activations [Tcap, K], 256-row boxes
  int T, Tcap, d, K, splits, num_sms;
  float* part;              // [splits][Tcap][d]
  int* err;
  const CUtensorMap* tm_x128 = nullptr;  // the activations in 128-row boxes: CTA pairs (P_WPART2)
};
struct ExpertArgs {
  const CUtensorMap *tm_gate, *tm_up, *tm_xp, *tm_down, *tm_hp;
  int d, fe, num_sms;
  const int4* egu_tiles;
  const int* egu_count;
  const int4* ed_tiles;
  const int* ed_count;
  const int* counts;
  const int* offsets;
  const float* row_weight;
  bf16* hp;
  bf16* yp;  // gate-weighted routed outputs, bf16
  int* err;
  // FP8 experts: per-row scales of the weight codes and of the token / hidden codes
  const float *s_gate = nullptr, *s_up = nullptr, *s_down = nullptr, *s_x = nullptr, *s_h = nullptr;
  int* sched = nullptr;  // [2] tile counters of the gate|up and down launches (zeroed by the grouping kernel)
  int* ready = nullptr;  // [token tiles] per-token-tile gate|up completions of run_experts (zeroed likewise)
  // run_experts only: the shared expert's down projection as extra tiles of the
  // same launch (tm_sdown == nullptr: none), output [T][d] fp32 into sd_part
  const CUtensorMap *tm_sdown = nullptr, *tm_hs64 = nullptr;
  int T = 0, sd_K = 0;
  float* sd_part = nullptr;
};
struct SharedArgs {
  const CUtensorMap *tm_u, *tm_gate, *tm_up, *tm_router;
  const CUtensorMap* tm_u64;  // the normed tokens in 64-row boxes (router tiles of 64 tokens), or null
  const CUtensorMap* tm_u32 = nullptr;  // ... in 32-row boxes (router tiles of 32 tokens), or null
  int T, d, fs, num_sms;
  int E, k, MW;       // router: experts (multiple of 16, <= 128), top-k, bitmask words per expert
  bf16* hs;
  float* logits;      // [Tcap, E] router logits (kept for inspection)
  int* idx;           // [T, k] picked experts
  float* w;           // [T, k] their renormalised probabilities
  unsigned* mask;     // [E][MW] per-expert token bitmasks, zero on entry
  int* err;
};
// Per-slot keys of the LM-head rows: row r is position r % canvas of slot
// r / canvas.  The candidate draw uses the slot's (seed, block, step,
// request); the self-conditioning state is stored under its request.
struct DrawKeys {
  int canvas;
  int req[DG_MAX_REQUESTS];
  int block[DG_MAX_REQUESTS];
  int step[DG_MAX_REQUESTS];
  unsigned long long seed[DG_MAX_REQUESTS];
};

// Rows one LM-head launch covers (its per-CTA statistics hold 8 token tiles);
// larger passes run the LM head in chunks of whole slots.
constexpr int kLmRowsMax = 1024;

struct LmArgs {
  const CUtensorMap* tm_x;
  const CUtensorMap* tm_embed;
  int T, d, num_sms;
  long long V;
  float4* part;
  float* logits;
  int* err;
  // candidate draw (draw == nullptr: argmax candidates only)
  float inv_tau = 1.f;       // 1 / temperature
  float2* draw = nullptr;    // [T][V/256]: (log-mass of the tile at 1/temperature, drawn id in the tile)
  DrawKeys keys = {};
  float2* sc_part = nullptr; // self-conditioning: per-CTA top-8 logits [grid][T][8] (logit, id bits)
  int row0 = 0;              // first row of tm_x this launch reads (its rows are row0 .. row0+T-1)
  const CUtensorMap* tm_embed128 = nullptr;  // the embedding in 128-row boxes: CTA pairs (P_LM2)
};

cudaError_t run_qkv(const QkvArgs& a, cudaStream_t st);
int wpart_splits(int d, int T, int K, int num_sms);
cudaError_t run_wpart(const WpartArgs& a, cudaStream_t st);
// gate|up and down of the bf16 routed experts in one launch (needs a.ready, a.sched)
cudaError_t run_experts(const ExpertArgs& a, cudaStream_t st);
cudaError_t run_experts_gate_up_fp8(const ExpertArgs& a, cudaStream_t st);
cudaError_t run_experts_down_fp8(const ExpertArgs& a, cudaStream_t st);
cudaError_t run_shared_gate_up(const SharedArgs& a, cudaStream_t st);
cudaError_t run_lm_head(const LmArgs& a, int* grid_out, cudaStream_t st);
size_t gemm_smem_bytes_max();

// ---- small kernels (kernels.cu) ----
struct SlotInfo {
  int n;                       // slots (requests) in this pass
  int Tr;                      // tokens per slot
  int req[DG_MAX_REQUESTS];    // request of each slot
  int pos0[DG_MAX_REQUESTS];   // position of the slot's first token
};

// ids[slot] points at the slot's Tr token ids
cudaError_t run_embed(const int* const* ids, const SlotInfo& s, const bf16* embed, int V, int d, float* x, int* tok_pos,
                      int* tok_req, const double* inv_freq, int half, float2* rope, int* err, cudaStream_t st);
// x[t] += sum_j yp[pair_row[t*k+j]] + sum_s part[s][t]; then (if an output is
// given) the RMSNorm of x[t] with gain g as bf16
cudaError_t run_residual_norm(float* x, const bf16* yp, const int* pair_row, int k, const float* part, int n_part,
                              int Tcap, const float* g, int T, int d, float eps, bf16* out, cudaStream_t st);
cudaError_t run_rmsnorm(const float* x, const float* g, int T, int d, float eps, bf16* out, cudaStream_t st);
cudaError_t run_topk(const float* logits, int T, int E, int k, int* idx, float* w, cudaStream_t st);
struct GroupArgs {
  int* idx;     // [T, k] selected experts (written by the router epilogue or the caller)
  float* w;     // [T, k] gate weights
  int T, k, E, FJ, MD, egu_cap, ed_cap;
  int* counts;
  int* offsets;
  int* pair_row;
  int* row_token;
  float* row_weight;
  int* row_pair;
  int4* egu_tiles;
  int* egu_count;
  int4* ed_tiles;
  int* ed_count;
  unsigned long long* route_stats;  // [0] += experts touched, [1] += launches (may be null)
  int* err;
  int* sched = nullptr;             // [2] tile counters of the expert GEMMs that follow, zeroed here
  int* ready = nullptr;             // [token tiles] counters of the fused expert launch, zeroed here
};
cudaError_t run_group(const GroupArgs& a, cudaStream_t st);
// the grouping above from the token bitmasks `mask` ([E][MW] words, MW fixed by
// the workspace so the layout never changes between passes) the router epilogue
// set, plus the gather of u rows into xp; clears all of `mask_next`
cudaError_t run_route(const bf16* u, int d, bf16* xp, unsigned* mask, unsigned* mask_next, int MW,
                      const GroupArgs& a, cudaStream_t st, uint8_t* xq = nullptr, float* xs = nullptr);
// Per-row E4M3 quantisation of bf16 rows [rows, n] (n % 8 == 0, n <= 4096):
// codes [rows, n] and fp32 scales [rows] (E4M3(x * 448 / amax), amax / 448).
cudaError_t run_quant_rows(const bf16* in, int n, int rows, uint8_t* out, float* scale, cudaStream_t st);
// Merge of the LM head's per-CTA partials into per-row statistics; with
// `draw` (the per-tile records of a candidate draw, NV tiles per row) also the
// row-level pick of the tile, whose drawn id goes to cand[row].
cudaError_t run_lm_combine(const float4* part, int G, int MT, int T, float* stats, int* argmax, int* err,
                           cudaStream_t st, const float2* draw = nullptr, int NV = 0, const DrawKeys* keys = nullptr,
                           int* cand = nullptr);
// Self-conditioning state: merge the LM head's per-CTA top-8 lists (sc_part,
// [G][T][8]) per row into the row's top-K softmax entries, written as (p, id
// bits) to sc_top[(keys.req[slot] * keys.canvas + pos) * 8 + k], k < K.  The
// rows' log-partitions come from `stats` (written by run_lm_combine).
cudaError_t run_selfcond_topk(const float2* sc_part, int G, int T, const float* stats, const DrawKeys& keys, int K,
                              float2* sc_top, int* err, cudaStream_t st);
// Soft embeddings of the self-conditioning input: row r (slot r / canvas,
// position r % canvas) gets sum_k p_k E[id_k] over its request's sc_top entries
// when on[slot], else zeros; rows T..: untouched.  out: bf16 [T, d].
struct SelfCondArgs {
  int canvas, T, d, vocab, K, n_slots;
  int req[DG_MAX_REQUESTS];
  int on[DG_MAX_REQUESTS];
  const float2* top;      // [max_req][canvas][8]
  const bf16* embed;      // [vocab, d]
  bf16* out;              // [T, d]
  int* err;
};
cudaError_t run_selfcond_embed(const SelfCondArgs& a, cudaStream_t st);
struct SampleArgs {
  int n_slots, canvas, vocab, min_accept, max_steps;
  float thr;
  int mode;               // DG_SAMPLER_THRESHOLD or DG_SAMPLER_ENTROPY_BUDGET
  float budget, stop_entropy;
  int* prev_argmax;       // [req][canvas] argmax of the previous step (budget rule)
  int req[DG_MAX_REQUESTS];
  int block[DG_MAX_REQUESTS];
  int step[DG_MAX_REQUESTS];
  unsigned long long seed[DG_MAX_REQUESTS];
  const float* entropy;   // [slot*canvas + i] * stride
  const float* logconf;   // [slot*canvas + i] * stride
  int stride;             // floats between consecutive positions
  const int* argmax;      // [slot*canvas + i]
  const int* cand;        // [slot*canvas + i] drawn candidates, or nullptr (argmax candidates)
  int* canvas_tok;        // [req][canvas]
  unsigned char* mask;    // [req][canvas]
  int* remaining;         // [req]
  int* err;
};
cudaError_t run_sample(const SampleArgs& a, cudaStream_t st);
cudaError_t run_philox_tokens(unsigned long long seed, int block, int step, int request, long long pos0, long long n,
                              int vocab, int* out, unsigned char* mask_clear, cudaStream_t st);
cudaError_t run_kv_copy(bf16* cache_k, bf16* cache_v, int Hkv, long long cap, int D, long long pos0, long long n,
                        const bf16* k_in, const bf16* v_in, bf16* k_out, bf16* v_out, cudaStream_t st);

// ---- attention (attention.cu) ----
struct AttnArgs {
  CUtensorMap tm_k;   // whole KV area as rows of 64 elements, boxes of D rows (one tiled 64-key K tile)
  CUtensorMap tm_vt;  // whole KV area as rows of cap elements, 64 x D boxes
  const bf16* q;      // [Hq][q_T][D]
  int q_T;
  bf16* o;            // [T][Hq*D]
  long long k_row0, req_rows_k;   // tm_k row of (request 0, this layer, head 0, pos 0); rows per request
  long long v_row0, req_rows_v;   // tm_vt row of (request 0, this layer, head 0, dim 0); rows per request
  long long cap;
  int Hq, Hkv, D, Tr, n_slots;
  int req[DG_MAX_REQUESTS];
  int n_keys[DG_MAX_REQUESTS];
  int n_split;                         // largest key split over the slots
  int slot_split[DG_MAX_REQUESTS];     // key splits of each slot (1 = direct output)
  float* part_o;     // [n_split][Hq][q_T][D]
  float2* part_ml;   // [n_split][Hq][q_T]
  int cluster;       // 1: every slot has n_split key splits, which form one thread-block
                     // cluster per query tile and merge through distributed shared memory
                     // (part_o / part_ml unused)
  float scale;
  int* err;
};
cudaError_t run_attention(const AttnArgs& a, cudaStream_t st);
int attention_split_cap();
size_t attention_smem_bytes(int D);

}  // namespace dg
