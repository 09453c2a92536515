// Host side of libdg: workspace planning, TMA descriptors, the decoder pass
// orchestration (prefill / denoising step / commit / generate) and the C ABI.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <map>
#include <string>
#include <utility>

#include "dg_internal.h"

using namespace dg;

namespace {

constexpr size_t kAlign = 1024;
constexpr int kLmGridMax = 256;
constexpr int kSplitCap = 8;
// A prefill pass carries up to this many consecutive 256-token segments of one
// request (block-causal: each attends to the cache before it and to itself),
// so the weights are streamed once per group instead of once per segment.
constexpr int kPrefillSlots = DG_MAX_REQUESTS;

// Passes carry at most this many canvas-sized slots.
int pass_slots(int max_req) { return max_req > kPrefillSlots ? max_req : kPrefillSlots; }

struct LayerMaps {
  CUtensorMap qkv, o, gate, up, down, sgate, sup, sdown, router;
};

struct ReqState {
  long long kv_len = 0;  // committed length, including a pending block
  bool pending = false;  // the last committed block's pass has not run yet (its tokens: "commit_tok")
  int block = 0;
  int step = 0;
  unsigned long long seed = 0;
  bool open = false;
  int last_slot = 0;
  long long stats_seq = -1;  // LM-head pass whose statistics are this request's last step
  bool sc_valid = false;  // "sc_top" holds this canvas's previous-step self-conditioning state
};

// Offsets of every buffer inside the caller's workspace.
struct Plan {
  std::map<std::string, std::pair<size_t, size_t>> buf;
  size_t total = 0;
  size_t add(const char* name, size_t bytes) {
    const size_t off = (total + kAlign - 1) / kAlign * kAlign;
    buf[name] = {off, bytes};
    total = off + bytes;
    return off;
  }
};

bool config_ok(const dg_config* c) {
  if (!c) return false;
  if (c->n_layers < 1 || c->d_model < 256 || c->d_model > 4096 || c->d_model % 256 != 0) return false;
  if (!(c->head_dim == 64 || c->head_dim == 128 || c->head_dim == 256)) return false;
  if (c->n_kv_heads < 1 || c->n_q_heads < 1 || c->n_q_heads % c->n_kv_heads != 0) return false;
  if ((c->n_q_heads * c->head_dim) % 128 != 0 || (c->n_kv_heads * c->head_dim) % 128 != 0) return false;
  if ((c->n_q_heads * c->head_dim) % 64 != 0) return false;
  if (c->n_experts < 16 || c->n_experts > 128 || c->n_experts % 16 != 0) return false;
  if (c->top_k < 1 || c->top_k > 8 || c->top_k > c->n_experts) return false;
  if (c->ffn_expert < 64 || c->ffn_expert % 64 != 0 || c->ffn_shared < 64 || c->ffn_shared % 64 != 0) return false;
  if (c->vocab < 256 || c->vocab % 256 != 0) return false;
  if (c->canvas < 1 || c->canvas > 256) return false;
  if (c->max_steps < 1 || c->min_accept < 0) return false;
  if (c->sampler != DG_SAMPLER_THRESHOLD && c->sampler != DG_SAMPLER_ENTROPY_BUDGET) return false;
  if (c->sampler == DG_SAMPLER_ENTROPY_BUDGET && !(c->entropy_budget >= 0.f && c->stop_entropy >= 0.f)) return false;
  if (!(c->temperature >= 0.f && c->temperature <= 1e30f)) return false;
  if (c->ffn_selfcond < 0 || c->ffn_selfcond % 64 != 0) return false;
  if (c->ffn_selfcond > 0 && (c->selfcond_topk < 1 || c->selfcond_topk > 8)) return false;
  if (c->expert_fp8 != 0 && c->expert_fp8 != 1) return false;
  if (c->expert_fp8 && c->ffn_expert > 4096) return false;  // one warp quantises a row in registers
  return true;
}

long long round_cap(long long cap) { return (cap + 63) / 64 * 64; }

void make_plan(const dg_config* c, int max_req, long long cap_user, Plan* p) {
  const long long cap = round_cap(cap_user);
  const int T = pass_slots(max_req) * c->canvas;
  const int Tcap = (T + 127) / 128 * 128;
  const long long rows = (long long)T * c->top_k;
  const int D = c->head_dim, d = c->d_model;
  const long long n_nt = c->n_experts + (rows + kExpertRows - 1) / kExpertRows;
  p->add("err", 64);
  p->add("kv", (size_t)max_req * c->n_layers * 2 * c->n_kv_heads * (size_t)cap * D * 2);
  p->add("x", (size_t)Tcap * d * 4);
  p->add("hn", (size_t)Tcap * d * 2);
  p->add("q", (size_t)c->n_q_heads * Tcap * D * 2);
  p->add("o", (size_t)Tcap * c->n_q_heads * D * 2);
  p->add("u", (size_t)Tcap * d * 2);
  p->add("idx", (size_t)T * c->top_k * 4);
  p->add("w", (size_t)T * c->top_k * 4);
  p->add("counts", (size_t)c->n_experts * 4);
  p->add("offsets", (size_t)(c->n_experts + 1) * 4);
  p->add("pair_row", (size_t)rows * 4);
  p->add("row_token", (size_t)rows * 4);
  p->add("row_weight", (size_t)rows * 4);
  p->add("row_pair", (size_t)rows * 4);
  p->add("tile_counts", 64);
  p->add("route_stats", 64);
  p->add("egu_tiles", (size_t)n_nt * (c->ffn_expert / 64) * 16);
  p->add("ed_tiles", (size_t)n_nt * (d / 128) * 16);
  p->add("xp", (size_t)rows * d * 2);
  p->add("hp", (size_t)rows * c->ffn_expert * 2);
  p->add("yp", (size_t)rows * d * 2);
  p->add("hs", (size_t)Tcap * c->ffn_shared * 2);
  p->add("attn_o", (size_t)kSplitCap * c->n_q_heads * Tcap * D * 4);
  p->add("attn_ml", (size_t)kSplitCap * c->n_q_heads * Tcap * 8);
  p->add("lm_part", (size_t)kLmGridMax * Tcap * 16);
  p->add("stats", (size_t)Tcap * 16);
  p->add("argmax", (size_t)Tcap * 4);
  p->add("draw", (size_t)max_req * c->canvas * (c->vocab / 256) * 8);
  p->add("cand", (size_t)max_req * c->canvas * 4);
  {
    const bool sc = c->ffn_selfcond > 0;
    p->add("sc_part", sc ? (size_t)kLmGridMax * max_req * c->canvas * 8 * 8 : 64);
    p->add("sc_top", sc ? (size_t)max_req * c->canvas * 8 * 8 : 64);
    p->add("hs_sc", sc ? (size_t)Tcap * c->ffn_selfcond * 2 : 64);
  }
  {
    const bool f8 = c->expert_fp8 != 0;
    p->add("xq", f8 ? (size_t)rows * d : 64);
    p->add("xs", f8 ? (size_t)rows * 4 : 64);
    p->add("hq", f8 ? (size_t)rows * c->ffn_expert : 64);
    p->add("hsq", f8 ? (size_t)rows * 4 : 64);
  }
  p->add("canvas", (size_t)max_req * c->canvas * 4);
  p->add("commit_tok", (size_t)max_req * c->canvas * 4);
  p->add("prev_argmax", (size_t)max_req * c->canvas * 4);
  p->add("mask", (size_t)max_req * c->canvas);
  p->add("remaining", (size_t)max_req * 4);
  p->add("tok_pos", (size_t)Tcap * 4);
  p->add("tok_req", (size_t)Tcap * 4);
  p->add("inv_freq", (size_t)D / 2 * 8);
  p->add("rope", (size_t)Tcap * (D / 2) * 8);
  p->add("router_logits", (size_t)Tcap * c->n_experts * 4);
  p->add("part", (size_t)kMaxPartSplits * Tcap * d * 4);
  p->add("route_mask", (size_t)2 * c->n_experts * ((T + 31) / 32) * 4);
  p->add("sched", 64);
  p->add("ready", (size_t)n_nt * 4);
  p->add("prompt", (size_t)cap_user * 4);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D bf16 tensor [rows, K] (K contiguous) read in boxes of 64 x box_rows with
// the 128-byte swizzle; rows past the end read as zeros.
bool make_map(CUtensorMap* m, const void* base, long long K, long long rows, int box_rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0 || (K * 2) % 16 != 0) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D byte tensor [rows, K] (E4M3 codes, K contiguous) read in boxes of 128 x
// box_rows bytes with the 128-byte swizzle; out-of-range elements read as zeros.
bool make_map_u8(CUtensorMap* m, const void* base, long long K, long long rows, int box_rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0 || K % 16 != 0) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)K};
  cuuint32_t box[2] = {128, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Opt-in per-kernel-class timing with CUDA events recorded on the handle's
// stream around each launch (dg_profile); a launch counter is always kept.
struct KernelProfiler {
  bool on = false;
  std::vector<std::pair<int, std::pair<cudaEvent_t, cudaEvent_t>>> pending;
  std::vector<cudaEvent_t> pool;
  double total_ms[16] = {0};
  long long count[16] = {0};
  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
  void flush() {
    for (auto& r : pending) {
      cudaEventSynchronize(r.second.second);
      float ms = 0.f;
      cudaEventElapsedTime(&ms, r.second.first, r.second.second);
      total_ms[r.first] += ms;
      count[r.first] += 1;
      pool.push_back(r.second.first);
      pool.push_back(r.second.second);
    }
    pending.clear();
  }
  ~KernelProfiler() {
    for (auto& r : pending) {
      cudaEventDestroy(r.second.first);
      cudaEventDestroy(r.second.second);
    }
    for (auto e : pool) cudaEventDestroy(e);
  }
};

const char* const kKernelClass[] = {"embed", "rmsnorm", "qkv", "attention", "oproj", "group",
                                    "experts_gate_up", "experts_down", "shared_gate_up", "shared_down", "lm_head",
                                    "lm_combine", "sample", "selfcond", "other", "experts"};
// K_EXP: the fused routed-expert launch (gate|up, SwiGLU and down); K_EGU /
// K_ED: the two launches of the FP8 experts
enum KClass { K_EMBED, K_RMSNORM, K_QKV, K_ATTN, K_OPROJ, K_GROUP, K_EGU, K_ED, K_SGU, K_SD, K_LM, K_LMC, K_SAMPLE,
              K_SC, K_OTHER, K_EXP, K_NCLASS };
static_assert(K_NCLASS <= 16, "profiler tables hold 16 classes");

struct dg_handle {
  dg_config cfg;
  KernelProfiler prof;
  long long launches = 0;
  int max_req = 0;
  long long cap = 0;
  cudaStream_t st = nullptr;
  int num_sms = 0;
  int T_max = 0, Tcap = 0;
  const bf16* embed = nullptr;
  const float* final_norm = nullptr;
  std::vector<dg_layer_weights> lw;
  uint8_t* ws = nullptr;
  Plan plan;
  int egu_cap = 0, ed_cap = 0;
  long long kv_req_stride = 0, kv_layer_stride = 0;
  std::vector<LayerMaps> maps;
  CUtensorMap tm_u32;
  CUtensorMap tm_hn, tm_o, tm_o128, tm_u, tm_u64, tm_xp, tm_hp, tm_hs, tm_hs64, tm_embed, tm_embed128, tm_k, tm_vt;
  CUtensorMap tm_sc_gate, tm_sc_up, tm_sc_down, tm_hs_sc;  // self-conditioning MLP and its hidden rows
  CUtensorMap tm_xq, tm_hq;                                // FP8 experts: token and hidden codes
  long long cap_user = 0;  // capacity the caller asked for (cap is rounded up to 64)
  ReqState req[DG_MAX_REQUESTS];
  int mask_flip = 0;  // which of the two routing bitmask buffers the next layer uses
  bool keep_router_logits = false;  // debug passes keep the router's fp32 logits for inspection
  long long lm_seq = 0;  // LM-head passes so far: the "stats" / "argmax" buffers hold the latest

  template <class T>
  T* B(const char* name) const {
    return reinterpret_cast<T*>(ws + plan.buf.at(name).first);
  }
};

#define CK(expr)                              \
  do {                                        \
    cudaError_t e__ = (expr);                 \
    if (e__ != cudaSuccess) return DG_E_CUDA; \
  } while (0)

// Launch `expr` (n kernels of class `cls`), counting it and, when profiling,
// bracketing it with events on the handle's stream.
#define LAUNCH(h, cls, n, expr)                                              \
  do {                                                                       \
    cudaEvent_t e0__ = nullptr, e1__ = nullptr;                              \
    if ((h)->prof.on) {                                                      \
      e0__ = (h)->prof.get();                                                \
      e1__ = (h)->prof.get();                                                \
      cudaEventRecord(e0__, (h)->st);                                        \
    }                                                                        \
    CK(expr);                                                                \
    (h)->launches += (n);                                                    \
    if ((h)->prof.on) {                                                      \
      cudaEventRecord(e1__, (h)->st);                                        \
      (h)->prof.pending.push_back({(int)(cls), {e0__, e1__}});               \
    }                                                                        \
  } while (0)

namespace {

// One decoder pass over s.n slots of s.Tr tokens.  n_layers layers; when
// `qkv_only_last` the last layer runs only its K/V projection (nothing reads
// the rest: commit and prefill); `want_lm` adds the final norm + LM head.
// One decoder pass over the slots of `s`.  With want_lm, the final norm and
// the LM head run over the first lm_rows tokens only (lm_rows < 0: all).
// With x_in (debugging): the residual stream entering layer `layer0` is taken
// from x_in [T, d] f32 instead of the token embeddings, and the layers run are
// layer0 .. layer0 + n_layers - 1.
int run_pass(dg_handle* h, const int* const* ids, const SlotInfo& s, int n_layers, bool qkv_only_last, bool want_lm,
             float* logits, int lm_rows = -1, const DrawKeys* keys = nullptr, float temperature = 0.f,
             const SelfCondArgs* sc = nullptr, int layer0 = 0, const float* x_in = nullptr) {
  const dg_config& c = h->cfg;
  const int T = s.n * s.Tr;
  const int TL = lm_rows < 0 ? T : lm_rows;
  const int d = c.d_model, D = c.head_dim, k = c.top_k;
  cudaStream_t st = h->st;
  int* err = h->B<int>("err");
  float* x = h->B<float>("x");
  bf16* hn = h->B<bf16>("hn");
  LAUNCH(h, K_EMBED, 1,
         run_embed(ids, s, h->embed, c.vocab, d, x, h->B<int>("tok_pos"), h->B<int>("tok_req"),
                   h->B<double>("inv_freq"), D / 2, h->B<float2>("rope"), err, st));
  // the routed outputs and the shared-expert partials of layer l are summed
  // into x by the norm kernel of layer l+1 (or the final norm)
  bf16* yp = h->B<bf16>("yp");
  const int* pair_row = h->B<int>("pair_row");
  float* part = h->B<float>("part");
  int pending_k = 0, pending_parts = 0;
  // K splits of the split-K projections are those of one slot, for the same
  // reason as the attention key splits
  const int so = wpart_splits(d, s.Tr, c.n_q_heads * D, h->num_sms);
  const int ss = wpart_splits(d, s.Tr, c.ffn_shared, h->num_sms);
  if (sc != nullptr) {
    // self-conditioning: soft embeddings -> gated MLP; its split-K partials are
    // added to the token embeddings by the first layer's norm kernel
    SelfCondArgs ea = *sc;
    ea.T = T;
    ea.out = h->B<bf16>("u");
    LAUNCH(h, K_SC, 1, run_selfcond_embed(ea, st));
    SharedArgs ga;
    memset(&ga, 0, sizeof(ga));
    ga.tm_u = &h->tm_u;
    ga.tm_gate = &h->tm_sc_gate;
    ga.tm_up = &h->tm_sc_up;
    ga.tm_router = nullptr;
    ga.T = T;
    ga.d = d;
    ga.fs = c.ffn_selfcond;
    ga.num_sms = h->num_sms;
    ga.E = 0;
    ga.hs = h->B<bf16>("hs_sc");
    ga.err = err;
    LAUNCH(h, K_SC, 1, run_shared_gate_up(ga, st));
    const int sp = wpart_splits(d, s.Tr, c.ffn_selfcond, h->num_sms);
    WpartArgs da;
    da.tm_w = &h->tm_sc_down;
    da.tm_x = &h->tm_hs_sc;
    da.T = T;
    da.Tcap = h->Tcap;
    da.d = d;
    da.K = c.ffn_selfcond;
    da.splits = sp;
    da.num_sms = h->num_sms;
    da.part = part;
    da.err = err;
    LAUNCH(h, K_SC, 1, run_wpart(da, st));
    pending_parts = sp;
  }
  if (x_in != nullptr) CK(cudaMemcpyAsync(x, x_in, (size_t)T * d * 4, cudaMemcpyDeviceToDevice, st));
  for (int l = layer0; l < layer0 + n_layers; ++l) {
    const dg_layer_weights& w = h->lw[l];
    const LayerMaps& m = h->maps[l];
    bf16* kv_l = h->B<bf16>("kv") + (size_t)l * h->kv_layer_stride;
    LAUNCH(h, K_RMSNORM, 1,
           run_residual_norm(x, yp, pair_row, pending_k, part, pending_parts, h->Tcap, (const float*)w.attn_norm, T,
                             d, c.norm_eps, hn, st));
    pending_k = pending_parts = 0;
    QkvArgs qa;
    qa.tm_x = &h->tm_hn;
    qa.tm_w = &m.qkv;
    qa.T = T;
    qa.d = d;
    qa.rows = (c.n_q_heads + 2 * c.n_kv_heads) * D;
    qa.D = D;
    qa.Hq = c.n_q_heads;
    qa.Hkv = c.n_kv_heads;
    qa.q_T = h->Tcap;
    qa.kv_cap = (int)h->cap;
    qa.num_sms = h->num_sms;
    qa.kv_req_stride = h->kv_req_stride;
    qa.tok_pos = h->B<int>("tok_pos");
    qa.tok_req = h->B<int>("tok_req");
    qa.rope = h->B<float2>("rope");
    qa.q = h->B<bf16>("q");
    qa.kv = kv_l;
    qa.err = err;
    qa.pair = 1;  // M = 256 tiles over CTA pairs
    LAUNCH(h, K_QKV, 1, run_qkv(qa, st));
    if (qkv_only_last && l == c.n_layers - 1) break;

    AttnArgs aa;
    aa.tm_k = h->tm_k;
    aa.tm_vt = h->tm_vt;
    aa.q = h->B<bf16>("q");
    aa.q_T = h->Tcap;
    aa.o = h->B<bf16>("o");
    aa.k_row0 = (long long)l * 2 * c.n_kv_heads * h->cap;
    aa.req_rows_k = (long long)c.n_layers * 2 * c.n_kv_heads * h->cap;
    aa.v_row0 = (long long)l * 2 * c.n_kv_heads * D + (long long)c.n_kv_heads * D;
    aa.req_rows_v = (long long)c.n_layers * 2 * c.n_kv_heads * D;
    aa.cap = h->cap;
    aa.Hq = c.n_q_heads;
    aa.Hkv = c.n_kv_heads;
    aa.D = D;
    aa.Tr = s.Tr;
    aa.n_slots = s.n;
    // Key splits are chosen per slot from that slot alone (enough CTAs for
    // one slot to fill the GPU, at least 256 keys per split), so a segment's
    // result does not depend on what else shares the pass.
    const int G = c.n_q_heads / c.n_kv_heads;
    const int slot_ctas = ((G * s.Tr + 127) / 128) * c.n_kv_heads;
    aa.n_split = 1;
    for (int i = 0; i < DG_MAX_REQUESTS; ++i) {
      aa.req[i] = i < s.n ? s.req[i] : 0;
      aa.n_keys[i] = i < s.n ? s.pos0[i] + s.Tr : 0;
      int split = 1;
      if (i < s.n) {
        split = h->num_sms / slot_ctas;
        const int by_keys = aa.n_keys[i] / 256;
        if (split > by_keys) split = by_keys;
        if (split > kSplitCap) split = kSplitCap;
        if (split < 1) split = 1;
      }
      aa.slot_split[i] = split;
      if (split > aa.n_split) aa.n_split = split;
    }
    aa.part_o = h->B<float>("attn_o");
    aa.part_ml = h->B<float2>("attn_ml");
    aa.scale = 1.0f / sqrtf((float)D);
    aa.err = err;
    // With the same key split in every slot the splits of a query tile run as
    // one thread-block cluster and merge through distributed shared memory;
    // otherwise their partials go through global memory and k_attn_combine.
    bool uniform = aa.n_split > 1;
    for (int i = 0; i < s.n; ++i) uniform = uniform && aa.slot_split[i] == aa.n_split;
    aa.cluster = uniform ? 1 : 0;
    LAUNCH(h, K_ATTN, aa.n_split > 1 && !aa.cluster ? 2 : 1, run_attention(aa, st));

    WpartArgs oa;
    oa.tm_w = &m.o;
    oa.tm_x = &h->tm_o;
    oa.T = T;
    oa.Tcap = h->Tcap;
    oa.d = d;
    oa.K = c.n_q_heads * D;
    oa.splits = so;
    oa.num_sms = h->num_sms;
    oa.part = part;
    oa.err = err;
    oa.tm_x128 = &h->tm_o128;  // CTA pairs
    LAUNCH(h, K_OPROJ, 1, run_wpart(oa, st));
    // x += attention output projection; FFN RMSNorm -> bf16 rows u
    LAUNCH(h, K_RMSNORM, 1,
           run_residual_norm(x, nullptr, nullptr, 0, part, so, h->Tcap, (const float*)w.ffn_norm, T, d, c.norm_eps,
                             h->B<bf16>("u"), st));
    const int MW = (h->T_max + 31) / 32;  // bitmask words per expert (fixed layout)
    const size_t mw = (size_t)c.n_experts * MW;
    unsigned* masks = h->B<unsigned>("route_mask");
    unsigned* mask_cur = masks + (size_t)h->mask_flip * mw;
    unsigned* mask_nxt = masks + (size_t)(h->mask_flip ^ 1) * mw;
    h->mask_flip ^= 1;
    // shared expert gate|up + router logits, top-k and token bitmasks
    SharedArgs sa;
    sa.tm_u = &h->tm_u;
    sa.tm_u64 = &h->tm_u64;
    sa.tm_u32 = &h->tm_u32;
    sa.tm_gate = &m.sgate;
    sa.tm_up = &m.sup;
    sa.tm_router = &m.router;
    sa.T = T;
    sa.d = d;
    sa.fs = c.ffn_shared;
    sa.num_sms = h->num_sms;
    sa.E = c.n_experts;
    sa.k = k;
    sa.MW = MW;
    sa.hs = h->B<bf16>("hs");
    sa.logits = h->keep_router_logits ? h->B<float>("router_logits") : nullptr;  // nothing else reads them
    sa.idx = h->B<int>("idx");
    sa.w = h->B<float>("w");
    sa.mask = mask_cur;
    sa.err = err;
    LAUNCH(h, K_SGU, 1, run_shared_gate_up(sa, st));
    GroupArgs ga;
    ga.idx = h->B<int>("idx");
    ga.w = h->B<float>("w");
    ga.T = T;
    ga.k = k;
    ga.E = c.n_experts;
    ga.FJ = c.ffn_expert / 64;
    ga.MD = d / 128;
    ga.egu_cap = h->egu_cap;
    ga.ed_cap = h->ed_cap;
    ga.counts = h->B<int>("counts");
    ga.offsets = h->B<int>("offsets");
    ga.pair_row = h->B<int>("pair_row");
    ga.row_token = h->B<int>("row_token");
    ga.row_weight = h->B<float>("row_weight");
    ga.row_pair = h->B<int>("row_pair");
    ga.egu_tiles = h->B<int4>("egu_tiles");
    ga.egu_count = h->B<int>("tile_counts");
    ga.ed_tiles = h->B<int4>("ed_tiles");
    ga.ed_count = h->B<int>("tile_counts") + 1;
    ga.route_stats = h->B<unsigned long long>("route_stats");
    ga.err = err;
    ga.sched = h->B<int>("sched");
    ga.ready = h->B<int>("ready");
    const bool f8 = c.expert_fp8 != 0;
    LAUNCH(h, K_GROUP, 1,
           run_route(h->B<bf16>("u"), d, h->B<bf16>("xp"), mask_cur, mask_nxt, MW, ga, st,
                     f8 ? h->B<uint8_t>("xq") : nullptr, f8 ? h->B<float>("xs") : nullptr));

    ExpertArgs ea;
    ea.tm_gate = &m.gate;
    ea.tm_up = &m.up;
    ea.tm_xp = &h->tm_xp;
    ea.tm_down = &m.down;
    ea.tm_hp = &h->tm_hp;
    ea.d = d;
    ea.fe = c.ffn_expert;
    ea.num_sms = h->num_sms;
    ea.egu_tiles = h->B<int4>("egu_tiles");
    ea.egu_count = h->B<int>("tile_counts");
    ea.ed_tiles = h->B<int4>("ed_tiles");
    ea.ed_count = h->B<int>("tile_counts") + 1;
    ea.counts = h->B<int>("counts");
    ea.offsets = h->B<int>("offsets");
    ea.row_weight = h->B<float>("row_weight");
    ea.hp = h->B<bf16>("hp");
    ea.yp = yp;
    ea.err = err;
    ea.sched = h->B<int>("sched");
    if (f8) {
      // E4M3 weight codes and token rows; the SwiGLU rows are quantised per row before down
      ea.tm_xp = &h->tm_xq;
      ea.tm_hp = &h->tm_hq;
      ea.s_gate = (const float*)w.w_gate_scale;
      ea.s_up = (const float*)w.w_up_scale;
      ea.s_down = (const float*)w.w_down_scale;
      ea.s_x = h->B<float>("xs");
      ea.s_h = h->B<float>("hsq");
      LAUNCH(h, K_EGU, 1, run_experts_gate_up_fp8(ea, st));
      LAUNCH(h, K_ED, 1, run_quant_rows(ea.hp, c.ffn_expert, T * k, h->B<uint8_t>("hq"), h->B<float>("hsq"), st));
      LAUNCH(h, K_ED, 1, run_experts_down_fp8(ea, st));
    } else {
      ea.ready = h->B<int>("ready");
      // the shared expert's down projection runs as tiles of the same launch,
      // unsplit along K: one fp32 slice for the residual norm
      ea.tm_sdown = &m.sdown;
      ea.tm_hs64 = &h->tm_hs64;
      ea.T = T;
      ea.sd_K = c.ffn_shared;
      ea.sd_part = part;
      LAUNCH(h, K_EXP, 1, run_experts(ea, st));
      pending_k = k;
      pending_parts = 1;
      continue;
    }

    WpartArgs da;
    da.tm_w = &m.sdown;
    da.tm_x = &h->tm_hs;
    da.T = T;
    da.Tcap = h->Tcap;
    da.d = d;
    da.K = c.ffn_shared;
    da.splits = ss;
    da.num_sms = h->num_sms;
    da.part = part;
    da.err = err;
    LAUNCH(h, K_SD, 1, run_wpart(da, st));
    pending_k = k;
    pending_parts = ss;
  }
  if (want_lm) {
    ++h->lm_seq;
    LAUNCH(h, K_RMSNORM, 1,
           run_residual_norm(x, yp, pair_row, pending_k, part, pending_parts, h->Tcap, h->final_norm, TL, d,
                             c.norm_eps, hn, st));
    const bool draw = keys != nullptr && temperature > 0.f;
    const bool keep_sc = keys != nullptr && c.ffn_selfcond > 0;  // record this step's state for the next
    const int NV = (int)(c.vocab / 256);
    // chunks of whole slots of at most kLmRowsMax rows; each chunk's draw keys
    // start at its first slot, so all row indexing inside a chunk is local
    const int chunk = kLmRowsMax / s.Tr * s.Tr;
    for (int r0 = 0; r0 < TL; r0 += chunk) {
      const int n = TL - r0 < chunk ? TL - r0 : chunk;
      DrawKeys ck;
      memset(&ck, 0, sizeof(ck));
      if (keys != nullptr) {
        const int slot0 = r0 / s.Tr;
        ck.canvas = keys->canvas;
        for (int i = 0; slot0 + i < DG_MAX_REQUESTS; ++i) {
          ck.req[i] = keys->req[slot0 + i];
          ck.block[i] = keys->block[slot0 + i];
          ck.step[i] = keys->step[slot0 + i];
          ck.seed[i] = keys->seed[slot0 + i];
        }
      }
      LmArgs la;
      la.tm_x = &h->tm_hn;
      la.tm_embed = &h->tm_embed;
      la.row0 = r0;
      la.T = n;
      la.d = d;
      la.num_sms = h->num_sms < kLmGridMax ? h->num_sms : kLmGridMax;
      la.V = c.vocab;
      la.part = h->B<float4>("lm_part");
      la.logits = logits ? logits + (size_t)r0 * c.vocab : nullptr;
      la.err = err;
      la.inv_tau = draw ? 1.0f / temperature : 1.0f;
      la.draw = draw ? h->B<float2>("draw") + (size_t)r0 * NV : nullptr;
      if (draw) la.keys = ck;
      la.sc_part = keep_sc ? h->B<float2>("sc_part") : nullptr;
      la.tm_embed128 = &h->tm_embed128;  // CTA pairs (unless the self-conditioning lists are kept)
      float* stats = h->B<float>("stats") + (size_t)r0 * 4;
      int grid = 0;
      LAUNCH(h, K_LM, 1, run_lm_head(la, &grid, st));
      LAUNCH(h, K_LMC, 1,
             run_lm_combine(h->B<float4>("lm_part"), grid, (n + 127) / 128, n, stats, h->B<int>("argmax") + r0, err,
                            st, la.draw, NV, draw ? &ck : nullptr, draw ? h->B<int>("cand") + r0 : nullptr));
      if (keep_sc)
        LAUNCH(h, K_SC, 1,
               run_selfcond_topk(la.sc_part, grid, n, stats, ck, c.selfcond_topk, h->B<float2>("sc_top"), err, st));
    }
  } else if (pending_k || pending_parts) {
    // a pass stopped after a full layer: fold its expert outputs into x
    LAUNCH(h, K_RMSNORM, 1,
           run_residual_norm(x, yp, pair_row, pending_k, part, pending_parts, h->Tcap, nullptr, T, d, c.norm_eps,
                             nullptr, st));
  }
  return DG_OK;
}

bool req_ok(const dg_handle* h, int r) { return h && r >= 0 && r < h->max_req; }

// Run the pass of a committed block on its own (its K/V at [kv_len - canvas,
// kv_len)) when nothing it could share a pass with is coming.
int flush_commit(dg_handle* h, int req) {
  ReqState& r = h->req[req];
  if (!r.pending) return DG_OK;
  const int C = h->cfg.canvas;
  SlotInfo s;
  memset(&s, 0, sizeof(s));
  s.n = 1;
  s.Tr = C;
  s.req[0] = req;
  s.pos0[0] = (int)(r.kv_len - C);
  const int* ids[1] = {h->B<int>("commit_tok") + (size_t)req * C};
  const int rc = run_pass(h, ids, s, h->cfg.n_layers, true, false, nullptr);
  if (rc == DG_OK) r.pending = false;
  return rc;
}

}  // namespace

extern "C" {

size_t dg_workspace_size(const dg_config* cfg, int max_requests, int64_t kv_capacity) {
  if (!config_ok(cfg) || max_requests < 1 || max_requests > DG_MAX_REQUESTS || kv_capacity < cfg->canvas) return 0;
  Plan p;
  make_plan(cfg, max_requests, kv_capacity, &p);
  return p.total;
}

const char* dg_strerror(int code) {
  switch (code) {
    case DG_OK: return "ok";
    case DG_E_ARG: return "invalid argument or unsupported shape";
    case DG_E_STATE: return "call not valid in the current request state";
    case DG_E_CAPACITY: return "KV capacity or workspace too small";
    case DG_E_CUDA: return "CUDA runtime error";
    case DG_E_DEVICE: return "a kernel reported a device-side error";
    case DG_E_UNSUPPORTED: return "no sm_100 device";
    default: return "unknown error";
  }
}

int dg_init(const dg_config* cfg, const dg_weights* wts, int max_requests, int64_t kv_capacity, void* workspace,
            size_t workspace_bytes, void* stream, dg_handle** out) {
  if (!out) return DG_E_ARG;
  *out = nullptr;
  if (!config_ok(cfg) || !wts || !wts->embed || !wts->final_norm || !wts->layers || !workspace) return DG_E_ARG;
  if (max_requests < 1 || max_requests > DG_MAX_REQUESTS || kv_capacity < cfg->canvas) return DG_E_ARG;
  if (kv_capacity > (1ll << 30)) return DG_E_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return DG_E_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DG_E_CUDA;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return DG_E_CUDA;
  if (prop.major != 10) return DG_E_UNSUPPORTED;
  if ((size_t)prop.sharedMemPerBlockOptin < gemm_smem_bytes_max() ||
      (size_t)prop.sharedMemPerBlockOptin < attention_smem_bytes(cfg->head_dim))
    return DG_E_UNSUPPORTED;

  dg_handle* h = new dg_handle();
  h->cfg = *cfg;
  h->max_req = max_requests;
  h->cap = round_cap(kv_capacity);
  h->cap_user = kv_capacity;
  h->st = static_cast<cudaStream_t>(stream);
  h->num_sms = prop.multiProcessorCount;
  h->T_max = pass_slots(max_requests) * cfg->canvas;
  h->Tcap = (h->T_max + 127) / 128 * 128;
  h->embed = static_cast<const bf16*>(wts->embed);
  h->final_norm = static_cast<const float*>(wts->final_norm);
  h->lw.assign(wts->layers, wts->layers + cfg->n_layers);
  make_plan(cfg, max_requests, kv_capacity, &h->plan);
  if (workspace_bytes < h->plan.total) {
    delete h;
    return DG_E_CAPACITY;
  }
  h->ws = static_cast<uint8_t*>(workspace);
  const dg_config& c = h->cfg;
  const int d = c.d_model, D = c.head_dim;
  h->kv_layer_stride = 2ll * c.n_kv_heads * h->cap * D;
  h->kv_req_stride = h->kv_layer_stride * c.n_layers;
  const long long rows = (long long)h->T_max * c.top_k;
  const long long n_nt = c.n_experts + (rows + kExpertRows - 1) / kExpertRows;
  h->egu_cap = (int)(n_nt * (c.ffn_expert / 64));
  h->ed_cap = (int)(n_nt * (d / 128));

  bool ok = true;
  const int qkv_rows = (c.n_q_heads + 2 * c.n_kv_heads) * D;
  const long long E = c.n_experts;
  h->maps.resize(c.n_layers);
  for (int l = 0; l < c.n_layers && ok; ++l) {
    const dg_layer_weights& w = h->lw[l];
    LayerMaps& m = h->maps[l];
    ok = ok && w.attn_norm && w.ffn_norm && w.w_router;
    ok = ok && make_map(&m.qkv, w.w_qkv, d, qkv_rows, 64);
    ok = ok && make_map(&m.o, w.w_o, (long long)c.n_q_heads * D, d, 128);
    if (c.expert_fp8) {
      ok = ok && w.w_gate_scale && w.w_up_scale && w.w_down_scale;
      ok = ok && make_map_u8(&m.gate, w.w_gate, d, E * c.ffn_expert, 64);
      ok = ok && make_map_u8(&m.up, w.w_up, d, E * c.ffn_expert, 64);
      ok = ok && make_map_u8(&m.down, w.w_down, c.ffn_expert, E * d, 128);
    } else {
      ok = ok && make_map(&m.gate, w.w_gate, d, E * c.ffn_expert, 64);
      ok = ok && make_map(&m.up, w.w_up, d, E * c.ffn_expert, 64);
      ok = ok && make_map(&m.down, w.w_down, c.ffn_expert, E * d, 128);
    }
    ok = ok && make_map(&m.sgate, w.ws_gate, d, c.ffn_shared, 32);
    ok = ok && make_map(&m.sup, w.ws_up, d, c.ffn_shared, 32);
    ok = ok && make_map(&m.router, w.w_router, d, E, (int)E);
    ok = ok && make_map(&m.sdown, w.ws_down, c.ffn_shared, d, 128);
  }
  ok = ok && make_map(&h->tm_hn, h->B<bf16>("hn"), d, h->Tcap, 128);
  ok = ok && make_map(&h->tm_o, h->B<bf16>("o"), (long long)c.n_q_heads * D, h->Tcap, 256);
  ok = ok && make_map(&h->tm_o128, h->B<bf16>("o"), (long long)c.n_q_heads * D, h->Tcap, 128);
  ok = ok && make_map(&h->tm_u, h->B<bf16>("u"), d, h->Tcap, 128);
  ok = ok && make_map(&h->tm_u64, h->B<bf16>("u"), d, h->Tcap, 64);
  ok = ok && make_map(&h->tm_u32, h->B<bf16>("u"), d, h->Tcap, 32);
  ok = ok && make_map(&h->tm_xp, h->B<bf16>("xp"), d, rows, kExpertBoxRows);
  ok = ok && make_map(&h->tm_hp, h->B<bf16>("hp"), c.ffn_expert, rows, kExpertBoxRows);
  ok = ok && make_map(&h->tm_hs, h->B<bf16>("hs"), c.ffn_shared, h->Tcap, 256);
  ok = ok && make_map(&h->tm_hs64, h->B<bf16>("hs"), c.ffn_shared, h->Tcap, kExpertRows);
  ok = ok && make_map(&h->tm_embed, h->embed, d, c.vocab, 256);
  ok = ok && make_map(&h->tm_embed128, h->embed, d, c.vocab, 128);
  {
    const long long kv_elems = (long long)max_requests * h->kv_req_stride;
    // K in the tiled layout: rows of 64 dims, a tile of 64 keys = D rows
    ok = ok && kv_elems / 64 < (1ll << 31);
    ok = ok && make_map(&h->tm_k, h->B<bf16>("kv"), 64, kv_elems / 64, D);
    ok = ok && make_map(&h->tm_vt, h->B<bf16>("kv"), h->cap, kv_elems / h->cap, D);
  }
  if (c.expert_fp8) {
    ok = ok && make_map_u8(&h->tm_xq, h->B<uint8_t>("xq"), d, rows, kExpertRows);
    ok = ok && make_map_u8(&h->tm_hq, h->B<uint8_t>("hq"), c.ffn_expert, rows, kExpertRows);
  }
  if (c.ffn_selfcond > 0) {
    const int f = c.ffn_selfcond;
    ok = ok && wts->sc_gate && wts->sc_up && wts->sc_down;
    ok = ok && make_map(&h->tm_sc_gate, wts->sc_gate, d, f, 32);
    ok = ok && make_map(&h->tm_sc_up, wts->sc_up, d, f, 32);
    ok = ok && make_map(&h->tm_sc_down, wts->sc_down, f, d, 128);
    ok = ok && make_map(&h->tm_hs_sc, h->B<bf16>("hs_sc"), f, h->Tcap, 256);
  }
  if (!ok) {
    delete h;
    return DG_E_ARG;
  }
  // RoPE inverse frequencies theta^(-2i/D), computed in double
  std::vector<double> inv(D / 2);
  for (int i = 0; i < D / 2; ++i) inv[i] = pow((double)c.rope_theta, -2.0 * i / (double)D);
  if (cudaMemcpyAsync(h->B<double>("inv_freq"), inv.data(), inv.size() * 8, cudaMemcpyHostToDevice, h->st) !=
          cudaSuccess ||
      cudaMemsetAsync(h->B<int>("err"), 0, 64, h->st) != cudaSuccess ||
      cudaMemsetAsync(h->B<int>("route_stats"), 0, 64, h->st) != cudaSuccess ||
      cudaMemsetAsync(h->B<int>("route_mask"), 0, h->plan.buf.at("route_mask").second, h->st) != cudaSuccess ||
      cudaMemsetAsync(h->B<int>("sched"), 0, 64, h->st) != cudaSuccess ||
      cudaMemsetAsync(h->B<bf16>("kv"), 0, h->plan.buf.at("kv").second, h->st) != cudaSuccess ||
      cudaMemsetAsync(h->B<int>("remaining"), 0, (size_t)max_requests * 4, h->st) != cudaSuccess ||
      cudaStreamSynchronize(h->st) != cudaSuccess) {
    delete h;
    return DG_E_CUDA;
  }
  *out = h;
  return DG_OK;
}

void dg_destroy(dg_handle* h) { delete h; }

int64_t dg_kv_len(const dg_handle* h, int req) { return req_ok(h, req) ? h->req[req].kv_len : -1; }

int dg_set_kv(dg_handle* h, int req, int layer, int64_t pos0, int64_t n, const void* d_k, const void* d_v) {
  if (!req_ok(h, req) || layer < 0 || layer >= h->cfg.n_layers || pos0 < 0 || n < 0 || !d_k || !d_v) return DG_E_ARG;
  if (pos0 + n > h->cap_user) return DG_E_CAPACITY;
  const int rc = flush_commit(h, req);
  if (rc != DG_OK) return rc;
  bf16* ck = h->B<bf16>("kv") + req * h->kv_req_stride + layer * h->kv_layer_stride;
  bf16* cv = ck + (size_t)h->cfg.n_kv_heads * h->cap * h->cfg.head_dim;
  CK(run_kv_copy(ck, cv, h->cfg.n_kv_heads, h->cap, h->cfg.head_dim, pos0, n, (const bf16*)d_k, (const bf16*)d_v,
                 nullptr, nullptr, h->st));
  return DG_OK;
}

int dg_get_kv(dg_handle* h, int req, int layer, int64_t pos0, int64_t n, void* d_k, void* d_v) {
  if (!req_ok(h, req) || layer < 0 || layer >= h->cfg.n_layers || pos0 < 0 || n < 0 || !d_k || !d_v) return DG_E_ARG;
  if (pos0 + n > h->cap_user) return DG_E_CAPACITY;
  const int rc = flush_commit(h, req);
  if (rc != DG_OK) return rc;
  bf16* ck = h->B<bf16>("kv") + req * h->kv_req_stride + layer * h->kv_layer_stride;
  bf16* cv = ck + (size_t)h->cfg.n_kv_heads * h->cap * h->cfg.head_dim;
  CK(run_kv_copy(ck, cv, h->cfg.n_kv_heads, h->cap, h->cfg.head_dim, pos0, n, nullptr, nullptr, (bf16*)d_k,
                 (bf16*)d_v, h->st));
  return DG_OK;
}

int dg_set_kv_len(dg_handle* h, int req, int64_t len) {
  if (!req_ok(h, req) || len < 0) return DG_E_ARG;
  if (h->req[req].open) return DG_E_STATE;
  if (len > h->cap_user) return DG_E_CAPACITY;
  const int rc = flush_commit(h, req);
  if (rc != DG_OK) return rc;
  h->req[req].kv_len = len;
  return DG_OK;
}

int dg_prefill(dg_handle* h, int req, const int32_t* d_tokens, int n) {
  if (!req_ok(h, req) || n < 0 || (n > 0 && !d_tokens)) return DG_E_ARG;
  ReqState& r = h->req[req];
  if (r.open) return DG_E_STATE;
  if (r.kv_len + n > h->cap_user) return DG_E_CAPACITY;
  int rc0 = flush_commit(h, req);
  if (rc0 != DG_OK) return rc0;
  const int seg = h->cfg.canvas;
  const int group = h->T_max / seg;  // full segments per pass
  int s0 = 0;
  while (s0 < n) {
    // consecutive full segments share a pass; a short last segment goes alone
    const int full = (n - s0) / seg;
    const int ns = full >= 1 ? (full < group ? full : group) : 1;
    const int len = full >= 1 ? seg : n - s0;
    SlotInfo s;
    memset(&s, 0, sizeof(s));
    s.n = ns;
    s.Tr = len;
    const int* ids[DG_MAX_REQUESTS];
    for (int i = 0; i < ns; ++i) {
      s.req[i] = req;
      s.pos0[i] = (int)r.kv_len + i * seg;
      ids[i] = d_tokens + s0 + i * seg;
    }
    int rc = run_pass(h, ids, s, h->cfg.n_layers, true, false, nullptr);
    if (rc != DG_OK) return rc;
    r.kv_len += (long long)ns * len;
    s0 += ns * len;
  }
  return DG_OK;
}

int dg_open_canvas(dg_handle* h, int req, uint64_t seed, int block) {
  if (!req_ok(h, req) || block < 0) return DG_E_ARG;
  ReqState& r = h->req[req];
  if (r.kv_len + h->cfg.canvas > h->cap_user) return DG_E_CAPACITY;
  const int C = h->cfg.canvas;
  LAUNCH(h, K_OTHER, 1,
         run_philox_tokens(seed, block, 0, req, 0, C, h->cfg.vocab, h->B<int>("canvas") + (size_t)req * C,
                           h->B<unsigned char>("mask") + (size_t)req * C, h->st));
  CK(cudaMemsetAsync(h->B<int>("remaining") + req, 0, 4, h->st));
  r.open = true;
  r.seed = seed;
  r.block = block;
  r.step = 0;
  r.sc_valid = false;
  return DG_OK;
}

static int sample_slots(dg_handle* h, int n_req, const int* reqs, const float* entropy, const float* logconf,
                        int stride, const int* argmax, const int* steps, const int* cand = nullptr) {
  const dg_config& c = h->cfg;
  SampleArgs a;
  memset(&a, 0, sizeof(a));
  a.n_slots = n_req;
  a.canvas = c.canvas;
  a.vocab = c.vocab;
  a.min_accept = c.min_accept;
  a.max_steps = c.max_steps;
  a.thr = c.entropy_thresh;
  a.mode = c.sampler;
  a.budget = c.entropy_budget;
  a.stop_entropy = c.stop_entropy;
  a.prev_argmax = h->B<int>("prev_argmax");
  for (int i = 0; i < n_req; ++i) {
    const ReqState& r = h->req[reqs[i]];
    a.req[i] = reqs[i];
    a.block[i] = r.block;
    a.step[i] = steps[i];
    a.seed[i] = r.seed;
  }
  a.entropy = entropy;
  a.logconf = logconf;
  a.stride = stride;
  a.argmax = argmax;
  a.cand = cand;
  a.canvas_tok = h->B<int>("canvas");
  a.mask = h->B<unsigned char>("mask");
  a.remaining = h->B<int>("remaining");
  a.err = h->B<int>("err");
  LAUNCH(h, K_SAMPLE, 1, run_sample(a, h->st));
  return DG_OK;
}

int dg_denoise_step(dg_handle* h, int n_req, const int* reqs, int32_t* d_remaining) {
  if (!h || n_req < 1 || n_req > h->max_req || !reqs) return DG_E_ARG;
  for (int i = 0; i < n_req; ++i) {
    if (!req_ok(h, reqs[i])) return DG_E_ARG;
    for (int j = 0; j < i; ++j)
      if (reqs[j] == reqs[i]) return DG_E_ARG;
    if (!h->req[reqs[i]].open) return DG_E_STATE;
  }
  const int C = h->cfg.canvas;
  // pending commits of these requests join the pass as extra slots after the
  // canvases (block-causal: a committed block's keys end where its canvas's
  // begin); the LM head covers the canvas slots only
  int n_pend = 0;
  for (int i = 0; i < n_req; ++i) n_pend += h->req[reqs[i]].pending ? 1 : 0;
  if (n_req + n_pend > h->T_max / C || n_req + n_pend > DG_MAX_REQUESTS) {
    for (int i = 0; i < n_req; ++i) {
      const int rc0 = flush_commit(h, reqs[i]);
      if (rc0 != DG_OK) return rc0;
    }
    n_pend = 0;
  }
  SlotInfo s;
  memset(&s, 0, sizeof(s));
  s.n = n_req + n_pend;
  s.Tr = C;
  const int* ids[DG_MAX_REQUESTS];
  int steps[DG_MAX_REQUESTS];
  int j = n_req;
  for (int i = 0; i < n_req; ++i) {
    const ReqState& r = h->req[reqs[i]];
    s.req[i] = reqs[i];
    s.pos0[i] = (int)r.kv_len;
    ids[i] = h->B<int>("canvas") + (size_t)reqs[i] * C;
    steps[i] = r.step + 1;
    if (r.pending) {
      s.req[j] = reqs[i];
      s.pos0[j] = (int)(r.kv_len - C);
      ids[j] = h->B<int>("commit_tok") + (size_t)reqs[i] * C;
      ++j;
    }
  }
  // candidate draw keys of the canvas slots (LM-head rows slot * C + position)
  DrawKeys keys;
  memset(&keys, 0, sizeof(keys));
  keys.canvas = C;
  for (int i = 0; i < n_req; ++i) {
    const ReqState& r = h->req[reqs[i]];
    keys.req[i] = reqs[i];
    keys.block[i] = r.block;
    keys.step[i] = steps[i];
    keys.seed[i] = r.seed;
  }
  const bool draw = h->cfg.temperature > 0.f;
  const bool selfcond = h->cfg.ffn_selfcond > 0;
  // self-conditioning input of the canvas slots whose request has a previous
  // step of this canvas (slots past n_req, the commit slots, get none)
  SelfCondArgs sca;
  memset(&sca, 0, sizeof(sca));
  bool any_sc = false;
  if (selfcond) {
    sca.canvas = C;
    sca.d = h->cfg.d_model;
    sca.vocab = h->cfg.vocab;
    sca.K = h->cfg.selfcond_topk;
    sca.n_slots = n_req;
    sca.top = h->B<float2>("sc_top");
    sca.embed = h->embed;
    sca.err = h->B<int>("err");
    for (int i = 0; i < n_req; ++i) {
      sca.req[i] = reqs[i];
      sca.on[i] = h->req[reqs[i]].sc_valid ? 1 : 0;
      any_sc = any_sc || sca.on[i];
    }
  }
  int rc = run_pass(h, ids, s, h->cfg.n_layers, false, true, nullptr, n_req * C,
                    (draw || selfcond) ? &keys : nullptr, h->cfg.temperature, any_sc ? &sca : nullptr);
  if (rc != DG_OK) return rc;
  for (int i = 0; i < n_req; ++i) {
    h->req[reqs[i]].pending = false;
    h->req[reqs[i]].sc_valid = selfcond;
  }
  float* stats = h->B<float>("stats");
  rc = sample_slots(h, n_req, reqs, stats, stats + 1, 4, h->B<int>("argmax"), steps,
                    draw ? h->B<int>("cand") : nullptr);
  if (rc != DG_OK) return rc;
  for (int i = 0; i < n_req; ++i) {
    h->req[reqs[i]].step = steps[i];
    h->req[reqs[i]].last_slot = i;
    h->req[reqs[i]].stats_seq = h->lm_seq;
    if (d_remaining)
      CK(cudaMemcpyAsync(d_remaining + i, h->B<int>("remaining") + reqs[i], 4, cudaMemcpyDeviceToDevice, h->st));
  }
  return DG_OK;
}

int dg_read_remaining(dg_handle* h, int req, int32_t* remaining) {
  if (!req_ok(h, req) || !remaining) return DG_E_ARG;
  CK(cudaMemcpyAsync(remaining, h->B<int>("remaining") + req, 4, cudaMemcpyDeviceToHost, h->st));
  CK(cudaStreamSynchronize(h->st));
  return DG_OK;
}

int dg_commit_block(dg_handle* h, int req) {
  if (!req_ok(h, req)) return DG_E_ARG;
  ReqState& r = h->req[req];
  if (!r.open) return DG_E_STATE;
  int rc = flush_commit(h, req);  // a block committed before this one without a step in between
  if (rc != DG_OK) return rc;
  // The block's pass is deferred: it rides along with the request's next
  // denoising step (one weight stream for both), or runs on its own as soon
  // as another call needs the cache.  The tokens are kept aside because the
  // next dg_open_canvas overwrites the canvas.
  const int C = h->cfg.canvas;
  CK(cudaMemcpyAsync(h->B<int>("commit_tok") + (size_t)req * C, h->B<int>("canvas") + (size_t)req * C, (size_t)C * 4,
                     cudaMemcpyDeviceToDevice, h->st));
  r.kv_len += C;
  r.pending = true;
  r.open = false;
  return DG_OK;
}

int dg_sync(dg_handle* h) {
  if (!h) return DG_E_ARG;
  CK(cudaStreamSynchronize(h->st));
  int e = 0;
  CK(cudaMemcpy(&e, h->B<int>("err"), 4, cudaMemcpyDeviceToHost));
  if (e != 0) {
    cudaMemset(h->B<int>("err"), 0, 4);
    return DG_E_DEVICE;
  }
  return DG_OK;
}

int dg_generate(dg_handle* h, int req, const int32_t* h_prompt, int n_prompt, int n_out, uint64_t seed,
                int32_t* h_out, int* steps_taken) {
  if (!req_ok(h, req) || n_prompt < 0 || (n_prompt > 0 && !h_prompt) || n_out < 0 || !h_out) return DG_E_ARG;
  const int C = h->cfg.canvas;
  if (n_out % C != 0) return DG_E_ARG;
  ReqState& r = h->req[req];
  if (r.open || r.kv_len != 0 || r.pending) return DG_E_STATE;
  if ((long long)n_prompt + n_out > h->cap_user) return DG_E_CAPACITY;
  int* prompt = h->B<int>("prompt");
  if (n_prompt > 0) CK(cudaMemcpyAsync(prompt, h_prompt, (size_t)n_prompt * 4, cudaMemcpyHostToDevice, h->st));
  int rc = dg_prefill(h, req, prompt, n_prompt);
  if (rc != DG_OK) return rc;
  for (int b = 0; b < n_out / C; ++b) {
    rc = dg_open_canvas(h, req, seed, b);
    if (rc != DG_OK) return rc;
    int steps = 0;
    int32_t rem = 1;
    while (rem > 0) {
      rc = dg_denoise_step(h, 1, &req, nullptr);
      if (rc != DG_OK) return rc;
      ++steps;
      rc = dg_read_remaining(h, req, &rem);
      if (rc != DG_OK) return rc;
      if (steps >= h->cfg.max_steps && rem > 0) return DG_E_DEVICE;
    }
    if (steps_taken) steps_taken[b] = steps;
    CK(cudaMemcpyAsync(h_out + (size_t)b * C, h->B<int>("canvas") + (size_t)req * C, (size_t)C * 4,
                       cudaMemcpyDeviceToHost, h->st));
    rc = dg_commit_block(h, req);
    if (rc != DG_OK) return rc;
  }
  rc = flush_commit(h, req);
  if (rc != DG_OK) return rc;
  return dg_sync(h);
}

int dg_get_canvas(dg_handle* h, int req, int32_t* d_tokens, uint8_t* d_mask, float* d_stats, int32_t* d_argmax) {
  if (!req_ok(h, req)) return DG_E_ARG;
  const int C = h->cfg.canvas;
  const ReqState& r = h->req[req];
  if (d_tokens)
    CK(cudaMemcpyAsync(d_tokens, h->B<int>("canvas") + (size_t)req * C, (size_t)C * 4, cudaMemcpyDeviceToDevice,
                       h->st));
  if (d_mask)
    CK(cudaMemcpyAsync(d_mask, h->B<unsigned char>("mask") + (size_t)req * C, (size_t)C, cudaMemcpyDeviceToDevice,
                       h->st));
  // the statistics buffers hold the latest LM-head pass only: another
  // request's step, an LM-head operation or a full debug pass since this
  // request's last step has overwritten them (NaN / -1 then)
  const bool current = r.stats_seq == h->lm_seq;
  if (d_stats) {
    if (current)
      CK(cudaMemcpyAsync(d_stats, h->B<float>("stats") + (size_t)r.last_slot * C * 4, (size_t)C * 16,
                         cudaMemcpyDeviceToDevice, h->st));
    else
      CK(cudaMemsetAsync(d_stats, 0xFF, (size_t)C * 16, h->st));
  }
  if (d_argmax) {
    if (current)
      CK(cudaMemcpyAsync(d_argmax, h->B<int>("argmax") + (size_t)r.last_slot * C, (size_t)C * 4,
                         cudaMemcpyDeviceToDevice, h->st));
    else
      CK(cudaMemsetAsync(d_argmax, 0xFF, (size_t)C * 4, h->st));
  }
  return DG_OK;
}

int dg_set_canvas(dg_handle* h, int req, const int32_t* d_tokens, const uint8_t* d_mask, int step) {
  if (!req_ok(h, req) || step < 0) return DG_E_ARG;
  ReqState& r = h->req[req];
  if (!r.open) return DG_E_STATE;
  const int C = h->cfg.canvas;
  if (d_tokens)
    CK(cudaMemcpyAsync(h->B<int>("canvas") + (size_t)req * C, d_tokens, (size_t)C * 4, cudaMemcpyDeviceToDevice,
                       h->st));
  if (d_mask)
    CK(cudaMemcpyAsync(h->B<unsigned char>("mask") + (size_t)req * C, d_mask, (size_t)C, cudaMemcpyDeviceToDevice,
                       h->st));
  r.step = step;
  return DG_OK;
}

// ---- operation-level entry points ----

int dg_op_philox_tokens(uint64_t seed, int block, int step, int request, int64_t pos0, int64_t n, int vocab,
                        int32_t* d_out, void* stream) {
  if (n < 0 || vocab < 1 || block < 0 || step < 0 || request < 0 || pos0 < 0 || (n > 0 && !d_out)) return DG_E_ARG;
  CK(run_philox_tokens(seed, block, step, request, pos0, n, vocab, d_out, nullptr, static_cast<cudaStream_t>(stream)));
  return DG_OK;
}

int dg_op_route_topk(const float* d_logits, int T, int E, int k, int32_t* d_idx, float* d_w, void* stream) {
  if (T < 0 || E < 1 || E > 256 || k < 1 || k > 8 || k > E || (T > 0 && (!d_logits || !d_idx || !d_w))) return DG_E_ARG;
  CK(run_topk(d_logits, T, E, k, d_idx, d_w, static_cast<cudaStream_t>(stream)));
  return DG_OK;
}

int dg_op_route_group(dg_handle* h, const int32_t* d_idx, const float* d_w, int T, int32_t* d_counts,
                      int32_t* d_offsets, int32_t* d_perm) {
  if (!h || T < 1 || T > h->T_max || !d_idx || !d_w) return DG_E_ARG;
  const dg_config& c = h->cfg;
  GroupArgs ga;
  ga.idx = const_cast<int*>(d_idx);
  ga.w = const_cast<float*>(d_w);
  ga.T = T;
  ga.k = c.top_k;
  ga.E = c.n_experts;
  ga.FJ = c.ffn_expert / 64;
  ga.MD = c.d_model / 128;
  ga.egu_cap = h->egu_cap;
  ga.ed_cap = h->ed_cap;
  ga.counts = h->B<int>("counts");
  ga.offsets = h->B<int>("offsets");
  ga.pair_row = h->B<int>("pair_row");
  ga.row_token = h->B<int>("row_token");
  ga.row_weight = h->B<float>("row_weight");
  ga.row_pair = h->B<int>("row_pair");
  ga.egu_tiles = h->B<int4>("egu_tiles");
  ga.egu_count = h->B<int>("tile_counts");
  ga.ed_tiles = h->B<int4>("ed_tiles");
  ga.ed_count = h->B<int>("tile_counts") + 1;
  ga.route_stats = nullptr;
  ga.err = h->B<int>("err");
  CK(run_group(ga, h->st));
  if (d_counts)
    CK(cudaMemcpyAsync(d_counts, ga.counts, (size_t)c.n_experts * 4, cudaMemcpyDeviceToDevice, h->st));
  if (d_offsets)
    CK(cudaMemcpyAsync(d_offsets, ga.offsets, (size_t)(c.n_experts + 1) * 4, cudaMemcpyDeviceToDevice, h->st));
  if (d_perm)
    CK(cudaMemcpyAsync(d_perm, ga.row_pair, (size_t)T * c.top_k * 4, cudaMemcpyDeviceToDevice, h->st));
  return DG_OK;
}

int dg_op_sample(dg_handle* h, int req, const float* d_entropy, const float* d_logconf, const int32_t* d_argmax,
                 int step) {
  if (!req_ok(h, req) || !d_entropy || !d_logconf || !d_argmax || step < 1) return DG_E_ARG;
  if (!h->req[req].open) return DG_E_STATE;
  int steps[1] = {step};
  int rc = sample_slots(h, 1, &req, d_entropy, d_logconf, 1, d_argmax, steps);
  if (rc == DG_OK) h->req[req].step = step;
  return rc;
}

int dg_op_lm_head(dg_handle* h, const float* d_x, int T, float* d_stats, int32_t* d_argmax, float* d_logits) {
  if (!h || T < 1 || T > h->T_max || !d_x) return DG_E_ARG;
  const dg_config& c = h->cfg;
  float* x = h->B<float>("x");
  CK(cudaMemcpyAsync(x, d_x, (size_t)T * c.d_model * 4, cudaMemcpyDeviceToDevice, h->st));
  CK(run_rmsnorm(x, h->final_norm, T, c.d_model, c.norm_eps, h->B<bf16>("hn"), h->st));
  LmArgs la;
  la.tm_x = &h->tm_hn;
  la.tm_embed = &h->tm_embed;
  la.T = T;
  la.d = c.d_model;
  la.num_sms = h->num_sms < kLmGridMax ? h->num_sms : kLmGridMax;
  la.V = c.vocab;
  la.part = h->B<float4>("lm_part");
  la.logits = d_logits;
  la.err = h->B<int>("err");
  ++h->lm_seq;
  int grid = 0;
  CK(run_lm_head(la, &grid, h->st));
  CK(run_lm_combine(la.part, grid, (T + 127) / 128, T, h->B<float>("stats"), h->B<int>("argmax"), la.err, h->st));
  if (d_stats) CK(cudaMemcpyAsync(d_stats, h->B<float>("stats"), (size_t)T * 16, cudaMemcpyDeviceToDevice, h->st));
  if (d_argmax) CK(cudaMemcpyAsync(d_argmax, h->B<int>("argmax"), (size_t)T * 4, cudaMemcpyDeviceToDevice, h->st));
  return DG_OK;
}

int dg_op_lm_sample(dg_handle* h, const float* d_x, int T, float temperature, uint64_t seed, int block, int step,
                    int request, float* d_stats, int32_t* d_argmax, int32_t* d_cand) {
  if (!h || !d_x || !d_cand || T < 1 || T > h->cfg.canvas || !(temperature > 0.f && temperature <= 1e30f) ||
      block < 0 || step < 0 || request < 0 || request >= h->max_req)
    return DG_E_ARG;
  const dg_config& c = h->cfg;
  float* x = h->B<float>("x");
  CK(cudaMemcpyAsync(x, d_x, (size_t)T * c.d_model * 4, cudaMemcpyDeviceToDevice, h->st));
  CK(run_rmsnorm(x, h->final_norm, T, c.d_model, c.norm_eps, h->B<bf16>("hn"), h->st));
  DrawKeys keys;
  memset(&keys, 0, sizeof(keys));
  keys.canvas = c.canvas;
  keys.req[0] = request;
  keys.block[0] = block;
  keys.step[0] = step;
  keys.seed[0] = seed;
  LmArgs la;
  la.tm_x = &h->tm_hn;
  la.tm_embed = &h->tm_embed;
  la.T = T;
  la.d = c.d_model;
  la.num_sms = h->num_sms < kLmGridMax ? h->num_sms : kLmGridMax;
  la.V = c.vocab;
  la.part = h->B<float4>("lm_part");
  la.logits = nullptr;
  la.err = h->B<int>("err");
  la.inv_tau = 1.0f / temperature;
  la.draw = h->B<float2>("draw");
  la.keys = keys;
  ++h->lm_seq;
  int grid = 0;
  CK(run_lm_head(la, &grid, h->st));
  CK(run_lm_combine(la.part, grid, (T + 127) / 128, T, h->B<float>("stats"), h->B<int>("argmax"), la.err, h->st,
                    la.draw, (int)(c.vocab / 256), &keys, h->B<int>("cand")));
  CK(cudaMemcpyAsync(d_cand, h->B<int>("cand"), (size_t)T * 4, cudaMemcpyDeviceToDevice, h->st));
  if (d_stats) CK(cudaMemcpyAsync(d_stats, h->B<float>("stats"), (size_t)T * 16, cudaMemcpyDeviceToDevice, h->st));
  if (d_argmax) CK(cudaMemcpyAsync(d_argmax, h->B<int>("argmax"), (size_t)T * 4, cudaMemcpyDeviceToDevice, h->st));
  return DG_OK;
}

int dg_op_selfcond(dg_handle* h, int request, const float* d_x, int T, float* d_sc, void* d_top) {
  if (!h || !d_x || !d_sc || T < 1 || T > h->cfg.canvas || !req_ok(h, request)) return DG_E_ARG;
  const dg_config& c = h->cfg;
  if (c.ffn_selfcond <= 0) return DG_E_ARG;
  const int d = c.d_model;
  float* x = h->B<float>("x");
  int* err = h->B<int>("err");
  CK(cudaMemcpyAsync(x, d_x, (size_t)T * d * 4, cudaMemcpyDeviceToDevice, h->st));
  CK(run_rmsnorm(x, h->final_norm, T, d, c.norm_eps, h->B<bf16>("hn"), h->st));
  DrawKeys keys;
  memset(&keys, 0, sizeof(keys));
  keys.canvas = c.canvas;
  keys.req[0] = request;
  LmArgs la;
  la.tm_x = &h->tm_hn;
  la.tm_embed = &h->tm_embed;
  la.T = T;
  la.d = d;
  la.num_sms = h->num_sms < kLmGridMax ? h->num_sms : kLmGridMax;
  la.V = c.vocab;
  la.part = h->B<float4>("lm_part");
  la.logits = nullptr;
  la.err = err;
  la.sc_part = h->B<float2>("sc_part");
  ++h->lm_seq;
  int grid = 0;
  CK(run_lm_head(la, &grid, h->st));
  CK(run_lm_combine(la.part, grid, (T + 127) / 128, T, h->B<float>("stats"), h->B<int>("argmax"), err, h->st));
  float2* top = h->B<float2>("sc_top");
  CK(run_selfcond_topk(la.sc_part, grid, T, h->B<float>("stats"), keys, c.selfcond_topk, top, err, h->st));
  if (d_top)
    CK(cudaMemcpyAsync(d_top, top + (size_t)request * c.canvas * 8, (size_t)T * 8 * sizeof(float2),
                       cudaMemcpyDeviceToDevice, h->st));
  // the pass's self-conditioning prologue on rows 0..T-1 as slot 0
  SelfCondArgs ea;
  memset(&ea, 0, sizeof(ea));
  ea.canvas = c.canvas;
  ea.T = T;
  ea.d = d;
  ea.vocab = c.vocab;
  ea.K = c.selfcond_topk;
  ea.n_slots = 1;
  ea.req[0] = request;
  ea.on[0] = 1;
  ea.top = top;
  ea.embed = h->embed;
  ea.out = h->B<bf16>("u");
  ea.err = err;
  CK(run_selfcond_embed(ea, h->st));
  SharedArgs ga;
  memset(&ga, 0, sizeof(ga));
  ga.tm_u = &h->tm_u;
  ga.tm_gate = &h->tm_sc_gate;
  ga.tm_up = &h->tm_sc_up;
  ga.T = T;
  ga.d = d;
  ga.fs = c.ffn_selfcond;
  ga.num_sms = h->num_sms;
  ga.hs = h->B<bf16>("hs_sc");
  ga.err = err;
  CK(run_shared_gate_up(ga, h->st));
  const int sp = wpart_splits(d, T, c.ffn_selfcond, h->num_sms);
  WpartArgs da;
  da.tm_w = &h->tm_sc_down;
  da.tm_x = &h->tm_hs_sc;
  da.T = T;
  da.Tcap = h->Tcap;
  da.d = d;
  da.K = c.ffn_selfcond;
  da.splits = sp;
  da.num_sms = h->num_sms;
  da.part = h->B<float>("part");
  da.err = err;
  CK(run_wpart(da, h->st));
  // sum of the partials (fold into a zeroed residual, no norm)
  CK(cudaMemsetAsync(x, 0, (size_t)T * d * 4, h->st));
  CK(run_residual_norm(x, nullptr, nullptr, 0, da.part, sp, h->Tcap, nullptr, T, d, c.norm_eps, nullptr, h->st));
  CK(cudaMemcpyAsync(d_sc, x, (size_t)T * d * 4, cudaMemcpyDeviceToDevice, h->st));
  return DG_OK;
}

int dg_debug_forward(dg_handle* h, int req, const int32_t* d_tokens, int T, int n_layers) {
  if (!req_ok(h, req) || !d_tokens || T < 1 || T > h->cfg.canvas || n_layers < 1 || n_layers > h->cfg.n_layers)
    return DG_E_ARG;
  const ReqState& r = h->req[req];
  if (r.kv_len + T > h->cap_user) return DG_E_CAPACITY;
  const int rc = flush_commit(h, req);
  if (rc != DG_OK) return rc;
  SlotInfo s;
  memset(&s, 0, sizeof(s));
  s.n = 1;
  s.Tr = T;
  s.req[0] = req;
  s.pos0[0] = (int)r.kv_len;
  const int* ids[1] = {d_tokens};
  h->keep_router_logits = true;
  const int rc2 = run_pass(h, ids, s, n_layers, false, n_layers == h->cfg.n_layers, nullptr);
  h->keep_router_logits = false;
  return rc2;
}

int dg_debug_forward_hidden(dg_handle* h, int req, const int32_t* d_tokens, const float* d_x, int T, int layer0,
                            int n_layers) {
  if (!req_ok(h, req) || !d_tokens || !d_x || T < 1 || T > h->cfg.canvas || layer0 < 0 || n_layers < 1 ||
      layer0 + n_layers > h->cfg.n_layers)
    return DG_E_ARG;
  const ReqState& r = h->req[req];
  if (r.kv_len + T > h->cap_user) return DG_E_CAPACITY;
  const int rc = flush_commit(h, req);
  if (rc != DG_OK) return rc;
  SlotInfo s;
  memset(&s, 0, sizeof(s));
  s.n = 1;
  s.Tr = T;
  s.req[0] = req;
  s.pos0[0] = (int)r.kv_len;
  const int* ids[1] = {d_tokens};
  h->keep_router_logits = true;
  const int rc2 = run_pass(h, ids, s, n_layers, false, layer0 + n_layers == h->cfg.n_layers, nullptr, -1, nullptr,
                           0.f, nullptr, layer0, d_x);
  h->keep_router_logits = false;
  return rc2;
}

int dg_profile(dg_handle* h, int enable) {
  if (!h) return DG_E_ARG;
  h->prof.flush();
  if (enable < 0) {
    for (int i = 0; i < K_NCLASS; ++i) {
      h->prof.total_ms[i] = 0.0;
      h->prof.count[i] = 0;
    }
    return DG_OK;
  }
  h->prof.on = enable != 0;
  return DG_OK;
}

int dg_profile_read(dg_handle* h, const char* kernel, double* total_ms, int64_t* launches) {
  if (!h || !kernel) return DG_E_ARG;
  h->prof.flush();
  for (int i = 0; i < K_NCLASS; ++i)
    if (strcmp(kernel, kKernelClass[i]) == 0) {
      if (total_ms) *total_ms = h->prof.total_ms[i];
      if (launches) *launches = h->prof.count[i];
      return DG_OK;
    }
  return DG_E_ARG;
}

int64_t dg_launch_count(const dg_handle* h) { return h ? h->launches : -1; }

int dg_debug_buffer(const dg_handle* h, const char* name, size_t* offset, size_t* bytes) {
  if (!h || !name) return DG_E_ARG;
  auto it = h->plan.buf.find(name);
  if (it == h->plan.buf.end()) return DG_E_ARG;
  if (offset) *offset = it->second.first;
  if (bytes) *bytes = it->second.second;
  return DG_OK;
}

}  // extern "C"
