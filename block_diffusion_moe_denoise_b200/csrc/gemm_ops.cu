// The dense contractions of the denoising pass on the tcgen05 GEMM engine,
// each with its epilogue fused:
//   qkv     RMSNorm'd tokens x W_qkv^T, rotate-half RoPE on q/k, q -> [Hq][T][D],
//           k/v -> KV cache slots of the canvas (or prefill segment)
//   wpart   split-K weight-row GEMM to fp32 partials (output projection and
//           shared-expert down projection; reduced by the residual + norm kernel)
//   egu     routed experts, gate|up for 64 hidden units per tile, SwiGLU in the
//           epilogue (weights as the 128-row operand, the expert's tokens as N)
//   ed      routed experts, down projection scaled by the pair's routing weight
//   sgu     shared expert gate|up + SwiGLU (tokens as the 128-row operand)
//   lm      tied LM head with per-row online max / argmax / sum e^(z-m) /
//           sum e^(z-m)(z-m) so the logits are never written
// Structure of a decoder layer and the MoE: DiffusionGemma pages ("26B MoE
// Architecture, but Only 3.8B Activated"; "The speed numbers and the hardware
// they require": 128 experts, 8 active plus one shared expert).
#include "dg_internal.h"
#include "umma_gemm.cuh"

namespace dg {

DG_DEVINL void store_bf16x16(__nv_bfloat16* dst, const float* v) {
  uint4 a, b;
  a.x = pack_bf16x2(v[0], v[1]);
  a.y = pack_bf16x2(v[2], v[3]);
  a.z = pack_bf16x2(v[4], v[5]);
  a.w = pack_bf16x2(v[6], v[7]);
  b.x = pack_bf16x2(v[8], v[9]);
  b.y = pack_bf16x2(v[10], v[11]);
  b.z = pack_bf16x2(v[12], v[13]);
  b.w = pack_bf16x2(v[14], v[15]);
  reinterpret_cast<uint4*>(dst)[0] = a;
  reinterpret_cast<uint4*>(dst)[1] = b;
}

// ---------------------------------------------------------------------------
// QKV projection + RoPE + KV-cache write.  Tile (token tile a, 128-column tile
// b).  The 128 W_qkv rows of a q/k tile are two 64-row boxes chosen so every
// rotate-half pair (i, i + D/2) lands in columns (c, c + 64) of the same
// accumulator row (head_dim 128/256), or inside one 64-column head at distance
// 32 (head_dim 64): the rotation stays in one thread.  cos/sin come from the
// per-pass table the embedding kernel writes.
// ---------------------------------------------------------------------------
struct P_QKV : ProblemBase {
  static constexpr int BN = 128, STAGES = 3, KB = 2, B_STAGE = BN * 128, TMEM_COLS = 256;
  struct Params {
    CUtensorMap tmA;  // normed tokens [Tcap, d]
    CUtensorMap tmB;  // w_qkv [(Hq+2Hkv)*D, d], 64-row boxes
    int T, nk, MT, NT, D, Hq, Hkv, q_T, kv_cap;
    long long kv_req_stride;
    const int* tok_pos;
    const int* tok_req;
    const float2* rope;  // [T][D/2] (cos, sin)
    __nv_bfloat16* q;
    __nv_bfloat16* kv;  // this layer's K block [Hkv][cap][D] of request 0; V^T [Hkv][D][cap] follows
    int* err;
  };
  // region (0 q, 1 k, 2 v), index of the tile inside its region, and the first
  // W_qkv row of each 64-row box
  DG_DEVINL static void rows_of(const Params& p, int b, int& kind, int& tb, int& r0, int& r1) {
    const int D = p.D;
    const int nq = p.Hq * D / 128, nkv = p.Hkv * D / 128;
    int base;
    if (b < nq) {
      kind = 0;
      tb = b;
      base = 0;
    } else if (b < nq + nkv) {
      kind = 1;
      tb = b - nq;
      base = p.Hq * D;
    } else {
      kind = 2;
      tb = b - nq - nkv;
      base = (p.Hq + p.Hkv) * D;
    }
    if (kind != 2 && D == 256) {
      r0 = base + (tb >> 1) * 256 + (tb & 1) * 64;
      r1 = r0 + 128;
    } else {
      r0 = base + tb * 128;
      r1 = r0 + 64;
    }
  }
  DG_DEVINL static void prefetch(const Params& p) {
    tma_prefetch_desc(&p.tmA);
    tma_prefetch_desc(&p.tmB);
  }
  DG_DEVINL static int num_tiles(const Params& p) { return p.MT * p.NT; }
  DG_DEVINL static Tile tile(const Params& p, int v) {
    Tile t;
    t.valid = 1;
    t.nk = p.nk;
    t.n_mma = BN;
    t.a = v % p.MT;  // token tile
    t.b = v / p.MT;  // 128-column tile of W_qkv
    return t;
  }
  DG_DEVINL static uint32_t tx_bytes(const Params&, const Tile&) { return kAStage + B_STAGE; }
  static constexpr bool PRELOAD = true;
  DG_DEVINL static void load_w(const Params& p, const Tile& t, int kb, uint32_t, uint32_t sb, uint64_t* bar) {
    int kind, tb, r0, r1;
    rows_of(p, t.b, kind, tb, r0, r1);
    tma_load_2d(sb, &p.tmB, kb * 64, r0, bar);
    tma_load_2d(sb + 64 * 128, &p.tmB, kb * 64, r1, bar);
  }
  DG_DEVINL static void load_x(const Params& p, const Tile& t, int kb, uint32_t sa, uint32_t, uint64_t* bar) {
    tma_load_2d(sa, &p.tmA, kb * 64, t.a * 128, bar);
  }
  DG_DEVINL static void load(const Params& p, const Tile& t, int kb, uint32_t sa, uint32_t sb, uint64_t* bar) {
    load_x(p, t, kb, sa, sb, bar);
    load_w(p, t, kb, sa, sb, bar);
  }
  DG_DEVINL static void epilogue_prefetch(const Params& p, const Tile& t, int row) {
    const int tok = t.a * 128 + row;
    if (tok >= p.T) return;
    prefetch_l1(p.tok_pos + tok);
    prefetch_l1(p.tok_req + tok);
    int kind, tb, r0, r1;
    rows_of(p, t.b, kind, tb, r0, r1);
    if (kind == 2) return;
    const int half = p.D >> 1;
    const int j = p.D == 256 ? (tb & 1) : 0;
    const char* cs = reinterpret_cast<const char*>(p.rope + (size_t)tok * half + (p.D == 64 ? 0 : j * 64));
    const int bytes = (p.D == 64 ? 32 : 64) * 8;
    for (int o = 0; o < bytes; o += 128) prefetch_l1(cs + o);
  }
  DG_DEVINL static void rotate16(const float* x1, const float* x2, const float2* cs, float* y1, float* y2) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float2 r = cs[i];
      y1[i] = x1[i] * r.x - x2[i] * r.y;
      y2[i] = x2[i] * r.x + x1[i] * r.y;
    }
  }
  DG_DEVINL static void epilogue(const Params& p, const Tile& t, uint32_t taddr, int, int, int row, uint8_t*) {
    const int tok = t.a * 128 + row;
    const bool ok = tok < p.T;
    const int pos = ok ? p.tok_pos[tok] : 0;
    const int req = ok ? p.tok_req[tok] : 0;
    const int D = p.D, half = D >> 1;
    int kind, tb, r0, r1;
    rows_of(p, t.b, kind, tb, r0, r1);
    // K: tiled cache layout (k_tile_offset); kpos = this position's row inside
    // its 64-position tile, block j of the dimensions 4096 elements further
    __nv_bfloat16* kbase = p.kv + (size_t)req * p.kv_req_stride + k_tile_offset(pos, 0, D);
    const size_t head_stride = (size_t)p.kv_cap * D;
    if (kind == 2) {
      // V is cached transposed, [Hkv][D][cap]: consecutive tokens of a warp
      // write consecutive positions of each dimension row
      __nv_bfloat16* vt = p.kv + (size_t)req * p.kv_req_stride + (size_t)p.Hkv * head_stride + pos;
      for (int c = 0; c < 128; c += 16) {
        float v[16];
        tmem_ld16(taddr + c, v);
        const int r = tb * 128 + c;  // = head * D + dim
        if (ok) {
#pragma unroll
          for (int i = 0; i < 16; ++i) vt[(size_t)(r + i) * p.kv_cap] = f2bf(v[i]);
        }
      }
      return;
    }
    const float2* cs_row = p.rope + (size_t)(ok ? tok : 0) * half;
    if (D == 64) {
      for (int hh = 0; hh < 2; ++hh) {
        const int head = tb * 2 + hh;
        // one 64-dim block: the tiled K row is contiguous like the q row
        __nv_bfloat16* dst = kind == 0 ? p.q + ((size_t)head * p.q_T + tok) * D : kbase + (size_t)head * head_stride;
        for (int c = 0; c < 32; c += 16) {
          float x1[16], x2[16], y1[16], y2[16];
          tmem_ld16(taddr + hh * 64 + c, x1);
          tmem_ld16(taddr + hh * 64 + 32 + c, x2);
          if (ok) {
            float2 cs[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) cs[i] = cs_row[c + i];
            rotate16(x1, x2, cs, y1, y2);
            store_bf16x16(dst + c, y1);
            store_bf16x16(dst + 32 + c, y2);
          }
        }
      }
      return;
    }
    const int j = D == 256 ? (tb & 1) : 0;
    const int head = D == 256 ? (tb >> 1) : tb;
    // dims j*64.. and half + j*64..: q rows are plain; K rows are 64-dim blocks
    // 4096 elements apart (tiled layout)
    __nv_bfloat16* dst = kind == 0 ? p.q + ((size_t)head * p.q_T + tok) * D : kbase + (size_t)head * head_stride;
    const size_t o1 = kind == 0 ? (size_t)j * 64 : (size_t)j * 4096;
    const size_t o2 = kind == 0 ? (size_t)(half + j * 64) : (size_t)((half >> 6) + j) * 4096;
    for (int c = 0; c < 64; c += 16) {
      float x1[16], x2[16], y1[16], y2[16];
      tmem_ld16(taddr + c, x1);
      tmem_ld16(taddr + 64 + c, x2);
      if (ok) {
        float2 cs[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) cs[i] = cs_row[j * 64 + c + i];
        rotate16(x1, x2, cs, y1, y2);
        store_bf16x16(dst + o1 + c, y1);
        store_bf16x16(dst + o2 + c, y2);
      }
    }
  }
};

// The QKV projection as M = 256 tiles over CTA pairs: a pair covers two token
// tiles (256 tokens) against one 128-column tile of W_qkv; each CTA loads its
// own 128 tokens and one of the column tile's two 64-row weight boxes, so the
// token rows stream through each SM once per 128 columns instead of the
// weight rows and token rows both (a quarter less traffic per SM).  The
// epilogue (each CTA: its 128 tokens x 128 columns) is P_QKV's.
struct P_QKV2 : P_QKV {
  static constexpr bool PAIR = true;
  // a CTA's B slot holds its 64 rows only: 48 KB per stage, four stages
  static constexpr int STAGES = 4, B_STAGE = BN * 128 / 2;
  DG_DEVINL static int num_tiles(const Params& p) { return ((p.MT + 1) / 2) * p.NT; }
  DG_DEVINL static Tile tile(const Params& p, int v) {
    Tile t;
    t.valid = 1;
    t.nk = p.nk;
    t.n_mma = BN;
    const int mt2 = (p.MT + 1) / 2;
    t.a = v % mt2;  // pair of token tiles
    t.b = v / mt2;  // 128-column tile of W_qkv
    return t;
  }
  DG_DEVINL static Tile local(const Params&, Tile t, int rank) {
    t.a = 2 * t.a + rank;  // this CTA's token tile
    t.half = rank;         // and weight box
    return t;
  }
  DG_DEVINL static uint32_t tx_bytes(const Params&, const Tile&) { return kAStage + B_STAGE; }
  DG_DEVINL static void load_w(const Params& p, const Tile& t, int kb, uint32_t, uint32_t sb, uint64_t* bar) {
    int kind, tb, r0, r1;
    rows_of(p, t.b, kind, tb, r0, r1);
    tma_load_2d_pair(sb, &p.tmB, kb * 64, t.half ? r1 : r0, bar);
  }
  DG_DEVINL static void load_x(const Params& p, const Tile& t, int kb, uint32_t sa, uint32_t, uint64_t* bar) {
    tma_load_2d_pair(sa, &p.tmA, kb * 64, t.a * 128, bar);
  }
  DG_DEVINL static void load(const Params& p, const Tile& t, int kb, uint32_t sa, uint32_t sb, uint64_t* bar) {
    load_x(p, t, kb, sa, sb, bar);
    load_w(p, t, kb, sa, sb, bar);
  }
};

// ---------------------------------------------------------------------------
// Split-K weight-row GEMM with fp32 partial output, shared by the output
// projection and the shared expert's down projection:
//   part[s][t][f] = sum_{c in K-slice s} X[t, c] W[f, c]
// Tile (128 output features a, 256 tokens b, K-slice s).  N = 256 keeps the
// tensor core fed (the weight slice read per MMA is amortised over all
// tokens); the K split gives enough CTAs.  The slices are summed, in slice
// order, into the residual stream by the next residual + norm kernel.
// ---------------------------------------------------------------------------
struct P_WPART : ProblemBase {
  static constexpr int BN = 256, STAGES = 4, B_STAGE = BN * 128, TMEM_COLS = 512;
  struct Params {
    CUtensorMap tmA;  // weights [d, K], 128-row boxes
    CUtensorMap tmB;  // activations [Tcap, K], 256-row boxes
    int T, nk, MT, NT, S, Tcap, d;
    float* part;  // [S][Tcap][d]
    int* err;
  };
  DG_DEVINL static void prefetch(const Params& p) {
    tma_prefetch_desc(&p.tmA);
    tma_prefetch_desc(&p.tmB);
  }
  DG_DEVINL static int num_tiles(const Params& p) { return p.MT * p.NT * p.S; }
  DG_DEVINL static Tile tile(const Params& p, int v) {
    Tile t;
    t.a = v % p.MT;              // feature tile
    const int rest = v / p.MT;
    t.b = rest % p.NT;           // token tile
    t.c = rest / p.NT;           // K slice
    const int per = (p.nk + p.S - 1) / p.S;
    t.d = t.c * per;             // first k-block
    t.nk = min(per, p.nk - t.d);
    t.valid = t.nk > 0;
    t.n_mma = round_up16(min(BN, p.T - t.b * BN));
    return t;
  }
  DG_DEVINL static uint32_t tx_bytes(const Params&, const Tile&) { return kAStage + B_STAGE; }
  static constexpr bool PRELOAD = true;
  DG_DEVINL static void load_w(const Params& p, const Tile& t, int kb, uint32_t sa, uint32_t, uint64_t* bar) {
    tma_load_2d(sa, &p.tmA, (t.d + kb) * 64, t.a * 128, bar);
  }
  DG_DEVINL static void load_x(const Params& p, const Tile& t, int kb, uint32_t, uint32_t sb, uint64_t* bar) {
    tma_load_2d(sb, &p.tmB, (t.d + kb) * 64, t.b * BN, bar);
  }
  DG_DEVINL static void load(const Params& p, const Tile& t, int kb, uint32_t sa, uint32_t sb, uint64_t* bar) {
    load_w(p, t, kb, sa, sb, bar);
    load_x(p, t, kb, sa, sb, bar);
  }
  DG_DEVINL static void epilogue(const Params& p, const Tile& t, uint32_t taddr, int, int, int row, uint8_t*) {
    const int f = t.a * 128 + row;
    float* dst = p.part + (size_t)t.c * p.Tcap * p.d + f;
    for (int c0 = 0; c0 < t.n_mma; c0 += 16) {
      float v[16];
      tmem_ld16(taddr + c0, v);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int tok = t.b * BN + c0 + j;
        if (tok < p.T) dst[(size_t)tok * p.d] = v[j];
      }
    }
  }
};

// P_WPART as M = 256 tiles over CTA pairs: a pair covers two 128-feature tiles
// against one 256-token tile (one K slice); each CTA loads its own 128 weight
// rows and half of the tokens (128 rows), a third less traffic per SM than a
// single-CTA tile.  Each CTA's accumulator is its 128 features x all 256
// tokens, so the epilogue is P_WPART's.  Needs an even number of feature tiles.
struct P_WPART2 : P_WPART {
  static constexpr bool PAIR = true;
  static constexpr int STAGES = 6, B_STAGE = BN * 128 / 2;  // 32 KB per stage and CTA
  DG_DEVINL static int num_tiles(const Params& p) { return (p.MT / 2) * p.NT * p.S; }
  DG_DEVINL static Tile tile(const Params& p, int v) {
    Tile t;
    const int mt2 = p.MT / 2;
    t.a = v % mt2;  // pair of feature tiles
    const int rest = v / mt2;
    t.b = rest % p.NT;  // token tile
    t.c = rest / p.NT;  // K slice
    const int per = (p.nk + p.S - 1) / p.S;
    t.d = t.c * per;
    t.nk = min(per, p.nk - t.d);
    t.valid = t.nk > 0;
    t.n_mma = BN;  // the full token tile; columns past T are not stored
    return t;
  }
  DG_DEVINL static Tile local(const Params&, Tile t, int rank) {
    t.a = 2 * t.a + rank;  // this CTA's feature tile
    t.half = rank;         // and half of the token tile
    return t;
  }
  DG_DEVINL static uint32_t tx_bytes(const Params&, const Tile&) { return kAStage + B_STAGE; }
  DG_DEVINL static void load_w(const Params& p, const Tile& t, int kb, uint32_t sa, uint32_t, uint64_t* bar) {
    tma_load_2d_pair(sa, &p.tmA, (t.d + kb) * 64, t.a * 128, bar);
  }
  DG_DEVINL static void load_x(const Params& p, const Tile& t, int kb, uint32_t, uint32_t sb, uint64_t* bar) {
    tma_load_2d_pair(sb, &p.tmB, (t.d + kb) * 64, t.b * BN + t.half * (BN / 2), bar);  // 128-row boxes
  }
  DG_DEVINL static void load(const Params& p, const Tile& t, int kb, uint32_t sa, uint32_t sb, uint64_t* bar) {
    load_w(p, t, kb, sa, sb, bar);
    load_x(p, t, kb, sa, sb, bar);
  }
};

// ---------------------------------------------------------------------------
// Routed experts, gate|up + SwiGLU (the first tile kind of P_EXP below).
// Tile (e, j, nt): hidden units j*64..+63 of expert e for its tokens
// nt*128..+127 (rows of the expert-grouped buffer; the token rows are loaded
// in 64-row boxes, one or two as the tile needs).  Tiles of 128 tokens read an
// expert's weights once per 128 of its tokens.
// A rows 0..63 = W_gate rows, 64..127 = W_up rows of the same hidden units.
// ---------------------------------------------------------------------------
struct P_EGU : ProblemBase {
  static constexpr int BN = kExpertTileRows, STAGES = 3, KB = 2, B_STAGE = BN * 128, TMEM_COLS = 2 * BN;
  static constexpr int kXchBytes = 64 * 17 * 4;
  static constexpr int EP_SMEM = kXchBytes + BN * 64 * 2;
  static constexpr bool DYNAMIC = true;
  struct Params {
    CUtensorMap tmG;  // w_gate as [E*fe, d]
    CUtensorMap tmU;  // w_up   as [E*fe, d]
    CUtensorMap tmX;  // expert-grouped tokens [rows_cap, d], kExpertBoxRows-row boxes
    int nk, fe;
    const int4* tiles;
    const int* n_tiles;
    const int* counts;
    const int* offsets;
    __nv_bfloat16* hp;  // [rows_cap, fe]
    int* sched;  // tile counter (zeroed by the grouping kernel)
    int* err;
  };
  DG_DEVINL static void prefetch(const Params& p) {
    tma_prefetch_desc(&p.tmG);
    tma_prefetch_desc(&p.tmU);
    tma_prefetch_desc(&p.tmX);
  }
  DG_DEVINL static int num_tiles(const Params& p) { return *p.n_tiles; }
  DG_DEVINL static Tile tile(const Params& p, int v) {
    const int4 tt = p.tiles[v];
    Tile t;
    t.a = tt.x;  // expert
    t.b = tt.y;  // hidden-unit block
    const int nt = tt.z;
    const int n_valid = min(BN, p.counts[t.a] - nt * BN);
    t.valid = n_valid > 0;
    t.c = n_valid;
    t.d = p.offsets[t.a] + nt * BN;  // first grouped row
    t.nk = p.nk;
    t.n_mma = round_up16(n_valid);
    return t;
  }
  // the token rows in kExpertBoxRows-row boxes, as many as the tile needs
  DG_DEVINL static uint32_t tx_bytes(const Params&, const Tile& t) {
    return kAStage + (uint32_t)((t.n_mma + kExpertBoxRows - 1) / kExpertBoxRows) * kExpertBoxRows * 128;
  }
  DG_DEVINL static void load(const Params& p, const Tile& t, int kb, uint32_t sa, uint32_t sb, uint64_t* bar) {
    const int r = t.a * p.fe + t.b * 64;
    tma_load_2d(sa, &p.tmG, kb * 64, r, bar);
    tma_load_2d(sa + 64 * 128, &p.tmU, kb * 64, r, bar);
    for (int i = 0; i < t.n_mma; i += kExpertBoxRows) tma_load_2d(sb + i * 128, &p.tmX, kb * 64, t.d + i, bar);
  }
  // The SwiGLU rows are transposed through shared memory: the 64 gate-row
  // threads each hold one hidden unit of 16 tokens per chunk; staged as
  // [token][64 units] they leave as full 128-byte row segments of hp (one
  // coalesced store per warp and token) instead of 2-byte stores per thread.
  DG_DEVINL static void epilogue(const Params& p, const Tile& t, uint32_t taddr, int, int lane, int row, uint8_t* ep) {
    float* xch = reinterpret_cast<float*>(ep);
    __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(ep + kXchBytes);  // [BN tokens][64 units]
    for (int c0 = 0; c0 < t.n_mma; c0 += 16) {
      float v[16];
      tmem_ld16(taddr + c0, v);
      if (row >= 64) {
#pragma unroll
        for (int i = 0; i < 16; ++i) xch[(row - 64) * 17 + i] = v[i];
      }
      named_bar_sync(1, 128);
      if (row < 64) {
#pragma unroll
        for (int i = 0; i < 16; ++i) stage[(c0 + i) * 64 + row] = f2bf(silu_f(v[i]) * xch[row * 17 + i]);
      }
      named_bar_sync(1, 128);
    }
    // row segments: token c, units 2*lane, 2*lane+1 (one warp per token)
    const int w = row >> 5;
    const uint32_t* st32 = reinterpret_cast<const uint32_t*>(stage);
    for (int c = w; c < t.c; c += 4) {
      uint32_t* dst = reinterpret_cast<uint32_t*>(p.hp + (size_t)(t.d + c) * p.fe + t.b * 64);
      dst[lane] = st32[c * 32 + lane];
    }
    named_bar_sync(1, 128);  // the staging tile is free for the next tile
  }
};

// ---------------------------------------------------------------------------
// Routed experts, down projection (the second tile kind of P_EXP below).
// Tile (e, m, nt): output features m*128..+127
// of expert e for its grouped rows nt*128..+127; each row scaled by its gate weight.
// ---------------------------------------------------------------------------
struct P_ED : ProblemBase {
  static constexpr int BN = kExpertTileRows, STAGES = 3, KB = 2, B_STAGE = BN * 128, TMEM_COLS = 2 * BN;
  static constexpr bool DYNAMIC = true;
  struct Params {
    CUtensorMap tmW;  // w_down as [E*d, fe]
    CUtensorMap tmH;  // hidden [rows_cap, fe], kExpertBoxRows-row boxes
    int nk, d;
    const int4* tiles;
    const int* n_tiles;
    const int* counts;
    const int* offsets;
    const float* row_weight;
    bf16* yp;   // [rows_cap, d], gate-weighted expert outputs
    int* sched;  // tile counter (zeroed by the grouping kernel)
    int* err;
  };
  DG_DEVINL static void prefetch(const Params& p) {
    tma_prefetch_desc(&p.tmW);
    tma_prefetch_desc(&p.tmH);
  }
  DG_DEVINL static int num_tiles(const Params& p) { return *p.n_tiles; }
  DG_DEVINL static Tile tile(const Params& p, int v) {
    const int4 tt = p.tiles[v];
    Tile t;
    t.a = tt.x;  // expert
    t.b = tt.y;  // 128-feature block
    const int nt = tt.z;
    const int n_valid = min(BN, p.counts[t.a] - nt * BN);
    t.valid = n_valid > 0;
    t.c = n_valid;
    t.d = p.offsets[t.a] + nt * BN;
    t.nk = p.nk;
    t.n_mma = round_up16(n_valid);
    return t;
  }
  DG_DEVINL static uint32_t tx_bytes(const Params&, const Tile& t) {
    return kAStage + (uint32_t)((t.n_mma + kExpertBoxRows - 1) / kExpertBoxRows) * kExpertBoxRows * 128;
  }
  DG_DEVINL static void load(const Params& p, const Tile& t, int kb, uint32_t sa, uint32_t sb, uint64_t* bar) {
    tma_load_2d(sa, &p.tmW, kb * 64, t.a * p.d + t.b * 128, bar);
    for (int i = 0; i < t.n_mma; i += kExpertBoxRows) tma_load_2d(sb + i * 128, &p.tmH, kb * 64, t.d + i, bar);
  }
  // The accumulator (thread = output feature, columns = tokens) is transposed
  // through shared memory 16 tokens at a time: staged fp32 as [token][128
  // features], each warp then scales whole token rows by their gate weight and
  // stores them as 256-byte row segments of yp (8 bytes per lane), instead of
  // 2-byte stores per thread and token.
  static constexpr int EP_SMEM = 16 * 128 * 4;
  DG_DEVINL static void epilogue(const Params& p, const Tile& t, uint32_t taddr, int q, int lane, int row,
                                 uint8_t* ep) {
    float* stg = reinterpret_cast<float*>(ep);  // [16 tokens][128 features]
    for (int c0 = 0; c0 < t.n_mma; c0 += 16) {
      float w[4];  // gate weights of the token rows this warp stores: c0 + q + 4 j
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = c0 + q + 4 * j;
        w[j] = c < t.c ? __ldcg(p.row_weight + t.d + c) : 0.f;
      }
      float v[16];
      tmem_ld16(taddr + c0, v);
#pragma unroll
      for (int i = 0; i < 16; ++i) stg[i * 128 + row] = v[i];
      named_bar_sync(1, 128);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = c0 + q + 4 * j;
        if (c < t.c) {
          const float4 a = *reinterpret_cast<const float4*>(stg + (q + 4 * j) * 128 + 4 * lane);
          uint2 o;
          o.x = pack_bf16x2(w[j] * a.x, w[j] * a.y);
          o.y = pack_bf16x2(w[j] * a.z, w[j] * a.w);
          *reinterpret_cast<uint2*>(p.yp + (size_t)(t.d + c) * p.d + t.b * 128 + 4 * lane) = o;
        }
      }
      named_bar_sync(1, 128);  // staging free for the next 16 tokens
    }
  }
};

// ---------------------------------------------------------------------------
// Routed experts, gate|up + SwiGLU and down projection, and the shared
// expert's down projection, in one persistent launch.  The tile queue holds
// the shared-down tiles (128 output features x 128 tokens over the whole
// shared hidden width, written straight to the fp32 partial the residual norm
// adds; they depend on nothing in the launch), then every gate|up tile (in
// expert order), then every down tile (in expert order).  (The shared-down
// tiles queued between the gate|up and the down tiles, or among the down
// tiles, measured slower on B200.)  A down tile reads the SwiGLU rows of one
// token tile of its expert, which that token tile's FJ gate|up tiles write;
// each of their epilogues adds one to ready[tt] (tt: the token tile's index
// over all experts) once its rows are stored, and the scheduler waits for FJ
// before handing the down tile on.  All gate|up tiles come before the down
// tiles in the queue, so no wait depends on a tile not yet taken (see the
// engine header).
// The down tiles of the first experts start while the last gate|up tiles
// still run: no gate|up tail and down ramp between two launches.
// ---------------------------------------------------------------------------
struct P_EXP : ProblemBase {
  static constexpr int BN = kExpertTileRows, STAGES = 3, KB = 2, B_STAGE = BN * 128, TMEM_COLS = 2 * BN;
  static constexpr int EP_SMEM = P_EGU::EP_SMEM > P_ED::EP_SMEM ? P_EGU::EP_SMEM : P_ED::EP_SMEM;
  static constexpr bool DYNAMIC = true;
  static constexpr bool ACQUIRE = true;
  static_assert(P_EGU::BN == BN && P_ED::BN == BN && P_EGU::KB == KB && P_ED::KB == KB &&
                    P_EGU::B_STAGE == B_STAGE && P_ED::B_STAGE == B_STAGE,
                "gate|up and down tiles share the ring layout");
  struct Params {
    P_EGU::Params gu;
    P_ED::Params dn;
    CUtensorMap tmSW;  // shared-expert down weights [d, fs], 128-row boxes
    CUtensorMap tmHS;  // shared SwiGLU rows [Tcap, fs], 64-row boxes
    int n_sd;          // shared-down tiles: (d / 128) x ceil(T / BN), 0 = none
    int sd_nk, sd_fb, T, d;
    float* part;       // [Tcap][d] shared-expert output (fp32)
    int* ready;  // [token tiles] finished gate|up tiles per token tile (zeroed by the grouping kernel)
    int FJ;      // gate|up tiles per token tile (fe / 64)
    int* sched;  // tile counter (zeroed by the grouping kernel)
    int* err;
  };
  DG_DEVINL static void prefetch(const Params& p) {
    P_EGU::prefetch(p.gu);
    P_ED::prefetch(p.dn);
    if (p.n_sd > 0) {
      tma_prefetch_desc(&p.tmSW);
      tma_prefetch_desc(&p.tmHS);
    }
  }
  DG_DEVINL static int num_tiles(const Params& p) { return *p.gu.n_tiles + p.n_sd + *p.dn.n_tiles; }
  // kinds: e = 0 gate|up, 1 down, 2 shared down
  DG_DEVINL static Tile tile(const Params& p, int v) {
    const int ng = *p.gu.n_tiles;
    Tile t;
    if (v >= p.n_sd && v < p.n_sd + ng) {
      t = P_EGU::tile(p.gu, v - p.n_sd);
      t.e = 0;
      t.f = p.gu.tiles[v - p.n_sd].w;
    } else if (v < p.n_sd) {
      const int u = v;
      t.a = u % p.sd_fb;  // 128-feature block
      t.b = u / p.sd_fb;  // BN-token tile
      t.c = min(BN, p.T - t.b * BN);
      t.valid = t.c > 0;
      t.d = 0;
      t.e = 2;
      t.f = 0;
      t.nk = p.sd_nk;
      t.n_mma = round_up16(t.c);
    } else {
      t = P_ED::tile(p.dn, v - ng - p.n_sd);
      t.e = 1;
      t.f = p.dn.tiles[v - ng - p.n_sd].w;
    }
    return t;
  }
  DG_DEVINL static uint32_t tx_bytes(const Params& p, const Tile& t) {
    if (t.e == 0) return P_EGU::tx_bytes(p.gu, t);
    if (t.e == 1) return P_ED::tx_bytes(p.dn, t);
    return kAStage + (uint32_t)((t.c + 63) / 64) * 64 * 128;  // shared down: 64-row boxes
  }
  DG_DEVINL static bool acquire(const Params& p, const Tile& t, volatile int* abort, int* err) {
    return t.e != 1 || counter_wait_bounded(p.ready + t.f, p.FJ, abort, err);
  }
  DG_DEVINL static void load(const Params& p, const Tile& t, int kb, uint32_t sa, uint32_t sb, uint64_t* bar) {
    if (t.e == 0) {
      P_EGU::load(p.gu, t, kb, sa, sb, bar);
    } else if (t.e == 1) {
      P_ED::load(p.dn, t, kb, sa, sb, bar);
    } else {
      tma_load_2d(sa, &p.tmSW, kb * 64, t.a * 128, bar);
      for (int i = 0; i < t.c; i += 64) tma_load_2d(sb + i * 128, &p.tmHS, kb * 64, t.b * BN + i, bar);
    }
  }
  DG_DEVINL static void epilogue(const Params& p, const Tile& t, uint32_t taddr, int q, int lane, int row,
                                 uint8_t* ep) {
    if (t.e == 1) {
      P_ED::epilogue(p.dn, t, taddr, q, lane, row, ep);
      return;
    }
    if (t.e == 2) {  // thread = output feature, columns = tokens
      float* dst = p.part + t.a * 128 + row;
      for (int c0 = 0; c0 < t.n_mma; c0 += 16) {
        float v[16];
        tmem_ld16(taddr + c0, v);
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (c0 + j < t.c) dst[(size_t)(t.b * BN + c0 + j) * p.d] = v[j];
      }
      return;
    }
    P_EGU::epilogue(p.gu, t, taddr, q, lane, row, ep);
    counter_release_fence();   // this thread's SwiGLU rows are visible to the TMA loads of the down tiles
    named_bar_sync(3, 128);    // ... every thread's
    if (row == 0) atomicAdd(p.ready + t.f, 1);
  }
};

// ---------------------------------------------------------------------------
// FP8 (E4M3) routed experts: the same tiles as P_EGU / P_ED with E4M3 weight
// codes (one fp32 scale per weight row) and E4M3 token rows (one fp32 scale per
// grouped row); a k-block is 128 elements (one 128-byte row), so a tile has
// half the k-blocks of its bf16 form.  The accumulator holds
// sum decode(q_w) decode(q_x); the epilogue applies both scales.
// ---------------------------------------------------------------------------
struct P_EGU8 : ProblemBase {
  static constexpr bool F8 = true;
  static constexpr int BN = kExpertRows, STAGES = 4, KB = 2, B_STAGE = BN * 128, TMEM_COLS = 128;
  static constexpr int EP_SMEM = 64 * 17 * 4;
  static constexpr bool DYNAMIC = true;
  struct Params {
    CUtensorMap tmG;  // w_gate codes as [E*fe, d] bytes
    CUtensorMap tmU;  // w_up codes as [E*fe, d] bytes
    CUtensorMap tmX;  // grouped token codes [rows_cap, d] bytes, 64-row boxes
    int nk, fe;
    const int4* tiles;
    const int* n_tiles;
    const int* counts;
    const int* offsets;
    const float* sg;    // [E*fe] gate row scales
    const float* su;    // [E*fe] up row scales
    const float* sx;    // [rows] token row scales
    __nv_bfloat16* hp;  // [rows_cap, fe]
    int* sched;  // tile counter (zeroed by the grouping kernel)
    int* err;
  };
  DG_DEVINL static void prefetch(const Params& p) {
    tma_prefetch_desc(&p.tmG);
    tma_prefetch_desc(&p.tmU);
    tma_prefetch_desc(&p.tmX);
  }
  DG_DEVINL static int num_tiles(const Params& p) { return *p.n_tiles; }
  DG_DEVINL static Tile tile(const Params& p, int v) {
    const int4 tt = p.tiles[v];
    Tile t;
    t.a = tt.x;
    t.b = tt.y;
    const int nt = tt.z;
    const int n_valid = min(BN, p.counts[t.a] - nt * BN);
    t.valid = n_valid > 0;
    t.c = n_valid;
    t.d = p.offsets[t.a] + nt * BN;
    t.nk = p.nk;
    t.n_mma = round_up16(n_valid);
    return t;
  }
  DG_DEVINL static uint32_t tx_bytes(const Params&, const Tile&) { return kAStage + B_STAGE; }
  DG_DEVINL static void load(const Params& p, const Tile& t, int kb, uint32_t sa, uint32_t sb, uint64_t* bar) {
    const int r = t.a * p.fe + t.b * 64;
    tma_load_2d(sa, &p.tmG, kb * 128, r, bar);
    tma_load_2d(sa + 64 * 128, &p.tmU, kb * 128, r, bar);
    tma_load_2d(sb, &p.tmX, kb * 128, t.d, bar);
  }
  DG_DEVINL static void epilogue(const Params& p, const Tile& t, uint32_t taddr, int, int, int row, uint8_t* ep) {
    float* xch = reinterpret_cast<float*>(ep);
    const int r = t.a * p.fe + t.b * 64 + (row & 63);
    const float sw = row < 64 ? p.sg[r] : p.su[r];
    for (int c0 = 0; c0 < t.n_mma; c0 += 16) {
      float v[16];
      tmem_ld16(taddr + c0, v);
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = c0 + i < t.c ? v[i] * sw * p.sx[t.d + c0 + i] : 0.f;
      if (row >= 64) {
#pragma unroll
        for (int i = 0; i < 16; ++i) xch[(row - 64) * 17 + i] = v[i];
      }
      named_bar_sync(1, 128);
      if (row < 64) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int c = c0 + i;
          if (c < t.c) {
            const float h = silu_f(v[i]) * xch[row * 17 + i];
            p.hp[(size_t)(t.d + c) * p.fe + t.b * 64 + row] = f2bf(h);
          }
        }
      }
      named_bar_sync(1, 128);
    }
  }
};

struct P_ED8 : ProblemBase {
  static constexpr bool F8 = true;
  static constexpr int BN = kExpertRows, STAGES = 4, KB = 2, B_STAGE = BN * 128, TMEM_COLS = 128;
  static constexpr bool DYNAMIC = true;
  struct Params {
    CUtensorMap tmW;  // w_down codes as [E*d, fe] bytes
    CUtensorMap tmH;  // hidden codes [rows_cap, fe] bytes, 64-row boxes
    int nk, d;
    const int4* tiles;
    const int* n_tiles;
    const int* counts;
    const int* offsets;
    const float* sw;   // [E*d] down row scales
    const float* sh;   // [rows] hidden row scales
    const float* row_weight;
    bf16* yp;   // [rows_cap, d], gate-weighted expert outputs
    int* sched;  // tile counter (zeroed by the grouping kernel)
    int* err;
  };
  DG_DEVINL static void prefetch(const Params& p) {
    tma_prefetch_desc(&p.tmW);
    tma_prefetch_desc(&p.tmH);
  }
  DG_DEVINL static int num_tiles(const Params& p) { return *p.n_tiles; }
  DG_DEVINL static Tile tile(const Params& p, int v) {
    const int4 tt = p.tiles[v];
    Tile t;
    t.a = tt.x;
    t.b = tt.y;
    const int nt = tt.z;
    const int n_valid = min(BN, p.counts[t.a] - nt * BN);
    t.valid = n_valid > 0;
    t.c = n_valid;
    t.d = p.offsets[t.a] + nt * BN;
    t.nk = p.nk;
    t.n_mma = round_up16(n_valid);
    return t;
  }
  DG_DEVINL static uint32_t tx_bytes(const Params&, const Tile&) { return kAStage + B_STAGE; }
  DG_DEVINL static void load(const Params& p, const Tile& t, int kb, uint32_t sa, uint32_t sb, uint64_t* bar) {
    tma_load_2d(sa, &p.tmW, kb * 128, t.a * p.d + t.b * 128, bar);
    tma_load_2d(sb, &p.tmH, kb * 128, t.d, bar);
  }
  // Transposed through shared memory as in P_ED: thread = output feature
  // stages v * (its weight row's scale), each warp then applies a token row's
  // scale and gate weight and stores 256-byte row segments of yp.  The
  // products are those of w_r * ((v * s_w) * s_h), in that order.
  static constexpr int EP_SMEM = 16 * 128 * 4;
  DG_DEVINL static void epilogue(const Params& p, const Tile& t, uint32_t taddr, int q, int lane, int row,
                                 uint8_t* ep) {
    float* stg = reinterpret_cast<float*>(ep);  // [16 tokens][128 features]
    const float sw = p.sw[(size_t)t.a * p.d + t.b * 128 + row];
    for (int c0 = 0; c0 < t.n_mma; c0 += 16) {
      float w[4], sh[4];  // gate weights and row scales of the token rows this warp stores: c0 + q + 4 j
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = c0 + q + 4 * j;
        w[j] = c < t.c ? __ldcg(p.row_weight + t.d + c) : 0.f;
        sh[j] = c < t.c ? __ldcg(p.sh + t.d + c) : 0.f;
      }
      float v[16];
      tmem_ld16(taddr + c0, v);
#pragma unroll
      for (int i = 0; i < 16; ++i) stg[i * 128 + row] = v[i] * sw;
      named_bar_sync(1, 128);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = c0 + q + 4 * j;
        if (c < t.c) {
          const float4 a = *reinterpret_cast<const float4*>(stg + (q + 4 * j) * 128 + 4 * lane);
          uint2 o;
          o.x = pack_bf16x2(w[j] * (a.x * sh[j]), w[j] * (a.y * sh[j]));
          o.y = pack_bf16x2(w[j] * (a.z * sh[j]), w[j] * (a.w * sh[j]));
          *reinterpret_cast<uint2*>(p.yp + (size_t)(t.d + c) * p.d + t.b * 128 + 4 * lane) = o;
        }
      }
      named_bar_sync(1, 128);  // staging free for the next 16 tokens
    }
  }
};

// ---------------------------------------------------------------------------
// Shared expert gate|up + SwiGLU, and the router, in one launch (both read the
// FFN-normed token rows).  Tokens are the 128-row operand.
//   router tile (mt):     N = E router rows; the epilogue thread owning a token
//                         row picks its top-k experts (descending logit, ties to
//                         the lower id), the softmax of the picked logits, and
//                         sets the token's bit in each picked expert's bitmask
//   shared tile (mt, j):  hidden units j*32..+31; B rows 0..31 = gate rows,
//                         32..63 = up rows (N = 64, so 2 x 33 tiles fill the GPU)
// Router tiles come first in the schedule: they have the longest main loop and
// the grouping kernel that follows waits on them.
// ---------------------------------------------------------------------------
struct P_SGU : ProblemBase {
  static constexpr int BN = 128, STAGES = 3, KB = 2, B_STAGE = BN * 128, TMEM_COLS = 256;
  static constexpr int kHid = 32;  // shared hidden units per tile
  struct Params {
    CUtensorMap tmX;  // normed tokens [Tcap, d]
    CUtensorMap tmG;  // ws_gate [fs, d], 32-row boxes
    CUtensorMap tmU;  // ws_up [fs, d], 32-row boxes
    CUtensorMap tmR;  // w_router [E, d], E-row boxes
    CUtensorMap tmXR;   // normed tokens in RR-row boxes (the router tiles' token rows)
    int T, nk, MT, FJ, fs, E, k, MW;
    int RR;             // tokens per router tile: 128, 64 or 32 (see router_tiles)
    __nv_bfloat16* hs;  // [Tcap, fs]
    float* logits;      // [Tcap, E], or nullptr: not written
    int* idx;           // [T, k]
    float* w;           // [T, k]
    unsigned* mask;     // [E][MW] token bitmasks (zero on entry)
    int* err;
  };
  static constexpr bool PRELOAD = true;
  DG_DEVINL static void prefetch(const Params& p) {
    tma_prefetch_desc(&p.tmX);
    tma_prefetch_desc(&p.tmG);
    tma_prefetch_desc(&p.tmU);
    if (p.E > 0) tma_prefetch_desc(&p.tmR);
  }
  // E == 0: a plain gated MLP (no router tile), as used for self-conditioning.
  // A router tile takes RR tokens (one RR-row box at the start of the A stage;
  // MMA rows RR..127 are ignored): with RR < 128 it streams RR + E rows per
  // k-block, fewer than a shared tile's 128 + 2 * kHid, so the router tiles,
  // whose top-k epilogue is longer, no longer outlast the shared tiles.
  DG_DEVINL static int router_tiles(const Params& p) { return p.E > 0 ? (p.T + p.RR - 1) / p.RR : 0; }
  DG_DEVINL static int num_tiles(const Params& p) { return router_tiles(p) + p.MT * p.FJ; }
  DG_DEVINL static Tile tile(const Params& p, int v) {
    Tile t;
    t.valid = 1;
    t.nk = p.nk;
    const int R = router_tiles(p);
    if (v < R) {
      t.a = v;
      t.b = -1;  // router tile
      t.n_mma = p.E;
    } else {
      t.a = (v - R) % p.MT;
      t.b = (v - R) / p.MT;
      t.n_mma = 2 * kHid;
    }
    return t;
  }
  DG_DEVINL static uint32_t tx_bytes(const Params& p, const Tile& t) {
    return (t.b < 0 ? (uint32_t)p.RR * 128 : kAStage) + (t.b < 0 ? p.E : 2 * kHid) * 128;
  }
  DG_DEVINL static void load_w(const Params& p, const Tile& t, int kb, uint32_t, uint32_t sb, uint64_t* bar) {
    if (t.b < 0) {
      tma_load_2d(sb, &p.tmR, kb * 64, 0, bar);
    } else {
      tma_load_2d(sb, &p.tmG, kb * 64, t.b * kHid, bar);
      tma_load_2d(sb + kHid * 128, &p.tmU, kb * 64, t.b * kHid, bar);
    }
  }
  DG_DEVINL static void load_x(const Params& p, const Tile& t, int kb, uint32_t sa, uint32_t, uint64_t* bar) {
    if (t.b < 0)
      tma_load_2d(sa, &p.tmXR, kb * 64, t.a * p.RR, bar);
    else
      tma_load_2d(sa, &p.tmX, kb * 64, t.a * 128, bar);
  }
  DG_DEVINL static void load(const Params& p, const Tile& t, int kb, uint32_t sa, uint32_t sb, uint64_t* bar) {
    load_x(p, t, kb, sa, sb, bar);
    load_w(p, t, kb, sa, sb, bar);
  }
  DG_DEVINL static void router_epilogue(const Params& p, int tok, bool row_valid, uint32_t taddr) {
    const bool ok = row_valid && tok < p.T;
    float tv[8];
    int ti[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      tv[r] = -INFINITY;
      ti[r] = 0x7fffffff;
    }
    for (int c0 = 0; c0 < p.E; c0 += 16) {
      float z[16];
      tmem_ld16(taddr + c0, z);
      if (!ok) continue;
      if (p.logits != nullptr) {  // kept for inspection only
        float4* lg = reinterpret_cast<float4*>(p.logits + (size_t)tok * p.E + c0);
#pragma unroll
        for (int i = 0; i < 16; i += 4) lg[i / 4] = make_float4(z[i], z[i + 1], z[i + 2], z[i + 3]);
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        // Experts arrive in ascending id order; strict comparisons keep the
        // earlier (lower) id ahead of an equal logit.  The list is sorted, so
        // the comparisons are monotone in r and every slot's new value follows
        // from the old list directly (no chain through the list).
        const float v = z[i];
        if (v > tv[7]) {
          bool gt[8];
#pragma unroll
          for (int r = 0; r < 8; ++r) gt[r] = v > tv[r];
#pragma unroll
          for (int r = 7; r > 0; --r) {
            tv[r] = gt[r] ? (gt[r - 1] ? tv[r - 1] : v) : tv[r];
            ti[r] = gt[r] ? (gt[r - 1] ? ti[r - 1] : c0 + i) : ti[r];
          }
          tv[0] = gt[0] ? v : tv[0];
          ti[0] = gt[0] ? c0 + i : ti[0];
        }
      }
    }
    if (!ok) return;
    float ex[8], sum = 0.f;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      ex[r] = r < p.k ? expf(tv[r] - tv[0]) : 0.f;
      sum += ex[r];
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      if (r < p.k) {
        // fewer than k picks only happen with NaN logits
        const bool valid = (unsigned)ti[r] < (unsigned)p.E;
        p.idx[(size_t)tok * p.k + r] = valid ? ti[r] : -1;
        p.w[(size_t)tok * p.k + r] = ex[r] / sum;
        if (valid)
          atomicOr(&p.mask[(size_t)ti[r] * p.MW + (tok >> 5)], 1u << (tok & 31));
        else
          atomicOr(p.err, DG_DEVERR_NAN);
      }
    }
  }
  DG_DEVINL static void epilogue(const Params& p, const Tile& t, uint32_t taddr, int, int, int row, uint8_t*) {
    if (t.b < 0) {
      router_epilogue(p, t.a * p.RR + row, row < p.RR, taddr);
      return;
    }
    const int tok = t.a * 128 + row;
    const bool ok = tok < p.T;
    for (int c0 = 0; c0 < kHid; c0 += 16) {
      float g[16], u[16];
      tmem_ld16(taddr + c0, g);
      tmem_ld16(taddr + kHid + c0, u);
      if (ok) {
        float h[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) h[i] = silu_f(g[i]) * u[i];
        store_bf16x16(p.hs + (size_t)tok * p.fs + t.b * kHid + c0, h);
      }
    }
  }
};

// ---------------------------------------------------------------------------
// LM head with fused online statistics.  Tile (mt, vt): tokens mt*128..+127,
// vocab rows vt*256..+255.  Each epilogue thread owns one token row and keeps,
// per token tile, the running (max m, argmax a, s = sum e^(z-m),
// t = sum e^(z-m)(z-m)) in shared memory across the CTA's tiles; the CTA's
// partial is written at the end and merged across CTAs by k_lm_combine.
//
// Candidate draw (draw != nullptr), the tile level of a two-level draw from
// softmax(z / temperature): for its row and the tile's 256 ids the thread sums
// w_v = exp(z_v/tau - max/tau), picks the first id whose running sum reaches
// u * sum (u from Philox, keyed by the row's slot), and stores the tile's
// log-mass max/tau + ln(sum) with that id.  k_lm_combine picks the tile.
//
// Self-conditioning (sc_part != nullptr): each thread also keeps its row's
// SC_K largest logits (ties to the lower id) over the CTA's tiles in shared
// memory; the grid is a multiple of MT so that a CTA only sees one token tile
// (mt = blockIdx.x % MT).  The CTA's lists go to sc_part and are merged by
// k_lm_combine.
// ---------------------------------------------------------------------------
struct LmStat {
  float m, s, t;
  int a;
};

// Sorted insertion into a descending top-8 list.  Values arrive in ascending
// id order, so the strict comparisons keep the lower id ahead of an equal one.
DG_DEVINL void top8_insert(float (&tv)[8], int (&ti)[8], float v, int id) {
  if (v > tv[7]) {
    bool gt[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) gt[r] = v > tv[r];
#pragma unroll
    for (int r = 7; r > 0; --r) {
      tv[r] = gt[r] ? (gt[r - 1] ? tv[r - 1] : v) : tv[r];
      ti[r] = gt[r] ? (gt[r - 1] ? ti[r - 1] : id) : ti[r];
    }
    tv[0] = gt[0] ? v : tv[0];
    ti[0] = gt[0] ? id : ti[0];
  }
}

struct P_LM : ProblemBase {
  static constexpr int BN = 256, STAGES = 4, B_STAGE = BN * 128, TMEM_COLS = 512;
  static constexpr int MT_MAX = 8;
  static constexpr int SC_K = 8;
  static constexpr int STAT_SMEM = MT_MAX * 128 * (int)sizeof(LmStat);
  static constexpr int EP_SMEM = STAT_SMEM + 128 * SC_K * 8;
  struct Params {
    CUtensorMap tmX;  // final-normed tokens [Tcap, d]
    CUtensorMap tmE;  // embedding [V, d]
    int T, nk, MT, NV;
    long long V;
    float4* part;    // [gridDim.x][MT*128]
    float* logits;   // optional [T, V]
    int* err;
    float inv_tau;
    float2* draw;    // optional [T][NV]
    DrawKeys keys;
    float2* sc_part; // optional [gridDim.x][T][SC_K] (logit, id as int bits)
    int row0;        // row of tmX holding this launch's row 0
  };
  DG_DEVINL static void prefetch(const Params& p) {
    tma_prefetch_desc(&p.tmX);
    tma_prefetch_desc(&p.tmE);
  }
  DG_DEVINL static int num_tiles(const Params& p) { return p.MT * p.NV; }
  DG_DEVINL static float draw_weight(float z, float inv_tau, float mt) {
    return exp2f((z * inv_tau - mt) * 1.4426950408889634f);
  }
  // Tile level of the candidate draw (all threads of the warp take part: the
  // TMEM loads are warp-collective); tm / ta = the tile's max logit and its column.
  DG_DEVINL static void draw_tile(const Params& p, const Tile& t, uint32_t taddr, int tok, bool ok, float tm,
                                  int ta) {
    const float it = p.inv_tau;
    const float mt = tm * it;
    float s = 0.f;
    for (int c0 = 0; c0 < 256; c0 += 32) {
      float z[32];
      tmem_ld16(taddr + c0, z);
      tmem_ld16(taddr + c0 + 16, z + 16);
#pragma unroll
      for (int i = 0; i < 32; ++i) s += draw_weight(z[i], it, mt);
    }
    float u = 0.5f;
    if (ok) {
      const int slot = tok / p.keys.canvas, pos = tok - slot * p.keys.canvas;
      const unsigned long long seed = p.keys.seed[slot];
      u = word_uniform(philox4x32_10((uint32_t)pos, (uint32_t)p.keys.step[slot], (uint32_t)p.keys.block[slot],
                                     (uint32_t)p.keys.req[slot] + 256u * (uint32_t)(t.b + 1), (uint32_t)seed,
                                     (uint32_t)(seed >> 32))
                           .x);
    }
    const float target = u * s;
    float cum = 0.f;
    int cand = -1;
    for (int c0 = 0; c0 < 256; c0 += 32) {
      float z[32];
      tmem_ld16(taddr + c0, z);
      tmem_ld16(taddr + c0 + 16, z + 16);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        cum += draw_weight(z[i], it, mt);
        if (cand < 0 && cum >= target) cand = c0 + i;
      }
    }
    if (cand < 0) cand = ta;  // rounding left the running sum short of the target
    if (ok) p.draw[(size_t)tok * p.NV + t.b] = make_float2(mt + logf(s), __int_as_float(t.b * 256 + cand));
  }
  DG_DEVINL static Tile tile(const Params& p, int v) {
    Tile t;
    t.valid = 1;
    t.nk = p.nk;
    t.n_mma = BN;
    t.a = v % p.MT;
    t.b = v / p.MT;
    return t;
  }
  DG_DEVINL static uint32_t tx_bytes(const Params&, const Tile&) { return kAStage + B_STAGE; }
  static constexpr bool PRELOAD = true;
  DG_DEVINL static void load_w(const Params& p, const Tile& t, int kb, uint32_t, uint32_t sb, uint64_t* bar) {
    tma_load_2d(sb, &p.tmE, kb * 64, t.b * 256, bar);
  }
  DG_DEVINL static void load_x(const Params& p, const Tile& t, int kb, uint32_t sa, uint32_t, uint64_t* bar) {
    tma_load_2d(sa, &p.tmX, kb * 64, p.row0 + t.a * 128, bar);
  }
  DG_DEVINL static void load(const Params& p, const Tile& t, int kb, uint32_t sa, uint32_t sb, uint64_t* bar) {
    load_x(p, t, kb, sa, sb, bar);
    load_w(p, t, kb, sa, sb, bar);
  }
  DG_DEVINL static float2* sc_list(uint8_t* ep, int row) {
    return reinterpret_cast<float2*>(ep + STAT_SMEM) + row * SC_K;
  }
  DG_DEVINL static void epilogue_init(const Params& p, int row, uint8_t* ep) {
    LmStat* st = reinterpret_cast<LmStat*>(ep);
    for (int mt = 0; mt < p.MT; ++mt) st[mt * 128 + row] = LmStat{-INFINITY, 0.f, 0.f, 0x7fffffff};
    if (p.sc_part != nullptr) {
      float2* l = sc_list(ep, row);
      for (int r = 0; r < SC_K; ++r) l[r] = make_float2(-INFINITY, __int_as_float(0x7fffffff));
    }
  }
  DG_DEVINL static void epilogue(const Params& p, const Tile& t, uint32_t taddr, int, int, int row, uint8_t* ep) {
    LmStat* st = reinterpret_cast<LmStat*>(ep);
    LmStat r = st[t.a * 128 + row];
    const int tok = t.a * 128 + row;
    const bool ok = tok < p.T;
    constexpr float kLog2e = 1.4426950408889634f;
    float tm = -INFINITY;  // this tile's max logit and its column
    int ta = 0;
    const bool sc = p.sc_part != nullptr;
    float tv[SC_K];
    int ti[SC_K];
    if (sc) {
      const float2* l = sc_list(ep, row);
#pragma unroll
      for (int r = 0; r < SC_K; ++r) {
        tv[r] = l[r].x;
        ti[r] = __float_as_int(l[r].y);
      }
    }
    for (int c0 = 0; c0 < 256; c0 += 32) {
      float z[32];
      tmem_ld16(taddr + c0, z);
      tmem_ld16(taddr + c0 + 16, z + 16);
      if (sc) {
#pragma unroll
        for (int i = 0; i < 32; ++i) top8_insert(tv, ti, z[i], t.b * 256 + c0 + i);
      }
      if (p.logits != nullptr && ok) {
        float* dst = p.logits + (size_t)tok * p.V + (size_t)t.b * 256 + c0;
#pragma unroll
        for (int i = 0; i < 32; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(z[i], z[i + 1], z[i + 2], z[i + 3]);
      }
      float cm = z[0];
      int ca = 0;
#pragma unroll
      for (int i = 1; i < 32; ++i)
        if (z[i] > cm) {
          cm = z[i];
          ca = i;
        }
      if (cm > r.m) {
        if (r.s > 0.f) {
          const float f = exp2f((r.m - cm) * kLog2e);
          r.t = f * (r.t + (r.m - cm) * r.s);
          r.s *= f;
        }
        r.m = cm;
        r.a = t.b * 256 + c0 + ca;
      }
      if (cm > tm) {
        tm = cm;
        ta = c0 + ca;
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float dz = z[i] - r.m;
        const float e = exp2f(dz * kLog2e);
        r.s += e;
        r.t = fmaf(e, dz, r.t);
      }
    }
    st[t.a * 128 + row] = r;
    if (sc) {
      float2* l = sc_list(ep, row);
#pragma unroll
      for (int r2 = 0; r2 < SC_K; ++r2) l[r2] = make_float2(tv[r2], __int_as_float(ti[r2]));
    }
    if (p.draw != nullptr) draw_tile(p, t, taddr, tok, ok, tm, ta);
  }
  DG_DEVINL static void finish(const Params& p, int row, uint8_t* ep) {
    const LmStat* st = reinterpret_cast<const LmStat*>(ep);
    for (int mt = 0; mt < p.MT; ++mt) {
      const LmStat r = st[mt * 128 + row];
      p.part[((size_t)blockIdx.x * p.MT + mt) * 128 + row] = make_float4(r.m, r.s, r.t, __int_as_float(r.a));
    }
    if (p.sc_part != nullptr) {
      const int tok = (blockIdx.x % p.MT) * 128 + row;
      if (tok < p.T) {
        const float2* l = sc_list(ep, row);
        float2* dst = p.sc_part + ((size_t)blockIdx.x * p.T + tok) * SC_K;
        for (int r = 0; r < SC_K; ++r) dst[r] = l[r];
      }
    }
  }
};

// The LM head as M = 256 tiles over CTA pairs: a pair covers two token tiles
// against one 256-row vocabulary tile; each CTA loads its 128 tokens and 128
// of the vocabulary rows, and its accumulator holds its tokens x all 256
// vocabulary columns, so P_LM's epilogue and statistics apply unchanged (a CTA
// sees one token tile, the other's partial stays empty).  Not with the
// self-conditioning lists (they assume a CTA sees one fixed token tile).
struct P_LM2 : P_LM {
  static constexpr bool PAIR = true;
  static constexpr int STAGES = 6, B_STAGE = BN * 128 / 2;  // 32 KB per stage and CTA
  DG_DEVINL static int num_tiles(const Params& p) { return ((p.MT + 1) / 2) * p.NV; }
  DG_DEVINL static Tile tile(const Params& p, int v) {
    Tile t;
    t.valid = 1;
    t.nk = p.nk;
    t.n_mma = BN;
    const int mt2 = (p.MT + 1) / 2;
    t.a = v % mt2;  // pair of token tiles
    t.b = v / mt2;  // vocabulary tile
    return t;
  }
  DG_DEVINL static Tile local(const Params&, Tile t, int rank) {
    t.a = 2 * t.a + rank;
    t.half = rank;
    return t;
  }
  DG_DEVINL static uint32_t tx_bytes(const Params&, const Tile&) { return kAStage + B_STAGE; }
  DG_DEVINL static void load_w(const Params& p, const Tile& t, int kb, uint32_t, uint32_t sb, uint64_t* bar) {
    tma_load_2d_pair(sb, &p.tmE, kb * 64, t.b * 256 + t.half * 128, bar);  // 128-row boxes
  }
  DG_DEVINL static void load_x(const Params& p, const Tile& t, int kb, uint32_t sa, uint32_t, uint64_t* bar) {
    tma_load_2d_pair(sa, &p.tmX, kb * 64, p.row0 + t.a * 128, bar);
  }
  DG_DEVINL static void load(const Params& p, const Tile& t, int kb, uint32_t sa, uint32_t sb, uint64_t* bar) {
    load_x(p, t, kb, sa, sb, bar);
    load_w(p, t, kb, sa, sb, bar);
  }
};

// ---------------------------------------------------------------------------
// host launchers
// ---------------------------------------------------------------------------
template <class P>
static cudaError_t launch_gemm(const typename P::Params& p, int grid, cudaStream_t st) {
  static bool configured = false;
  const size_t smem = GemmSmem<P>::total;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(k_umma_gemm<P>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  if (grid <= 0) return cudaSuccess;
  if constexpr (P::PAIR)  // grid = 2 x pairs, launched as clusters of two
    return launch_pdl_cluster(k_umma_gemm<P>, dim3(grid), dim3(gemm_threads<P>()), smem, st, dim3(2, 1, 1), p);
  else
    return launch_pdl(k_umma_gemm<P>, dim3(grid), dim3(gemm_threads<P>()), smem, st, p);
}

static int grid_for(int tiles, int sms) { return tiles < sms ? tiles : sms; }

cudaError_t run_qkv(const QkvArgs& a, cudaStream_t st) {
  P_QKV::Params p;
  p.tmA = *a.tm_x;
  p.tmB = *a.tm_w;
  p.T = a.T;
  p.nk = a.d / 64;
  p.MT = (a.T + 127) / 128;
  p.NT = a.rows / 128;
  p.D = a.D;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.q_T = a.q_T;
  p.kv_cap = a.kv_cap;
  p.kv_req_stride = a.kv_req_stride;
  p.tok_pos = a.tok_pos;
  p.tok_req = a.tok_req;
  p.rope = a.rope;
  p.q = a.q;
  p.kv = a.kv;
  p.err = a.err;
  if (a.pair) return launch_gemm<P_QKV2>(p, 2 * grid_for(((p.MT + 1) / 2) * p.NT, a.num_sms / 2), st);
  return launch_gemm<P_QKV>(p, grid_for(p.MT * p.NT, a.num_sms), st);
}

// K split so that feature tiles x token tiles x splits fills the GPU once.
int wpart_splits(int d, int T, int K, int num_sms) {
  const int tiles = (d / 128) * ((T + 255) / 256);
  int s = num_sms / tiles;
  const int nk = K / 64;
  if (s > nk) s = nk;
  if (s > kMaxPartSplits) s = kMaxPartSplits;
  if (s < 1) return 1;
  // every split must own at least one k-block (an empty split writes no partial)
  const int per = (nk + s - 1) / s;
  return (nk + per - 1) / per;
}

cudaError_t run_wpart(const WpartArgs& a, cudaStream_t st) {
  P_WPART::Params p;
  p.tmA = *a.tm_w;
  p.tmB = *a.tm_x;
  p.T = a.T;
  p.nk = a.K / 64;
  p.MT = a.d / 128;
  p.NT = (a.T + P_WPART::BN - 1) / P_WPART::BN;
  p.S = a.splits;
  p.Tcap = a.Tcap;
  p.d = a.d;
  p.part = a.part;
  p.err = a.err;
  if (a.tm_x128 != nullptr && p.MT % 2 == 0) {  // CTA pairs (the activations in 128-row boxes)
    p.tmB = *a.tm_x128;
    return launch_gemm<P_WPART2>(p, 2 * grid_for((p.MT / 2) * p.NT * p.S, a.num_sms / 2), st);
  }
  return launch_gemm<P_WPART>(p, grid_for(p.MT * p.NT * p.S, a.num_sms), st);
}

cudaError_t run_experts_gate_up_fp8(const ExpertArgs& a, cudaStream_t st) {
  P_EGU8::Params g;
  g.tmG = *a.tm_gate;
  g.tmU = *a.tm_up;
  g.tmX = *a.tm_xp;
  g.nk = (a.d + 127) / 128;
  g.fe = a.fe;
  g.tiles = a.egu_tiles;
  g.n_tiles = a.egu_count;
  g.counts = a.counts;
  g.offsets = a.offsets;
  g.sg = a.s_gate;
  g.su = a.s_up;
  g.sx = a.s_x;
  g.hp = a.hp;
  g.err = a.err;
  g.sched = a.sched;
  return launch_gemm<P_EGU8>(g, a.num_sms, st);
}

cudaError_t run_experts_down_fp8(const ExpertArgs& a, cudaStream_t st) {
  P_ED8::Params dn;
  dn.tmW = *a.tm_down;
  dn.tmH = *a.tm_hp;
  dn.nk = (a.fe + 127) / 128;
  dn.d = a.d;
  dn.tiles = a.ed_tiles;
  dn.n_tiles = a.ed_count;
  dn.counts = a.counts;
  dn.offsets = a.offsets;
  dn.sw = a.s_down;
  dn.sh = a.s_h;
  dn.row_weight = a.row_weight;
  dn.yp = a.yp;
  dn.err = a.err;
  dn.sched = a.sched + 1;
  return launch_gemm<P_ED8>(dn, a.num_sms, st);
}

cudaError_t run_experts(const ExpertArgs& a, cudaStream_t st) {
  if (a.ready == nullptr || a.sched == nullptr) return cudaErrorInvalidValue;
  P_EXP::Params x;
  x.gu.tmG = *a.tm_gate;
  x.gu.tmU = *a.tm_up;
  x.gu.tmX = *a.tm_xp;
  x.gu.nk = a.d / 64;
  x.gu.fe = a.fe;
  x.gu.tiles = a.egu_tiles;
  x.gu.n_tiles = a.egu_count;
  x.gu.counts = a.counts;
  x.gu.offsets = a.offsets;
  x.gu.hp = a.hp;
  x.gu.err = a.err;
  x.gu.sched = a.sched;
  x.dn.tmW = *a.tm_down;
  x.dn.tmH = *a.tm_hp;
  x.dn.nk = a.fe / 64;
  x.dn.d = a.d;
  x.dn.tiles = a.ed_tiles;
  x.dn.n_tiles = a.ed_count;
  x.dn.counts = a.counts;
  x.dn.offsets = a.offsets;
  x.dn.row_weight = a.row_weight;
  x.dn.yp = a.yp;
  x.dn.err = a.err;
  x.dn.sched = a.sched;
  x.n_sd = 0;
  x.sd_nk = x.sd_fb = 0;
  x.T = a.T;
  x.d = a.d;
  x.part = a.sd_part;
  if (a.tm_sdown != nullptr) {  // the shared expert's down projection rides along
    if (a.sd_K % 64 != 0 || a.d % 128 != 0 || a.T < 1 || a.sd_part == nullptr) return cudaErrorInvalidValue;
    x.tmSW = *a.tm_sdown;
    x.tmHS = *a.tm_hs64;
    x.sd_fb = a.d / 128;
    x.sd_nk = a.sd_K / 64;
    x.n_sd = x.sd_fb * ((a.T + P_EXP::BN - 1) / P_EXP::BN);
  } else {
    x.tmSW = *a.tm_down;  // unused
    x.tmHS = *a.tm_hp;
  }
  x.ready = a.ready;
  x.FJ = a.fe / 64;
  x.sched = a.sched;
  x.err = a.err;
  return launch_gemm<P_EXP>(x, a.num_sms, st);
}

cudaError_t run_shared_gate_up(const SharedArgs& a, cudaStream_t st) {
  if (a.E != 0 && (a.E < 16 || a.E > P_SGU::BN || a.E % 16 != 0 || a.k < 1 || a.k > 8 || a.tm_router == nullptr))
    return cudaErrorInvalidValue;
  if (a.fs % P_SGU::kHid != 0) return cudaErrorInvalidValue;
  P_SGU::Params g;
  g.tmX = *a.tm_u;
  g.tmG = *a.tm_gate;
  g.tmU = *a.tm_up;
  g.tmR = a.E > 0 ? *a.tm_router : *a.tm_gate;  // unused without a router
  g.T = a.T;
  g.nk = a.d / 64;
  g.MT = (a.T + 127) / 128;
  g.FJ = a.fs / P_SGU::kHid;
  g.fs = a.fs;
  g.E = a.E;
  g.k = a.k;
  g.MW = a.MW;
  g.hs = a.hs;
  g.logits = a.logits;
  g.idx = a.idx;
  g.w = a.w;
  g.mask = a.mask;
  g.err = a.err;
  // router tiles of 32 or 64 tokens while they and the shared tiles still fit in one wave
  const int shared_tiles = g.MT * g.FJ;
  g.RR = 128;
  g.tmXR = *a.tm_u;
  if (a.E > 0 && a.tm_u32 != nullptr && (a.T + 31) / 32 + shared_tiles <= a.num_sms) {
    g.RR = 32;
    g.tmXR = *a.tm_u32;
  } else if (a.E > 0 && a.tm_u64 != nullptr && (a.T + 63) / 64 + shared_tiles <= a.num_sms) {
    g.RR = 64;
    g.tmXR = *a.tm_u64;
  }
  const int router = a.E > 0 ? (a.T + g.RR - 1) / g.RR : 0;  // P_SGU::router_tiles
  return launch_gemm<P_SGU>(g, grid_for(router + g.MT * g.FJ, a.num_sms), st);
}

cudaError_t run_lm_head(const LmArgs& a, int* grid_out, cudaStream_t st) {
  P_LM::Params p;
  p.tmX = *a.tm_x;
  p.tmE = *a.tm_embed;
  p.T = a.T;
  p.nk = a.d / 64;
  p.MT = (a.T + 127) / 128;
  p.NV = (int)(a.V / 256);
  p.V = a.V;
  p.part = a.part;
  p.logits = a.logits;
  p.err = a.err;
  p.inv_tau = a.inv_tau;
  p.draw = a.draw;
  p.keys = a.keys;
  p.sc_part = a.sc_part;
  p.row0 = a.row0;
  static_assert(P_LM::MT_MAX * 128 == kLmRowsMax, "LM-head chunk size");
  if (p.MT > P_LM::MT_MAX || a.row0 < 0) return cudaErrorInvalidValue;
  if (p.draw != nullptr && (p.keys.canvas < 1 || (p.T + p.keys.canvas - 1) / p.keys.canvas > DG_MAX_REQUESTS))
    return cudaErrorInvalidValue;
  if (a.tm_embed128 != nullptr && p.sc_part == nullptr) {  // CTA pairs
    p.tmE = *a.tm_embed128;
    const int grid = 2 * grid_for(((p.MT + 1) / 2) * p.NV, a.num_sms / 2);
    if (grid < 2) return cudaErrorInvalidValue;
    *grid_out = grid;
    return launch_gemm<P_LM2>(p, grid, st);
  }
  int grid = grid_for(p.MT * p.NV, a.num_sms);
  if (p.sc_part != nullptr) grid = grid / p.MT * p.MT;  // one token tile per CTA
  if (grid < 1) return cudaErrorInvalidValue;
  *grid_out = grid;
  return launch_gemm<P_LM>(p, grid, st);
}

size_t gemm_smem_bytes_max() {
  size_t m = GemmSmem<P_QKV>::total;
  m = m > GemmSmem<P_WPART>::total ? m : GemmSmem<P_WPART>::total;
  m = m > GemmSmem<P_EGU>::total ? m : GemmSmem<P_EGU>::total;
  m = m > GemmSmem<P_ED>::total ? m : GemmSmem<P_ED>::total;
  m = m > GemmSmem<P_EXP>::total ? m : GemmSmem<P_EXP>::total;
  m = m > GemmSmem<P_QKV2>::total ? m : GemmSmem<P_QKV2>::total;
  m = m > GemmSmem<P_WPART2>::total ? m : GemmSmem<P_WPART2>::total;
  m = m > GemmSmem<P_LM2>::total ? m : GemmSmem<P_LM2>::total;
  m = m > GemmSmem<P_SGU>::total ? m : GemmSmem<P_SGU>::total;
  m = m > GemmSmem<P_LM>::total ? m : GemmSmem<P_LM>::total;
  m = m > GemmSmem<P_EGU8>::total ? m : GemmSmem<P_EGU8>::total;
  m = m > GemmSmem<P_ED8>::total ? m : GemmSmem<P_ED8>::total;
  return m;
}

}  // namespace dg
