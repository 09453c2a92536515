// Canvas attention on tcgen05: every canvas (or prefill segment) query
// attends, with no mask, to all committed keys of its request and to every
// key of its own segment (DiffusionGemma pages: bidirectional decoder pass
// over the canvas, "What DiffusionGemma is"; every token sees every other
// token in its context, "26B MoE Architecture, but Only 3.8B Activated").
//
// One CTA = 128 query rows of one (request slot, KV head) -- the G = Hq/Hkv
// query heads of a KV head are stacked as G*Tr rows so one K/V tile serves
// them all -- over one range of keys (split-KV when the query tiles alone
// cannot fill the GPU; partial (O, max, sum) are merged by k_attn_combine).
//   warps 0, 6 TMA producers: 64-key K tiles [64 x D] (warp 0) and V^T tiles
//              [D x 64] (warp 6) in separate three-slot rings (the cache keeps V
//              transposed so both MMAs read K-major operands); a K slot is
//              refilled as soon as the S MMA that read it completes, a V slot
//              once its PV MMA completes
//   warp 1     S issuer: S = Q K^T into one of two TMEM buffers (N = 64, Q read
//              from tensor memory)
//   warp 7     P V issuer: O += P V^T into TMEM (N = D); two issuing threads keep
//              the S stream from waiting behind P V and the other way round
//   warps 2-5  one query row per thread: Q row into tensor memory, then per
//              tile the exp2-domain online softmax on the S row read from TMEM,
//              P row (bf16) written into the swizzled shared tile PV reads.
//              The running max is only moved (and O, l rescaled in TMEM) when
//              it grows by more than 2^8, so rescales are rare; O and l always
//              share the same reference max, so the result is exact.
// Every wait is bounded (mbar_wait_bounded).
#include "common.cuh"
#include "dg_internal.h"

namespace dg {

constexpr int kAQ = 128;        // query rows per CTA
constexpr int kAK = 64;         // keys per tile
constexpr int kAStages = 3;     // K/V ring depth
constexpr float kRescaleLog2 = 8.0f;
constexpr int kMaxSplits = 8;   // key splits of one query tile (also the largest cluster)
constexpr int kVWarp = 6;                 // V^T producer
constexpr int kPVWarp = 7;                // issuer of the P V MMAs
constexpr int kAttnThreads = 32 * (kPVWarp + 1);

// Tensor memory (512 columns): O fp32 in [0, D), the two S buffers at 256 and
// 320, Q (bf16 pairs, the A operand of S = Q K^T) in [384, 384 + D/2).
constexpr uint32_t kTmS = 256, kTmQ = 384;

template <int D>
struct AttnSmem {
  static constexpr int kK = kAK * D * 2;            // K tile: D/64 blocks of [64 x 128 B]
  static constexpr int kV = D * kAK * 2;            // V^T tile: [D x 128 B]
  static constexpr int kP = kAQ * kAK * 2;          // P tile: [128 x 128 B]
  static constexpr size_t k_off = 0;
  static constexpr size_t v_off = k_off + (size_t)kAStages * kK;
  static constexpr size_t p_off = v_off + (size_t)kAStages * kV;
  // after the last MMA the K and V rings hold the finished O rows (fp32,
  // 128 x D) and, with the cluster merge, each row's (max, sum) behind them
  static constexpr size_t ml_off = k_off + (size_t)kAQ * D * 4;
  static_assert(ml_off + kAQ * 8 <= p_off, "O staging exceeds the K and V rings");
  static constexpr size_t bar_off = p_off + 2 * (size_t)kP;
  static constexpr int kBars = 4 * kAStages + 9;
  static constexpr size_t misc_off = bar_off + kBars * 8;
  // at least 120 KB so two CTAs (each owning all 512 TMEM columns) never share an SM
  static constexpr size_t total = misc_off + 16 + 1024 > 120 * 1024 ? misc_off + 16 + 1024 : 120 * 1024;
};
static_assert(AttnSmem<256>::total <= 227 * 1024, "attention shared memory exceeds the per-CTA limit");

DG_DEVINL void tmem_st16_raw(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

DG_DEVINL void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1) k_attn_tc(const __grid_constant__ AttnArgs a) {
  using S = AttnSmem<D>;
  extern __shared__ uint8_t dyn_smem[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~(uintptr_t)1023);
  uint8_t* sK = base + S::k_off;
  uint8_t* sV = base + S::v_off;
  uint8_t* sP = base + S::p_off;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + S::bar_off);
  uint64_t* k_full = bars;
  uint64_t* k_empty = bars + kAStages;
  uint64_t* v_full = bars + 2 * kAStages;
  uint64_t* v_empty = bars + 3 * kAStages;
  uint64_t* s_full = bars + 4 * kAStages;       // [2]
  uint64_t* s_empty = s_full + 2;               // [2]
  uint64_t* p_full = s_empty + 2;               // [2]
  uint64_t* pv_done = p_full + 2;               // [2]
  uint64_t* q_ready = pv_done + 2;              // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + S::misc_off);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + S::misc_off + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.Hq / a.Hkv;
  const int slot = blockIdx.y / a.Hkv, g = blockIdx.y % a.Hkv;
  const int rows = G * a.Tr;
  const int r0 = blockIdx.x * kAQ;
  const int n_keys = a.n_keys[slot];
  const int n_split = a.slot_split[slot];
  if ((int)blockIdx.z >= n_split) {  // this slot uses fewer key splits
    pdl_trigger();
    pdl_wait();
    if (a.cluster) {  // not launched this way (uniform splits), but never leave a cluster waiting
      float2* ml = reinterpret_cast<float2*>(base + S::ml_off);
      if (threadIdx.x < kAQ) ml[threadIdx.x] = make_float2(-INFINITY, 0.f);
      __syncthreads();
      cluster_sync_all();
      cluster_sync_all();
    }
    return;
  }
  int per = (n_keys + n_split - 1) / n_split;
  per = (per + kAK - 1) / kAK * kAK;
  const int k_begin = blockIdx.z * per;
  const int k_end = min(n_keys, k_begin + per);
  const int n_tiles = k_end > k_begin ? (k_end - k_begin + kAK - 1) / kAK : 0;
  int* err = a.err;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kAStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_empty[b], 128);
      mbar_init(&p_full[b], 128);
      mbar_init(&pv_done[b], 1);
    }
    mbar_init(q_ready, 128);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&a.tm_k);
    tma_prefetch_desc(&a.tm_vt);
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_trigger();
  pdl_wait();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_o = tmem, tm_s0 = tmem + kTmS, tm_q = tmem + kTmQ;

  // cache rows of this (request, layer, kv head) in the two tensor maps
  const long long krow0 = a.k_row0 + (long long)a.req[slot] * a.req_rows_k + (long long)g * a.cap;
  const long long vrow0 = a.v_row0 + (long long)a.req[slot] * a.req_rows_v + (long long)g * D;

  if (warp == 0 || warp == kVWarp) {
    if (lane == 0) {
      // K(j) waits for S(j - depth) to free its slot, V(j) for PV(j - depth)
      auto load_k = [&](int j) -> bool {
        const int st = j % kAStages;
        if (!mbar_wait_bounded(&k_empty[st], ((j / kAStages) & 1) ^ 1, abort_flag, err)) return false;
        mbar_arrive_expect_tx(&k_full[st], S::kK);
        const uint32_t k_dst = smem_u32(sK + (size_t)st * S::kK);
        const int key0 = k_begin + j * kAK;
        // the tiled K cache holds the 64 keys x D dims of a tile as D
        // consecutive 128-byte rows: one box, [D/64][64 keys][128 B] in smem
        tma_load_2d(k_dst, &a.tm_k, 0, (int)((krow0 + key0) * (D / 64)), &k_full[st]);
        return true;
      };
      auto load_v = [&](int j) -> bool {
        const int st = j % kAStages;
        if (!mbar_wait_bounded(&v_empty[st], ((j / kAStages) & 1) ^ 1, abort_flag, err)) return false;
        mbar_arrive_expect_tx(&v_full[st], S::kV);
        tma_load_2d(smem_u32(sV + (size_t)st * S::kV), &a.tm_vt, k_begin + j * kAK, (int)vrow0, &v_full[st]);
        return true;
      };
      // warp 0 streams K, the last warp V: a V load waits for PV(j - depth),
      // which must not hold back the K stream (and the other way round)
      bool ok = true;
      if (warp == 0) {
        for (int j = 0; ok && j < n_tiles; ++j) ok = load_k(j);
      } else {
        // the Q rows and the first K tiles go first: V(0) is needed only after S(0) and its softmax
        ok = n_tiles == 0 || mbar_wait_bounded(q_ready, 0, abort_flag, err);
        for (int j = 0; ok && j < n_tiles; ++j) ok = load_v(j);
      }
    }
  } else if (warp == 1) {
    // S MMAs: S(j) as soon as its S buffer is free and its K tile landed,
    // independently of the P V stream (separate issuing thread)
    if (lane == 0 && n_tiles > 0) {
      const uint32_t idesc_s = umma_idesc_bf16(128, kAK);
      bool ok = mbar_wait_bounded(q_ready, 0, abort_flag, err);
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int b = j & 1, stage = j % kAStages;
        if (!mbar_wait_bounded(&s_empty[b], ((j >> 1) & 1) ^ 1, abort_flag, err)) break;
        if (!mbar_wait_bounded(&k_full[stage], (j / kAStages) & 1, abort_flag, err)) break;
        tc_fence_after();
        const uint32_t k0 = smem_u32(sK + (size_t)stage * S::kK);
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16_ts(tm_s0 + b * kAK, tm_q + (uint32_t)(kb * 32 + k * 8),
                         umma_sdesc_k128(k0 + kb * (kAK * 128) + 32 * k), idesc_s, (kb | k) != 0 ? 1u : 0u);
        umma_commit(&k_empty[stage]);
        umma_commit(&s_full[b]);
      }
    }
  } else if (warp == kPVWarp) {
    // O += P(j) V(j)^T as soon as the softmax has written P(j)
    if (lane == 0 && n_tiles > 0) {
      const uint32_t idesc_o = umma_idesc_bf16(128, D);
      const uint32_t p0 = smem_u32(sP);
      for (int j = 0; j < n_tiles; ++j) {
        const int b = j & 1, stage = j % kAStages;
        if (!mbar_wait_bounded(&v_full[stage], (j / kAStages) & 1, abort_flag, err)) break;
        if (!mbar_wait_bounded(&p_full[b], (j >> 1) & 1, abort_flag, err)) break;
        tc_fence_after();
        const uint32_t v0 = smem_u32(sV + (size_t)stage * S::kV);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_bf16(tm_o, umma_sdesc_k128(p0 + b * S::kP + 32 * k), umma_sdesc_k128(v0 + 32 * k), idesc_o,
                    (j | k) != 0 ? 1u : 0u);
        umma_commit(&v_empty[stage]);
        umma_commit(&pv_done[b]);
      }
    }
  } else {
    // ---- softmax / epilogue warps: one query row per thread ----
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const int qr = r0 + row;
    const bool valid = qr < rows;
    const int h = g * G + (valid ? qr / a.Tr : 0);
    const int t = slot * a.Tr + (valid ? qr % a.Tr : 0);
    // Q row -> tensor memory lane `row`, bf16 pairs in columns kTmQ + [0, D/2).
    // The rows are read coalesced (kRW lanes per row, up to 256 bytes per row
    // and instruction) and transposed through the P buffers (free until the
    // first softmax) kRW 16-byte chunks per round: lane-per-row loads touched
    // 32 sectors per instruction and were bound by the L2 request rate.
    {
      constexpr int kNC = D / 8;                 // 16-byte chunks of a row
      constexpr int kRW = kNC < 16 ? kNC : 16;   // chunks per round
      constexpr int kRPI = 32 / kRW;             // rows per load instruction
      static_assert(kRW % 4 == 0 && kNC % kRW == 0 && 4 * 32 * kRW * 16 <= 2 * S::kP, "Q staging");
      const unsigned long long my_src =
          valid ? reinterpret_cast<unsigned long long>(a.q + ((size_t)h * a.q_T + t) * D) : 0ull;
      uint4* stq = reinterpret_cast<uint4*>(sP) + (size_t)q * 32 * kRW;  // this warp: [32 rows][kRW chunks]
      const int cl = lane % kRW, rl = lane / kRW;
#pragma unroll 1
      for (int rd = 0; rd < kNC / kRW; ++rd) {
        uint4 v[kRW];
#pragma unroll
        for (int k = 0; k < kRW; ++k) {
          const uint4* src = reinterpret_cast<const uint4*>(__shfl_sync(0xffffffffu, my_src, kRPI * k + rl));
          v[k] = src != nullptr ? __ldcg(src + rd * kRW + cl) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int k = 0; k < kRW; ++k) {
          const int rk = kRPI * k + rl;
          stq[rk * kRW + (cl ^ (rk % kRW))] = v[k];
        }
        __syncwarp();
#pragma unroll
        for (int cg = 0; cg < kRW / 4; ++cg) {
          uint32_t r[16];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint4 w = stq[lane * kRW + ((cg * 4 + u) ^ (lane % kRW))];
            r[4 * u] = w.x;
            r[4 * u + 1] = w.y;
            r[4 * u + 2] = w.z;
            r[4 * u + 3] = w.w;
          }
          tmem_st16_raw(tm_q + lane_off + (rd * kRW + cg * 4) * 4, r);
        }
        __syncwarp();
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(q_ready);
    }
    const float sl2 = a.scale * 1.4426950408889634f;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles && ok; ++j) {
      const int b = j & 1;
      if (!mbar_wait_bounded(&s_full[b], (j >> 1) & 1, abort_flag, err)) { ok = false; break; }
      tc_fence_after();
      float s[kAK];
      {
        uint32_t r[kAK / 16][16];
#pragma unroll
        for (int c = 0; c < kAK / 16; ++c) tmem_ld16_issue(tm_s0 + lane_off + b * kAK + c * 16, r[c]);
#pragma unroll
        for (int c = 0; c < kAK / 16; ++c) tmem_ld_wait16(r[c]);
#pragma unroll
        for (int c = 0; c < kAK / 16; ++c)
#pragma unroll
          for (int i = 0; i < 16; ++i) s[c * 16 + i] = __uint_as_float(r[c][i]);
      }
      tc_fence_before();
      mbar_arrive(&s_empty[b]);
      const int key0 = k_begin + j * kAK;
      if (key0 + kAK > k_end) {   // ragged last tile: keys past the range get no weight
#pragma unroll
        for (int c = 0; c < kAK; ++c)
          if (key0 + c >= k_end) s[c] = -INFINITY;
      }
      // raw-score max, then scaled (sl2 > 0 keeps the order); the tile has
      // at least one key in range, so mx is finite
      float mx = s[0];
#pragma unroll
      for (int c = 1; c < kAK; ++c) mx = fmaxf(mx, s[c]);
      mx *= sl2;
      const bool need = mx > m_used + kRescaleLog2;
      const float m_new = need ? mx : m_used;
      // P buffer b is free once PV(j-2) is done
      if (j >= 2 && !mbar_wait_bounded(&pv_done[b], ((j - 2) >> 1) & 1, abort_flag, err)) { ok = false; break; }
      if (__any_sync(0xffffffffu, need) && j >= 1) {
        // O holds PV(0..j-1): wait for PV(j-1), then rescale this warp's rows
        if (!mbar_wait_bounded(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        const float f = need ? exp2f(m_used - m_new) : 1.f;
        for (int c = 0; c < D; c += 16) {
          float o[16];
          tmem_ld16(tm_o + lane_off + c, o);
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] *= f;
          tmem_st16(tm_o + lane_off + c, o);
        }
        l *= f;
      }
      m_used = m_new;
      uint8_t* prow = sP + b * S::kP + row * 128;
      float rs = 0.f;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        float p[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          p[i] = ex2_fast(fmaf(s[ch * 8 + i], sl2, -m_used));
          rs += p[i];
        }
        uint4 v;
        v.x = pack_bf16x2(p[0], p[1]);
        v.y = pack_bf16x2(p[2], p[3]);
        v.z = pack_bf16x2(p[4], p[5]);
        v.w = pack_bf16x2(p[6], p[7]);
        *reinterpret_cast<uint4*>(prow + ((ch ^ (row & 7)) << 4)) = v;
      }
      l += rs;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[b]);
    }
    // final O
    if (ok && n_tiles > 0 &&
        mbar_wait_bounded(&pv_done[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1, abort_flag, err)) {
      tc_fence_after();
      // Each warp stages its 32 finished rows in shared memory (the K and V
      // rings: every MMA that read them has completed) and then writes them
      // row by row, each lane storing 16 consecutive bytes of the row, so every
      // store instruction covers whole 128-byte lines.  Chunk c of local row i
      // is kept at position c ^ (i mod nch) (conflict-free both ways).
      const bool direct = n_split == 1;
      const bool merge = a.cluster != 0;
      const int nch = direct ? D / 8 : D / 4;  // 16-byte chunks per output row (bf16 / fp32)
      uint4* stg = reinterpret_cast<uint4*>(sK) + (size_t)q * 32 * (D / 4);
      const float inv = direct ? (l > 0.f ? 1.f / l : 0.f) : 1.f;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 64) {
        uint32_t r[4][16];
#pragma unroll
        for (int u = 0; u < 4; ++u) tmem_ld16_issue(tm_o + lane_off + c0 + 16 * u, r[u]);
#pragma unroll
        for (int u = 0; u < 4; ++u) tmem_ld_wait16(r[u]);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int col = c0 + 16 * u;
          if (direct) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              uint4 w;
              const uint32_t* x = r[u] + 8 * hh;
              w.x = pack_bf16x2(__uint_as_float(x[0]) * inv, __uint_as_float(x[1]) * inv);
              w.y = pack_bf16x2(__uint_as_float(x[2]) * inv, __uint_as_float(x[3]) * inv);
              w.z = pack_bf16x2(__uint_as_float(x[4]) * inv, __uint_as_float(x[5]) * inv);
              w.w = pack_bf16x2(__uint_as_float(x[6]) * inv, __uint_as_float(x[7]) * inv);
              const int ch = col / 8 + hh;
              stg[lane * nch + (ch ^ (lane & (nch - 1)))] = w;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int ch = col / 4 + i;
              stg[lane * nch + (ch ^ (lane & (nch - 1)))] =
                  make_uint4(r[u][4 * i], r[u][4 * i + 1], r[u][4 * i + 2], r[u][4 * i + 3]);
            }
          }
        }
      }
      __syncwarp();
      if (!merge) {
        // each lane knows its own row's destination; the warp writes row i from lane i's pointer
        unsigned long long my_dst = 0ull;
        if (valid)
          my_dst = direct ? reinterpret_cast<unsigned long long>(a.o + (size_t)t * a.Hq * D + (size_t)h * D)
                          : reinterpret_cast<unsigned long long>(
                                a.part_o + (((size_t)blockIdx.z * a.Hq + h) * a.q_T + t) * D);
#pragma unroll 4
        for (int i = 0; i < 32; ++i) {
          uint4* dst = reinterpret_cast<uint4*>(__shfl_sync(0xffffffffu, my_dst, i));
          if (dst == nullptr) continue;
          for (int c = lane; c < nch; c += 32) dst[c] = stg[i * nch + (c ^ (i & (nch - 1)))];
        }
      }
      if (merge) {
        reinterpret_cast<float2*>(base + S::ml_off)[row] = make_float2(m_used, l);
      } else if (!direct && valid) {
        const size_t prow_i = ((size_t)blockIdx.z * a.Hq + h) * a.q_T + t;
        a.part_ml[prow_i] = make_float2(m_used, l);
      }
    } else if (a.cluster) {  // no keys in this split (or an aborted wait): zero weight in the merge
      reinterpret_cast<float2*>(base + S::ml_off)[row] = make_float2(-INFINITY, 0.f);
    } else if (n_tiles == 0 && n_split > 1 && valid) {
      const size_t prow_i = ((size_t)blockIdx.z * a.Hq + h) * a.q_T + t;
      a.part_ml[prow_i] = make_float2(-INFINITY, 0.f);
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (a.cluster) {
    // The n_split CTAs of this query tile (one cluster) have staged their
    // partial O rows and (max, sum); CTA z merges rows [z*rp, (z+1)*rp) from all
    // of them, as O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s with M the
    // largest max, in split order, and writes them in bf16.
    cluster_sync_all();
    {
      const int ns = gridDim.z;
      const int rp = (kAQ + ns - 1) / ns;
      const int i0 = (int)blockIdx.z * rp, i1 = min(kAQ, i0 + rp);
      const uint32_t stg = smem_u32(base + S::k_off), mls = smem_u32(base + S::ml_off);
      // per merged row: the split weights 2^(m_s - M), 1 / L and the output row.
      // The arithmetic (and its order) is that of k_attn_combine, so a query
      // tile's result does not depend on which of the two merges it took.
      float* wsm = reinterpret_cast<float*>(base + S::p_off);  // [kAQ][kMaxSplits + 1]
      bf16** osm = reinterpret_cast<bf16**>(base + S::p_off + kAQ * (kMaxSplits + 1) * 4);  // [kAQ]
      const int row = (warp & 3) * 32 + lane;
      if (warp >= 2 && warp <= 5 && row >= i0 && row < i1) {
        float2 ml[kMaxSplits];
#pragma unroll
        for (int s2 = 0; s2 < kMaxSplits; ++s2)
          ml[s2] = s2 < ns ? ld_dsmem_f2(dsmem_addr(mls + row * 8, s2)) : make_float2(-INFINITY, 0.f);
        float M = -INFINITY;
#pragma unroll
        for (int s2 = 0; s2 < kMaxSplits; ++s2) M = fmaxf(M, ml[s2].y > 0.f ? ml[s2].x : -INFINITY);
        float w[kMaxSplits], x[kMaxSplits];
#pragma unroll
        for (int s2 = 0; s2 < kMaxSplits; ++s2) {
          w[s2] = ml[s2].y > 0.f ? exp2f(ml[s2].x - M) : 0.f;
          x[s2] = __fmul_rn(w[s2], ml[s2].y);
        }
        // the combine kernel's butterfly sum over lanes 0..7 (the other lanes hold 0)
        const float L = __fadd_rn(__fadd_rn(__fadd_rn(x[0], x[4]), __fadd_rn(x[2], x[6])),
                                  __fadd_rn(__fadd_rn(x[1], x[5]), __fadd_rn(x[3], x[7])));
#pragma unroll
        for (int s2 = 0; s2 < kMaxSplits; ++s2) wsm[row * (kMaxSplits + 1) + s2] = w[s2];
        wsm[row * (kMaxSplits + 1) + kMaxSplits] = L > 0.f ? 1.f / L : 0.f;
        const int qr = r0 + row;  // the output row (h, t) of merged row `row`
        const int hr = g * G + (qr < rows ? qr / a.Tr : 0), tr = slot * a.Tr + (qr < rows ? qr % a.Tr : 0);
        osm[row] = a.o + (size_t)tr * a.Hq * D + (size_t)hr * D;
      }
      // the merge itself is bound by the latency of distributed-shared-memory
      // loads: all eight warps take rows, doubling the loads in flight
      __syncthreads();
      constexpr int nch = D / 4;   // 16-byte chunks of an fp32 row
      constexpr int kRows = 2;     // rows merged side by side (loads in flight)
      constexpr int kWarps = kAttnThreads / 32;
#pragma unroll 1
      for (int ib = i0 + warp; ib < i1; ib += kWarps * kRows) {
#pragma unroll
        for (int c0 = 0; c0 < nch; c0 += 32) {
          const int c = c0 + lane;
          float4 v[kRows][kMaxSplits];
          float wr[kRows][kMaxSplits];
#pragma unroll
          for (int rr = 0; rr < kRows; ++rr) {
            const int i = ib + kWarps * rr;
#pragma unroll
            for (int s2 = 0; s2 < kMaxSplits; ++s2) {
              wr[rr][s2] = (i < i1 && r0 + i < rows) ? wsm[i * (kMaxSplits + 1) + s2] : 0.f;
              if (s2 < ns && wr[rr][s2] != 0.f && c < nch)
                v[rr][s2] = ld_dsmem_f4(
                    dsmem_addr(stg + (uint32_t)(i * nch + (c ^ (i & 31 & (nch - 1)))) * 16u, s2));
            }
          }
#pragma unroll
          for (int rr = 0; rr < kRows; ++rr) {
            const int i = ib + kWarps * rr;
            if (i >= i1 || r0 + i >= rows || c >= nch) continue;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int s2 = 0; s2 < kMaxSplits; ++s2)
              if (s2 < ns && wr[rr][s2] != 0.f) {
                acc.x = __fmaf_rn(wr[rr][s2], v[rr][s2].x, acc.x);
                acc.y = __fmaf_rn(wr[rr][s2], v[rr][s2].y, acc.y);
                acc.z = __fmaf_rn(wr[rr][s2], v[rr][s2].z, acc.z);
                acc.w = __fmaf_rn(wr[rr][s2], v[rr][s2].w, acc.w);
              }
            const float inv = wsm[i * (kMaxSplits + 1) + kMaxSplits];
            reinterpret_cast<uint2*>(osm[i])[c] = make_uint2(pack_bf16x2(__fmul_rn(acc.x, inv), __fmul_rn(acc.y, inv)),
                                                             pack_bf16x2(__fmul_rn(acc.z, inv), __fmul_rn(acc.w, inv)));
          }
        }
      }
    }
    __syncwarp();
    cluster_sync_all();  // no CTA leaves while another still reads its shared memory
  }
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// Merge of the split-KV partials: O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s.
// One warp per (token, head); lane s reads split s's (max, sum), each lane then
// owns 8 consecutive output elements and loads every split's values at once.
// Tokens of slots that used a single split were written by the attention kernel.
struct SlotSplits {
  int s[DG_MAX_REQUESTS];
};

__global__ void k_attn_combine(const float* __restrict__ part_o, const float2* __restrict__ part_ml,
                               SlotSplits splits, int Tr, int Hq, int q_T, int T, int D, bf16* __restrict__ o) {
  pdl_trigger();
  pdl_wait();
  const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= T * Hq) return;
  const int t = w / Hq, h = w % Hq;
  const int n_split = splits.s[t / Tr];
  if (n_split == 1) return;  // written directly by the attention kernel
  float2 ml = make_float2(-INFINITY, 0.f);
  if (lane < n_split) ml = __ldcg(part_ml + ((size_t)lane * Hq + h) * q_T + t);
  float M = ml.y > 0.f ? ml.x : -INFINITY;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  const float wl = ml.y > 0.f ? exp2f(ml.x - M) : 0.f;
  // explicit roundings: the in-kernel cluster merge repeats exactly these operations
  float L = __fmul_rn(wl, ml.y);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) L = __fadd_rn(L, __shfl_xor_sync(0xffffffffu, L, off));
  float wts[kMaxSplits];
#pragma unroll
  for (int s = 0; s < kMaxSplits; ++s) wts[s] = __shfl_sync(0xffffffffu, wl, s);
  const int c = lane * 8;
  if (c >= D) return;
  float4 va[kMaxSplits], vb[kMaxSplits];
#pragma unroll
  for (int s = 0; s < kMaxSplits; ++s)
    if (s < n_split && wts[s] != 0.f) {
      const float4* src = reinterpret_cast<const float4*>(part_o + (((size_t)s * Hq + h) * q_T + t) * D + c);
      va[s] = __ldcg(src);
      vb[s] = __ldcg(src + 1);
    }
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int s = 0; s < kMaxSplits; ++s)
    if (s < n_split && wts[s] != 0.f) {
      acc[0] = __fmaf_rn(wts[s], va[s].x, acc[0]);
      acc[1] = __fmaf_rn(wts[s], va[s].y, acc[1]);
      acc[2] = __fmaf_rn(wts[s], va[s].z, acc[2]);
      acc[3] = __fmaf_rn(wts[s], va[s].w, acc[3]);
      acc[4] = __fmaf_rn(wts[s], vb[s].x, acc[4]);
      acc[5] = __fmaf_rn(wts[s], vb[s].y, acc[5]);
      acc[6] = __fmaf_rn(wts[s], vb[s].z, acc[6]);
      acc[7] = __fmaf_rn(wts[s], vb[s].w, acc[7]);
    }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  uint4 u;
  u.x = pack_bf16x2(__fmul_rn(acc[0], inv), __fmul_rn(acc[1], inv));
  u.y = pack_bf16x2(__fmul_rn(acc[2], inv), __fmul_rn(acc[3], inv));
  u.z = pack_bf16x2(__fmul_rn(acc[4], inv), __fmul_rn(acc[5], inv));
  u.w = pack_bf16x2(__fmul_rn(acc[6], inv), __fmul_rn(acc[7], inv));
  *reinterpret_cast<uint4*>(o + (size_t)t * Hq * D + (size_t)h * D + c) = u;
}

int attention_split_cap() { return kMaxSplits; }

template <int D>
static cudaError_t launch_attn(const AttnArgs& a, cudaStream_t st) {
  const size_t smem = AttnSmem<D>::total;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(k_attn_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int G = a.Hq / a.Hkv;
  dim3 grid((G * a.Tr + kAQ - 1) / kAQ, a.Hkv * a.n_slots, a.n_split);
  if (a.cluster) {  // the key splits of a query tile merge in-kernel (uniform splits only)
    for (int i = 0; i < a.n_slots; ++i)
      if (a.slot_split[i] != a.n_split) return cudaErrorInvalidValue;
    const cudaError_t e_ = launch_pdl_cluster(k_attn_tc<D>, dim3(grid), dim3(kAttnThreads), smem, st,
                                              dim3(1, 1, a.n_split), a);
    if (e_ != cudaSuccess) return e_;
    return cudaGetLastError();
  }
  {
    const cudaError_t e_ = launch_pdl(k_attn_tc<D>, dim3(grid), dim3(kAttnThreads), smem, st, a);
    if (e_ != cudaSuccess) return e_;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || a.n_split == 1) return e;
  const int T = a.n_slots * a.Tr;
  const int warps = T * a.Hq;
  SlotSplits sp;
  for (int i = 0; i < DG_MAX_REQUESTS; ++i) sp.s[i] = i < a.n_slots ? a.slot_split[i] : 1;
  {
    const cudaError_t e_ = launch_pdl(k_attn_combine, dim3((warps + 7) / 8), dim3(256), 0, st, a.part_o, a.part_ml, sp,
                                      a.Tr, a.Hq, a.q_T, T, D, a.o);
    if (e_ != cudaSuccess) return e_;
  }
  return cudaGetLastError();
}

size_t attention_smem_bytes(int D) {
  switch (D) {
    case 64: return AttnSmem<64>::total;
    case 128: return AttnSmem<128>::total;
    default: return AttnSmem<256>::total;
  }
}

cudaError_t run_attention(const AttnArgs& a, cudaStream_t st) {
  if (a.n_split < 1 || a.n_split > attention_split_cap()) return cudaErrorInvalidValue;
  for (int i = 0; i < a.n_slots; ++i)
    if (a.slot_split[i] < 1 || a.slot_split[i] > a.n_split) return cudaErrorInvalidValue;
  switch (a.D) {
    case 64: return launch_attn<64>(a, st);
    case 128: return launch_attn<128>(a, st);
    case 256: return launch_attn<256>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dg
