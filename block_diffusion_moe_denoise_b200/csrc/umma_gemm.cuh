// Persistent, warp-specialised tcgen05 GEMM engine for sm_100a.
//
//   D[128 x N] = A[128 x K] * B[N x K]^T      (bf16 operands, fp32 accumulator in TMEM)
//
// Both operands are K-major tiles staged in shared memory by TMA with the
// 128-byte swizzle, 64 bf16 (one 128-byte row) per k-block.  A ring stage holds
// P::KB consecutive k-blocks: every stage costs a pair of barrier round trips
// (producer <-> MMA issuer), which dominates at small N, so small-N problems
// take two k-blocks per stage.  Roles:
//   warp 0 (one lane)   TMA producer: fills a STAGES-deep ring of (A, B) tiles
//   warp 1 (one lane)   MMA issuer: 4 x tcgen05.mma (K = 16 each) per k-block,
//                       tcgen05.commit frees the ring slot / signals the accumulator
//   warps 2..5          epilogue: tcgen05.ld of the accumulator rows they own
//                       (warp w reads TMEM lanes 32*(w%4) .. +31) and the fused
//                       problem-specific epilogue
//   warp 6 (one lane)   DYNAMIC problems only: tile scheduler (see below)
// The accumulator is double-buffered in TMEM (2 x BN columns) so the epilogue
// of one tile overlaps the main loop of the next.  Tiles are assigned
// statically (tile v to CTA v mod gridDim.x), so every role walks the same list.
//
// A problem class P supplies: BN, STAGES, KB, B_STAGE (bytes per k-block), EP_SMEM (bytes),
// TMEM_COLS, Params, num_tiles(), tile(), tx_bytes(), load(), epilogue(),
// finish(), epilogue_prefetch() (called before the accumulator wait, so an
// epilogue can pull its inputs into L1 while the main loop runs), and, with
// PRELOAD, load_w()/load_x(): the weight and activation halves of load().
// Every wait is bounded (see mbar_wait_bounded).
//
// Tile scheduling.  By default tile v goes to CTA v mod gridDim.x.  A problem
// with DYNAMIC = true instead hands out tiles from a global counter (p.sched,
// zero at launch): a seventh warp (the scheduler, one lane) takes indices with
// an atomic add, builds each tile's descriptor and publishes it through a
// small shared-memory ring that the producer, the MMA thread and the epilogue
// threads read in the same order, so a CTA that drew cheap tiles simply takes
// more of them (the expert GEMMs, whose tiles differ in cost and do not divide
// evenly over the SMs).  The atomic, the descriptor's dependent loads and any
// dependency wait (below) take one to two microseconds of round trips to L2;
// in a separate warp they overlap the producer's loads of the previous tile
// instead of draining the ring between two short tiles.
//
// CTA pairs.  With PAIR = true the grid is launched as clusters of two CTAs
// and one tile is an M = 256 MMA tile (tcgen05 .cta_group::2): each CTA loads
// half of A (its 128 rows) and half of B (N/2 rows) into its own ring, both
// halves completing on the even CTA's full barrier; the even CTA alone issues
// the MMAs, whose commits arrive on the empty and accumulator barriers of
// both; each CTA's epilogue reads its own 128 accumulator rows and releases
// the accumulator on the even CTA's barrier.  P::local(t, rank) turns a pair
// tile into the CTA's half (its tile coordinates and t.half).
//
// Dependent tiles.  With ACQUIRE = true P::acquire(p, t) runs before a tile is
// loaded (in the scheduler, which then hands the tile on through the ring's
// release/acquire barriers; in the producer with a static schedule); it may
// wait (bounded) for data that earlier tiles of the same launch write.  Every wait ends as long as the tiles it depends on
// come earlier in the tile order: a CTA processes its claimed tiles in claim
// order and claims increasing indices, so every tile queued in front of a
// tile X has a smaller index than X, and by induction over the index all of
// them finish; the MMA and epilogue roles never wait on the producer's later
// tiles.
#pragma once

#include "common.cuh"

namespace dg {

struct Tile {
  int valid;
  int nk;     // k-blocks of 64
  int n_mma;  // MMA N (multiple of 16, <= BN)
  int a, b, c, d, e, f;  // problem-specific coordinates
  int half;              // PAIR problems: this CTA's rank in its pair (0 issues the MMAs)
};

constexpr int kAStage = 128 * 128;  // 128 rows x 128 bytes
constexpr int kSchedRing = 2;       // tiles in flight between the scheduler and the other roles (DYNAMIC);
                                    // deeper rings claim tiles too far ahead (measured slower: 3, 4, 8)

// Threads of a block: producer, MMA and four epilogue warps, plus the scheduler
// warp of DYNAMIC problems.
template <class P>
constexpr int gemm_threads() { return P::DYNAMIC ? 224 : 192; }

template <class P>
struct GemmSmem {
  static constexpr int kStages = P::STAGES;
  static constexpr size_t a_stage = (size_t)P::KB * kAStage;
  static constexpr size_t b_stage = (size_t)P::KB * P::B_STAGE;
  static constexpr size_t a_off = 0;
  static constexpr size_t b_off = a_off + (size_t)kStages * a_stage;
  static constexpr size_t ep_off = b_off + (size_t)kStages * b_stage;
  static constexpr size_t bar_off = (ep_off + P::EP_SMEM + 15) & ~(size_t)15;
  static constexpr size_t misc_off = bar_off + (2 * kStages + 4 + 2 * kSchedRing) * 8;
  static constexpr size_t total = misc_off + 16 + sizeof(Tile) * kSchedRing + 1024;  // + alignment slack
};

template <class P>
__global__ void __launch_bounds__(224, 1) k_umma_gemm(const __grid_constant__ typename P::Params p) {
  static_assert(!(P::PRELOAD && P::DYNAMIC), "a preloaded first tile needs the static schedule");
  static_assert(!(P::PAIR && (P::DYNAMIC || P::F8)), "CTA pairs: static schedule, bf16");
  using S = GemmSmem<P>;
  extern __shared__ uint8_t dyn_smem[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = base + S::a_off;
  uint8_t* sB = base + S::b_off;
  uint8_t* ep_smem = base + S::ep_off;
  uint64_t* full = reinterpret_cast<uint64_t*>(base + S::bar_off);
  uint64_t* empty = full + P::STAGES;
  uint64_t* tfull = empty + P::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* sched_full = tempty + 2;                 // [kSchedRing], DYNAMIC only
  uint64_t* sched_empty = sched_full + kSchedRing;   // [kSchedRing]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + S::misc_off);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + S::misc_off + 4);
  Tile* sched_tile = reinterpret_cast<Tile*>(base + S::misc_off + 16);  // [kSchedRing], DYNAMIC only;
                                                                         // valid < 0 ends the list

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // PAIR: rank in the pair; tiles are dealt to pairs
  const uint32_t rank = P::PAIR ? cluster_ctarank() : 0;
  const int unit = P::PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int n_units = P::PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  auto tile_of = [&](int v) {
    Tile t = P::tile(p, v);
    if constexpr (P::PAIR) t = P::local(p, t, (int)rank);
    return t;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < P::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], P::PAIR ? 256 : 128);  // the epilogue threads (of both CTAs of a pair)
    }
    if constexpr (P::DYNAMIC)
      for (int r = 0; r < kSchedRing; ++r) {
        mbar_init(&sched_full[r], 1);
        mbar_init(&sched_empty[r], 130);  // the producer, the MMA thread and the 128 epilogue threads
      }
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) P::prefetch(p);
  if (warp == 1) {
    if constexpr (P::PAIR)
      tmem_alloc_pair(tmem_slot, P::TMEM_COLS);
    else
      tmem_alloc(tmem_slot, P::TMEM_COLS);
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (P::PAIR) cluster_sync_all();  // the partner's barriers exist before anything signals them
  tc_fence_after();
  pdl_trigger();
  const uint32_t tmem = *tmem_slot;
  int* err = p.err;

  if (warp == 0) {
    if (lane == 0) {
      // Weight tiles do not depend on the preceding kernel: for problems whose
      // tile list is static (P::PRELOAD) the first ring slots of this CTA's
      // first tile are filled with them before the dependency wait, so the
      // weight stream starts while the predecessor drains.
      int pre = 0;  // stages of the first tile armed before the wait
      if constexpr (P::PRELOAD) {
        if (unit < P::num_tiles(p)) {
          const Tile t0 = tile_of(unit);
          if (t0.valid) {
            const int n_st = (t0.nk + P::KB - 1) / P::KB;
            pre = n_st < P::STAGES ? n_st : P::STAGES;
            for (int st = 0; st < pre; ++st) {
              const int kb = st * P::KB;
              const int nsub = t0.nk - kb < P::KB ? t0.nk - kb : P::KB;
              if (rank == 0)  // a pair's even CTA expects both halves
                mbar_arrive_expect_tx(&full[st], P::tx_bytes(p, t0) * (uint32_t)nsub * (P::PAIR ? 2u : 1u));
              for (int j = 0; j < nsub; ++j)
                P::load_w(p, t0, kb + j, smem_u32(sA + st * S::a_stage + (size_t)j * kAStage),
                          smem_u32(sB + st * S::b_stage + (size_t)j * P::B_STAGE), &full[st]);
            }
          }
        }
      }
      pdl_wait();
      const int n_tiles = P::num_tiles(p);
      uint32_t stage = 0, phase = 0;
      for (int i = 0, v = unit;; ++i, v += n_units) {
        Tile t;
        if constexpr (P::DYNAMIC) {  // descriptor (dependencies already met) from the scheduler
          const int slot = i % kSchedRing;
          if (!mbar_wait_bounded(&sched_full[slot], (i / kSchedRing) & 1, abort_flag, err)) break;
          t = sched_tile[slot];
          mbar_arrive(&sched_empty[slot]);
          if (t.valid < 0) break;
        } else {
          if (v >= n_tiles) break;
          t = tile_of(v);
          // a tile whose operands another tile of this launch produces waits for them
          if constexpr (P::ACQUIRE)
            if (t.valid && !P::acquire(p, t, abort_flag, err)) break;
        }
        if (!t.valid) continue;
        const uint32_t tx = P::tx_bytes(p, t);
        bool ok = true;
        for (int kb = 0; kb < t.nk; kb += P::KB) {
          const int nsub = t.nk - kb < P::KB ? t.nk - kb : P::KB;
          uint8_t* sa = sA + stage * S::a_stage;
          uint8_t* sb = sB + stage * S::b_stage;
          if (pre > 0) {  // slot already armed and holding its weight tiles
            --pre;
            for (int j = 0; j < nsub; ++j)
              P::load_x(p, t, kb + j, smem_u32(sa + (size_t)j * kAStage), smem_u32(sb + (size_t)j * P::B_STAGE),
                        &full[stage]);
          } else {
            if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, err)) { ok = false; break; }
            if (rank == 0) mbar_arrive_expect_tx(&full[stage], tx * (uint32_t)nsub * (P::PAIR ? 2u : 1u));
            for (int j = 0; j < nsub; ++j)
              P::load(p, t, kb + j, smem_u32(sa + (size_t)j * kAStage), smem_u32(sb + (size_t)j * P::B_STAGE),
                      &full[stage]);
          }
          if (++stage == P::STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
      }
    } else {
      pdl_wait();
    }
  } else if (warp == 1) {
    pdl_wait();
    const int n_tiles = P::num_tiles(p);
    if (lane == 0 && rank == 0) {  // a pair's odd CTA issues no MMAs
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
      for (int i = 0, v = unit;; ++i, v += n_units) {
        Tile t;
        if constexpr (P::DYNAMIC) {
          const int slot = i % kSchedRing;
          if (!mbar_wait_bounded(&sched_full[slot], (i / kSchedRing) & 1, abort_flag, err)) break;
          t = sched_tile[slot];
          mbar_arrive(&sched_empty[slot]);
          if (t.valid < 0) break;
        } else {
          if (v >= n_tiles) break;
          t = tile_of(v);
        }
        if (!t.valid) continue;
        if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1, abort_flag, err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * P::BN;
        constexpr uint32_t kM = P::PAIR ? 256 : 128;
        const uint32_t idesc =
            P::F8 ? umma_idesc_e4m3(kM, (uint32_t)t.n_mma) : umma_idesc_bf16(kM, (uint32_t)t.n_mma);
        bool ok = true;
        for (int kb = 0; kb < t.nk; kb += P::KB) {
          const int nsub = t.nk - kb < P::KB ? t.nk - kb : P::KB;
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * S::a_stage);
          const uint32_t b0 = smem_u32(sB + stage * S::b_stage);
#pragma unroll
          for (int j = 0; j < P::KB; ++j) {
            if (j < nsub) {
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const uint64_t ad = umma_sdesc_k128(a0 + j * kAStage + 32 * k);
                const uint64_t bd = umma_sdesc_k128(b0 + j * P::B_STAGE + 32 * k);
                if constexpr (P::F8)
                  umma_e4m3(d_tmem, ad, bd, idesc, (kb | j | k) != 0 ? 1u : 0u);
                else if constexpr (P::PAIR)
                  umma_bf16_pair(d_tmem, ad, bd, idesc, (kb | j | k) != 0 ? 1u : 0u);
                else
                  umma_bf16(d_tmem, ad, bd, idesc, (kb | j | k) != 0 ? 1u : 0u);
              }
            }
          }
          if constexpr (P::PAIR)
            umma_commit_pair(&empty[stage]);
          else
            umma_commit(&empty[stage]);
          if (++stage == P::STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        if constexpr (P::PAIR)
          umma_commit_pair(&tfull[acc]);
        else
          umma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
    }
  } else if (warp < 6) {
    pdl_wait();
    const int n_tiles = P::num_tiles(p);
    const int q = warp & 3;            // TMEM lane quadrant of this warp
    const int row = q * 32 + lane;     // accumulator row (M index) owned by this thread
    P::epilogue_init(p, row, ep_smem);
    uint32_t acc = 0, acc_phase = 0;
    for (int i = 0, v = unit;; ++i, v += n_units) {
      Tile t;
      if constexpr (P::DYNAMIC) {
        const int slot = i % kSchedRing;
        if (!mbar_wait_bounded(&sched_full[slot], (i / kSchedRing) & 1, abort_flag, err)) break;
        t = sched_tile[slot];
        mbar_arrive(&sched_empty[slot]);
        if (t.valid < 0) break;
      } else {
        if (v >= n_tiles) break;
        t = tile_of(v);
      }
      if (!t.valid) continue;
      P::epilogue_prefetch(p, t, row);
      if (!mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, err)) break;
      tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + acc * P::BN;
      P::epilogue(p, t, taddr, q, lane, row, ep_smem);
      tc_fence_before();
      if (rank == 0)
        mbar_arrive(&tempty[acc]);
      else
        mbar_arrive_remote(&tempty[acc], 0);  // the pair's MMAs are issued from the even CTA
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
    P::finish(p, row, ep_smem);
  } else {
    // scheduler (DYNAMIC only): claim, describe, wait for dependencies, publish
    pdl_wait();
    if constexpr (P::DYNAMIC) {
      if (lane == 0) {
        const int n_tiles = P::num_tiles(p);
        for (int i = 0;; ++i) {
          const int slot = i % kSchedRing;
          if (!mbar_wait_bounded(&sched_empty[slot], ((i / kSchedRing) & 1) ^ 1, abort_flag, err)) break;
          const int v = atomicAdd(p.sched, 1);
          Tile t{};
          t.valid = -1;
          if (v < n_tiles) {
            t = tile_of(v);
            if constexpr (P::ACQUIRE)
              if (t.valid && !P::acquire(p, t, abort_flag, err)) t.valid = -1;  // abort: end the list
          }
          sched_tile[slot] = t;
          mbar_arrive(&sched_full[slot]);
          if (t.valid < 0) break;
        }
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if constexpr (P::PAIR) cluster_sync_all();  // the partner is done with both CTAs' memory
  tc_fence_after();
  if (warp == 1) {
    if constexpr (P::PAIR)
      tmem_dealloc_pair(tmem, P::TMEM_COLS);
    else
      tmem_dealloc(tmem, P::TMEM_COLS);
  }
}

// Default no-op hooks for problems that need none.
struct ProblemBase {
  static constexpr int EP_SMEM = 0;
  static constexpr bool PRELOAD = false;  // true: static tiles, load_w / load_x split of load
  static constexpr int KB = 1;            // k-blocks per ring stage
  static constexpr bool F8 = false;       // E4M3 operands (kind::f8f6f4): a k-block is 128 elements
  static constexpr bool DYNAMIC = false;  // tiles from the global counter p.sched (see above)
  static constexpr bool ACQUIRE = false;  // acquire(): the producer waits before loading a tile
  static constexpr bool PAIR = false;     // M = 256 tiles over a cluster of two CTAs (see above)
  template <class Params>
  DG_DEVINL static Tile local(const Params&, Tile t, int rank) {
    t.half = rank;
    return t;
  }
  template <class Params>
  DG_DEVINL static void epilogue_init(const Params&, int, uint8_t*) {}
  template <class Params>
  DG_DEVINL static void finish(const Params&, int, uint8_t*) {}
  template <class Params>
  DG_DEVINL static void epilogue_prefetch(const Params&, const Tile&, int) {}
  template <class Params>
  DG_DEVINL static bool acquire(const Params&, const Tile&, volatile int*, int*) { return true; }
  template <class Params>
  DG_DEVINL static void load_w(const Params&, const Tile&, int, uint32_t, uint32_t, uint64_t*) {}
  template <class Params>
  DG_DEVINL static void load_x(const Params&, const Tile&, int, uint32_t, uint32_t, uint64_t*) {}
};

DG_DEVINL void prefetch_l1(const void* ptr) { asm volatile("prefetch.global.L1 [%0];" ::"l"(ptr)); }

DG_DEVINL int round_up16(int n) { return (n + 15) & ~15; }

}  // namespace dg
