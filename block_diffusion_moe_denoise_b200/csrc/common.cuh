// Shared device helpers for the sm_100a kernels: bf16 conversion, the device
// error word, bounded mbarrier waits, TMA tile loads and the tcgen05
// (5th-generation tensor core + tensor memory) instructions used by the GEMMs.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define DG_DEVINL __device__ __forceinline__

// Bits of the device error word (atomicOr'ed by kernels, read by the host).
enum : int {
  DG_DEVERR_TOKEN = 1,         // token id outside [0, vocab)
  DG_DEVERR_TIMEOUT = 2,       // a bounded barrier wait gave up
  DG_DEVERR_CAPACITY = 4,      // a device-side list overflowed
  DG_DEVERR_NAN = 8,           // non-finite value in a reduction
};

// Upper bound on one barrier wait (ns).  Far above any legitimate wait in a
// single kernel; after it the kernel records DG_DEVERR_TIMEOUT and unwinds.
#define DG_WAIT_LIMIT_NS 2000000000ull

// Programmatic dependent launch: every kernel of the pass is launched so that
// it may start while its predecessor in the stream drains.  A kernel lets its
// successor be scheduled (pdl_trigger) and then waits for the predecessor to
// complete and its writes to be visible (pdl_wait) before touching anything
// the predecessor produced.  Every CTA waits unconditionally, so completion
// stays transitive along the stream.  A kernel that starts early this way can
// still find lines of a buffer in its SM's L1 that are older than what its
// predecessors wrote there (measured: the residual norm, reading the shared
// expert's output written by the routed-expert launch, picked up stale values
// in about one canvas segment in four); CUDA-core kernels therefore read
// data produced earlier in the pass with ld.global.cg (__ldcg, L2 only).  TMA
// loads do not go through L1.
DG_DEVINL void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
DG_DEVINL void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

DG_DEVINL uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

DG_DEVINL uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

DG_DEVINL float bf2f(__nv_bfloat16 v) { return __bfloat162float(v); }
DG_DEVINL __nv_bfloat16 f2bf(float v) { return __float2bfloat16_rn(v); }

DG_DEVINL uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

DG_DEVINL float silu_f(float v) { return v / (1.0f + __expf(-v)); }

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
DG_DEVINL void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

DG_DEVINL void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

DG_DEVINL void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

DG_DEVINL void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

DG_DEVINL void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// A waiting thread may be suspended inside try_wait; the hint caps that
// suspension (ns).  Measured on B200 with a TMA ring streaming from L2: the
// hardware default costs ~15% of the per-stage handoff rate, a 20 ns cap
// (re-polled by the caller's loop) does not.
constexpr uint32_t kWaitHintNs = 20;

DG_DEVINL bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kWaitHintNs)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete.  Gives up when
// `*abort` becomes nonzero (another role of the CTA gave up) or after
// DG_WAIT_LIMIT_NS; on its own timeout it sets `*abort` and the error word.
DG_DEVINL bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort, int* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > DG_WAIT_LIMIT_NS) {
      *abort = 1;
      if (err) atomicOr(err, DG_DEVERR_TIMEOUT);
      return false;
    }
  }
}

// Wait (bounded like mbar_wait_bounded) until the counter reaches target;
// acquire ordering, then a proxy fence so that TMA loads issued afterwards see
// the data the counted writers stored before their release.
DG_DEVINL bool counter_wait_bounded(const int* ctr, int target, volatile int* abort, int* err) {
  auto load = [&]() {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
    return v;
  };
  if (load() < target) {
    const uint64_t t0 = globaltimer_ns();
    while (load() < target) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > DG_WAIT_LIMIT_NS) {
        *abort = 1;
        if (err) atomicOr(err, DG_DEVERR_TIMEOUT);
        return false;
      }
      __nanosleep(64);
    }
  }
  asm volatile("fence.proxy.async.global;" ::: "memory");
  return true;
}

// Release side of counter_wait_bounded for data written by this thread.
DG_DEVINL void counter_release_fence() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
  __threadfence();
}

// ---------------------------------------------------------------------------
// TMA (bulk tensor copies global -> shared, completion on an mbarrier)
// ---------------------------------------------------------------------------
DG_DEVINL void tma_load_2d(uint32_t dst_smem, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst_smem),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// TMA load by either CTA of a pair into its own shared memory, completing on
// the mbarrier at `bar`'s offset in the pair's even CTA.
DG_DEVINL void tma_load_2d_pair(uint32_t dst_smem, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b32 lb;\n\t"
      "mapa.shared::cluster.u32 lb, %4, 0;\n\t"
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [lb];\n\t}"
      ::"r"(dst_smem), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

DG_DEVINL void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------------------
// Distributed shared memory of the CTAs of a cluster.
DG_DEVINL uint32_t dsmem_addr(uint32_t local_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_addr), "r"(rank));
  return r;
}
DG_DEVINL float4 ld_dsmem_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
DG_DEVINL float ld_dsmem_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
DG_DEVINL float2 ld_dsmem_f2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared::cluster.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr) : "memory");
  return v;
}
// Every thread of every CTA of the cluster; orders this CTA's earlier shared
// memory writes before the other CTAs' later reads of them.
DG_DEVINL void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory allocation, MMA, commit, loads, fences
// ---------------------------------------------------------------------------
DG_DEVINL void tmem_alloc(uint32_t* dst_smem_slot, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem_slot)),
               "r"(ncols));
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
}

DG_DEVINL void tmem_dealloc(uint32_t taddr, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}

DG_DEVINL void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
DG_DEVINL void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, bf16 inputs, fp32 accumulator.
DG_DEVINL void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, E4M3 inputs (K = 32 per
// instruction, the same 32 bytes of each 128-byte row as a bf16 K = 16 step),
// fp32 accumulator.
DG_DEVINL void umma_e4m3(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T: A (M = 128 rows, one per lane, bf16
// pairs per 32-bit column, K-major) read from tensor memory.
DG_DEVINL void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when all previously issued MMAs of this thread complete.
DG_DEVINL void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// ---- CTA pairs (tcgen05 .cta_group::2): one MMA of M = 256 spans two CTAs of
// a cluster; each holds half of A (128 rows) and half of B (N/2 rows) in its
// own shared memory at the same offsets and its 128 rows x N of D in its own
// tensor memory.  The even CTA of the pair issues the MMAs.
DG_DEVINL uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Both CTAs' warps with the same warp index allocate together.
DG_DEVINL void tmem_alloc_pair(uint32_t* dst_smem_slot, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem_slot)),
               "r"(ncols));
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
}

DG_DEVINL void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}

DG_DEVINL void umma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives once (when the pair's earlier MMAs complete) on the mbarrier at this
// shared-memory offset in both CTAs of the pair.
DG_DEVINL void umma_commit_pair(uint64_t* bar) {
  const uint16_t both = 3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(both)
      : "memory");
}

// Arrival on the mbarrier at this offset in CTA `rank` of the cluster.
DG_DEVINL void mbar_arrive_remote(uint64_t* bar, uint32_t rank) {
  asm volatile(
      "{\n\t.reg .b32 ra;\n\t"
      "mapa.shared::cluster.u32 ra, %0, %1;\n\t"
      "mbarrier.arrive.release.cluster.shared::cluster.b64 _, [ra];\n\t}" ::"r"(smem_u32(bar)),
      "r"(rank)
      : "memory");
}

// Instruction descriptor for kind::f16 with bf16 A/B, fp32 D, both K-major,
// M = 128, N = n (multiple of 16, 16..256).
DG_DEVINL uint32_t umma_idesc_bf16(uint32_t m, uint32_t n) {
  return (1u << 4)            // D format: f32
         | (1u << 7)          // A format: bf16
         | (1u << 10)         // B format: bf16
         | ((n >> 3) << 17)   // N >> 3
         | ((m >> 4) << 24);  // M >> 4
}

// Instruction descriptor for kind::f8f6f4 with E4M3 A/B (format code 0), fp32 D,
// both K-major, M = 128, N = n (multiple of 16, 16..256).
DG_DEVINL uint32_t umma_idesc_e4m3(uint32_t m, uint32_t n) {
  return (1u << 4)            // D format: f32
         | (0u << 7)          // A format: e4m3
         | (0u << 10)         // B format: e4m3
         | ((n >> 3) << 17)   // N >> 3
         | ((m >> 4) << 24);  // M >> 4
}

// Shared-memory matrix descriptor for a K-major operand tile stored as rows of
// 128 bytes (64 bf16) with the 128-byte swizzle, 8-row groups 1024 bytes apart.
// `addr` must lie in a 1024-byte aligned tile (plus a k offset of 32*j bytes).
DG_DEVINL uint64_t umma_sdesc_k128(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFF);          // start address
  d |= (uint64_t)1 << 16;                         // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;               // stride byte offset: 8 rows * 128 B
  d |= (uint64_t)1 << 46;                         // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                         // layout: 128-byte swizzle
  return d;
}

DG_DEVINL void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Split form of tmem_ld16: issue several loads, then one wait.  The wait
// names the destination registers as in/out operands so that no use of them
// can be scheduled before it.
DG_DEVINL void tmem_ld16_issue(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

DG_DEVINL void tmem_ld_wait16(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15])
               :
               : "memory");
}

// 2^x with the hardware approximation (single MUFU op, denormals flushed).
DG_DEVINL float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

DG_DEVINL void tmem_st16(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
      "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
      "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])));
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

DG_DEVINL void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------
// K cache layout.  Per (request, layer, KV head) the keys are stored in tiles
// of 64 positions, and inside a tile by 64-dimension block:
//   [cap / 64][D / 64][64 positions][64 dims]
// so one 64-position K tile of every dimension is a single contiguous run of
// D rows of 128 bytes -- one TMA box instead of D / 64 of them -- that lands
// in shared memory as the [D / 64][64][128 B] operand the S MMAs read.
// Element offset of (position, dim) from the head's base; cap % 64 == 0.
// ---------------------------------------------------------------------------
DG_DEVINL size_t k_tile_offset(long long pos, int dim, int D) {
  return (size_t)(pos >> 6) * 64 * D + (size_t)(dim >> 6) * 4096 + (size_t)(pos & 63) * 64 + (dim & 63);
}

// ---------------------------------------------------------------------------
// misc
// ---------------------------------------------------------------------------
DG_DEVINL float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

DG_DEVINL int warp_sum_int(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

DG_DEVINL float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// ---------------------------------------------------------------------------
// Philox-4x32-10 (Salmon et al., SC'11): ten rounds of two 32x32->64-bit
// multiplies with the high halves XORed into the odd words and the round key,
// key bumped by the Weyl constants between rounds.  Returns all four words.
// ---------------------------------------------------------------------------
DG_DEVINL uint4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, uint32_t k0, uint32_t k1) {
  constexpr uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u, W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += W0;
      k1 += W1;
    }
    const uint32_t lo0 = M0 * c0, hi0 = __umulhi(M0, c0);
    const uint32_t lo1 = M1 * c2, hi1 = __umulhi(M1, c2);
    const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  return make_uint4(c0, c1, c2, c3);
}

// A 32-bit word as an odd multiple of 2^-24 in (0, 1): (2 (w >> 9) + 1) / 2^24,
// exact in float32 and never 0 or 1.
DG_DEVINL float word_uniform(uint32_t w) { return (float)(2u * (w >> 9) + 1u) * 5.9604644775390625e-8f; }
