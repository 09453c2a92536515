// Canvas attention: every canvas (or prefill segment) query attends, with no
// mask, to all committed keys of its request and to every key of its own
// segment (DiffusionGemma pages: bidirectional decoder pass over the canvas,
// "What DiffusionGemma is"; every token sees every other token in its
// context, "26B MoE Architecture, but Only 3.8B Activated").
//
// FlashAttention-style single pass with online softmax (exp2 domain), GQA:
// the G = Hq/Hkv query heads of a KV head are stacked as G*Tr query rows so one
// CTA's K/V tiles serve all of them.  64 query rows x 64-key tiles per CTA,
// 4 warps x 16 rows, bf16 mma.sync m16n8k16 with fp32 accumulation, K/V tiles
// double-buffered through cp.async into XOR-swizzled shared memory.  The key
// range is split across CTAs (split-KV) when the query tiles alone cannot fill
// the GPU; partial (O, max, sum) are merged by k_attn_combine.
#include "common.cuh"
#include "dg_internal.h"

namespace dg {

DG_DEVINL void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0) : "memory");
}
DG_DEVINL void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
DG_DEVINL void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

DG_DEVINL void ldsm_x4(uint32_t* r, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
DG_DEVINL void ldsm_x4_t(uint32_t* r, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
DG_DEVINL void mma_bf16_16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

constexpr int kBQ = 64, kBK = 64;

// byte offset of 16-byte chunk `ch` of row `r` in a [rows][D] bf16 tile whose
// chunk index is XOR-swizzled with (r mod 8)
template <int D>
DG_DEVINL uint32_t swz(int r, int ch) {
  return (uint32_t)(r * D * 2 + ((ch ^ (r & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(128, 1) k_attn(const AttnArgs a) {
  constexpr int CH = D / 8;  // 16-byte chunks per row
  extern __shared__ __align__(128) uint8_t asmem[];
  const uint32_t sQ = smem_u32(asmem);
  const uint32_t sK0 = sQ + kBQ * D * 2;
  const uint32_t sV0 = sK0 + 2 * kBK * D * 2;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.Hq / a.Hkv;
  const int slot = blockIdx.y / a.Hkv, g = blockIdx.y % a.Hkv;
  const int rows = G * a.Tr;
  const int r0 = blockIdx.x * kBQ;
  const int n_keys = a.n_keys[slot];
  int per = (n_keys + a.n_split - 1) / a.n_split;
  per = (per + kBK - 1) / kBK * kBK;
  const int k_begin = blockIdx.z * per;
  const int k_end = min(n_keys, k_begin + per);
  const int n_tiles = k_end > k_begin ? (k_end - k_begin + kBK - 1) / kBK : 0;
  const bf16* Kg = a.kv + (size_t)a.req[slot] * a.req_stride + (size_t)g * a.cap * D;
  const bf16* Vg = Kg + (size_t)a.Hkv * a.cap * D;

  // Q tile
  for (int c = tid; c < kBQ * CH; c += 128) {
    const int r = c / CH, ch = c % CH;
    const int qr = r0 + r;
    const bool ok = qr < rows;
    const int h = g * G + (ok ? qr / a.Tr : 0);
    const int t = slot * a.Tr + (ok ? qr % a.Tr : 0);
    cp_async16(sQ + swz<D>(r, ch), a.q + ((size_t)h * a.q_T + t) * D + ch * 8, ok);
  }
  auto load_kv = [&](int it, int buf) {
    const int key0 = k_begin + it * kBK;
    const uint32_t sk = sK0 + buf * kBK * D * 2, sv = sV0 + buf * kBK * D * 2;
    for (int c = tid; c < kBK * CH; c += 128) {
      const int r = c / CH, ch = c % CH;
      const int key = key0 + r;
      const bool ok = key < k_end;
      const size_t off = (size_t)(ok ? key : k_begin) * D + ch * 8;
      cp_async16(sk + swz<D>(r, ch), Kg + off, ok);
      cp_async16(sv + swz<D>(r, ch), Vg + off, ok);
    }
  };
  if (n_tiles > 0) load_kv(0, 0);
  cp_async_commit();

  float o[D / 8][4];
#pragma unroll
  for (int j = 0; j < D / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
  const float sl2 = a.scale * 1.4426950408889634f;

  for (int it = 0; it < n_tiles; ++it) {
    const int buf = it & 1;
    if (it + 1 < n_tiles) {
      load_kv(it + 1, buf ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint32_t sk = sK0 + buf * kBK * D * 2, sv = sV0 + buf * kBK * D * 2;

    float s[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t af[4];
      {
        const int r = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        ldsm_x4(af, sQ + swz<D>(r, kk * 2 + (lane >> 4)));
      }
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t bf[4];
        const int key = np * 16 + (lane & 7) + (lane >> 4) * 8;
        ldsm_x4(bf, sk + swz<D>(key, kk * 2 + ((lane >> 3) & 1)));
        mma_bf16_16816(s[2 * np], af, bf[0], bf[1]);
        mma_bf16_16816(s[2 * np + 1], af, bf[2], bf[3]);
      }
    }
    // online softmax (rows lane/4 and lane/4 + 8 of this warp's 16)
    const int key0 = k_begin + it * kBK;
    float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = key0 + j * 8 + (lane & 3) * 2 + (e & 1);
        const float v = key < k_end ? s[j][e] * sl2 : -INFINITY;
        s[j][e] = v;
        if (e < 2) mx_a = fmaxf(mx_a, v);
        else mx_b = fmaxf(mx_b, v);
      }
    }
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
    const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
    const float mu_a = mn_a == -INFINITY ? 0.f : mn_a, mu_b = mn_b == -INFINITY ? 0.f : mn_b;
    const float al_a = exp2f(m_a - mu_a), al_b = exp2f(m_b - mu_b);
    m_a = mn_a;
    m_b = mn_b;
    float rs_a = 0.f, rs_b = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      s[j][0] = exp2f(s[j][0] - mu_a);
      s[j][1] = exp2f(s[j][1] - mu_a);
      s[j][2] = exp2f(s[j][2] - mu_b);
      s[j][3] = exp2f(s[j][3] - mu_b);
      rs_a += s[j][0] + s[j][1];
      rs_b += s[j][2] + s[j][3];
    }
    l_a = l_a * al_a + rs_a;
    l_b = l_b * al_b + rs_b;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      o[j][0] *= al_a;
      o[j][1] *= al_a;
      o[j][2] *= al_b;
      o[j][3] *= al_b;
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t pf[4];
      pf[0] = pack_bf16x2(s[2 * kk][0], s[2 * kk][1]);
      pf[1] = pack_bf16x2(s[2 * kk][2], s[2 * kk][3]);
      pf[2] = pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pf[3] = pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
      const int key = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int dp = 0; dp < D / 16; ++dp) {
        uint32_t bf[4];
        ldsm_x4_t(bf, sv + swz<D>(key, dp * 2 + (lane >> 4)));
        mma_bf16_16816(o[2 * dp], pf, bf[0], bf[1]);
        mma_bf16_16816(o[2 * dp + 1], pf, bf[2], bf[3]);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);

#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int qr = r0 + warp * 16 + (lane >> 2) + half * 8;
    if (qr >= rows) continue;
    const int h = g * G + qr / a.Tr;
    const int t = slot * a.Tr + qr % a.Tr;
    const float l = half ? l_b : l_a;
    const float m = half ? m_b : m_a;
    if (a.n_split == 1) {
      const float inv = l > 0.f ? 1.f / l : 0.f;
      uint32_t* dst = reinterpret_cast<uint32_t*>(a.o + (size_t)t * a.Hq * D + (size_t)h * D);
#pragma unroll
      for (int j = 0; j < D / 8; ++j)
        dst[(j * 8 + (lane & 3) * 2) >> 1] = pack_bf16x2(o[j][2 * half] * inv, o[j][2 * half + 1] * inv);
    } else {
      const size_t row = ((size_t)blockIdx.z * a.Hq + h) * a.q_T + t;
      float2* dst = reinterpret_cast<float2*>(a.part_o + row * D);
#pragma unroll
      for (int j = 0; j < D / 8; ++j) dst[(j * 8 + (lane & 3) * 2) >> 1] = make_float2(o[j][2 * half], o[j][2 * half + 1]);
      if ((lane & 3) == 0) a.part_ml[row] = make_float2(m, l);
    }
  }
}

// Merge of the split-KV partials: O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s.
__global__ void k_attn_combine(const float* __restrict__ part_o, const float2* __restrict__ part_ml, int n_split,
                               int Hq, int q_T, int T, int D, bf16* __restrict__ o) {
  const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= T * Hq) return;
  const int t = w / Hq, h = w % Hq;
  float M = -INFINITY;
  for (int s = 0; s < n_split; ++s) {
    const float2 ml = part_ml[((size_t)s * Hq + h) * q_T + t];
    if (ml.y > 0.f) M = fmaxf(M, ml.x);
  }
  float L = 0.f;
  float wts[16];
  for (int s = 0; s < n_split; ++s) {
    const float2 ml = part_ml[((size_t)s * Hq + h) * q_T + t];
    wts[s] = ml.y > 0.f ? exp2f(ml.x - M) : 0.f;
    L += wts[s] * ml.y;
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  for (int c = lane * 2; c < D; c += 64) {
    float ax = 0.f, ay = 0.f;
    for (int s = 0; s < n_split; ++s) {
      if (wts[s] == 0.f) continue;
      const float2 v = *reinterpret_cast<const float2*>(part_o + (((size_t)s * Hq + h) * q_T + t) * D + c);
      ax += wts[s] * v.x;
      ay += wts[s] * v.y;
    }
    *reinterpret_cast<uint32_t*>(o + (size_t)t * Hq * D + (size_t)h * D + c) = pack_bf16x2(ax * inv, ay * inv);
  }
}

int attention_split_cap() { return 16; }

template <int D>
static cudaError_t launch_attn(const AttnArgs& a, cudaStream_t st) {
  const size_t smem = (size_t)(kBQ + 4 * kBK) * D * 2;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(k_attn<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int G = a.Hq / a.Hkv;
  dim3 grid((G * a.Tr + kBQ - 1) / kBQ, a.Hkv * a.n_slots, a.n_split);
  k_attn<D><<<grid, 128, smem, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || a.n_split == 1) return e;
  const int T = a.n_slots * a.Tr;
  const int warps = T * a.Hq;
  k_attn_combine<<<(warps + 7) / 8, 256, 0, st>>>(a.part_o, a.part_ml, a.n_split, a.Hq, a.q_T, T, D, a.o);
  return cudaGetLastError();
}

cudaError_t run_attention(const AttnArgs& a, cudaStream_t st) {
  if (a.n_split < 1 || a.n_split > attention_split_cap()) return cudaErrorInvalidValue;
  switch (a.D) {
    case 64: return launch_attn<64>(a, st);
    case 128: return launch_attn<128>(a, st);
    case 256: return launch_attn<256>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dg
