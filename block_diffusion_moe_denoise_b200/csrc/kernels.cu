// CUDA-core kernels of the denoising pass: everything that is not a dense
// contraction.  Warp-shuffle reductions, 16-byte vector loads/stores.
#include <cuda_fp8.h>
#include <float.h>
#include <string.h>

#include "common.cuh"
#include "dg_internal.h"

namespace dg {

// ---------------------------------------------------------------------------
// Embedding gather: x[t, :] = E[id_t, :] (fp32 residual stream), and each
// token's absolute position and request.
// ---------------------------------------------------------------------------
struct EmbedParams {
  SlotInfo s;
  const int* ids[DG_MAX_REQUESTS];
};

__global__ void k_embed(EmbedParams p, const bf16* __restrict__ embed, int V, int d, float* __restrict__ x,
                        int* tok_pos, int* tok_req, const double* __restrict__ inv_freq, int half,
                        float2* __restrict__ rope, int* err) {
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.x;
  const int slot = t / p.s.Tr;
  const int i = t - slot * p.s.Tr;
  int id = p.ids[slot][i];
  if (id < 0 || id >= V) {
    if (threadIdx.x == 0) atomicOr(err, DG_DEVERR_TOKEN);
    id = 0;
  }
  const int pos = p.s.pos0[slot] + i;
  if (threadIdx.x == 0) {
    tok_pos[t] = pos;
    tok_req[t] = p.s.req[slot];
  }
  // RoPE (cos, sin) of this token's position for every frequency: the angle in
  // fp64, reduced to [-pi, pi] before the fp32 sincos; shared by all layers.
  for (int f = threadIdx.x; f < half; f += blockDim.x) {
    double a = (double)pos * inv_freq[f];
    a -= rint(a * 0.15915494309189535) * 6.283185307179586;
    float sn, cs;
    sincosf((float)a, &sn, &cs);
    rope[(size_t)t * half + f] = make_float2(cs, sn);
  }
  const uint4* src = reinterpret_cast<const uint4*>(embed + (size_t)id * d);
  float4* dst = reinterpret_cast<float4*>(x + (size_t)t * d);
  for (int c = threadIdx.x; c < d / 8; c += blockDim.x) {
    const uint4 v = src[c];
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
    const float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
    const float2 e = __bfloat1622float2(h[2]), f = __bfloat1622float2(h[3]);
    dst[2 * c] = make_float4(a.x, a.y, b.x, b.y);
    dst[2 * c + 1] = make_float4(e.x, e.y, f.x, f.y);
  }
}

cudaError_t run_embed(const int* const* ids, const SlotInfo& s, const bf16* embed, int V, int d, float* x,
                      int* tok_pos, int* tok_req, const double* inv_freq, int half, float2* rope, int* err,
                      cudaStream_t st) {
  EmbedParams p;
  p.s = s;
  for (int i = 0; i < DG_MAX_REQUESTS; ++i) p.ids[i] = i < s.n ? ids[i] : nullptr;
  const int T = s.n * s.Tr;
  if (T == 0) return cudaSuccess;
  {
    const cudaError_t e_ = launch_pdl(k_embed, dim3(T), dim3(128), 0, st, p, embed, V, d, x, tok_pos, tok_req, inv_freq, half, rope, err);
    if (e_ != cudaSuccess) return e_;
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// RMSNorm: out = bf16(x / sqrt(mean(x^2) + eps) * g), one warp per row.
// ---------------------------------------------------------------------------
__global__ void k_rmsnorm(const float* __restrict__ x, const float* __restrict__ g, int T, int d, float eps,
                          bf16* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= T) return;
  const float4* xr = reinterpret_cast<const float4*>(x + (size_t)row * d);
  float ss = 0.f;
  for (int c = lane; c < d / 4; c += 32) {
    const float4 v = __ldcg(xr + c);
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  ss = warp_sum(ss);
  const float rs = rsqrtf(ss / (float)d + eps);
  const float4* g4 = reinterpret_cast<const float4*>(g);
  uint2* o = reinterpret_cast<uint2*>(out + (size_t)row * d);
  for (int c = lane; c < d / 4; c += 32) {
    const float4 v = __ldcg(xr + c);
    const float4 w = g4[c];
    o[c] = make_uint2(pack_bf16x2(v.x * rs * w.x, v.y * rs * w.y), pack_bf16x2(v.z * rs * w.z, v.w * rs * w.w));
  }
}

cudaError_t run_rmsnorm(const float* x, const float* g, int T, int d, float eps, bf16* out, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  {
    const cudaError_t e_ = launch_pdl(k_rmsnorm, dim3((T + 7) / 8), dim3(256), 0, st, x, g, T, d, eps, out);
    if (e_ != cudaSuccess) return e_;
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Residual update + RMSNorm, one CTA per token row, 8 consecutive features per
// thread so every input row is read with all loads in flight at once:
//   x[t] += sum_j Yp[row(t, j)] + sum_s part[s][t]
//   out[t] = bf16(x[t] / sqrt(mean(x[t]^2) + eps) * g)
// The routed experts' outputs (slot order) and the split-K partials (slice
// order) are added in a fixed order, so the result is deterministic.
// ---------------------------------------------------------------------------
// One CTA per SM at most by registers on purpose: the GEMM launched after it
// (programmatic dependent launch) must find room on every SM to become
// resident and start its weight loads while this kernel still runs.
__global__ void __launch_bounds__(512) k_residual_norm(float* __restrict__ x, const bf16* __restrict__ yp,
                                                        const int* __restrict__ pair_row, int k,
                                                        const float* __restrict__ part, int n_part,
                                                        size_t part_stride, const float* __restrict__ g, int d,
                                                        float eps, bf16* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[32];
  const int t = blockIdx.x;
  const int c = threadIdx.x * 2;  // first of this thread's two float4 columns
  float4* xr = reinterpret_cast<float4*>(x + (size_t)t * d);
  int rows[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) rows[j] = j < k ? __ldcg(pair_row + (size_t)t * k + j) : 0;
  float4 v[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    v[h] = __ldcg(xr + c + h);
    uint2 y[8];  // 4 bf16
    float4 q[kMaxPartSplits];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < k) y[j] = __ldcg(reinterpret_cast<const uint2*>(yp + (size_t)rows[j] * d) + c + h);
#pragma unroll
    for (int j = 0; j < kMaxPartSplits; ++j)
      if (j < n_part) q[j] = __ldcg(reinterpret_cast<const float4*>(part + j * part_stride + (size_t)t * d) + c + h);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < k) {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&y[j].x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&y[j].y));
        v[h].x += a.x;
        v[h].y += a.y;
        v[h].z += b.x;
        v[h].w += b.y;
      }
#pragma unroll
    for (int j = 0; j < kMaxPartSplits; ++j)
      if (j < n_part) {
        v[h].x += q[j].x;
        v[h].y += q[j].y;
        v[h].z += q[j].z;
        v[h].w += q[j].w;
      }
  }
  if (k || n_part) {
    xr[c] = v[0];
    xr[c + 1] = v[1];
  }
  if (out == nullptr) return;
  float ss = 0.f;
#pragma unroll
  for (int h = 0; h < 2; ++h) ss += v[h].x * v[h].x + v[h].y * v[h].y + v[h].z * v[h].z + v[h].w * v[h].w;
  ss = warp_sum(ss);
  const int nw = blockDim.x >> 5;
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float r = threadIdx.x < nw ? red[threadIdx.x] : 0.f;
    r = warp_sum(r);
    if (threadIdx.x == 0) red[0] = r;
  }
  __syncthreads();
  const float rs = rsqrtf(red[0] / (float)d + eps);
  const float4* g4 = reinterpret_cast<const float4*>(g);
  uint4 o;
  {
    const float4 w0 = g4[c], w1 = g4[c + 1];
    o.x = pack_bf16x2(v[0].x * rs * w0.x, v[0].y * rs * w0.y);
    o.y = pack_bf16x2(v[0].z * rs * w0.z, v[0].w * rs * w0.w);
    o.z = pack_bf16x2(v[1].x * rs * w1.x, v[1].y * rs * w1.y);
    o.w = pack_bf16x2(v[1].z * rs * w1.z, v[1].w * rs * w1.w);
  }
  reinterpret_cast<uint4*>(out + (size_t)t * d)[threadIdx.x] = o;
}

cudaError_t run_residual_norm(float* x, const bf16* yp, const int* pair_row, int k, const float* part, int n_part,
                              int Tcap, const float* g, int T, int d, float eps, bf16* out, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  if (n_part > kMaxPartSplits || k > 8 || d % 256 != 0 || d > 4096) return cudaErrorInvalidValue;
  {
    const cudaError_t e_ = launch_pdl(k_residual_norm, dim3(T), dim3(d / 8), 0, st, x, yp, pair_row, k, part, n_part,
                                      (size_t)Tcap * d, g, d, eps, out);
    if (e_ != cudaSuccess) return e_;
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Router top-k: one warp per token over E <= 256 fp32 logits.  Picks the k
// largest in descending order (ties to the lower expert id) and the softmax of
// the picked logits.
// ---------------------------------------------------------------------------
DG_DEVINL void topk_warp(const float* vals, int E, int k, int* idx_out, float* w_out) {
  const int lane = threadIdx.x & 31;
  float v[8];
  unsigned taken = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = lane + 32 * j;
    v[j] = e < E ? vals[e] : -INFINITY;
    if (e >= E) taken |= 1u << j;
  }
  float sel_v[8];
  int sel_i[8];
  for (int r = 0; r < k; ++r) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane + 32 * j;
      if (!(taken & (1u << j)) && (v[j] > bv || (v[j] == bv && e < bi))) {
        bv = v[j];
        bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (bi != 0x7fffffff && (bi & 31) == lane) taken |= 1u << (bi >> 5);
    sel_v[r] = bv;
    sel_i[r] = bi;
  }
  if (lane == 0) {
    float sum = 0.f, e[8];
    for (int r = 0; r < k; ++r) {
      e[r] = expf(sel_v[r] - sel_v[0]);
      sum += e[r];
    }
    for (int r = 0; r < k; ++r) {
      idx_out[r] = sel_i[r];
      w_out[r] = e[r] / sum;
    }
  }
}

__global__ void k_topk(const float* __restrict__ logits, int T, int E, int k, int* idx, float* w) {
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  topk_warp(logits + (size_t)t * E, E, k, idx + (size_t)t * k, w + (size_t)t * k);
}

cudaError_t run_topk(const float* logits, int T, int E, int k, int* idx, float* w, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  {
    const cudaError_t e_ = launch_pdl(k_topk, dim3((T + 7) / 8), dim3(256), 0, st, logits, T, E, k, idx, w);
    if (e_ != cudaSuccess) return e_;
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Expert grouping (single CTA, the operation-level entry point): per-expert
// counts, exclusive offsets and the row of every (token, slot) pair in
// expert-grouped order (tokens ascending inside an expert, via per-expert token
// bitmasks).  The decoder pass uses k_group_gather, which also builds the GEMM
// tile lists and gathers the rows.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) k_group(GroupArgs a) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ int gsm[];
  const int E = a.E, T = a.T, k = a.k;
  const int MW = (T + 31) >> 5;
  int* cnt = gsm;                 // [E]
  int* off = cnt + E;             // [E+1]
  unsigned* mask = reinterpret_cast<unsigned*>(off + E + 1);  // [E][MW]
  const int tid = threadIdx.x;
  for (int i = tid; i < E; i += blockDim.x) cnt[i] = 0;
  for (int i = tid; i < E * MW; i += blockDim.x) mask[i] = 0u;
  __syncthreads();
  const int P = T * k;
  for (int p = tid; p < P; p += blockDim.x) {
    const int e = a.idx[p];
    const int t = p / k;
    if (e < 0 || e >= E) {
      atomicOr(a.err, DG_DEVERR_TOKEN);
      continue;
    }
    atomicAdd(&cnt[e], 1);
    atomicOr(&mask[e * MW + (t >> 5)], 1u << (t & 31));
  }
  __syncthreads();
  if (tid == 0) {
    off[0] = 0;
    for (int e = 0; e < E; ++e) off[e + 1] = off[e] + cnt[e];
    if (a.route_stats) {
      int touched = 0;
      for (int e = 0; e < E; ++e) touched += cnt[e] > 0;
      atomicAdd(&a.route_stats[0], (unsigned long long)touched);
      atomicAdd(&a.route_stats[1], 1ull);
    }
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    a.counts[e] = cnt[e];
    a.offsets[e] = off[e];
  }
  if (tid == 0) a.offsets[E] = off[E];
  for (int p = tid; p < P; p += blockDim.x) {
    const int e = a.idx[p];
    if (e < 0 || e >= E) continue;
    const int t = p / k;
    const unsigned* m = mask + e * MW;
    int rank = __popc(m[t >> 5] & ((1u << (t & 31)) - 1u));
    for (int wi = 0; wi < (t >> 5); ++wi) rank += __popc(m[wi]);
    const int row = off[e] + rank;
    a.pair_row[p] = row;
    a.row_token[row] = t;
    a.row_weight[row] = a.w[p];
    a.row_pair[row] = p;
  }
}

cudaError_t run_group(const GroupArgs& a, cudaStream_t st) {
  const int MW = (a.T + 31) >> 5;
  const size_t smem = (size_t)(2 * a.E + 1 + a.E * MW) * sizeof(int);
  static size_t configured = 0;
  if (smem > configured) {
    cudaError_t e = cudaFuncSetAttribute(k_group, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = smem;
  }
  {
    const cudaError_t e_ = launch_pdl(k_group, dim3(1), dim3(1024), smem, st, a);
    if (e_ != cudaSuccess) return e_;
  }
  return cudaGetLastError();
}

// Exclusive scan of 8 consecutive values per lane across a warp (256 values);
// rewrites vals8 with the exclusive prefixes and returns the total.
DG_DEVINL int warp_excl_scan8(int* vals8, int lane) {
  int run = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int v = vals8[i];
    vals8[i] = run;
    run += v;
  }
  int incl = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  const int base = incl - run;
#pragma unroll
  for (int i = 0; i < 8; ++i) vals8[i] += base;
  return __shfl_sync(0xffffffffu, incl, 31);
}

// ---------------------------------------------------------------------------
// Per-row E4M3 quantisation by one warp (row of n bf16 values, n % 8 == 0,
// n <= 4096): amax = max |x|; codes = E4M3(x * (448 / amax)) rounded to
// nearest even with saturation; scale = amax / 448 (both divisions and the
// product IEEE round-to-nearest in fp32); a zero row gives zero codes and
// scale 0.
// ---------------------------------------------------------------------------
DG_DEVINL void quant_row_warp(const bf16* __restrict__ src, int n, uint8_t* __restrict__ dst, float* scale,
                              int lane) {
  constexpr int kMaxChunks = 16;  // 4096 / 8 / 32
  const int n8 = n / 8;
  uint4 r[kMaxChunks];
  float amax = 0.f;
#pragma unroll
  for (int b = 0; b < kMaxChunks; ++b) {
    const int c = lane + 32 * b;
    if (c < n8) {
      r[b] = reinterpret_cast<const uint4*>(src)[c];
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&r[b]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h2[i]);
        amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
  }
  amax = warp_max(amax);
  const bool nz = amax > 0.f;
  const float s_inv = nz ? __fdiv_rn(448.f, amax) : 0.f;
#pragma unroll
  for (int b = 0; b < kMaxChunks; ++b) {
    const int c = lane + 32 * b;
    if (c < n8) {
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&r[b]);
      uint32_t w[2];
#pragma unroll
      for (int i = 0; i < 4; i += 2) {
        const float2 f0 = __bfloat1622float2(h2[i]), f1 = __bfloat1622float2(h2[i + 1]);
        const __nv_fp8x2_storage_t q0 =
            __nv_cvt_float2_to_fp8x2(make_float2(__fmul_rn(f0.x, s_inv), __fmul_rn(f0.y, s_inv)), __NV_SATFINITE,
                                     __NV_E4M3);
        const __nv_fp8x2_storage_t q1 =
            __nv_cvt_float2_to_fp8x2(make_float2(__fmul_rn(f1.x, s_inv), __fmul_rn(f1.y, s_inv)), __NV_SATFINITE,
                                     __NV_E4M3);
        w[i / 2] = (uint32_t)q0 | ((uint32_t)q1 << 16);
      }
      reinterpret_cast<uint2*>(dst)[c] = make_uint2(w[0], w[1]);
    }
  }
  if (lane == 0) *scale = nz ? __fdiv_rn(amax, 448.f) : 0.f;
}

__global__ void k_quant_rows(const bf16* __restrict__ in, int n, int rows, uint8_t* __restrict__ out,
                             float* __restrict__ scale) {
  pdl_trigger();
  pdl_wait();
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= rows) return;
  quant_row_warp(in + (size_t)r * n, n, out + (size_t)r * n, scale + r, threadIdx.x & 31);
}

cudaError_t run_quant_rows(const bf16* in, int n, int rows, uint8_t* out, float* scale, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  if (n % 8 != 0 || n > 4096) return cudaErrorInvalidValue;
  {
    const cudaError_t e_ = launch_pdl(k_quant_rows, dim3((rows + 7) / 8), dim3(256), 0, st, in, n, rows, out, scale);
    if (e_ != cudaSuccess) return e_;
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Routing after the router GEMM (every CTA): per-expert counts from the token
// bitmasks the router epilogue set and their
// exclusive scans (tiny, recomputed by each CTA); CTA 0 publishes counts,
// offsets, tile lists and statistics.  Each CTA then places its share of the
// (token, slot) pairs -- row = offset[e] + number of earlier tokens routed to
// e, so tokens ascend inside an expert -- and copies the token's normalised
// row into the expert-grouped buffer.  It also clears the other mask buffer
// (used by the previous layer, read by nobody now) for the next layer.
// ---------------------------------------------------------------------------
template <bool kF8>
__global__ void __launch_bounds__(512) k_group_gather(GroupArgs a, const unsigned* __restrict__ mask,
                                                      unsigned* __restrict__ mask_next, int MW,
                                                      const bf16* __restrict__ u, int d, bf16* __restrict__ xp,
                                                      uint8_t* __restrict__ xq, float* __restrict__ xs) {
  pdl_trigger();
  pdl_wait();
  __shared__ int cnt[256];
  __shared__ int off[257];
  __shared__ int toff[257];
  const int E = a.E, T = a.T, k = a.k, P = T * k;
  const int used = (T + 31) >> 5;  // words of each expert's mask this pass can have set
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int e = tid; e < E; e += blockDim.x) {
    int c = 0;
    for (int wi = 0; wi < used; ++wi) c += __popc(__ldcg(mask + (size_t)e * MW + wi));
    cnt[e] = c;
  }
  __syncthreads();
  if (warp == 0) {
    int v[8], tv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane * 8 + i;
      v[i] = e < E ? cnt[e] : 0;
      constexpr int kTileRows = kF8 ? kExpertRows : kExpertTileRows;  // token rows per expert tile
      tv[i] = e < E ? (cnt[e] + kTileRows - 1) / kTileRows : 0;
    }
    const int tot = warp_excl_scan8(v, lane);
    const int ttot = warp_excl_scan8(tv, lane);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane * 8 + i;
      if (e < E) {
        off[e] = v[i];
        toff[e] = tv[i];
      }
    }
    if (lane == 0) {
      off[E] = tot;
      toff[E] = ttot;
      if (blockIdx.x == 0) {
        const int egu = ttot * a.FJ, ed = ttot * a.MD;
        if (egu > a.egu_cap || ed > a.ed_cap || tot != P) atomicOr(a.err, DG_DEVERR_CAPACITY);
        *a.egu_count = min(egu, a.egu_cap);
        *a.ed_count = min(ed, a.ed_cap);
      }
    }
  }
  __syncthreads();
  if (blockIdx.x == 0) {
    int touched = 0;
    for (int e = tid; e < E; e += blockDim.x) {
      a.counts[e] = cnt[e];
      a.offsets[e] = off[e];
      touched += cnt[e] > 0;
    }
    if (tid == 0) a.offsets[E] = off[E];
    if (a.route_stats) {
      touched = warp_sum_int(touched);
      if (lane == 0) atomicAdd(&a.route_stats[0], (unsigned long long)touched);
      if (tid == 0) atomicAdd(&a.route_stats[1], 1ull);
    }
    for (int e = warp; e < E; e += blockDim.x >> 5) {
      const int n_nt = toff[e + 1] - toff[e];
      for (int i = lane; i < n_nt * (a.FJ + a.MD); i += 32) {
        const int nt = i / (a.FJ + a.MD), r = i % (a.FJ + a.MD);
        // .w: the token tile's index over all experts (its readiness counter)
        if (r < a.FJ) {
          const int slot = (toff[e] + nt) * a.FJ + r;
          if (slot < a.egu_cap) a.egu_tiles[slot] = make_int4(e, r, nt, toff[e] + nt);
        } else {
          const int slot = (toff[e] + nt) * a.MD + (r - a.FJ);
          if (slot < a.ed_cap) a.ed_tiles[slot] = make_int4(e, r - a.FJ, nt, toff[e] + nt);
        }
      }
    }
  }
  // the expert GEMMs that follow draw their tiles from these counters
  if (blockIdx.x == 0 && tid < 2 && a.sched != nullptr) a.sched[tid] = 0;
  if (blockIdx.x == 0 && a.ready != nullptr) {
    const int n_tt = min(toff[E], a.egu_cap / max(1, a.FJ));  // token tiles the lists can hold
    for (int i = tid; i < n_tt; i += blockDim.x) a.ready[i] = 0;
  }
  // clear the other mask buffer, sliced across CTAs
  for (int i = blockIdx.x * blockDim.x + tid; i < E * MW; i += gridDim.x * blockDim.x) mask_next[i] = 0u;
  // this CTA's pairs, one warp per pair
  const int per = (P + gridDim.x - 1) / gridDim.x;
  const int p0 = blockIdx.x * per, p1 = min(P, p0 + per);
  for (int p = p0 + warp; p < p1; p += blockDim.x >> 5) {
    const int e = __ldcg(a.idx + p);
    const int t = p / k;
    int rank = 0;
    if (e >= 0 && e < E) {
      const unsigned* m = mask + (size_t)e * MW;
      const int wt = t >> 5;
      for (int wi = lane; wi <= wt; wi += 32) {
        const unsigned mw = __ldcg(m + wi);
        const unsigned bits = wi < wt ? mw : (mw & ((1u << (t & 31)) - 1u));
        rank += __popc(bits);
      }
      rank = warp_sum_int(rank);
    }
    const int row = (e >= 0 && e < E) ? off[e] + rank : 0;
    if (lane == 0) {
      a.pair_row[p] = row;
      a.row_token[row] = t;
      a.row_weight[row] = __ldcg(a.w + p);
      a.row_pair[row] = p;
    }
    if constexpr (kF8) {  // FP8 experts: the row is quantised on the way (same codes for every copy)
      quant_row_warp(u + (size_t)t * d, d, xq + (size_t)row * d, xs + row, lane);
      continue;
    }
    // rows of up to 3072 features in flight at once (12 chunks of 16 bytes per lane)
    const uint4* src = reinterpret_cast<const uint4*>(u + (size_t)t * d);
    uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)row * d);
    const int n16 = d / 8;
    for (int c0 = lane; c0 < n16; c0 += 32 * 12) {
      uint4 r[12];
#pragma unroll
      for (int b = 0; b < 12; ++b)
        if (c0 + b * 32 < n16) r[b] = __ldcg(src + c0 + b * 32);
#pragma unroll
      for (int b = 0; b < 12; ++b)
        if (c0 + b * 32 < n16) dst[c0 + b * 32] = r[b];
    }
  }
}

cudaError_t run_route(const bf16* u, int d, bf16* xp, unsigned* mask, unsigned* mask_next, int MW,
                      const GroupArgs& a, cudaStream_t st, uint8_t* xq, float* xs) {
  if (a.T < 1 || a.T > DG_MAX_REQUESTS * 256 || a.E > 256 || MW * 32 < a.T) return cudaErrorInvalidValue;
  if (xq != nullptr && (d % 8 != 0 || d > 4096 || xs == nullptr)) return cudaErrorInvalidValue;
  // one pair per warp where the GPU allows (16 warps per CTA, one CTA per SM)
  const int P = a.T * a.k;
  const int grid = (P + 15) / 16 < 148 ? (P + 15) / 16 : 148;
  {
    const cudaError_t e_ = xq != nullptr ? launch_pdl(k_group_gather<true>, dim3(grid), dim3(512), 0, st, a, mask,
                                                      mask_next, MW, u, d, xp, xq, xs)
                                         : launch_pdl(k_group_gather<false>, dim3(grid), dim3(512), 0, st, a, mask,
                                                      mask_next, MW, u, d, xp, xq, xs);
    if (e_ != cudaSuccess) return e_;
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Merge of the LM head's per-CTA partials, in CTA order:
//   m = max, s = sum e^(z-m), t = sum e^(z-m)(z-m), argmax lowest id on ties.
//   logZ = m + ln s, H = ln s - t/s, logconf = -ln s.
// ---------------------------------------------------------------------------
struct LmPart {
  float m, s, t;
  int a;
};

DG_DEVINL LmPart lm_merge(LmPart x, LmPart y) {
  if (!(y.s > 0.f)) return x;
  if (!(x.s > 0.f)) return y;
  if (y.m > x.m || (y.m == x.m && y.a < x.a)) {
    const LmPart tmp = x;
    x = y;
    y = tmp;
  }
  // x holds the larger max (ties: the lower argmax)
  const float f = expf(y.m - x.m);
  x.t += f * (y.t + (y.m - x.m) * y.s);
  x.s += f * y.s;
  return x;
}

// With `draw`: the row level of the candidate draw.  Lane l owns a contiguous
// run of the row's tiles; the tile masses exp(lambda_j - max) are summed per
// lane, scanned across lanes in lane order, and the tile whose running sum
// first reaches u * total is picked (u = word 1 of the row's re-noise Philox
// block); its drawn id is the candidate.
__global__ void k_lm_combine(const float4* __restrict__ part, int G, int MT, int T, float* stats, int* argmax,
                             int* err, const float2* __restrict__ draw, int NV, DrawKeys keys, int* cand) {
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  const size_t stride = (size_t)MT * 128;
  LmPart r{-INFINITY, 0.f, 0.f, 0x7fffffff};
  for (int c = lane; c < G; c += 32) {
    const float4 v = __ldcg(part + (size_t)c * stride + t);
    if (v.y != v.y) atomicOr(err, DG_DEVERR_NAN);
    r = lm_merge(r, LmPart{v.x, v.y, v.z, __float_as_int(v.w)});
  }
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    LmPart q;
    q.m = __shfl_xor_sync(0xffffffffu, r.m, o);
    q.s = __shfl_xor_sync(0xffffffffu, r.s, o);
    q.t = __shfl_xor_sync(0xffffffffu, r.t, o);
    q.a = __shfl_xor_sync(0xffffffffu, r.a, o);
    // both lanes of a pair merge in the same (lower lane first) order
    r = (lane & o) ? lm_merge(q, r) : lm_merge(r, q);
  }
  if (lane == 0) {
    const float ls = logf(r.s);
    const float4 o = make_float4(ls - r.t / r.s, -ls, r.m, r.m + ls);
    if (!(r.s > 0.f) || o.x != o.x) atomicOr(err, DG_DEVERR_NAN);
    reinterpret_cast<float4*>(stats)[t] = o;
    argmax[t] = r.a;
  }
  if (draw == nullptr) return;
  constexpr float kLog2e = 1.4426950408889634f;
  const float2* dr = draw + (size_t)t * NV;
  const int per = (NV + 31) / 32;
  const int j0 = min(lane * per, NV), j1 = min(j0 + per, NV);
  float M = -INFINITY;
  for (int j = j0; j < j1; ++j) M = fmaxf(M, dr[j].x);
  M = warp_max(M);
  float cs = 0.f;
  for (int j = j0; j < j1; ++j) cs += exp2f((dr[j].x - M) * kLog2e);
  float incl = cs;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  const float total = __shfl_sync(0xffffffffu, incl, 31);
  const int slot = t / keys.canvas, pos = t - slot * keys.canvas;
  const unsigned long long seed = keys.seed[slot];
  const float u = word_uniform(philox4x32_10((uint32_t)pos, (uint32_t)keys.step[slot], (uint32_t)keys.block[slot],
                                             (uint32_t)keys.req[slot], (uint32_t)seed, (uint32_t)(seed >> 32))
                                   .y);
  const float target = u * total;
  const unsigned hit = __ballot_sync(0xffffffffu, incl >= target && cs > 0.f);
  const int L = hit ? __ffs(hit) - 1 : 31;
  int J = -1;
  if (lane == L) {
    const float local = target - (incl - cs);
    float cum = 0.f;
    int last = -1;
    for (int j = j0; j < j1; ++j) {
      const float w = exp2f((dr[j].x - M) * kLog2e);
      cum += w;
      if (w > 0.f) last = j;
      if (J < 0 && cum >= local) J = j;
    }
    if (J < 0) J = last;  // rounding left the running sum short of the target
    if (J < 0) {
      atomicOr(err, DG_DEVERR_NAN);
      J = 0;
    }
    const int c = __float_as_int(dr[J].y);
    if (c < 0 || c >= NV * 256) atomicOr(err, DG_DEVERR_TOKEN);
    cand[t] = c;
  }
}

cudaError_t run_lm_combine(const float4* part, int G, int MT, int T, float* stats, int* argmax, int* err,
                           cudaStream_t st, const float2* draw, int NV, const DrawKeys* keys, int* cand) {
  if (T == 0) return cudaSuccess;
  DrawKeys k;
  memset(&k, 0, sizeof(k));
  if (draw != nullptr) {
    if (keys == nullptr || cand == nullptr || NV < 1 || keys->canvas < 1 ||
        (T + keys->canvas - 1) / keys->canvas > DG_MAX_REQUESTS)
      return cudaErrorInvalidValue;
    k = *keys;
  }
  {
    const cudaError_t e_ = launch_pdl(k_lm_combine, dim3((T + 7) / 8), dim3(256), 0, st, part, G, MT, T, stats, argmax,
                                      err, draw, NV, k, cand);
    if (e_ != cudaSuccess) return e_;
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Self-conditioning.  k_selfcond_topk: one warp per LM-head row merges the
// top-8 logit lists of the CTAs that saw the row (the grid is a multiple of
// the token-tile count MT and CTA c handles tile c % MT; lane l takes the
// l-th, (l+32)-th, ... of them), then K rounds of
// a warp-wide max, ties to the lower id) and stores the K largest softmax
// entries p = exp(z - logZ) with their ids in the row's request slot.
// k_selfcond_embed: one CTA per pass row, 8 columns per thread, accumulates
// sum_k p_k E[id_k] in fp32 (k ascending) and stores bf16.
// ---------------------------------------------------------------------------
DG_DEVINL void sc_insert(float (&tv)[8], int (&ti)[8], float v, int id) {
  // list sorted by (value descending, id ascending); gt[r]: the new entry goes before entry r
  bool gt[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) gt[r] = v > tv[r] || (v == tv[r] && id < ti[r]);
  if (!gt[7]) return;
#pragma unroll
  for (int r = 7; r > 0; --r) {
    tv[r] = gt[r] ? (gt[r - 1] ? tv[r - 1] : v) : tv[r];
    ti[r] = gt[r] ? (gt[r - 1] ? ti[r - 1] : id) : ti[r];
  }
  tv[0] = gt[0] ? v : tv[0];
  ti[0] = gt[0] ? id : ti[0];
}

__global__ void k_selfcond_topk(const float2* __restrict__ sc_part, int G, int T, const float* __restrict__ stats,
                                DrawKeys keys, int K, float2* sc_top, int* err) {
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  float tv[8];
  int ti[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    tv[r] = -INFINITY;
    ti[r] = 0x7fffffff;
  }
  // only the CTAs of this row's token tile wrote it (CTA c holds tile c % MT)
  const int MT = (T + 127) / 128;
  for (int c = t / 128 + lane * MT; c < G; c += 32 * MT) {
    const float2* l = sc_part + ((size_t)c * T + t) * 8;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const float2 e = l[r];
      sc_insert(tv, ti, e.x, __float_as_int(e.y));
    }
  }
  const float4 st = reinterpret_cast<const float4*>(stats)[t];  // (entropy, logconf, max, logZ)
  const float logZ = st.w;
  const int slot = t / keys.canvas, pos = t - slot * keys.canvas;
  float2* out = sc_top + ((size_t)keys.req[slot] * keys.canvas + pos) * 8;
  for (int k = 0; k < K; ++k) {
    float bv = tv[0];
    int bi = ti[0];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (tv[0] == bv && ti[0] == bi) {  // this lane held it: pop
#pragma unroll
      for (int r = 0; r < 7; ++r) {
        tv[r] = tv[r + 1];
        ti[r] = ti[r + 1];
      }
      tv[7] = -INFINITY;
      ti[7] = 0x7fffffff;
    }
    if (lane == 0) {
      const float pk = expf(bv - logZ);
      if (bi < 0 || bi == 0x7fffffff || pk != pk) atomicOr(err, DG_DEVERR_NAN);
      out[k] = make_float2(pk, __int_as_float(bi));
    }
  }
}

cudaError_t run_selfcond_topk(const float2* sc_part, int G, int T, const float* stats, const DrawKeys& keys, int K,
                              float2* sc_top, int* err, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  if (K < 1 || K > 8 || keys.canvas < 1 || (T + keys.canvas - 1) / keys.canvas > DG_MAX_REQUESTS)
    return cudaErrorInvalidValue;
  {
    const cudaError_t e_ = launch_pdl(k_selfcond_topk, dim3((T + 7) / 8), dim3(256), 0, st, sc_part, G, T, stats,
                                      keys, K, sc_top, err);
    if (e_ != cudaSuccess) return e_;
  }
  return cudaGetLastError();
}

__global__ void k_selfcond_embed(const __grid_constant__ SelfCondArgs a) {
  pdl_trigger();
  pdl_wait();
  const int r = blockIdx.x;
  const int slot = r / a.canvas, pos = r - slot * a.canvas;
  const bool on = slot < a.n_slots && a.on[slot];
  const float2* top = on ? a.top + ((size_t)a.req[slot] * a.canvas + pos) * 8 : nullptr;
  for (int c = threadIdx.x; c < a.d / 8; c += blockDim.x) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    if (on) {
      for (int k = 0; k < a.K; ++k) {
        const float2 e = top[k];
        const int id = __float_as_int(e.y);
        if (id < 0 || id >= a.vocab) {
          if (c == threadIdx.x) atomicOr(a.err, DG_DEVERR_TOKEN);
          continue;
        }
        const uint4 v = *reinterpret_cast<const uint4*>(a.embed + (size_t)id * a.d + c * 8);
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(b2[i]);
          acc[2 * i] = fmaf(e.x, f.x, acc[2 * i]);
          acc[2 * i + 1] = fmaf(e.x, f.y, acc[2 * i + 1]);
        }
      }
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(a.out + (size_t)r * a.d + c * 8) = o;
  }
}

cudaError_t run_selfcond_embed(const SelfCondArgs& a, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  if (a.d % 8 != 0 || a.K < 1 || a.K > 8 || a.canvas < 1 || a.n_slots > DG_MAX_REQUESTS) return cudaErrorInvalidValue;
  const int threads = a.d / 8 < 512 ? (a.d / 8 + 31) / 32 * 32 : 512;
  {
    const cudaError_t e_ = launch_pdl(k_selfcond_embed, dim3(a.T), dim3(threads), 0, st, a);
    if (e_ != cudaSuccess) return e_;
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Re-noise token: word 0 of Philox-4x32-10 (common.cuh) at counter
// (position, step, block, request), key = seed, mapped to [0, vocab) by
// multiply-shift.
// ---------------------------------------------------------------------------
DG_DEVINL int renoise_token(unsigned long long seed, int block, int step, uint32_t pos, int request, int vocab) {
  const uint32_t x0 = philox4x32_10(pos, (uint32_t)step, (uint32_t)block, (uint32_t)request, (uint32_t)seed,
                                    (uint32_t)(seed >> 32)).x;
  return (int)(((unsigned long long)x0 * (unsigned long long)vocab) >> 32);
}

__global__ void k_philox_tokens(unsigned long long seed, int block, int step, int request, long long pos0, long long n,
                                int vocab, int* out, unsigned char* mask_clear) {
  pdl_trigger();
  pdl_wait();
  const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (i >= n) return;
  out[i] = renoise_token(seed, block, step, (uint32_t)(pos0 + i), request, vocab);
  if (mask_clear) mask_clear[i] = 0;
}

cudaError_t run_philox_tokens(unsigned long long seed, int block, int step, int request, long long pos0, long long n,
                              int vocab, int* out, unsigned char* mask_clear, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  {
    const cudaError_t e_ = launch_pdl(k_philox_tokens, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, seed, block, step, request, pos0, n, vocab, out,
                                                               mask_clear);
    if (e_ != cudaSuccess) return e_;
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Accept / freeze / re-noise rule, one CTA per canvas, one thread per position.
// Threshold rule: accept an open position whose entropy is <= thr or that is
// among the min_accept most confident open positions.  Entropy-budget rule
// (the pages' default sampler, "How the sampler actually works"): accept the
// open positions from most to least confident while their running entropy
// stays within the budget (at least the first); accept them all once the
// argmax of every open position repeats the previous step's and their mean
// entropy is below stop_entropy.  Both accept everything at the step cap.
// ---------------------------------------------------------------------------
__global__ void k_sample(SampleArgs a) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ float ssm[];
  float* lc_s = ssm;                                             // [canvas]
  int* un_s = reinterpret_cast<int*>(ssm + a.canvas);            // [canvas]
  float* h_s = ssm + 2 * a.canvas;                               // [canvas] entropy, by position
  float* hr_s = ssm + 3 * a.canvas;                              // [canvas] entropy, by confidence rank
  __shared__ int stop_s;
  const int slot = blockIdx.x;
  const int req = a.req[slot];
  const int i = threadIdx.x;
  const int C = a.canvas;
  const bool valid = i < C;
  const size_t p = (size_t)slot * C + i;
  int acc = 1;
  float H = 0.f, lc = -INFINITY;
  int am = 0;
  if (valid) {
    acc = a.mask[(size_t)req * C + i] ? 1 : 0;
    H = a.entropy[p * a.stride];
    lc = a.logconf[p * a.stride];
    am = a.argmax[p];
    if (H != H || lc != lc) atomicOr(a.err, DG_DEVERR_NAN);
    lc_s[i] = lc;
    un_s[i] = !acc;
    h_s[i] = H;
  }
  const int nU = __syncthreads_count(valid && !acc);
  const bool force = a.step[slot] >= a.max_steps;
  // rank among the positions not yet accepted: descending logconf, ties to the lower position
  int rank = 0;
  if (valid && !acc) {
    for (int j = 0; j < C; ++j) {
      const float o = lc_s[j];
      rank += (un_s[j] && (o > lc || (o == lc && j < i))) ? 1 : 0;
    }
  }
  bool take;
  if (a.mode == DG_SAMPLER_ENTROPY_BUDGET) {
    // converged: every open position kept its previous argmax and their mean
    // entropy (fp64, summed in position order) is below stop_entropy
    int* prev = a.prev_argmax + (size_t)req * C;
    const bool same = !valid || acc || (a.step[slot] > 1 && prev[i] == am);
    const int all_same = __syncthreads_and(same);
    if (valid && !acc) hr_s[rank] = H;
    if (i == 0) {
      double sum = 0.0;
      for (int j = 0; j < C; ++j)
        if (un_s[j]) sum += (double)h_s[j];
      stop_s = nU > 0 && all_same && sum / (double)nU < (double)a.stop_entropy;
    }
    __syncthreads();
    // running entropy of the rank-ordered open positions (fp64, in rank
    // order): a position is taken when no earlier prefix beyond the first
    // position went over the budget
    bool within = false;
    if (valid && !acc) {
      double cum = 0.0;
      within = true;
      for (int r = 0; r <= rank; ++r) {
        cum += (double)hr_s[r];
        if (r > 0 && cum > (double)a.budget) within = false;
      }
    }
    take = valid && !acc && (force || stop_s || within);
    if (valid) prev[i] = am;
  } else {
    const int n_top = min(a.min_accept, nU);
    take = valid && !acc && (force || H <= a.thr || rank < n_top);
  }
  if (take) {
    if (am < 0 || am >= a.vocab) {
      atomicOr(a.err, DG_DEVERR_TOKEN);
      am = 0;
    }
    int tok = am;
    if (a.cand != nullptr) {
      tok = a.cand[p];
      if (tok < 0 || tok >= a.vocab) {
        atomicOr(a.err, DG_DEVERR_TOKEN);
        tok = 0;
      }
    }
    a.canvas_tok[(size_t)req * C + i] = tok;
    a.mask[(size_t)req * C + i] = 1;
  } else if (valid && !acc) {
    a.canvas_tok[(size_t)req * C + i] =
        renoise_token(a.seed[slot], a.block[slot], a.step[slot], (uint32_t)i, req, a.vocab);
  }
  const int rem = __syncthreads_count(valid && !acc && !take);
  if (i == 0) a.remaining[req] = rem;
}

cudaError_t run_sample(const SampleArgs& a, cudaStream_t st) {
  if (a.n_slots == 0) return cudaSuccess;
  const int threads = (a.canvas + 31) / 32 * 32;
  {
    const cudaError_t e_ = launch_pdl(k_sample, dim3(a.n_slots), dim3(threads), (size_t)a.canvas * 16, st, a);
    if (e_ != cudaSuccess) return e_;
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// KV copy between the cache layout (K tiled as in k_tile_offset per head,
// V^T [Hkv][D][cap]) and dense [Hkv][n][D] arrays, either direction.
// ---------------------------------------------------------------------------
__global__ void k_k_copy(bf16* cache_k, int Hkv, long long cap, int D, long long pos0, long long n, const bf16* k_in,
                         bf16* k_out) {
  pdl_trigger();
  pdl_wait();
  const long long r = blockIdx.x;  // (head, i)
  const int head = (int)(r / n);
  const long long i = r - (long long)head * n;
  const size_t head_off = (size_t)head * cap * D;
  const size_t dense_off = ((size_t)head * n + i) * D;
  for (int c = threadIdx.x; c < D / 8; c += blockDim.x) {  // 8 dims, inside one 64-dim block
    const size_t cache_off = head_off + k_tile_offset(pos0 + i, c * 8, D);
    if (k_in)
      *reinterpret_cast<uint4*>(cache_k + cache_off) = reinterpret_cast<const uint4*>(k_in + dense_off)[c];
    else
      reinterpret_cast<uint4*>(k_out + dense_off)[c] = *reinterpret_cast<const uint4*>(cache_k + cache_off);
  }
}

__global__ void k_vt_copy(bf16* cache_vt, int Hkv, long long cap, int D, long long pos0, long long n,
                          const bf16* v_in, bf16* v_out) {
  pdl_trigger();
  pdl_wait();
  const long long total = (long long)Hkv * D * n;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const long long i = e % n;             // position fastest: coalesced in the cache
    const long long hd = e / n;            // head * D + dim
    const long long head = hd / D, dim = hd % D;
    const size_t c_off = (size_t)hd * cap + pos0 + i;
    const size_t d_off = ((size_t)head * n + i) * D + dim;
    if (v_in)
      cache_vt[c_off] = v_in[d_off];
    else
      v_out[d_off] = cache_vt[c_off];
  }
}

cudaError_t run_kv_copy(bf16* cache_k, bf16* cache_v, int Hkv, long long cap, int D, long long pos0, long long n,
                        const bf16* k_in, const bf16* v_in, bf16* k_out, bf16* v_out, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  {
    const cudaError_t e_ = launch_pdl(k_k_copy, dim3((unsigned)(Hkv * n)), dim3(32), 0, st, cache_k, Hkv, cap, D, pos0, n, k_in, k_out);
    if (e_ != cudaSuccess) return e_;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long total = (long long)Hkv * D * n;
  const unsigned blocks = (unsigned)((total + 255) / 256 < 65535 ? (total + 255) / 256 : 65535);
  {
    const cudaError_t e_ = launch_pdl(k_vt_copy, dim3(blocks), dim3(256), 0, st, cache_v, Hkv, cap, D, pos0, n, v_in, v_out);
    if (e_ != cudaSuccess) return e_;
  }
  return cudaGetLastError();
}

}  // namespace dg
