// LM-head statistics without any device allocation by the caller or by us.
//
// Some callers cannot hand the library a workspace or call cudaMalloc: a
// serving runtime that has already given all free HBM to its own caching
// allocator (a cudaMalloc there fails or fragments the pool), or a
// latency-critical loop where cudaMalloc's implicit device synchronisation is
// not acceptable.  dg_op_lm_head_noalloc serves them: it runs the same final
// RMSNorm + tied LM head + fused (max, argmax, log-partition, entropy,
// logconf) kernels as dg_op_lm_head, with the scratch those kernels need (the
// normalised bf16 rows and the per-CTA partial statistics) in the file-scope
// array below instead of a caller workspace.
//
// The array is a fixed 3 MiB held by every GPU that loads the library until
// the process exits.  Its device address is looked up once per device
// (cudaGetSymbolAddress) by the first call on that device, which therefore
// must come before any stream capture.  Every call shares the array and it
// keeps the last call's contents: nothing in it needs to start at zero (each
// call writes every scratch value it later reads), but calls that overlap on
// the GPU (other streams, other threads) race on it and must be serialised by
// the caller.
#include <mutex>

#include "dg_internal.h"

namespace {

constexpr int kMaxTokens = DG_NOALLOC_MAX_TOKENS;
constexpr int kMaxDModel = DG_NOALLOC_MAX_DMODEL;
constexpr int kMaxCtas = 256;
constexpr size_t kRowsBytes = (size_t)kMaxTokens * kMaxDModel * 2;    // normalised bf16 rows
constexpr size_t kPartBytes = (size_t)kMaxCtas * kMaxTokens * 16;     // per-CTA partial statistics
constexpr size_t kErrBytes = 256;
constexpr size_t kScratchBytes = kRowsBytes + kPartBytes + kErrBytes;

static __device__ __align__(256) unsigned char g_lm_scratch[kScratchBytes];

struct DeviceScratch {
  bool ready = false;
  unsigned char* ptr = nullptr;  // device address of g_lm_scratch on this device
  int num_sms = 0;
};

constexpr int kMaxDevices = 64;
DeviceScratch g_dev[kMaxDevices];
std::mutex g_mu;

// Once per device, with that device current: resolve the array's device address.
int scratch_for_current_device(DeviceScratch** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DG_E_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceScratch& s = g_dev[dev];
  if (!s.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_lm_scratch) != cudaSuccess || p == nullptr) return DG_E_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
      return DG_E_CUDA;
    s.ptr = static_cast<unsigned char*>(p);
    s.num_sms = sms;
    s.ready = true;
  }
  *out = &s;
  return DG_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once per process (std::call_once:
// first calls from several host threads do not race on the pointer).
EncodeTiledFn encoder() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// TMA descriptor of a bf16 [rows, K] tensor read in 64 x box_rows boxes with
// the 128-byte swizzle (host-side encoding only; allocates nothing).
bool encode_2d(CUtensorMap* m, const void* base, long long K, long long rows, int box_rows) {
  const EncodeTiledFn fn = encoder();
  if (fn == nullptr) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

extern "C" int dg_op_lm_head_noalloc(const float* d_x, const float* d_final_norm, const void* d_embed, int T,
                                     int d_model, int vocab, float norm_eps, float* d_stats, int32_t* d_argmax,
                                     int32_t* d_err, void* stream) {
  if (!d_x || !d_final_norm || !d_embed || !d_stats || !d_argmax) return DG_E_ARG;
  if (T < 1 || T > kMaxTokens || d_model < 64 || d_model > kMaxDModel || d_model % 64 != 0) return DG_E_ARG;
  if (vocab < 256 || vocab % 256 != 0) return DG_E_ARG;
  DeviceScratch* s = nullptr;
  int rc = scratch_for_current_device(&s);
  if (rc != DG_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  dg::bf16* rows = reinterpret_cast<dg::bf16*>(s->ptr);
  float4* part = reinterpret_cast<float4*>(s->ptr + kRowsBytes);
  int* err = d_err ? reinterpret_cast<int*>(d_err) : reinterpret_cast<int*>(s->ptr + kRowsBytes + kPartBytes);

  CUtensorMap tm_rows, tm_embed;
  const int Tcap = (T + 127) / 128 * 128;
  if (!encode_2d(&tm_rows, rows, d_model, Tcap, 128) || !encode_2d(&tm_embed, d_embed, d_model, vocab, 256))
    return DG_E_ARG;
  if (cudaMemsetAsync(err, 0, sizeof(int), st) != cudaSuccess) return DG_E_CUDA;
  if (dg::run_rmsnorm(d_x, d_final_norm, T, d_model, norm_eps, rows, st) != cudaSuccess) return DG_E_CUDA;
  dg::LmArgs la;
  la.tm_x = &tm_rows;
  la.tm_embed = &tm_embed;
  la.T = T;
  la.d = d_model;
  la.num_sms = s->num_sms < kMaxCtas ? s->num_sms : kMaxCtas;
  la.V = vocab;
  la.part = part;
  la.logits = nullptr;
  la.err = err;
  int grid = 0;
  if (dg::run_lm_head(la, &grid, st) != cudaSuccess) return DG_E_CUDA;
  if (dg::run_lm_combine(part, grid, Tcap / 128, T, d_stats, reinterpret_cast<int*>(d_argmax), err, st) !=
      cudaSuccess)
    return DG_E_CUDA;
  return DG_OK;
}
