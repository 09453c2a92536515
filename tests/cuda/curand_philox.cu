// Test-only probe: raw 32-bit words of cuRAND's device Philox4_32_10
// generator, an implementation independent of both the oracle and the
// library, used to pin the oracle's Philox-4x32-10 (Salmon et al., SC'11,
// "Parallel Random Numbers: As Easy as 1, 2, 3") bit for bit.
//
// For each i the generator is initialised with curand_init(seed, subseq[i],
// offset[i]) and curand4() returns the four words of one counter block.
#include <cuda_runtime.h>
#include <curand_kernel.h>

__global__ void k_curand_philox_words(unsigned long long seed, const unsigned long long* __restrict__ subseq,
                                      const unsigned long long* __restrict__ offset, int n, uint4* __restrict__ out) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  curandStatePhilox4_32_10_t s;
  curand_init(seed, subseq[i], offset[i], &s);
  out[i] = curand4(&s);
}

extern "C" int curand_philox_words(unsigned long long seed, const unsigned long long* d_subseq,
                                   const unsigned long long* d_offset, int n, void* d_out, void* stream) {
  if (n <= 0) return 0;
  k_curand_philox_words<<<(n + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      seed, d_subseq, d_offset, n, static_cast<uint4*>(d_out));
  return static_cast<int>(cudaGetLastError());
}
