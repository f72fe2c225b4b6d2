// Longest-first order of a batch's requests for the tensor-core attention
// kernel: the grid's request axis reads it, so the longest requests start
// first and the launch's ragged tail is made of short ones.
#include "va_common.cuh"

namespace va {
namespace {

// Longest-first order of the requests: order[y] = the request with the y-th
// largest kv_len, ties by index.  One CTA sorts keys (descending kv_len,
// ascending index) bitonically in shared memory; batches beyond kMaxSorted
// keep their natural order (their grids are many waves deep, so the ragged
// tail that the order shortens is a small share of the launch).
constexpr int kMaxSorted = 16384;
constexpr int kOrderThreads = 1024;

__global__ void __launch_bounds__(kOrderThreads)
request_order_kernel(const int32_t* __restrict__ kv_len, int B, int n, int32_t* __restrict__ order) {
  extern __shared__ unsigned long long keys[];
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    unsigned long long k = ~0ull;  // padding sorts last
    if (i < B) {
      const int v = kv_len[i];
      const unsigned int len = v < 0 ? 0u : (unsigned int)v;
      k = ((unsigned long long)(0x7fffffffu - min(len, 0x7fffffffu)) << 32) | (unsigned int)i;
    }
    keys[i] = k;
  }
  __syncthreads();
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int j = i ^ stride;
        if (j > i) {
          const bool up = (i & size) == 0;
          const unsigned long long a = keys[i], c = keys[j];
          if ((a > c) == up) { keys[i] = c; keys[j] = a; }
        }
      }
      __syncthreads();
    }
  }
  for (int i = threadIdx.x; i < B; i += blockDim.x) order[i] = (int32_t)(keys[i] & 0xffffffffu);
}

__global__ void identity_order_kernel(int B, int32_t* __restrict__ order) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < B) order[i] = i;
}

}  // namespace

cudaError_t launch_request_order(const int32_t* kv_len, int B, int32_t* order, cudaStream_t st) {
  if (B == 0) return cudaSuccess;
  if (B > kMaxSorted) {
    identity_order_kernel<<<(B + 255) / 256, 256, 0, st>>>(B, order);
    return cudaGetLastError();
  }
  int n = 1;
  while (n < B) n <<= 1;
  const size_t smem = (size_t)n * sizeof(unsigned long long);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(request_order_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const int threads = n < kOrderThreads ? (n < 32 ? 32 : n) : kOrderThreads;  // one key per thread
  request_order_kernel<<<1, threads, smem, st>>>(kv_len, B, n, order);
  return cudaGetLastError();
}

}  // namespace va
