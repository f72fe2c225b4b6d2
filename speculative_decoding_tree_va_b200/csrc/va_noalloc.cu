// va_verify_attn_noalloc: the split-KV verify step for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) when they run the
// verify step: a serving loop whose device memory is planned once at start-up
// and may not grow, or a latency-critical path where an allocation (which can
// synchronise the device) is not acceptable.  va_verify_attn needs such a
// caller to hand over a workspace for the split-KV partials; this entry point
// instead keeps the partials in a fixed array of this library, so the caller
// passes only inputs and outputs.
//
// The array has kScratchBytes (VA_NOALLOC_SCRATCH_BYTES) on every device that
// loads the library, for as long as the process lives.  Every call shares it
// and it keeps the last call's contents; the split kernels write every partial
// they later read (empty splits write zeros and -inf), so nothing needs
// clearing between calls.  Two calls whose work overlaps on the GPU (on
// different streams, or on devices sharing nothing else) race on the array.
#include <mutex>

#include "va_common.cuh"

namespace {

constexpr size_t kScratchBytes = VA_NOALLOC_SCRATCH_BYTES;
static_assert(kScratchBytes % 256 == 0, "scratch size must keep 256-byte alignment");

// Device-resident scratch.  In host code this name is only a stand-in for the
// symbol: its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char va_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 128;
void* g_scratch_addr[kMaxDevices];
cudaError_t g_scratch_err[kMaxDevices];
std::once_flag g_scratch_once[kMaxDevices];

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Device address of the scratch array on the current device, looked up once
// per device (with that device current) and cached.
cudaError_t scratch_address(void** addr) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(g_scratch_once[dev], [dev] {
    g_scratch_err[dev] = cudaGetSymbolAddress(&g_scratch_addr[dev], va_noalloc_scratch);
  });
  if (g_scratch_err[dev] != cudaSuccess) return g_scratch_err[dev];
  *addr = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" int va_verify_attn_noalloc(const va_attn_args* args, va_stream_t stream) {
  // Argument checks and the split count are exactly those of va_verify_attn;
  // the workspace fields of args are ignored.
  const int S = va_num_splits(args);
  if (S < 0) return -S;
  if (args->B == 0) return VA_OK;
  const size_t rows = (size_t)args->B * args->T * args->H;
  const size_t lse_off = align256((size_t)S * rows * VA_D_LATENT * sizeof(float));
  const size_t need = lse_off + align256((size_t)S * rows * sizeof(float));
  if (S > 1 && need > kScratchBytes) return VA_ERR_UNSUPPORTED;  // larger than the fixed array

  cudaStream_t st = (cudaStream_t)stream;
  const bool tc = va::uses_tensor_cores(*args);
  float* o_part = nullptr;
  float* lse_part = nullptr;
  if (S > 1) {
    void* base = nullptr;
    if (scratch_address(&base) != cudaSuccess) return VA_ERR_CUDA;
    o_part = (float*)base;
    lse_part = (float*)((char*)base + lse_off);
  }
  cudaError_t e = tc ? va::launch_attn_tc(*args, S, o_part, lse_part, st)
                     : va::launch_attn_simt(*args, S, o_part, lse_part, st);
  if (e == cudaErrorNotSupported) return VA_ERR_UNSUPPORTED;
  if (e != cudaSuccess) return VA_ERR_CUDA;
  if (S > 1) {
    e = va::launch_merge(o_part, lse_part, S, (long long)rows, args->dtype, args->out, args->lse,
                         st);
    if (e != cudaSuccess) return VA_ERR_CUDA;
  }
  return VA_OK;
}
