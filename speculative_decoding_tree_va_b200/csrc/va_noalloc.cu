// va_verify_attn_noalloc: the split-KV verify step for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) when they run the
// verify step: a serving loop whose device memory is planned once at start-up
// and may not grow, or a latency-critical path where an allocation (which can
// synchronise the device) is not acceptable.  va_verify_attn needs such a
// caller to hand over a workspace for the split-KV partials (and, for bf16
// queries against an FP8 cache, the widened cache pages); this entry point
// instead keeps them in a fixed array of this library, so the caller passes
// only inputs and outputs.
//
// The array has kScratchBytes (VA_NOALLOC_SCRATCH_BYTES) on every device that
// loads the library, for as long as the process lives.  Every call shares it
// and it keeps the last call's contents; every part of the workspace is
// written before it is read within the call (the request order, the split
// partials -- empty splits write zeros and -inf -- and the widened pages), so
// nothing needs clearing between calls.  Two calls whose work overlaps on the GPU (on
// different streams, or on devices sharing nothing else) race on the array.
#include <atomic>
#include <mutex>

#include "va_common.cuh"

namespace {

constexpr size_t kScratchBytes = VA_NOALLOC_SCRATCH_BYTES;
static_assert(kScratchBytes % 256 == 0, "scratch size must keep 256-byte alignment");

// Device-resident scratch.  In host code this name is only a stand-in for the
// symbol: its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char va_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 128;
std::atomic<void*> g_scratch_addr[kMaxDevices];  // nullptr until a lookup succeeds
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device, looked up with
// that device current and cached once the lookup has succeeded.  A failed
// lookup (for instance one attempted during stream capture) is not cached:
// the call fails with its error, the runtime's last-error state is cleared,
// and the next call on that device tries again.
cudaError_t scratch_address(void** addr) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return e;
  }
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (!p) {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    p = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (!p) {
      e = cudaGetSymbolAddress(&p, va_noalloc_scratch);
      if (e != cudaSuccess || !p) {
        (void)cudaGetLastError();
        return e != cudaSuccess ? e : cudaErrorInvalidSymbol;
      }
      g_scratch_addr[dev].store(p, std::memory_order_release);
    }
  }
  *addr = p;
  return cudaSuccess;
}

}  // namespace

extern "C" int va_verify_attn_noalloc(const va_attn_args* args, va_stream_t stream) {
  // Argument checks, the split count and the workspace layout are exactly
  // those of va_verify_attn; the workspace fields of args are ignored.
  const int S = va_num_splits(args);
  if (S < 0) return -S;
  if (args->B == 0) return VA_OK;
  const size_t need = va::workspace_layout(*args, S).total;
  if (need > kScratchBytes) return VA_ERR_UNSUPPORTED;  // larger than the fixed array
  void* base = nullptr;
  if (need && scratch_address(&base) != cudaSuccess) return VA_ERR_CUDA;
  return va::run_verify(*args, S, base, (cudaStream_t)stream);
}
