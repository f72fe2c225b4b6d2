// Split-KV merge (the flash+merge production note on page "The Milestone
// Commit...", section "How Decisions Were Made").
//
// One warp per output row.  Lane c < S reads lse_c; the warp reduces the max
// and the sum of exp(lse_c - max) with shuffles, then every lane combines 16
// of the 512 latent columns (four float4 groups, 128 columns apart, so each
// group access is one coalesced 512-byte line per warp).  HBM-bound: reads
// S * 2052 bytes per row, writes the row once.
#include "va_common.cuh"

namespace va {
namespace {

constexpr int kWarps = 8;

template <typename Tout>
__device__ __forceinline__ void store4(Tout* dst, float4 v);
template <>
__device__ __forceinline__ void store4<float>(float* dst, float4 v) {
  *reinterpret_cast<float4*>(dst) = v;
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* dst, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
  __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(dst) = u;
}

template <typename Tout>
__global__ void __launch_bounds__(kWarps * 32)
merge_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part, int S,
             long long rows, Tout* __restrict__ out, float* __restrict__ lse,
             const int32_t* __restrict__ req_bad, int rows_per_req,
             int32_t* __restrict__ req_status) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  if (req_bad) {  // a flagged request's rows come out empty, whatever its other splits hold
    const long long b = row / rows_per_req;
    const int32_t st = req_bad[b];
    if (st != 0) {
      Tout* orow = out + row * kDc + lane * 4;
#pragma unroll
      for (int g = 0; g < 4; ++g) store4<Tout>(orow + g * 128, make_float4(0.f, 0.f, 0.f, 0.f));
      if (lane == 0) {
        lse[row] = -INFINITY;
        if (req_status && row == b * rows_per_req) req_status[b] = st;
      }
      return;
    }
  }
  // S <= 64: lanes hold chunks lane and lane + 32.
  const float l0 = lane < S ? lse_part[(long long)lane * rows + row] : -INFINITY;
  const float l1 = lane + 32 < S ? lse_part[(long long)(lane + 32) * rows + row] : -INFINITY;
  float mx = fmaxf(l0, l1);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  Tout* orow = out + row * kDc + lane * 4;
  if (mx == -INFINITY) {
#pragma unroll
    for (int g = 0; g < 4; ++g) store4<Tout>(orow + g * 128, make_float4(0.f, 0.f, 0.f, 0.f));
    if (lane == 0) lse[row] = -INFINITY;
    return;
  }
  float z = (l0 == -INFINITY ? 0.f : exp2f((l0 - mx) * kLog2e)) +
            (l1 == -INFINITY ? 0.f : exp2f((l1 - mx) * kLog2e));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  const float L = mx + logf(z);
  float4 acc[4];
#pragma unroll
  for (int g = 0; g < 4; ++g) acc[g] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int c = 0; c < S; ++c) {
    const float lc = __shfl_sync(0xffffffffu, c < 32 ? l0 : l1, c & 31);
    if (lc == -INFINITY) continue;
    const float w = exp2f((lc - L) * kLog2e);
    const float* src = o_part + ((long long)c * rows + row) * kDc + lane * 4;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const float4 v = __ldcs(reinterpret_cast<const float4*>(src + g * 128));
      acc[g].x = fmaf(w, v.x, acc[g].x);
      acc[g].y = fmaf(w, v.y, acc[g].y);
      acc[g].z = fmaf(w, v.z, acc[g].z);
      acc[g].w = fmaf(w, v.w, acc[g].w);
    }
  }
#pragma unroll
  for (int g = 0; g < 4; ++g) store4<Tout>(orow + g * 128, acc[g]);
  if (lane == 0) lse[row] = L;
}

}  // namespace

cudaError_t launch_merge(const float* o_part, const float* lse_part, int S, long long rows,
                         int out_dtype, void* out, float* lse, cudaStream_t st,
                         const int32_t* req_bad, int rows_per_req, int32_t* req_status) {
  if (rows == 0) return cudaSuccess;
  const long long blocks = (rows + kWarps - 1) / kWarps;
  if (out_dtype == VA_F32)
    merge_kernel<float><<<(unsigned)blocks, kWarps * 32, 0, st>>>(
        o_part, lse_part, S, rows, (float*)out, lse, req_bad, rows_per_req, req_status);
  else
    merge_kernel<__nv_bfloat16><<<(unsigned)blocks, kWarps * 32, 0, st>>>(
        o_part, lse_part, S, rows, (__nv_bfloat16*)out, lse, req_bad, rows_per_req, req_status);
  return cudaGetLastError();
}

}  // namespace va
