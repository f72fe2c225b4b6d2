// Widening of an FP8 E4M3 latent cache into bf16 scratch pages, so that bf16
// queries against an FP8 cache run on the tensor-core kernel.
//
// Every finite E4M3 value is exactly a bf16 value (4 significant bits, and
// exponents from 2^-9 to 2^8), so the widened pages hold the codes' values
// unchanged; the cache scale is not applied here but folded into the score
// scale and the output normalisation of the attention kernel.  The result is
// therefore the attention over kv_scale * value(code) with no extra rounding.
//
// Request b's logical page i goes to scratch page b * max_pages + i, and a
// new page table records that index (or -1 for a page index outside the
// pool, which the attention kernel flags, as it would the original entry).
// Slots at or past kv_len in a request's last page are written as zeros, so
// whatever codes sit there (NaN included) cannot reach the products.
#include <cuda_fp8.h>

#include "va_common.cuh"

namespace va {
namespace {

constexpr int kThreads = 256;
constexpr int kChunksC = kPage * kDc / 16;  // 16-code chunks of one c_kv page
constexpr int kChunksR = kPage * kDr / 16;  // ... of one k_pe page

// 16 codes -> 16 bf16 values (exact), written as two 16-byte stores.
__device__ __forceinline__ void widen16(__nv_bfloat16* dst, const uint8_t* src) {
  const uint4 u = *reinterpret_cast<const uint4*>(src);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2 lo(__nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[i] & 0xffffu), __NV_E4M3));
    const __half2 hi(__nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[i] >> 16), __NV_E4M3));
    const float2 a = __half22float2(lo), b = __half22float2(hi);
    const __nv_bfloat162 ba = __floats2bfloat162_rn(a.x, a.y);
    const __nv_bfloat162 bb = __floats2bfloat162_rn(b.x, b.y);
    o[2 * i] = *reinterpret_cast<const uint32_t*>(&ba);
    o[2 * i + 1] = *reinterpret_cast<const uint32_t*>(&bb);
  }
  reinterpret_cast<uint4*>(dst)[0] = make_uint4(o[0], o[1], o[2], o[3]);
  reinterpret_cast<uint4*>(dst)[1] = make_uint4(o[4], o[5], o[6], o[7]);
}

// One CTA per (logical page i, request b).
__global__ void __launch_bounds__(kThreads)
kv_widen_kernel(const uint8_t* __restrict__ c_kv, const uint8_t* __restrict__ k_pe, int num_pages,
                const int32_t* __restrict__ page_table, int max_pages,
                const int32_t* __restrict__ kv_len_arr, int T, __nv_bfloat16* __restrict__ w_ckv,
                __nv_bfloat16* __restrict__ w_kpe, int32_t* __restrict__ w_table) {
  const int i = blockIdx.x, b = blockIdx.y;
  const size_t slot = (size_t)b * max_pages + i;
  const int n = kv_len_arr[b];
  // Requests the attention kernel rejects (bad kv_len) and pages it never
  // reads get no scratch page.
  const bool req_ok = n >= T && n <= max_pages * kPage;
  if (!req_ok || i * kPage >= n) {
    if (threadIdx.x == 0) w_table[slot] = -1;
    return;
  }
  const int phys = page_table[slot];
  if (phys < 0 || phys >= num_pages) {
    if (threadIdx.x == 0) w_table[slot] = -1;
    return;
  }
  if (threadIdx.x == 0) w_table[slot] = (int32_t)slot;
  const int live = min(kPage, n - i * kPage);  // slots of this page below kv_len
  const uint8_t* sc = c_kv + (size_t)phys * kPage * kDc;
  const uint8_t* sr = k_pe + (size_t)phys * kPage * kDr;
  __nv_bfloat16* dc = w_ckv + slot * kPage * kDc;
  __nv_bfloat16* dr = w_kpe + slot * kPage * kDr;
  for (int c = threadIdx.x; c < kChunksC + kChunksR; c += kThreads) {
    const bool lat = c < kChunksC;
    const int e = (lat ? c : c - kChunksC) * 16;  // element offset inside the page
    const int row = lat ? e / kDc : e / kDr;
    __nv_bfloat16* d = (lat ? dc : dr) + e;
    if (row < live) {
      widen16(d, (lat ? sc : sr) + e);
    } else {
      reinterpret_cast<uint4*>(d)[0] = make_uint4(0, 0, 0, 0);
      reinterpret_cast<uint4*>(d)[1] = make_uint4(0, 0, 0, 0);
    }
  }
}

}  // namespace

cudaError_t launch_kv_widen(const va_attn_args& a, void* w_ckv, void* w_kpe, int32_t* w_table,
                            cudaStream_t st) {
  if (a.B == 0) return cudaSuccess;
  dim3 grid((unsigned)a.max_pages, (unsigned)a.B);
  kv_widen_kernel<<<grid, kThreads, 0, st>>>(
      (const uint8_t*)a.c_kv, (const uint8_t*)a.k_pe, a.num_pages, a.page_table, a.max_pages,
      a.kv_len, a.T, (__nv_bfloat16*)w_ckv, (__nv_bfloat16*)w_kpe, w_table);
  return cudaGetLastError();
}

}  // namespace va
