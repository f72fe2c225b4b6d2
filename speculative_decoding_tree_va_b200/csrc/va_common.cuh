// Shared device helpers of libverifyattn (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/verifyattn.h"

namespace va {

constexpr int kDc = VA_D_LATENT;
constexpr int kDr = VA_D_ROPE;
constexpr int kDqk = kDc + kDr;
constexpr int kPage = VA_PAGE_SIZE;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Bit i of a tree-mask row (W words).
__device__ __forceinline__ bool mask_bit(const uint64_t* row, int i) {
  return (row[i >> 6] >> (i & 63)) & 1ull;
}

// Split-KV partition, as fixed in the public header: split s covers
// [e(s), e(s+1)), where e(0) = 0, e(S) = kv_len and, in between, e(s) is
// s * kv_len / S rounded to the nearest multiple of 256 (ties up), at most
// kv_len.  Every split's length is within 256 keys of kv_len / S.
__host__ __device__ __forceinline__ int split_edge(int kv_len, int S, int s) {
  if (s >= S) return kv_len;
  const long long A = VA_SPLIT_ALIGN;
  const long long e = (2LL * s * kv_len + S * A) / (2LL * S * A) * A;
  return (int)(e < kv_len ? e : kv_len);
}
__host__ __device__ __forceinline__ void split_range(int kv_len, int S, int s, int* lo, int* hi) {
  *lo = split_edge(kv_len, S, s);
  *hi = split_edge(kv_len, S, s + 1);
}

// The kernel a va_verify_attn call runs on: bf16 queries go to the tensor
// cores unless the caller asks for CUDA cores; fp32 queries to CUDA cores.
inline bool uses_tensor_cores(const va_attn_args& a) {
  return a.dtype == VA_BF16 && !(a.flags & VA_FLAG_BF16_CUDA_CORES);
}

// A tensor-core call with an FP8 cache first widens the pages it reads into
// bf16 scratch pages (part of the workspace).
inline bool widens_fp8_cache(const va_attn_args& a) {
  return uses_tensor_cores(a) && (a.flags & VA_FLAG_KV_FP8_E4M3);
}

// Workspace layout of one call: on the tensor-core path, the requests'
// longest-first order (int32 [B]); then the split-KV partials (S > 1 and not
// a partials-only call, whose partials go to the caller's arrays) and the
// call's own per-request status (int32 [B], same condition); then the
// widened cache (widens_fp8_cache): bf16 [B * max_pages, 64, 512], bf16
// [B * max_pages, 64, 64] and an int32 [B, max_pages] page table.  Every part
// starts on a 256-byte boundary.  Offsets are in bytes; `total` is 0 when
// nothing is needed.
struct WorkspaceLayout {
  size_t order, o_part, lse_part, status, w_ckv, w_kpe, w_table, total;
};

inline size_t align256(size_t x) { return (x + 255) / 256 * 256; }

inline WorkspaceLayout workspace_layout(const va_attn_args& a, int S, bool partials_here = true) {
  WorkspaceLayout w{0, 0, 0, 0, 0, 0, 0, 0};
  const size_t rows = (size_t)a.B * a.T * a.H;
  size_t off = 0;
  if (uses_tensor_cores(a)) {
    w.order = off;
    off += align256((size_t)a.B * sizeof(int32_t));
  }
  if (S > 1 && partials_here) {
    w.o_part = off;
    off += align256((size_t)S * rows * kDc * sizeof(float));
    w.lse_part = off;
    off += align256((size_t)S * rows * sizeof(float));
    w.status = off;
    off += align256((size_t)a.B * sizeof(int32_t));
  }
  if (widens_fp8_cache(a)) {
    const size_t pages = (size_t)a.B * a.max_pages;
    w.w_ckv = off;
    off += align256(pages * kPage * kDc * 2);
    w.w_kpe = off;
    off += align256(pages * kPage * kDr * 2);
    w.w_table = off;
    off += align256(pages * sizeof(int32_t));
  }
  w.total = off;
  return w;
}

// Which splits of the S-way key partition one launch computes: [first,
// first + count).  Partials go to o_part / lse_part indexed by the split's
// position in the launch (0 .. count-1).
struct SplitRange {
  int S, first, count;
};

// Balanced plan of the CUDA-core kernel for a full call (automatic split
// count) whose (request, 32-row tile) segments are fewer than the SMs: each
// segment's key range is cut into VT virtual 32-key tiles (VT = 2 max_pages,
// the page table's capacity; tiles past kv_len are empty), the Q * VT tiles of
// all segments in order are divided into G contiguous ranges of equal length,
// one CTA each, and every CTA that covers part of a segment writes one
// partial for it (slot = CTA - first CTA of the segment).  `slots` is the
// largest number of CTAs that share a segment; the last CTA of a segment
// marks its unused slots empty (lse -inf), and the merge combines `slots`
// partials per row.  G = 0: not used (one CTA per segment and split).
struct Balance {
  int G = 0, VT = 0, NRT = 0, slots = 0;
  long long U = 0;
};
// The CTA whose range holds virtual tile u: CTA c covers [c U / G, (c+1) U / G).
__host__ __device__ __forceinline__ int balance_cta_of(long long u, long long U, int G) {
  return (int)((u * G + G - 1) / U);
}
inline Balance plan_balance(const va_attn_args& a, int sms) {
  Balance bal;
  if (uses_tensor_cores(a) || a.num_splits != 0 || a.B < 1) return bal;
  const int nrt = (a.T * a.H + 31) / 32;
  const long long q = (long long)a.B * nrt;
  if (q >= sms) return bal;  // one CTA per segment already fills the SMs
  const int vt = 2 * a.max_pages;
  const long long U = q * vt;
  constexpr int kMinTilesPerCta = 4;
  int G = sms;
  if (U < (long long)G * kMinTilesPerCta) G = (int)(U / kMinTilesPerCta);
  if (G <= q) return bal;  // no gain over one CTA per segment
  for (; G > q; --G) {  // at most VA_MAX_SPLITS partials per row
    int slots = 0;
    for (long long s = 0; s < q; ++s) {
      const int n = balance_cta_of((s + 1) * vt - 1, U, G) - balance_cta_of(s * vt, U, G) + 1;
      slots = n > slots ? n : slots;
    }
    if (slots <= VA_MAX_SPLITS) {
      if (slots < 2) return bal;
      bal.G = G;
      bal.VT = vt;
      bal.NRT = nrt;
      bal.slots = slots;
      bal.U = U;
      return bal;
    }
  }
  return bal;
}

// Launchers implemented in the .cu files (internal C++ linkage).
cudaError_t launch_build_tree(const double* lp, const int32_t* tok, int B, int L, int K,
                              int budget, int32_t* parents, int32_t* tokens, int32_t* depth,
                              int32_t* n_nodes, cudaStream_t st);
cudaError_t launch_tree_accept(const int32_t* parents, const int32_t* tokens,
                               const int32_t* target_next, int B, int T, int32_t* path,
                               int32_t* accept_len, int32_t* next_token, cudaStream_t st);
cudaError_t launch_tree_mask(const int32_t* parents, int B, int T, uint64_t* mask,
                             int32_t* status, cudaStream_t st);
// Expired bounded waits of each attention kernel on the current device
// (0xFFFFFFFF if the counter cannot be read).
unsigned int tc_timeouts();
unsigned int simt_timeouts();

cudaError_t launch_attn_simt(const va_attn_args& a, SplitRange sp, float* o_part,
                             float* lse_part, cudaStream_t st, const Balance& bal);
// req_bad (nullable): per-request status of the attention launches; every row
// of a request with a non-zero status is written as 0 / -inf, and the status
// is copied into req_status (nullable) at that request.
cudaError_t launch_merge(const float* o_part, const float* lse_part, int S, long long rows,
                         int out_dtype, void* out, float* lse, cudaStream_t st,
                         const int32_t* req_bad = nullptr, int rows_per_req = 1,
                         int32_t* req_status = nullptr);
cudaError_t launch_request_order(const int32_t* kv_len, int B, int32_t* order, cudaStream_t st);
cudaError_t launch_attn_tc(const va_attn_args& a, SplitRange sp, const int32_t* order,
                           float* o_part, float* lse_part, cudaStream_t st, float out_scale);
cudaError_t launch_kv_widen(const va_attn_args& a, void* w_ckv, void* w_kpe, int32_t* w_table,
                            cudaStream_t st);

// Everything va_verify_attn launches once its arguments are checked and its
// split count S is known, with the workspace at `ws` laid out as above.
int run_verify(const va_attn_args& a, int S, void* ws, cudaStream_t st);

// A partials-only call: splits [first, first + count) of the S-way partition
// into the caller's o_part / lse_part, no merge; `ws` laid out for
// (S, partials_here = false).
int run_partials(const va_attn_args& a, SplitRange sp, void* ws, float* o_part, float* lse_part,
                 cudaStream_t st);

}  // namespace va
