// CUDA-core (FFMA) tree-verify attention: the fp32 path, a second,
// independent GPU path for bf16 inputs, and the path for a latent cache kept
// as FP8 E4M3 codes (either query type).
//
// Computes, per row (b, t, h), the masked softmax over the request's prefix
// and the row's tree ancestors in the absorbed latent space (page "The
// Milestone Commit...", section "The Context", item 2), online over key tiles
// so nothing but the running max / sum / output is kept per row.
//
// Layout: one CTA = 32 consecutive rows (row = t*H + h) of one request and one
// key split; 8 warps, warp w owns rows 4w..4w+3.  Key tiles of 32 keys
// (all 576 q.k dims, fp32 in shared memory, double-buffered with cp.async for
// fp32 inputs) are shared by the 32 rows.  Scores: lane = key.  Output: lane
// owns 16 of the 512 latent columns (4 groups of 4, 128 apart) for the
// warp's 4 rows, so every row's softmax state lives in one warp.
//
// FP8 cache: codes are widened to fp32 while they are staged; the cache scale
// is folded into the score scale and into the output normalisation, so the
// inner loops are those of the other types.
#include <cuda_fp8.h>

#include "va_common.cuh"

namespace va {
namespace {

constexpr int kRows = 32;       // rows per CTA
constexpr int kKeys = 32;       // keys per tile
constexpr int kThreads = 256;
constexpr int kQStride = kDqk;       // q rows are read as warp-wide broadcasts
constexpr int kKStride = kDqk + 4;   // +4 floats: lane-strided float4 reads avoid bank conflicts
constexpr size_t kSmemQ = (size_t)kRows * kQStride * sizeof(float);
constexpr size_t kSmemK = (size_t)kKeys * kKStride * sizeof(float);
constexpr size_t kSmemTotal = kSmemQ + 2 * kSmemK;

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n"); }

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Load 16 bytes of `src` (8 bf16 or 4 fp32 values) as fp32 into dst.
__device__ __forceinline__ void load_row_chunk(float* dst, const float* src) {
  cp_async16(dst, src);
}
__device__ __forceinline__ void load_row_chunk(float* dst, const __nv_bfloat16* src) {
  uint4 u = *reinterpret_cast<const uint4*>(src);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
  float4 a, b;
  float2 f;
  f = __bfloat1622float2(h[0]); a.x = f.x; a.y = f.y;
  f = __bfloat1622float2(h[1]); a.z = f.x; a.w = f.y;
  f = __bfloat1622float2(h[2]); b.x = f.x; b.y = f.y;
  f = __bfloat1622float2(h[3]); b.z = f.x; b.w = f.y;
  reinterpret_cast<float4*>(dst)[0] = a;
  reinterpret_cast<float4*>(dst)[1] = b;
}

// Load 16 FP8 E4M3 codes as fp32 into dst.  The hardware conversion to fp16
// is exact for every finite code (E4M3 values are a subset of fp16's), and
// so is fp16 -> fp32.  Code k of the 16 bytes lands in dst[k].
__device__ __forceinline__ void load_row_chunk(float* dst, const uint8_t* src) {
  const uint4 u = *reinterpret_cast<const uint4*>(src);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2 lo(__nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[i] & 0xffffu), __NV_E4M3));
    const __half2 hi(__nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[i] >> 16), __NV_E4M3));
    const float2 a = __half22float2(lo), b = __half22float2(hi);
    reinterpret_cast<float4*>(dst)[i] = make_float4(a.x, a.y, b.x, b.y);
  }
}

template <typename Tin>
struct Elems {  // values per 16-byte chunk
  static constexpr int v = 16 / sizeof(Tin);
};

// Stage keys [j0, j0 + 32) of request b (all inside one page) into sK.
// Keys at or past `hi`, and keys whose page index is out of range, are
// staged as zeros (the latter also flags the request).
template <typename Tin>
__device__ void stage_keys(float* sK, const Tin* __restrict__ c_kv, const Tin* __restrict__ k_pe,
                           int phys, int j0, int hi, int tid) {
  constexpr int V = Elems<Tin>::v;
  constexpr int kChunksC = kDc / V, kChunksR = kDr / V, kChunks = kChunksC + kChunksR;
  for (int c = tid; c < kKeys * kChunks; c += kThreads) {
    const int key = c / kChunks;
    const int part = c - key * kChunks;
    float* dst = sK + key * kKStride + (part < kChunksC ? part * V : kDc + (part - kChunksC) * V);
    const int j = j0 + key;
    if (j < hi && phys >= 0) {
      const size_t krow = (size_t)phys * kPage + (j & (kPage - 1));
      const Tin* src = part < kChunksC ? c_kv + krow * kDc + part * V
                                       : k_pe + krow * kDr + (part - kChunksC) * V;
      load_row_chunk(dst, src);
    } else {
#pragma unroll
      for (int e = 0; e < V; e += 4) *reinterpret_cast<float4*>(dst + e) = make_float4(0, 0, 0, 0);
    }
  }
}

// Tq: query element type; Tkv: cache element type (Tq, or uint8_t E4M3
// codes); Tout: output element type.  scale_log2 already holds the cache
// scale; out_scale (the cache scale, 1 for an unscaled cache) multiplies the
// normalised output.
template <typename Tq, typename Tkv, typename Tout>
__global__ void __launch_bounds__(kThreads, 1)
attn_simt_kernel(const Tq* __restrict__ q_nope, const Tq* __restrict__ q_pe,
                 const Tkv* __restrict__ c_kv, const Tkv* __restrict__ k_pe, int num_pages,
                 const int32_t* __restrict__ page_table, int max_pages,
                 const int32_t* __restrict__ kv_len_arr, const uint64_t* __restrict__ tree_mask,
                 int H, int T, float scale_log2, float out_scale, int S, int split0,
                 Tout* __restrict__ out,
                 float* __restrict__ lse_out, float* __restrict__ o_part,
                 float* __restrict__ lse_part, int32_t* __restrict__ req_status, int B) {
  extern __shared__ __align__(16) float smem[];
  float* sQ = smem;
  float* sK0 = sQ + kRows * kQStride;
  float* sK1 = sK0 + kKeys * kKStride;
  __shared__ int bad_page;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.y;
  const int split = blockIdx.z;
  const int R = T * H;
  const int row0 = blockIdx.x * kRows;
  const int W = (T + 63) >> 6;

  const int kv_len = kv_len_arr[b];
  const bool req_ok = kv_len >= T && kv_len <= max_pages * kPage;
  int lo = 0, hi = 0;
  if (req_ok) split_range(kv_len, S, split0 + split, &lo, &hi);
  const int P = kv_len - T;
  if (tid == 0) bad_page = 0;
  __syncthreads();

  // q rows -> shared (fp32).  Rows past R are zero.
  {
    constexpr int V = Elems<Tq>::v;
    constexpr int kChunksC = kDc / V, kChunks = kChunksC + kDr / V;
    for (int c = tid; c < kRows * kChunks; c += kThreads) {
      const int r = c / kChunks, part = c - r * kChunks;
      float* dst = sQ + r * kQStride + (part < kChunksC ? part * V : kDc + (part - kChunksC) * V);
      const int row = row0 + r;
      if (row < R) {
        const size_t g = (size_t)b * R + row;
        const Tq* src = part < kChunksC ? q_nope + g * kDc + part * V
                                         : q_pe + g * kDr + (part - kChunksC) * V;
        load_row_chunk(dst, src);
      } else {
#pragma unroll
        for (int e = 0; e < V; e += 4) *reinterpret_cast<float4*>(dst + e) = make_float4(0, 0, 0, 0);
      }
    }
  }

  // Per-row state of this warp's 4 rows (replicated across lanes).
  float m[4], l[4];
  uint64_t mw0[4], mw1[4];
  bool live[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int row = row0 + warp * 4 + r;
    m[r] = -INFINITY;
    l[r] = 0.f;
    live[r] = false;
    mw0[r] = mw1[r] = 0;
    if (row < R && req_ok) {
      const int t = row / H;
      const uint64_t* mrow = tree_mask + ((size_t)b * T + t) * W;
      mw0[r] = mrow[0];
      mw1[r] = W > 1 ? mrow[1] : 0ull;
      live[r] = mask_bit(mrow, t);
    }
  }
  float acc[4][16];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 16; ++c) acc[r][c] = 0.f;

  const int ntiles = (hi > lo) ? (hi - lo + kKeys - 1) / kKeys : 0;
  auto phys_of = [&](int j0) -> int {
    const int pg = page_table[(size_t)b * max_pages + j0 / kPage];
    if (pg < 0 || pg >= num_pages) { bad_page = 1; return -1; }
    return pg;
  };
  if (ntiles > 0) stage_keys<Tkv>(sK0, c_kv, k_pe, phys_of(lo), lo, hi, tid);
  cp_async_commit();

  for (int it = 0; it < ntiles; ++it) {
    float* sK = (it & 1) ? sK1 : sK0;
    cp_async_wait_all();
    __syncthreads();
    if (it + 1 < ntiles) {
      const int jn = lo + (it + 1) * kKeys;
      stage_keys<Tkv>((it & 1) ? sK0 : sK1, c_kv, k_pe, phys_of(jn), jn, hi, tid);
    }
    cp_async_commit();

    // scores: lane = key, 4 rows
    const int j = lo + it * kKeys + lane;
    float s[4] = {0.f, 0.f, 0.f, 0.f};
    {
      const float* kr = sK + lane * kKStride;
      const float* q0 = sQ + (warp * 4) * kQStride;
#pragma unroll 4
      for (int d = 0; d < kDqk; d += 4) {
        const float4 kv = *reinterpret_cast<const float4*>(kr + d);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float4 qv = *reinterpret_cast<const float4*>(q0 + r * kQStride + d);
          s[r] = fmaf(qv.x, kv.x, s[r]);
          s[r] = fmaf(qv.y, kv.y, s[r]);
          s[r] = fmaf(qv.z, kv.z, s[r]);
          s[r] = fmaf(qv.w, kv.w, s[r]);
        }
      }
    }
    float alpha[4], pk[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      bool vis = live[r] && j < hi;
      if (vis && j >= P) {
        const int i = j - P;
        vis = ((i < 64 ? (mw0[r] >> i) : (mw1[r] >> (i - 64))) & 1ull) != 0;
      }
      const float x = vis ? s[r] * scale_log2 : -INFINITY;
      const float mnew = fmaxf(m[r], warp_max(x));
      float p = 0.f;
      alpha[r] = 1.f;
      if (mnew != -INFINITY) {
        p = exp2f(x - mnew);
        alpha[r] = exp2f(m[r] - mnew);  // m = -inf -> 0
      }
      l[r] = l[r] * alpha[r] + warp_sum(p);
      m[r] = mnew;
      pk[r] = p;
    }
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 16; ++c) acc[r][c] *= alpha[r];
    // PV: V = the staged c_kv columns; p of key k comes from lane k
#pragma unroll 4
    for (int k = 0; k < kKeys; ++k) {
      float pr[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) pr[r] = __shfl_sync(0xffffffffu, pk[r], k);
      const float* vr = sK + k * kKStride + lane * 4;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const float4 v = *reinterpret_cast<const float4*>(vr + g * 128);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          acc[r][g * 4 + 0] = fmaf(pr[r], v.x, acc[r][g * 4 + 0]);
          acc[r][g * 4 + 1] = fmaf(pr[r], v.y, acc[r][g * 4 + 1]);
          acc[r][g * 4 + 2] = fmaf(pr[r], v.z, acc[r][g * 4 + 2]);
          acc[r][g * 4 + 3] = fmaf(pr[r], v.w, acc[r][g * 4 + 3]);
        }
      }
    }
  }
  cp_async_wait_all();
  __syncthreads();
  if (tid == 0 && req_status && (!req_ok || bad_page)) req_status[b] = VA_ERR_INVALID_ARG;

  // epilogue
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int row = row0 + warp * 4 + r;
    if (row >= R) continue;
    const bool empty = !(l[r] > 0.f) || !req_ok || bad_page;
    const float inv = empty ? 0.f : out_scale / l[r];
    const float lse = empty ? -INFINITY : (m[r] + log2f(l[r])) * kLn2;
    const size_t g = (size_t)b * R + row;
    if (!o_part) {
      Tout* o = out + g * kDc + lane * 4;
#pragma unroll
      for (int gq = 0; gq < 4; ++gq)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[gq * 128 + e] = from_f32<Tout>(acc[r][gq * 4 + e] * inv);
      if (lane == 0) lse_out[g] = lse;
    } else {
      const size_t rows_total = (size_t)B * R;
      float* o = o_part + ((size_t)split * rows_total + g) * kDc + lane * 4;
#pragma unroll
      for (int gq = 0; gq < 4; ++gq)
        *reinterpret_cast<float4*>(o + gq * 128) =
            make_float4(acc[r][gq * 4 + 0] * inv, acc[r][gq * 4 + 1] * inv,
                        acc[r][gq * 4 + 2] * inv, acc[r][gq * 4 + 3] * inv);
      if (lane == 0) lse_part[(size_t)split * rows_total + g] = lse;
    }
  }
}

template <typename Tq, typename Tkv, typename Tout>
cudaError_t launch_typed(const va_attn_args& a, SplitRange sp, float* o_part, float* lse_part,
                         cudaStream_t st) {
  auto kern = attn_simt_kernel<Tq, Tkv, Tout>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemTotal);
  if (e != cudaSuccess) return e;
  const int R = a.T * a.H;
  dim3 grid((R + kRows - 1) / kRows, a.B, sp.count);
  const float kv_scale = (a.flags & VA_FLAG_KV_FP8_E4M3) ? a.kv_scale : 1.f;
  const float scale_log2 = (a.scale * kv_scale) * kLog2e;
  kern<<<grid, kThreads, kSmemTotal, st>>>(
      (const Tq*)a.q_nope, (const Tq*)a.q_pe, (const Tkv*)a.c_kv, (const Tkv*)a.k_pe,
      a.num_pages, a.page_table, a.max_pages, a.kv_len, a.tree_mask, a.H, a.T, scale_log2,
      kv_scale, sp.S, sp.first, (Tout*)a.out, a.lse, o_part, lse_part, a.req_status, a.B);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_simt(const va_attn_args& a, SplitRange S, float* o_part,
                             float* lse_part, cudaStream_t st) {
  if (a.B == 0) return cudaSuccess;
  const bool fp8 = (a.flags & VA_FLAG_KV_FP8_E4M3) != 0;
  if (a.dtype == VA_F32)
    return fp8 ? launch_typed<float, uint8_t, float>(a, S, o_part, lse_part, st)
               : launch_typed<float, float, float>(a, S, o_part, lse_part, st);
  return fp8 ? launch_typed<__nv_bfloat16, uint8_t, __nv_bfloat16>(a, S, o_part, lse_part, st)
             : launch_typed<__nv_bfloat16, __nv_bfloat16, __nv_bfloat16>(a, S, o_part, lse_part, st);
}

}  // namespace va
