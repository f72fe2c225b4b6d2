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
// key split, 8 warps; key tiles of 32 keys (all 576 q.k dims, fp32 in shared
// memory, double-buffered; the staged Q shares the second key buffer, which
// is free until the second tile).  A staged tile is its 32 c_kv rows
// ([32][512], dense) followed by its 32 k_pe rows ([32][64]): for an fp32
// cache both parts are contiguous in the page, so warp 0 stages a tile with
// nine bulk copies completed on an mbarrier (bounded wait), and the staging
// costs the other warps nothing.  Per tile:
//  * S = Q.K^T (32 x 32): warp w takes 72 of the 576 dims of every row and
//    key: c_kv columns [64w, 64w + 64) and k_pe columns [8w, 8w + 8).  Lane
//    (i, j) keeps the Q of rows i + 8a (a = 0..3) on its 18 of them in
//    registers for the whole key range -- the column quads 64w + 16m + 4j
//    (m = 0..3) and k_pe pair 8w + 2j, so the four j lanes read adjacent
//    16-byte chunks of a key row, conflict-free without padding -- and
//    reads only K from shared memory (one 16-byte load feeds 16 FFMAs
//    across its 4 rows).  The four dim sub-slices of a warp are summed by a
//    two-step shuffle butterfly; each lane visits its 8 keys of a group in
//    the order c ^ (4 j0 + 2 j1) (j = j0 + 2 j1), which makes the entries it
//    keeps and gives the same at every lane, so the butterfly needs no
//    selects.  The 8 warps' partial tiles are summed through shared memory.
//  * softmax: 8 lanes per row, 4 keys each; the running max moves (and O is
//    rescaled) only when a tile raises it by more than 2^8.
//  * O += P.V (32 x 512): warp w owns columns [64w, 64w + 64), each lane an
//    8-row x 8-column register tile, so two 16-byte loads of P and two of V
//    feed 64 FFMAs.
// All lanes of a warp read the same key row in both products, so the dense
// rows cause no bank conflicts there.
//
// FP8 cache: codes are widened to fp32 while they are staged; the cache scale
// is folded into the score scale and into the output normalisation, so the
// inner loops are those of the other types.
#include <cuda_fp8.h>

#include "va_bulk.cuh"
#include "va_common.cuh"

namespace va {

__device__ unsigned int g_simt_timeouts = 0;  // count of staging waits that expired

namespace {

constexpr int kRows = 32;       // rows per CTA
constexpr int kKeys = 32;       // keys per tile
constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kSub = kDqk / kWarps / 4;   // dims per lane (four sub-slices per warp): 18
constexpr int kSpStride = 36;              // partial-score tile [key][row], padded
constexpr int kPStride = kRows + 4;        // probabilities [key][row], padded
constexpr float kRescaleLog2 = 8.0f;       // lazy max: rescale only past 2^8
constexpr int kTileFloats = kKeys * kDqk;  // one staged tile: [32][512] c_kv, then [32][64] k_pe
constexpr size_t kSmemK = (size_t)kTileFloats * sizeof(float);
constexpr size_t kSmemSp = (size_t)kWarps * kKeys * kSpStride * sizeof(float);
constexpr size_t kSmemP = (size_t)kKeys * kPStride * sizeof(float);
constexpr size_t kSmemTotal = 2 * kSmemK + kSmemSp + kSmemP + 3 * kRows * sizeof(float);
static_assert(kDqk % (8 * kWarps) == 0, "dims split evenly into float2 steps per lane");
static_assert(kRows <= kKeys, "the staged Q fits in a key buffer");
static_assert(kKeys % 8 == 0 && kKeys / 8 <= 8, "8-key groups in Q.K^T; 8 softmax lanes per row");
static_assert(kKeys == 32, "bulk staging: lanes 0-7 of warp 0 copy 4 c_kv rows each");
static_assert(kRows == kKeys, "the staged Q uses the tile layout");
static_assert(kDc == 64 * kWarps && kDr == 8 * kWarps && kSub == 18,
              "per warp: 64 c_kv columns and 8 k_pe columns, 8 + 1 pairs per lane");

// Row `key` of the c_kv part / the k_pe part of a staged tile.
__device__ __forceinline__ float* c_row(float* t, int key) { return t + key * kDc; }
__device__ __forceinline__ float* r_row(float* t, int key) { return t + kKeys * kDc + key * kDr; }

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n"); }


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

// Two fp32 fused multiply-adds in one instruction (sm_100 packed f32x2),
// each rounded to nearest exactly like fmaf: d = a * b + c per element.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(d)
      : "l"(*reinterpret_cast<unsigned long long*>(&a)),
        "l"(*reinterpret_cast<unsigned long long*>(&b)),
        "l"(*reinterpret_cast<unsigned long long*>(&c)));
  return *reinterpret_cast<float2*>(&d);
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
    float* dst =
        part < kChunksC ? c_row(sK, key) + part * V : r_row(sK, key) + (part - kChunksC) * V;
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

// Key staging for element types that are widened on the way into shared
// memory (bf16, FP8 codes): the next tile's 16-byte chunks are loaded into
// registers in two halves, one before the current tile's Q.K^T and one before
// its P.V, and each half is converted and stored after the products it
// overlaps.  Keys at or past `hi`, and keys of an out-of-range page, become
// zeros.
template <typename Tin>
struct RegStage {
  static constexpr int V = Elems<Tin>::v;
  static constexpr int kChunksC = kDc / V, kChunks = kChunksC + kDr / V;
  static constexpr int kTotal = kKeys * kChunks;
  static constexpr int kPer = (kTotal / 2 + kThreads - 1) / kThreads;  // per half
  static_assert(kTotal % 2 == 0, "halves of equal size");
  uint4 buf[kPer];

  // half h covers chunks [h kTotal/2, (h + 1) kTotal/2)
  __device__ __forceinline__ void load(const Tin* __restrict__ c_kv, const Tin* __restrict__ k_pe,
                                       int phys, int j0, int hi, int tid, int h) {
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int c = h * (kTotal / 2) + tid + i * kThreads;
      buf[i] = make_uint4(0, 0, 0, 0);
      if (c < (h + 1) * (kTotal / 2)) {
        const int key = c / kChunks, part = c - key * kChunks;
        const int j = j0 + key;
        if (j < hi && phys >= 0) {
          const size_t krow = (size_t)phys * kPage + (j & (kPage - 1));
          const Tin* src = part < kChunksC ? c_kv + krow * kDc + part * V
                                           : k_pe + krow * kDr + (part - kChunksC) * V;
          buf[i] = *reinterpret_cast<const uint4*>(src);
        }
      }
    }
  }
  __device__ __forceinline__ void store(float* sK, int tid, int h) const {
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int c = h * (kTotal / 2) + tid + i * kThreads;
      if (c < (h + 1) * (kTotal / 2)) {
        const int key = c / kChunks, part = c - key * kChunks;
        float* dst =
            part < kChunksC ? c_row(sK, key) + part * V : r_row(sK, key) + (part - kChunksC) * V;
        load_row_chunk(dst, reinterpret_cast<const Tin*>(&buf[i]));
      }
    }
  }
};

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
                 Balance bal, int stall_copies, Tout* __restrict__ out,
                 float* __restrict__ lse_out, float* __restrict__ o_part,
                 float* __restrict__ lse_part, int32_t* __restrict__ req_status, int B) {
  extern __shared__ __align__(16) float smem[];
  float* sK0 = smem;
  float* sK1 = sK0 + kTileFloats;           // also the staged Q until tile 1 is staged
  float* sQ = sK1;
  float* sSp = sK1 + kTileFloats;           // [warp][key][row] partial scores
  float* sP = sSp + kWarps * kKeys * kSpStride;  // [key][row] probabilities
  float* sAlpha = sP + kKeys * kPStride;    // [row] rescale factor of this tile
  float* sM = sAlpha + kRows;               // [row] final running max (log2 domain)
  float* sL = sM + kRows;                   // [row] final sum
  __shared__ int bad_page;
  __shared__ int aborted;                   // a staging wait expired
  __shared__ __align__(8) uint64_t kv_full; // bulk-staged tile t completes phase t
  // an fp32 cache is staged by bulk copies; other types are widened on the way
  constexpr bool kBulk = sizeof(Tkv) == 4;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int R = T * H;
  const int W = (T + 63) >> 6;
  const size_t rows_total = (size_t)B * R;
  if (tid == 0) {
    aborted = 0;
    if (kBulk) {
      bulk::mbar_init(&kv_full, 1);
      bulk::fence_mbar_init();
    }
  }

  // Segments of this CTA: one (blockIdx: row tile, request, split) without a
  // balanced plan, else the pieces of its virtual-tile range [u0, u1).
  int seg_begin = 0, seg_end = 1;
  long long u0 = 0, u1 = 0;
  if (bal.G) {
    u0 = (long long)blockIdx.x * bal.U / bal.G;
    u1 = (long long)(blockIdx.x + 1) * bal.U / bal.G;
    seg_begin = (int)(u0 / bal.VT);
    seg_end = u1 > u0 ? (int)((u1 - 1) / bal.VT) + 1 : seg_begin;
  }
  uint32_t staged = 0;  // bulk stages issued and waited for before this segment
  for (int seg = seg_begin; seg < seg_end; ++seg) {
    int b, row0, split, t0 = 0, t1 = 0;
    bool seg_last = false;  // this CTA ends the segment (balanced plan)
    if (bal.G) {
      b = seg / bal.NRT;
      row0 = (seg - b * bal.NRT) * kRows;
      const long long s0 = (long long)seg * bal.VT;
      split = (int)blockIdx.x - balance_cta_of(s0, bal.U, bal.G);
      seg_last = (int)blockIdx.x == balance_cta_of(s0 + bal.VT - 1, bal.U, bal.G);
      t0 = (int)((u0 > s0 ? u0 : s0) - s0);
      t1 = (int)((u1 < s0 + bal.VT ? u1 : s0 + bal.VT) - s0);
    } else {
      b = blockIdx.y;
      row0 = blockIdx.x * kRows;
      split = blockIdx.z;
    }
    const int kv_len = kv_len_arr[b];
    const bool req_ok = kv_len >= T && kv_len <= max_pages * kPage;
    int lo = 0, hi = 0;
    if (req_ok) {
      if (bal.G) {
        lo = t0 * kKeys < kv_len ? t0 * kKeys : kv_len;
        hi = t1 * kKeys < kv_len ? t1 * kKeys : kv_len;
      } else {
        split_range(kv_len, S, split0 + split, &lo, &hi);
      }
    }
    const int P = kv_len - T;
    __syncthreads();  // the previous segment's epilogue is done with sM / sL
    if (tid == 0) bad_page = 0;
    __syncthreads();

    // q rows -> shared (fp32).  Rows past R are zero.  (Nothing is staged once
    // a wait has expired: a copy could still be landing.)
    if (!aborted) {
      constexpr int V = Elems<Tq>::v;
      constexpr int kChunksC = kDc / V, kChunks = kChunksC + kDr / V;
      for (int c = tid; c < kRows * kChunks; c += kThreads) {
        const int r = c / kChunks, part = c - r * kChunks;
        float* dst =
            part < kChunksC ? c_row(sQ, r) + part * V : r_row(sQ, r) + (part - kChunksC) * V;
        const int row = row0 + r;
        if (row < R) {
          const size_t g = (size_t)b * R + row;
          const Tq* src = part < kChunksC ? q_nope + g * kDc + part * V
                                           : q_pe + g * kDr + (part - kChunksC) * V;
          load_row_chunk(dst, src);
        } else {
#pragma unroll
          for (int e = 0; e < V; e += 4)
            *reinterpret_cast<float4*>(dst + e) = make_float4(0, 0, 0, 0);
        }
      }
    }

    // Softmax role: row sr of the CTA, keys sk + 8 e (e = 0..3) of each tile;
    // the row's 8 lanes keep identical copies of its running max and sum.
    const int sr = tid >> 3, sk = tid & 7;
    float m_used = -INFINITY, l = 0.f;
    uint64_t mw0 = 0, mw1 = 0;
    bool live = false;
    {
      const int row = row0 + sr;
      if (row < R && req_ok) {
        const int t = row / H;
        const uint64_t* mrow = tree_mask + ((size_t)b * T + t) * W;
        mw0 = mrow[0];
        mw1 = W > 1 ? mrow[1] : 0ull;
        live = mask_bit(mrow, t);
      }
    }
    // Q.K^T role: rows qi + 8a (a = 0..3), this warp's dims of sub-slice qj, all keys.
    const int qi = lane & 7, qj = lane >> 3;
    // P.V role: rows 8 pi .. 8 pi + 7; columns 64 warp + 4 pj + {0..3} and +32.
    const int pi = lane >> 3, pj = lane & 7;
    const int col0 = 64 * warp + 4 * pj;
    float2 acc[8][4];  // columns (col0 + 2c, +1) for c < 2, (col0 + 32 + 2(c-2), +1) after
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[r][c] = make_float2(0.f, 0.f);

    // after an expired wait the CTA computes nothing more (its mbarrier phase
    // is unknown): its remaining segments come out empty
    const int ntiles = (hi > lo && !aborted) ? (hi - lo + kKeys - 1) / kKeys : 0;
    // Page-table entries are read one tile ahead of their use, so the global
    // load's latency does not sit between a tile's barrier and its staging.
    auto page_of = [&](int j0) -> int { return page_table[(size_t)b * max_pages + j0 / kPage]; };
    auto checked = [&](int pg) -> int {
      if (pg < 0 || pg >= num_pages) { bad_page = 1; return -1; }
      return pg;
    };
    auto phys_of = [&](int j0) -> int { return checked(page_of(j0)); };
    int pg_ahead = ntiles > 1 ? page_of(lo + kKeys) : 0;  // entry of the tile being staged next
    // Bulk staging of keys [j0, j0 + 32) (one page) into dst, called by every
    // thread alike: lanes 0-7 of warp 0 copy 4 c_kv rows each (8 KB), lane 8
    // the 32 k_pe rows (8 KB).  All 32 rows are copied: rows at or past `hi`
    // lie in the same page, hold finite values, and get probability exactly
    // 0.  A bad page instead zeroes the tile with plain stores and completes
    // the phase without copies.
    auto stage_bulk = [&](float* dst, int phys, int j0) {
      if constexpr (kBulk) {
        if (phys >= 0) {
          if (warp == 0) {
            bulk::fence_proxy_async();
            if (lane == 0)
              bulk::mbar_arrive_expect_tx(&kv_full, kTileFloats * (uint32_t)sizeof(float));
            __syncwarp();
            const size_t krow = (size_t)phys * kPage + (j0 & (kPage - 1));
            constexpr int kRowsPerCopy = kKeys / 8;
            if (stall_copies) {
              // test hook: the barrier expects the bytes, no copy brings them
            } else if (lane < 8)
              bulk::copy_g2s(c_row(dst, kRowsPerCopy * lane),
                             c_kv + (krow + kRowsPerCopy * lane) * kDc,
                             kRowsPerCopy * kDc * sizeof(float), &kv_full);
            else if (lane == 8)
              bulk::copy_g2s(r_row(dst, 0), k_pe + krow * kDr, kKeys * kDr * sizeof(float),
                             &kv_full);
          }
        } else {
          for (int c = tid; c < kTileFloats / 4; c += kThreads)
            reinterpret_cast<float4*>(dst)[c] = make_float4(0.f, 0.f, 0.f, 0.f);
          bulk::fence_proxy_async();
          if (tid == 0) bulk::mbar_arrive_expect_tx(&kv_full, 0);
        }
      }
    };
    RegStage<Tkv> reg;
    if (ntiles > 0) {
      if constexpr (kBulk) stage_bulk(sK0, phys_of(lo), lo);
      else stage_keys<Tkv>(sK0, c_kv, k_pe, phys_of(lo), lo, hi, tid);
    }
    // this lane's Q: rows qi + 8 a, c_kv column quads 64 warp + 16 m + 4 qj
    // (m = 0..3) and k_pe pair 8 warp + 2 qj, kept in registers for every key
    // tile
    float2 qr[4][kSub / 2];  // (even dim, odd dim) pairs; [8] is the k_pe pair
    cp_async_commit();
    cp_async_wait_all();
    if (kBulk) bulk::fence_proxy_async();  // the staged Q's buffer later takes bulk copies
    __syncthreads();
    {
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const float* qc = c_row(sQ, qi + 8 * a) + 64 * warp + 4 * qj;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const float4 q4 = *reinterpret_cast<const float4*>(qc + 16 * m);
          qr[a][2 * m] = make_float2(q4.x, q4.y);
          qr[a][2 * m + 1] = make_float2(q4.z, q4.w);
        }
        qr[a][8] = *reinterpret_cast<const float2*>(r_row(sQ, qi + 8 * a) + 8 * warp + 2 * qj);
      }
    }

    for (int it = 0; it < ntiles; ++it) {
      float* sK = (it & 1) ? sK1 : sK0;
      float* sKn = (it & 1) ? sK0 : sK1;
      // tile it staged; the previous tile's P.V (and, at the first tile, every
      // read of the staged Q) is done, so the other buffer is free
      if constexpr (kBulk) {
        const bool ok = bulk::mbar_wait(&kv_full, (staged + it) & 1);
        if (__syncthreads_or(!ok)) {
          if (tid == 0) {
            aborted = 1;
            atomicAdd(&g_simt_timeouts, 1u);
          }
          bulk::settle();  // copies already issued land before the CTA moves on
          break;
        }
      } else {
        __syncthreads();
      }
      const bool more = it + 1 < ntiles;
      const int jn = lo + (it + 1) * kKeys;
      const int physn = more ? checked(pg_ahead) : -1;
      if (it + 2 < ntiles) pg_ahead = page_of(jn + kKeys);
      if (more) {
        if constexpr (kBulk) stage_bulk(sKn, physn, jn);
        else reg.load(c_kv, k_pe, physn, jn, hi, tid, 0);
      }

      // ---- partial scores of this warp's dim slice: the lane's Q rows stay in
      // registers (qr), only K comes from shared memory; the warp's four dim
      // sub-slices are summed with shuffles before the cross-warp reduction
      {
        const bool b0 = (qj & 1) != 0, b1 = (qj >> 1) != 0;
        const int kmask = 4 * b0 + 2 * b1;  // this lane visits key c of a group as c ^ kmask
        float* sp = sSp + warp * kKeys * kSpStride;
#pragma unroll
        for (int half = 0; half < kKeys / 8; ++half) {
          // even and odd dims accumulate in the two halves of a packed pair
          float2 acc2[4][8];
#pragma unroll
          for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int c = 0; c < 8; ++c) acc2[a][c] = make_float2(0.f, 0.f);
          // rows of the key pairs (c & 6) ^ kmask of this group; c & 1 is a
          // compile-time offset from them
          const float* kcb[4];
          const float* krb[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            kcb[i] = c_row(sK, 8 * half + ((2 * i) ^ kmask)) + 64 * warp + 4 * qj;
            krb[i] = r_row(sK, 8 * half + ((2 * i) ^ kmask)) + 8 * warp + 2 * qj;
          }
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float* kcc = kcb[c >> 1] + (c & 1) * kDc;
            float2 kv[kSub / 2];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              const float4 k4 = *reinterpret_cast<const float4*>(kcc + 16 * m);
              kv[2 * m] = make_float2(k4.x, k4.y);
              kv[2 * m + 1] = make_float2(k4.z, k4.w);
            }
            kv[8] = *reinterpret_cast<const float2*>(krb[c >> 1] + (c & 1) * kDr);
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
              for (int m2 = 0; m2 < kSub / 2; ++m2)
                acc2[a][c] = fma2(qr[a][m2], kv[m2], acc2[a][c]);
          }
          // acc8[a][c]: row qi + 8a, key 8 half + (c ^ kmask), over this lane's dims
          float acc8[4][8];
#pragma unroll
          for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int c = 0; c < 8; ++c) acc8[a][c] = acc2[a][c].x + acc2[a][c].y;
          // Lanes qi + 8 qj, qj = 0..3, hold the same rows over four dim
          // sub-slices.  Step 1 (lane ^ 8 flips j0): entry c < 4 of both lanes
          // is a key with bit 2 = j0 of this lane, entry 4 + c of the partner
          // the same key; step 2 (lane ^ 16 flips j1) likewise on bit 1.
          float r1[4][4];
#pragma unroll
          for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int c = 0; c < 4; ++c)
              r1[a][c] = acc8[a][c] + __shfl_xor_sync(0xffffffffu, acc8[a][4 + c], 8);
#pragma unroll
          for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const float v = r1[a][c] + __shfl_xor_sync(0xffffffffu, r1[a][2 + c], 16);
              // key 8 half + (c ^ kmask) = 8 half + 4 b0 + 2 b1 + c of row qi + 8 a,
              // over the warp's dims
              sp[(8 * half + 4 * b0 + 2 * b1 + c) * kSpStride + qi + 8 * a] = v;
            }
        }
      }
      // the other buffer is free (see the top of the loop): the first half of
      // the next tile goes in, the second half's loads overlap P.V
      if (!kBulk && more) {
        reg.store(sKn, tid, 0);
        reg.load(c_kv, k_pe, physn, jn, hi, tid, 1);
      }
      __syncthreads();  // partial scores visible

      // ---- online softmax of row sr, keys sk + 8 e
      {
        constexpr int kE = kKeys / 8;
        const int jt = lo + it * kKeys;
        float x[kE];
#pragma unroll
        for (int e = 0; e < kE; ++e) {
          const int key = sk + 8 * e;
          float sum = 0.f;
#pragma unroll
          for (int w = 0; w < kWarps; ++w) sum += sSp[(w * kKeys + key) * kSpStride + sr];
          const int j = jt + key;
          bool vis = live && j < hi;
          if (vis && j >= P) {
            const int i = j - P;
            vis = ((i < 64 ? (mw0 >> i) : (mw1 >> (i - 64))) & 1ull) != 0;
          }
          x[e] = vis ? sum * scale_log2 : -INFINITY;
        }
        float tmax = x[0];
#pragma unroll
        for (int e = 1; e < kE; ++e) tmax = fmaxf(tmax, x[e]);
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
        float alpha = 1.f;
        if (tmax > m_used + kRescaleLog2 || (m_used == -INFINITY && tmax != -INFINITY)) {
          alpha = m_used == -INFINITY ? 1.f : exp2f(m_used - tmax);  // O and l are 0 before
          m_used = tmax;
        }
        float psum = 0.f;
#pragma unroll
        for (int e = 0; e < kE; ++e) {
          const float p = m_used != -INFINITY ? exp2f(x[e] - m_used) : 0.f;
          psum += p;
          sP[(sk + 8 * e) * kPStride + sr] = p;
        }
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
        l = l * alpha + psum;
        if (sk == 0) sAlpha[sr] = alpha;
      }
      __syncthreads();  // probabilities and rescale factors visible

      // ---- O += P.V on this lane's 8 x 8 tile
      {
        const float4 a0 = *reinterpret_cast<const float4*>(sAlpha + 8 * pi);
        const float4 a1 = *reinterpret_cast<const float4*>(sAlpha + 8 * pi + 4);
        const float al[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        bool any = false;
#pragma unroll
        for (int r = 0; r < 8; ++r) any |= al[r] != 1.f;
        if (any) {
#pragma unroll
          for (int r = 0; r < 8; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              acc[r][c].x *= al[r];
              acc[r][c].y *= al[r];
            }
        }
#pragma unroll 4
        for (int k = 0; k < kKeys; ++k) {
          const float4 p0 = *reinterpret_cast<const float4*>(sP + k * kPStride + 8 * pi);
          const float4 p1 = *reinterpret_cast<const float4*>(sP + k * kPStride + 8 * pi + 4);
          const float4 v0 = *reinterpret_cast<const float4*>(c_row(sK, k) + col0);
          const float4 v1 = *reinterpret_cast<const float4*>(c_row(sK, k) + col0 + 32);
          const float pr[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
          const float2 vv[4] = {make_float2(v0.x, v0.y), make_float2(v0.z, v0.w),
                                make_float2(v1.x, v1.y), make_float2(v1.z, v1.w)};
#pragma unroll
          for (int r = 0; r < 8; ++r) {
            const float2 pp = make_float2(pr[r], pr[r]);
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[r][c] = fma2(pp, vv[c], acc[r][c]);
          }
        }
      }
      if (!kBulk && more) reg.store(sKn, tid, 1);
    }
    if (kBulk) staged += ntiles;
    cp_async_wait_all();
    if (sk == 0) {
      sM[sr] = m_used;
      sL[sr] = l;
    }
    __syncthreads();
    if (tid == 0 && req_status && (!req_ok || bad_page || aborted))
      req_status[b] = aborted ? VA_ERR_CUDA : VA_ERR_INVALID_ARG;

    // epilogue: lane writes rows 8 pi + r, columns col0 .. +3 and col0 + 32 .. +3
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int rr = 8 * pi + r;
      const int row = row0 + rr;
      if (row >= R) continue;
      const float lr = sL[rr];
      const bool empty = !(lr > 0.f) || !req_ok || bad_page || aborted;
      // an expired wait leaves the accumulators undefined: multiply by 0 only
      // what is known to be finite
      const float inv = empty ? 0.f : out_scale / lr;
      if (aborted) {
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = make_float2(0.f, 0.f);
      }
      const float lse = empty ? -INFINITY : (sM[rr] + log2f(lr)) * kLn2;
      const size_t g = (size_t)b * R + row;
      if (!o_part) {
        Tout* o = out + g * kDc + col0;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          o[2 * e] = from_f32<Tout>(acc[r][e].x * inv);
          o[2 * e + 1] = from_f32<Tout>(acc[r][e].y * inv);
          o[32 + 2 * e] = from_f32<Tout>(acc[r][2 + e].x * inv);
          o[32 + 2 * e + 1] = from_f32<Tout>(acc[r][2 + e].y * inv);
        }
        if (warp == 0 && pj == 0) lse_out[g] = lse;
      } else {
        float* o = o_part + ((size_t)split * rows_total + g) * kDc + col0;
        *reinterpret_cast<float4*>(o) = make_float4(acc[r][0].x * inv, acc[r][0].y * inv,
                                                    acc[r][1].x * inv, acc[r][1].y * inv);
        *reinterpret_cast<float4*>(o + 32) = make_float4(acc[r][2].x * inv, acc[r][2].y * inv,
                                                         acc[r][3].x * inv, acc[r][3].y * inv);
        if (warp == 0 && pj == 0) lse_part[(size_t)split * rows_total + g] = lse;
      }
    }
    // the CTA that ends a segment marks the slots no CTA wrote as empty
    if (seg_last) {
      const int rows = R - row0 < kRows ? R - row0 : kRows;
      for (int i = tid; i < (bal.slots - split - 1) * rows; i += kThreads) {
        const int sl = split + 1 + i / rows;
        lse_part[(size_t)sl * rows_total + (size_t)b * R + row0 + i % rows] = -INFINITY;
      }
    }
  }  // segments
}

template <typename Tq, typename Tkv, typename Tout>
cudaError_t launch_typed(const va_attn_args& a, SplitRange sp, float* o_part, float* lse_part,
                         cudaStream_t st, const Balance& bal) {
  auto kern = attn_simt_kernel<Tq, Tkv, Tout>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemTotal);
  if (e != cudaSuccess) return e;
  const int R = a.T * a.H;
  const dim3 grid = bal.G ? dim3(bal.G, 1, 1) : dim3((R + kRows - 1) / kRows, a.B, sp.count);
  const float kv_scale = (a.flags & VA_FLAG_KV_FP8_E4M3) ? a.kv_scale : 1.f;
  const float scale_log2 = (a.scale * kv_scale) * kLog2e;
  kern<<<grid, kThreads, kSmemTotal, st>>>(
      (const Tq*)a.q_nope, (const Tq*)a.q_pe, (const Tkv*)a.c_kv, (const Tkv*)a.k_pe,
      a.num_pages, a.page_table, a.max_pages, a.kv_len, a.tree_mask, a.H, a.T, scale_log2,
      kv_scale, sp.S, sp.first, bal, (a.flags & VA_FLAG_TEST_STALL_COPIES) ? 1 : 0, (Tout*)a.out,
      a.lse, o_part, lse_part, a.req_status, a.B);
  return cudaGetLastError();
}

}  // namespace

unsigned int simt_timeouts() {
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_simt_timeouts, sizeof(v)) != cudaSuccess) return 0xFFFFFFFFu;
  return v;
}

cudaError_t launch_attn_simt(const va_attn_args& a, SplitRange S, float* o_part,
                             float* lse_part, cudaStream_t st, const Balance& bal) {
  if (a.B == 0) return cudaSuccess;
  if (bal.G && (!o_part || !lse_part || S.count != bal.slots)) return cudaErrorInvalidValue;
  const bool fp8 = (a.flags & VA_FLAG_KV_FP8_E4M3) != 0;
  if (a.dtype == VA_F32)
    return fp8 ? launch_typed<float, uint8_t, float>(a, S, o_part, lse_part, st, bal)
               : launch_typed<float, float, float>(a, S, o_part, lse_part, st, bal);
  return fp8 ? launch_typed<__nv_bfloat16, uint8_t, __nv_bfloat16>(a, S, o_part, lse_part, st, bal)
             : launch_typed<__nv_bfloat16, __nv_bfloat16, __nv_bfloat16>(a, S, o_part, lse_part, st,
                                                                         bal);
}

}  // namespace va
