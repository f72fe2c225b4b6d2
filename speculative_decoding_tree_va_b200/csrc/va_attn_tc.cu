// Tensor-core (tcgen05) bf16 tree-verify MLA-absorb attention for sm_100a.
//
// What it computes (page "The Milestone Commit...", section "The Context",
// item 2; MLA absorb from section "Input Knowledge Required"): for every
// tree-node query row, a masked softmax over the request's paged prefix and
// the row's ancestors in the tree tail, in the 512-d latent space plus the
// 64-d rope key, giving the normalised latent output and its log-sum-exp.
// The flash-decode split for long prefixes (section "How Decisions Were
// Made", production notes) is a grid dimension; va_merge combines splits.
//
// Design (B200-native; the pages' block-per-(batch, head, query) kernel for
// sm_120 is not used):
//  * All H*T query rows of a request share each key, so QK^T and PV are
//    dense bf16 contractions on the 5th-gen tensor cores.  A 64-row x 512
//    fp32 output accumulator is 128 KB, half of one SM's tensor memory, so
//    a CTA pair (cluster of 2) runs tcgen05.mma.cta_group::2 with M = 128:
//    each CTA holds 64 query rows, and the pair splits every B operand.
//  * Key tiles of 256 keys (4 pages).  QK: N = 256 keys, CTA r supplies keys
//    [128r, 128r+128).  PV: two MMAs of N = 256 latent columns; CTA r
//    supplies columns [256c + 128r, +128) of chunk c.  TMEM per CTA:
//    S0 | S1 (128 columns each, double-buffered scores) | O (256 columns).
//  * Data arrives by TMA (128-byte swizzle) into a ring of 16 KB slots,
//    page-table indexed, one 64-token page per box; pages past the request
//    are addressed out of bounds and read as zeros.
//  * Warp roles: warp 0 TMA producer, warp 1 MMA issuer (leader CTA only),
//    warps 2-9 softmax + epilogue.  The MMA order QK(i+1) before PV(i) lets
//    the softmax of tile i overlap the tensor core.  The producer and MMA
//    warps wait on barriers with all 32 lanes converged and issue from one
//    elected lane (a single lane polling in a diverged warp slowed MMA issue
//    about fourfold).
//  * Online softmax in the log2 domain.  The running max is only moved (and
//    O rescaled in TMEM) when a tile raises it by more than 2^8; otherwise
//    probabilities up to 2^8 go through bf16/fp32 unchanged (exact maths,
//    fewer TMEM round trips).  The tree mask is applied only on tiles that
//    reach the tree tail or the end of the key range.
//  * Every barrier wait is bounded (1 s): on expiry the CTA sets an abort
//    flag, every later wait returns at once, and the request is flagged.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "va_common.cuh"

namespace va {

__device__ unsigned int g_tc_timeouts = 0;  // count of barrier waits that expired

namespace {

constexpr int kThreads = 320;          // 10 warps: producer, MMA, 8 softmax
constexpr int kSoftThreads = 256;      // softmax + epilogue warps 2-9
constexpr int kRing = 7;               // KV ring slots
constexpr int kSlotBytes = 16384;      // one slot: two 8 KB TMA boxes
constexpr int kChunkBytes = 8192;      // [64 rows x 64 bf16] swizzled chunk
constexpr int kQBytes = 9 * kChunkBytes;   // 64 rows x 576
constexpr int kPBytes = 4 * kChunkBytes;   // 64 rows x 256 keys
constexpr int kTileKeys = 256;
constexpr int kTmemS1 = 128, kTmemO = 256;
constexpr float kRescaleLog2 = 8.0f;
constexpr unsigned long long kTimeoutNs = 1000000000ull;

struct TcParams {
  const void* c_kv;
  const void* k_pe;
  const int32_t* page_table;
  const int32_t* kv_len;
  const int32_t* order;  // grid row y -> request (longest first)
  const uint64_t* tree_mask;
  void* out;
  float* lse;
  float* o_part;
  float* lse_part;
  int32_t* req_status;
  int B, H, T, R, max_pages, num_pages;
  int S, split0;  // S-way key partition; grid z = splits split0, split0 + 1, ...
  int stall_mma;  // test hook: issue no tensor-core work (the waits expire)
  float scale_log2;
  float out_scale;  // multiplies the normalised output (an FP8 cache's scale; else 1)
};

struct __align__(16) Ctl {
  uint64_t full[kRing];   // leader: expect_tx arrival + both CTAs' TMA bytes
  uint64_t empty[kRing];
  uint64_t q_full;
  uint64_t s_full[2];
  uint64_t p_ready;
  uint64_t o_done;
  uint64_t mma_drain;
  uint32_t tmem_base;
  int abort;
  int bad_page;
  float xmax[2][4][64];  // [tile parity][key quarter][row]
  float xsum[4][64];
  float xsumr[4][64];
};

constexpr size_t kSmemBytes = 1024 + kQBytes + kPBytes + (size_t)kRing * kSlotBytes + sizeof(Ctl);

// ---------------------------------------------------------------- PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      "selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}
// Bounded wait on phase `parity` of a local barrier.  Returns false (and
// marks the CTA aborted) if it did not complete within kTimeoutNs.
__device__ __noinline__ bool mbar_wait(uint64_t* barp, uint32_t parity, volatile int* abort) {
  const uint32_t bar = smem_u32(barp);
  if (mbar_try(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (;;) {
#pragma unroll 1
    for (int k = 0; k < 32; ++k)
      if (mbar_try(bar, parity)) return true;
    if (*abort) return false;
    if (global_ns() - t0 > kTimeoutNs) {
      *abort = 1;
      atomicAdd(&g_tc_timeouts, 1u);
      return false;
    }
  }
}
// Warp-wide bounded wait: every lane of the warp calls it together and gets
// the same answer.  The producer and the MMA issuer wait like this, with the
// whole warp converged, and hand the issue to one elected lane: a lone lane
// that polls barriers in a diverged warp was measured to slow tcgen05.mma
// issue to ~270 clocks per instruction, against 64 with the warp converged.
__device__ __noinline__ bool warp_wait_slow(uint32_t bar, uint32_t parity, volatile int* abort) {
  const unsigned long long t0 = global_ns();
  for (;;) {
#pragma unroll 1
    for (int k = 0; k < 32; ++k)
      if (__all_sync(0xffffffffu, mbar_try(bar, parity))) return true;
    const bool give_up = __shfl_sync(
        0xffffffffu, (*abort != 0) || (global_ns() - t0 > kTimeoutNs) ? 1 : 0, 0) != 0;
    if (give_up) {
      if ((threadIdx.x & 31) == 0 && !*abort) {
        *abort = 1;
        atomicAdd(&g_tc_timeouts, 1u);
      }
      __syncwarp();
      return false;
    }
  }
}
__device__ __forceinline__ bool warp_wait(uint64_t* barp, uint32_t parity, volatile int* abort) {
  const uint32_t bar = smem_u32(barp);
  if (__all_sync(0xffffffffu, mbar_try(bar, parity))) return true;
  return warp_wait_slow(bar, parity, abort);
}
// One lane of a converged warp (elect.sync).
__device__ __forceinline__ bool elect_one() {
  uint32_t e;
  asm volatile("{\n.reg .pred p;\nelect.sync _|p, 0xffffffff;\nselp.u32 %0, 1, 0, p;\n}" : "=r"(e));
  return e != 0;
}
// Last-resort wait used only after an abort (bounded, never marks anything).
__device__ __noinline__ void mbar_wait_final(uint64_t* barp, uint32_t parity) {
  const uint32_t bar = smem_u32(barp);
  const unsigned long long t0 = global_ns();
  while (!mbar_try(bar, parity))
    if (global_ns() - t0 > kTimeoutNs) return;
}
// After an abort: give copies already in flight time to land (bounded).
__device__ __noinline__ void settle() {
  const unsigned long long t0 = global_ns();
  while (global_ns() - t0 < 200000ull) { }
}
// Barrier operations keep the default (CTA-scope) memory semantics.  The
// data they publish is either written by TMA (counted by the transaction
// bytes) or made visible to the tensor cores' async proxy by an explicit
// proxy fence before the arrival; cluster-scope release on every arrival
// was measured to cut the TMA stream to about a third.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar_local, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
               ::"r"(bar_local), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}
// 2-D TMA load into this CTA's shared memory, completion counted on the
// pair leader's barrier (cta_group::2 form).  No cluster multicast.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map,
                                            uint32_t bar_leader, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_leader), "r"(x), "r"(y)
      : "memory");
}
// 3-D TMA load: coordinates (x in chunk, pool row, 64-column chunk).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map,
                                            uint32_t bar_leader, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_leader), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem] * B[smem], issued once for the CTA pair.
__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}
// Arrive (once) on the same barrier offset in both CTAs of the pair when all
// previously issued MMAs of this thread have completed.
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)), "h"((uint16_t)0x3) : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  const uint32_t* r = reinterpret_cast<const uint32_t*>(v);
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
        "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
        "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]),
        "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
        "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void named_arrive(int id, int n) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// 2^x (hardware approximation, subnormal results flushed to zero; 2^-inf = 0).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2), sm_100
// version bits = 1.  lbo/sbo in bytes.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
// Instruction descriptor, kind::f16: bf16 A and B, fp32 D, M = 128, N = 256.
__host__ __device__ constexpr uint32_t idesc_bf16(bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(256 >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// -------------------------------------------------------------------- kernel

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_qn, const __grid_constant__ CUtensorMap tm_qp,
               const __grid_constant__ CUtensorMap tm_ckv,
               const __grid_constant__ CUtensorMap tm_kpe,
               const __grid_constant__ CUtensorMap tm_ckv3, const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = base;
  uint8_t* sP = sQ + kQBytes;
  uint8_t* sRing = sP + kPBytes;
  Ctl& c = *reinterpret_cast<Ctl*>(sRing + (size_t)kRing * kSlotBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  // Requests run longest first: grid row y takes the request of rank y in
  // descending kv_len (ties by index), so the ragged tail of the launch is
  // made of short row tiles.
  const int b = p.order[blockIdx.y];
  const int split = blockIdx.z;  // position in this launch; the key range is split0 + split
  const int tile_m = blockIdx.x >> 1;
  const int row0 = tile_m * 128 + (int)rank * 64;  // first query row of this CTA

  const int kv_len = p.kv_len[b];
  const bool req_ok = kv_len >= p.T && kv_len <= p.max_pages * kPage;
  int lo = 0, hi = 0;
  if (req_ok) split_range(kv_len, p.S, p.split0 + split, &lo, &hi);
  const int P = kv_len - p.T;
  const int ntiles = hi > lo ? (hi - lo + kTileKeys - 1) / kTileKeys : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRing; ++s) {
      mbar_init(&c.full[s], 1);
      mbar_init(&c.empty[s], 1);
    }
    mbar_init(&c.q_full, 1);
    mbar_init(&c.s_full[0], 1);
    mbar_init(&c.s_full[1], 1);
    mbar_init(&c.p_ready, 16);  // 8 softmax warps x 2 CTAs
    mbar_init(&c.o_done, 1);
    mbar_init(&c.mma_drain, 1);
    c.abort = 0;
    c.bad_page = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], 512;"
                 ::"r"(smem_u32(&c.tmem_base)));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = c.tmem_base;
  volatile int* abort = &c.abort;

  // Ring protocol.  Every 16 KB slot is two 8 KB TMA boxes (K: one per page;
  // V: one 3-D box).  The producer and the MMA issuer walk the same slot
  // sequence -- for tile t: K chunks kc = 0..8 of tile t, then the V slots of
  // tile t-1 -- so every ring position is taken by both in order and a
  // barrier phase can never be waited on twice ahead.  A slot is full when
  // the leader's expect_tx arrival and both CTAs' TMA bytes are in.

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // The warp walks the slot sequence converged; one elected lane issues.
    if (ntiles > 0) {
      if (elect_one()) {
        const uint32_t q_bar = map_to_rank(smem_u32(&c.q_full), 0);
        if (rank == 0) mbar_arrive_expect_tx(smem_u32(&c.q_full), 2 * kQBytes);
        const int qrow = b * p.R + row0;
        for (int ch = 0; ch < 8; ++ch)
          tma_load_2d(smem_u32(sQ + ch * kChunkBytes), &tm_qn, q_bar, ch * 64, qrow);
        tma_load_2d(smem_u32(sQ + 8 * kChunkBytes), &tm_qp, q_bar, 0, qrow);
      }
      __syncwarp();

      const int npages_valid = (kv_len + kPage - 1) / kPage;
      const int oob_row = p.num_pages * kPage;  // first row past the pool: zero fill
      auto page_row = [&](int pg) -> int {  // logical page -> first pool row
        if (pg >= npages_valid) return oob_row;
        const int ph = p.page_table[(size_t)b * p.max_pages + pg];
        if (ph < 0 || ph >= p.num_pages) return oob_row;  // flagged by the page scan
        return ph * kPage;
      };
      int slot = 0;
      uint32_t phase = 0;
      auto advance = [&]() { if (++slot == kRing) { slot = 0; phase ^= 1; } };
      bool go = true;
      for (int t = 0; t <= ntiles && go; ++t) {
        if (t < ntiles) {  // K chunks: this CTA's two pages of the tile
          const int kb = lo + t * kTileKeys;
          const int r0 = page_row(kb / kPage + 2 * (int)rank);
          const int r1 = page_row(kb / kPage + 2 * (int)rank + 1);
          for (int kc = 0; kc < 9 && go; ++kc) {
            go = warp_wait(&c.empty[slot], phase ^ 1, abort);
            if (!go) break;
            if (elect_one()) {
              const uint32_t bar = map_to_rank(smem_u32(&c.full[slot]), 0);
              if (rank == 0) mbar_arrive_expect_tx(smem_u32(&c.full[slot]), 2 * kSlotBytes);
              const uint32_t dst = smem_u32(sRing + (size_t)slot * kSlotBytes);
              const CUtensorMap* map = kc < 8 ? &tm_ckv : &tm_kpe;
              const int x0 = kc < 8 ? kc * 64 : 0;
              tma_load_2d(dst, map, bar, x0, r0);
              tma_load_2d(dst + kChunkBytes, map, bar, x0, r1);
            }
            __syncwarp();
            advance();
          }
        }
        if (t > 0 && go) {  // V slots of tile t-1: [64 keys x 2 chunks x 64 latent columns]
          const int kb = lo + (t - 1) * kTileKeys;
          for (int pg = 0; pg < 4 && go; ++pg) {
            const int k0 = kb + pg * kPage;
            if (k0 >= hi) break;
            const int r = page_row(k0 / kPage);
            for (int nc = 0; nc < 2 && go; ++nc) {
              go = warp_wait(&c.empty[slot], phase ^ 1, abort);
              if (!go) break;
              if (elect_one()) {
                const uint32_t bar = map_to_rank(smem_u32(&c.full[slot]), 0);
                if (rank == 0) mbar_arrive_expect_tx(smem_u32(&c.full[slot]), 2 * kSlotBytes);
                tma_load_3d(smem_u32(sRing + (size_t)slot * kSlotBytes), &tm_ckv3, bar, 0, r,
                            nc * 4 + (int)rank * 2);
              }
              __syncwarp();
              advance();
            }
          }
        }
      }
      // every page index this split reads is checked while the last loads
      // are consumed (out-of-range pages were read as zeros)
      int bad = 0;
      for (int pg = lo / kPage + lane; pg < (hi + kPage - 1) / kPage; pg += 32) {
        const int ph = p.page_table[(size_t)b * p.max_pages + pg];
        bad |= (ph < 0 || ph >= p.num_pages);
      }
      if (__any_sync(0xffffffffu, bad) && lane == 0) c.bad_page = 1;
      // drain: every slot's last load must be consumed before the CTA may exit
      for (int s2 = 0; s2 < kRing && go; ++s2) {
        go = warp_wait(&c.empty[slot], phase ^ 1, abort);
        advance();
      }
      if (*abort) settle();  // loads already issued land before teardown
    }
    __syncwarp();
    named_arrive(2, 32 + kSoftThreads);  // publishes bad_page to the epilogue
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The warp walks the slot sequence converged; one elected lane issues
    // each slot's MMAs and its commit.
    if (rank == 0 && ntiles > 0 && !p.stall_mma) {
      constexpr uint32_t kIdQK = idesc_bf16(false), kIdPV = idesc_bf16(true);
      const uint32_t sq = smem_u32(sQ), sp = smem_u32(sP), sr = smem_u32(sRing);
      int slot = 0;
      uint32_t phase = 0;
      auto advance = [&]() { if (++slot == kRing) { slot = 0; phase ^= 1; } };
      // Descriptors are built once; a K step only adds its byte offset / 16
      // to the start-address field (no carry: every operand lies inside the
      // 256 KB shared window, whose addresses fit the 14-bit field).
      const uint64_t dq0 = sw128_desc(sq, 16, 1024);           // Q, K-major
      const uint64_t dp0 = sw128_desc(sp, 16, 1024);           // P, K-major
      const uint64_t dk0 = sw128_desc(sr, 16, 1024);           // K slot, K-major
      const uint64_t dv0 = sw128_desc(sr, kChunkBytes, 1024);  // V slot, MN-major
      bool ok = warp_wait(&c.q_full, 0, abort);
      auto qk = [&](int t) {
        const uint32_t d = tmem + ((t & 1) ? kTmemS1 : 0);
        for (int kc = 0; kc < 9 && ok; ++kc) {
          ok = warp_wait(&c.full[slot], phase, abort);
          if (!ok) break;
          if (elect_one()) {
            tc_fence_after();
            const uint64_t da = dq0 + (uint64_t)((kc * kChunkBytes) >> 4);
            const uint64_t db = dk0 + (uint64_t)((slot * kSlotBytes) >> 4);
            mma_bf16_pair(d, da, db, kIdQK, kc != 0);
            mma_bf16_pair(d, da + 2, db + 2, kIdQK, 1u);
            mma_bf16_pair(d, da + 4, db + 4, kIdQK, 1u);
            mma_bf16_pair(d, da + 6, db + 6, kIdQK, 1u);
            mma_commit_pair(&c.empty[slot]);
          }
          __syncwarp();
          advance();
        }
        if (elect_one()) mma_commit_pair(&c.s_full[t & 1]);
        __syncwarp();
      };
      auto pv = [&](int t) {
        const int kb = lo + t * kTileKeys;
        if (ok) ok = warp_wait(&c.p_ready, t & 1, abort);
        if (!ok) return;
        for (int pg = 0; pg < 4 && ok; ++pg) {
          if (kb + pg * kPage >= hi) break;
          const int nk = min(4, (hi - (kb + pg * kPage) + 15) >> 4);  // 16-key steps in range
          const uint64_t da = dp0 + (uint64_t)((pg * kChunkBytes) >> 4);
          for (int nc = 0; nc < 2 && ok; ++nc) {
            ok = warp_wait(&c.full[slot], phase, abort);
            if (!ok) break;
            if (elect_one()) {
              tc_fence_after();
              const uint32_t d = tmem + kTmemO + nc * 128;
              const uint64_t db = dv0 + (uint64_t)((slot * kSlotBytes) >> 4);
              const uint32_t acc0 = (t == 0 && pg == 0) ? 0u : 1u;
              mma_bf16_pair(d, da, db, kIdPV, acc0);
              if (nk > 1) mma_bf16_pair(d, da + 2, db + 128, kIdPV, 1u);
              if (nk > 2) mma_bf16_pair(d, da + 4, db + 256, kIdPV, 1u);
              if (nk > 3) mma_bf16_pair(d, da + 6, db + 384, kIdPV, 1u);
              mma_commit_pair(&c.empty[slot]);
            }
            __syncwarp();
            advance();
          }
        }
        if (elect_one()) mma_commit_pair(&c.o_done);
        __syncwarp();
      };
      for (int t = 0; t < ntiles && ok; ++t) {
        qk(t);
        if (t > 0) pv(t - 1);
      }
      if (ok) pv(ntiles - 1);
      if (!ok) {
        // aborted: issue nothing more, and let every MMA already issued
        // finish before the pair tears down and frees tensor memory
        if (elect_one()) mma_commit_pair(&c.mma_drain);
        __syncwarp();
        mbar_wait_final(&c.mma_drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    // Eight warps.  Warp w reads TMEM lane quadrant q = w & 3 (rows
    // 32 (q & 1) .. +31 of this CTA; key half h = q >> 1 of each tile) and
    // takes the sub-half sh = (w - 2) >> 2 of it: keys [64 part, +64) of the
    // tile with part = 2 h + sh.  The four parts of a row combine their maxima
    // and sums through shared memory.
    const int q = warp & 3;             // TMEM lane quadrant of this warp
    const int m = 32 * (q & 1) + lane;  // row within the CTA
    const int h = q >> 1;               // key half of each tile
    const int sh = (warp - 2) >> 2;     // sub-half
    const int part = 2 * h + sh;        // key quarter: also the P chunk and the O columns' half
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    const int row = row0 + m;
    const bool row_in = row < p.R;
    const int W = (p.T + 63) >> 6;
    uint64_t mw0 = 0, mw1 = 0;
    bool live = false;
    if (row_in && req_ok) {
      const int t = row / p.H;
      const uint64_t* mrow = p.tree_mask + ((size_t)b * p.T + t) * W;
      mw0 = mrow[0];
      mw1 = W > 1 ? mrow[1] : 0ull;
      live = mask_bit(mrow, t);
    }
    const uint32_t p_ready_leader = map_to_rank(smem_u32(&c.p_ready), 0);
    float m_used = -INFINITY, l = 0.f, lr = 0.f;  // lr: sum of the bf16-rounded probabilities

    for (int t = 0; t < ntiles; ++t) {
      const int kb = lo + t * kTileKeys;
      const int j0 = kb + 64 * part;  // key of this thread's first column
      mbar_wait(&c.s_full[t & 1], (t >> 1) & 1, abort);
      tc_fence_after();
      __syncwarp();  // tcgen05.ld is warp-collective
      float x[64];
      const uint32_t s_addr = tmem + lane_base + ((t & 1) ? kTmemS1 : 0) + 64 * sh;
      tmem_ld32(s_addr, *reinterpret_cast<float(*)[32]>(&x[0]));
      tmem_ld32(s_addr + 32, *reinterpret_cast<float(*)[32]>(&x[32]));
      tmem_wait_ld();
      const bool need_mask = !live || (kb + kTileKeys > P) || (kb + kTileKeys > hi);
      float tmax = -INFINITY;
      if (!need_mask) {
#pragma unroll
        for (int i = 0; i < 64; ++i) { x[i] *= p.scale_log2; tmax = fmaxf(tmax, x[i]); }
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const int j = j0 + i;
          bool vis = live && j < hi;
          if (vis && j >= P) {
            const int nd = j - P;
            vis = ((nd < 64 ? (mw0 >> nd) : (mw1 >> (nd - 64))) & 1ull) != 0;
          }
          x[i] = vis ? x[i] * p.scale_log2 : -INFINITY;
          tmax = fmaxf(tmax, x[i]);
        }
      }
      // combine the four key quarters of the row
      c.xmax[t & 1][part][m] = tmax;
      named_sync(1, kSoftThreads);
      tmax = fmaxf(fmaxf(c.xmax[t & 1][0][m], c.xmax[t & 1][1][m]),
                   fmaxf(c.xmax[t & 1][2][m], c.xmax[t & 1][3][m]));

      bool rescale = false;
      float alpha = 1.f;
      if (tmax > m_used + kRescaleLog2 || (m_used == -INFINITY && tmax != -INFINITY)) {
        if (m_used != -INFINITY) {
          alpha = ex2(m_used - tmax);
          rescale = true;
        }
        m_used = tmax;
      }
      uint32_t pk[32];
      float sum = 0.f;
      if (m_used == -INFINITY) {
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = 0u;
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p0 = ex2(x[2 * i] - m_used);
          const float p1 = ex2(x[2 * i + 1] - m_used);
          sum += p0 + p1;
          pk[i] = pack_bf16(p0, p1);
        }
      }

      // PV(t-1) must be done before P is overwritten or O rescaled
      if (t > 0) {
        mbar_wait(&c.o_done, (t - 1) & 1, abort);
        tc_fence_after();
      }
      // tcgen05.ld/st are warp-collective: the whole warp takes this branch
      // if any of its rows needs it (factor 1 for the others).  This warp
      // rescales the O columns of its sub-half (TMEM chunks 4 sh .. 4 sh + 3).
      __syncwarp();
      if (t > 0 && __any_sync(0xffffffffu, rescale)) {
        const float f = rescale ? alpha : 1.f;
#pragma unroll 1
        for (int cc = 4 * sh; cc < 4 * sh + 4; ++cc) {
          float o[32];
          const uint32_t oa = tmem + lane_base + kTmemO + cc * 32;
          tmem_ld32(oa, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= f;
          tmem_st32(oa, o);
        }
        tmem_wait_st();
      }
      // P -> shared, K-major 128B-swizzled [64 rows x 64 keys] chunk `part`
#pragma unroll
      for (int k16 = 0; k16 < 8; ++k16) {  // 16-byte units of the 128-byte row
        uint8_t* dst = sP + part * kChunkBytes + (m >> 3) * 1024 + (m & 7) * 128 +
                       ((k16 ^ (m & 7)) << 4);
        *reinterpret_cast<uint4*>(dst) =
            make_uint4(pk[4 * k16], pk[4 * k16 + 1], pk[4 * k16 + 2], pk[4 * k16 + 3]);
      }
      fence_proxy_async();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(p_ready_leader);
      // the sum of the rounded probabilities (the normaliser of the output)
      // is taken after P is handed to the tensor cores, off their path
      float sumr = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i)
        sumr += __uint_as_float(pk[i] << 16) + __uint_as_float(pk[i] & 0xffff0000u);
      l = l * alpha + sum;
      lr = lr * alpha + sumr;
    }

    // ---------------------------------------------------------------- epilogue
    if (ntiles > 0) {
      mbar_wait(&c.o_done, (ntiles - 1) & 1, abort);
      tc_fence_after();
    }
    c.xsum[part][m] = l;
    c.xsumr[part][m] = lr;
    named_sync(1, kSoftThreads);
    named_sync(2, 32 + kSoftThreads);
    const float lsum = (c.xsum[0][m] + c.xsum[1][m]) + (c.xsum[2][m] + c.xsum[3][m]);
    const float lsumr = (c.xsumr[0][m] + c.xsumr[1][m]) + (c.xsumr[2][m] + c.xsumr[3][m]);
    const bool bad = !req_ok || c.bad_page || *abort;
    const bool empty = bad || !(lsum > 0.f) || !(lsumr > 0.f) || ntiles == 0;
    const float inv = empty ? 0.f : p.out_scale / lsumr;
    const float lse = empty ? -INFINITY : (m_used + log2f(lsum)) * kLn2;
    __syncwarp();
    {
      // every lane runs the (warp-collective) TMEM loads; only rows inside
      // the request store.  This warp writes the latent columns of the O
      // accumulator sh (nc = sh): [256 sh + 128 h, +128).
      const size_t g = (size_t)b * p.R + (row_in ? row : 0);
      const size_t rows_total = (size_t)p.B * p.R;
      const int nc = sh;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        float o[32];
        if (ntiles > 0) {
          tmem_ld32(tmem + lane_base + kTmemO + nc * 128 + cc * 32, o);
          tmem_wait_ld();
        }
        const int col = nc * 256 + h * 128 + cc * 32;
        if (!row_in) {
          // nothing to store for rows past the request
        } else if (!p.o_part) {
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + g * kDc + col;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 u;
            u.x = pack_bf16(empty ? 0.f : o[8 * v + 0] * inv, empty ? 0.f : o[8 * v + 1] * inv);
            u.y = pack_bf16(empty ? 0.f : o[8 * v + 2] * inv, empty ? 0.f : o[8 * v + 3] * inv);
            u.z = pack_bf16(empty ? 0.f : o[8 * v + 4] * inv, empty ? 0.f : o[8 * v + 5] * inv);
            u.w = pack_bf16(empty ? 0.f : o[8 * v + 6] * inv, empty ? 0.f : o[8 * v + 7] * inv);
            reinterpret_cast<uint4*>(dst)[v] = u;
          }
        } else {
          float* dst = p.o_part + ((size_t)split * rows_total + g) * kDc + col;
#pragma unroll
          for (int v = 0; v < 8; ++v)
            reinterpret_cast<float4*>(dst)[v] =
                empty ? make_float4(0.f, 0.f, 0.f, 0.f)
                      : make_float4(o[4 * v] * inv, o[4 * v + 1] * inv, o[4 * v + 2] * inv,
                                    o[4 * v + 3] * inv);
        }
        __syncwarp();  // reconverge before the next warp-collective load
      }
      if (part == 0 && row_in) {
        if (!p.o_part) p.lse[g] = lse;
        else p.lse_part[(size_t)split * rows_total + g] = lse;
      }
    }
    if (threadIdx.x == 64 && p.req_status && (!req_ok || c.bad_page))
      p.req_status[b] = VA_ERR_INVALID_ARG;
    if (threadIdx.x == 64 && p.req_status && *abort) p.req_status[b] = VA_ERR_CUDA;
  }

  // ------------------------------------------------------------------ teardown
  __syncwarp();  // role branches diverge inside warps 0 and 1; reconverge first
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, 512;" ::"r"(tmem));
  }
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// c_kv as 3-D (64 columns of a chunk, pool row, chunk): a [64 x 64 x 2] box
// lands as two consecutive swizzled [64 rows x 64 columns] chunks.
bool encode_ckv3(CUtensorMap* map, const void* ptr, uint64_t rows) {
  auto fn = get_encoder();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, rows, kDc / 64};
  cuuint64_t strides[2] = {(cuuint64_t)kDc * 2, 128};
  cuuint32_t box[3] = {64, 64, 2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D bf16 map over a row-major [rows, cols] tensor with [64 x 64] boxes and
// 128-byte swizzle (the layout the UMMA descriptors above expect).
bool encode_2d(CUtensorMap* map, const void* ptr, uint64_t rows, uint64_t cols) {
  auto fn = get_encoder();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_attn_tc(const va_attn_args& a, SplitRange sp, const int32_t* order,
                           float* o_part, float* lse_part, cudaStream_t st, float out_scale) {
  if (a.B == 0) return cudaSuccess;
  const long long R = (long long)a.T * a.H;
  const long long rows_total = (long long)a.B * R;
  if (rows_total > 0x7fffffffLL) return cudaErrorNotSupported;
  CUtensorMap tqn, tqp, tckv, tkpe, tckv3;
  if (!encode_2d(&tqn, a.q_nope, rows_total, kDc) || !encode_2d(&tqp, a.q_pe, rows_total, kDr) ||
      !encode_2d(&tckv, a.c_kv, (uint64_t)a.num_pages * kPage, kDc) ||
      !encode_2d(&tkpe, a.k_pe, (uint64_t)a.num_pages * kPage, kDr) ||
      !encode_ckv3(&tckv3, a.c_kv, (uint64_t)a.num_pages * kPage))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  TcParams p;
  p.c_kv = a.c_kv;
  p.k_pe = a.k_pe;
  p.page_table = a.page_table;
  p.kv_len = a.kv_len;
  p.order = order;
  p.tree_mask = a.tree_mask;
  p.out = a.out;
  p.lse = a.lse;
  p.o_part = o_part;
  p.lse_part = lse_part;
  p.req_status = a.req_status;
  p.B = a.B;
  p.H = a.H;
  p.T = a.T;
  p.R = (int)R;
  p.max_pages = a.max_pages;
  p.num_pages = a.num_pages;
  p.S = sp.S;
  p.split0 = sp.first;
  p.stall_mma = (a.flags & VA_FLAG_TEST_STALL_MMA) ? 1 : 0;
  p.scale_log2 = a.scale * kLog2e;
  p.out_scale = out_scale;
  dim3 grid((unsigned)(2 * ((R + 127) / 128)), (unsigned)a.B, (unsigned)sp.count);
  attn_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(tqn, tqp, tckv, tkpe, tckv3, p);
  return cudaGetLastError();
}

unsigned int tc_timeouts() {
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_tc_timeouts, sizeof(v)) != cudaSuccess) return 0xFFFFFFFFu;
  return v;
}

}  // namespace va
