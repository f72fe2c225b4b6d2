/*
 * libverifyattn -- tree-verify MLA-absorb attention for DDTree speculative
 * decoding, for NVIDIA B200 (sm_100a).
 *
 * The verify step of a greedy DDTree decode step (page "The Milestone
 * Commit: Cementing Phase 1 of a Custom CUDA Speculative Decoding Engine",
 * section "The Context", items 1-3): a best-first draft tree is built from
 * the drafter's per-depth top-k, every tree node becomes a query, and each
 * node attends -- per head, in the absorbed MLA latent space (512-d c_kv plus
 * a 64-d rope key) -- to its request's cached prefix and to its own
 * ancestors in the tree tail, through a masked softmax that yields a latent
 * output and its log-sum-exp.  The pages' C ABI hands raw device pointers
 * and the caller's CUDA stream across the boundary (page "The Capstone
 * Commit: Validating a Native CUDA DDTree Inference Engine", section "The
 * Message Itself"); this header keeps that shape.
 *
 * Conventions for every call:
 *   - Pointers marked [device] are CUDA device pointers owned by the caller;
 *     the library never allocates, frees or keeps them.  [host] pointers are
 *     read during the call only.
 *   - Work is enqueued on `stream` (NULL = legacy default stream) and runs
 *     asynchronously; nothing synchronises the host.
 *   - A call returns VA_OK once its kernels are enqueued.  Argument errors
 *     are reported before anything is launched (VA_ERR_INVALID_ARG,
 *     VA_ERR_UNSUPPORTED); a failed launch returns VA_ERR_CUDA.  Errors found
 *     on the device (a malformed tree, a bad kv_len or page index) are
 *     written to the optional per-request status arrays.
 *   - Device pointers must be 16-byte aligned; all tensors are dense,
 *     row-major, innermost dimension last.
 *   - Thread safety: calls may be issued from several host threads on
 *     different streams; calls that share output buffers race on the GPU.
 */
#ifndef VERIFYATTN_H_
#define VERIFYATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; declared here so the header needs no CUDA. */
typedef struct CUstream_st* va_stream_t;

enum va_status {
  VA_OK = 0,
  VA_ERR_INVALID_ARG = 1,  /* bad size, NULL or misaligned pointer      */
  VA_ERR_UNSUPPORTED = 2,  /* valid request this build does not handle  */
  VA_ERR_CUDA = 3,         /* a CUDA launch or driver call failed       */
  VA_ERR_INVALID_TREE = 4  /* (device status) malformed parent array    */
};

enum va_dtype { VA_F32 = 0, VA_BF16 = 1 };

#define VA_D_LATENT 512   /* c_kv / q_nope / output width                 */
#define VA_D_ROPE 64      /* k_pe / q_pe width                            */
#define VA_PAGE_SIZE 64   /* tokens per KV page                           */
#define VA_MAX_QLEN 65    /* T = tree budget 64 + root (pages: MAX_QLEN)  */
#define VA_MAX_DEPTH 15   /* deepest tree the builder produces            */
#define VA_MAX_TOPK 16    /* widest drafter top-k the builder accepts     */
#define VA_SPLIT_ALIGN 256/* split-KV chunk granularity, in keys          */
#define VA_MAX_SPLITS 64
#define VA_MAX_BATCH 65535 /* requests per va_verify_attn call              */

/* Largest tree-verify query length T (root included): 65.  The pages'
 * library reports the same limit when it loads ("Verified lib loads
 * (MAX_QLEN=65)", page "The Capstone Commit...", section "The Message
 * Itself"). */
int va_max_qlen(void);

/* Static, human-readable name of a va_status value. */
const char* va_status_string(int status);

/*
 * Best-first draft-tree builder (page "The Milestone Commit...", section
 * "The Context", item 1: a GPU best-first builder replacing the per-request
 * CPU heap; page "Strategic Pivots in CUDA Kernel Engineering...", section
 * "Why This Message Was Written": ties resolved as in tuple comparison).
 *
 *   lp      [device] double [B, L, K]  per-depth top-K drafter log-probs,
 *                                      row d = depth d+1, descending in K
 *   tok     [device] int32  [B, L, K]  matching token ids
 *   parents [device] int32  [B, T]     out: parent node, -1 for the root and
 *                                      for absent nodes of underfull trees
 *   tokens  [device] int32  [B, T]     out: token id (-1 root / absent)
 *   depth   [device] int32  [B, T]     out: depth (0 root, -1 absent)
 *   n_nodes [device] int32  [B]        out: node count incl. the root
 *   T = budget + 1, 1 <= T <= VA_MAX_QLEN, 1 <= L <= VA_MAX_DEPTH,
 *   1 <= K <= VA_MAX_TOPK.
 * A node's score is its parent's score plus its own log-prob, in fp64.  The
 * frontier pops the highest score; equal scores go to the lower parent node
 * index, then the lower rank.  Node indices are pop order, so parent < child.
 * lp and tok are read only; the builder does not check lp is sorted.
 */
int va_build_tree(const double* lp, const int32_t* tok, int B, int L, int K, int budget,
                  int32_t* parents, int32_t* tokens, int32_t* depth, int32_t* n_nodes,
                  va_stream_t stream);

/*
 * Tree visibility (ancestor) mask (page "Strategic Pivots in CUDA Kernel
 * Engineering...", section "The Message": a tree visibility mask from the
 * builder).
 *
 *   parents     [device] int32  [B, T]     parent[0] = -1; for i >= 1 either
 *                                          -1 (absent node) or 0 <= p < i with
 *                                          node p present
 *   mask        [device] uint64 [B, T, W]  out, W = ceil(T / 64): bit i of
 *                                          row t (word i / 64) is set iff node
 *                                          i is t or an ancestor of t
 *   tree_status [device] int32  [B]        out (nullable): VA_OK or
 *                                          VA_ERR_INVALID_TREE
 * Absent nodes get an all-zero row (their own bit clear).  A malformed
 * request gets all-zero rows and VA_ERR_INVALID_TREE.  1 <= T <= 65, B >= 0.
 */
int va_build_tree_mask(const int32_t* parents, int B, int T, uint64_t* mask,
                       int32_t* tree_status, va_stream_t stream);

/*
 * Greedy tree accept (page "The Milestone Commit...", section "The Context",
 * item 3: the verified tree is walked with next-token / next-sibling pointers
 * to find the accepted tokens).
 *
 *   parents, tokens [device] int32 [B, T]   the draft tree (va_build_tree)
 *   target_next     [device] int32 [B, T]   the target model's greedy token
 *                                           after the path to each node
 *   path            [device] int32 [B, T]   out: accepted nodes, root first,
 *                                           then -1
 *   accept_len      [device] int32 [B]      out: tokens committed this step
 *                                           = accepted draft tokens + 1
 *   next_token      [device] int32 [B]      out: target_next of the last
 *                                           accepted node
 * From the root, move to the child whose token equals target_next of the
 * current node (lowest index among equal tokens) until none does.  Only
 * links with 0 <= parent < index count; absent nodes are never accepted.
 */
int va_tree_accept(const int32_t* parents, const int32_t* tokens, const int32_t* target_next,
                   int B, int T, int32_t* path, int32_t* accept_len, int32_t* next_token,
                   va_stream_t stream);

/* Arguments of va_verify_attn.  Zero-initialise, then fill. */
typedef struct va_attn_args {
  int dtype;          /* VA_F32 (CUDA-core FFMA path) or VA_BF16 (tcgen05 path) */
  int B, H, T;        /* requests, heads, query length (1 <= T <= 65)           */
  float scale;        /* softmax scale on q.k (e.g. 1/sqrt(192))                */
  const void* q_nope; /* [device] [B, T, H, 512] dtype, latent (absorbed) query */
  const void* q_pe;   /* [device] [B, T, H, 64]  dtype, rope query              */
  const void* c_kv;   /* [device] [num_pages, 64, 512] dtype, latent KV pool    */
  const void* k_pe;   /* [device] [num_pages, 64, 64]  dtype, rope key pool     */
  int num_pages;      /* pages in the pool                                      */
  int page_size;      /* must be VA_PAGE_SIZE                                   */
  const int32_t* page_table; /* [device] [B, max_pages] logical -> physical   */
  int max_pages;      /* row stride of page_table                               */
  const int32_t* kv_len;     /* [device] [B] keys of request b = P_b + T; the
                                tree tail is the last T keys (node i at P_b+i) */
  const uint64_t* tree_mask; /* [device] [B, T, ceil(T/64)] from
                                va_build_tree_mask                             */
  void* out;          /* [device] [B, T, H, 512] dtype, normalised latent out   */
  float* lse;         /* [device] [B, T, H] float, natural-log sum-exp          */
  int32_t* req_status;/* [device] [B] nullable: VA_ERR_INVALID_ARG when kv_len
                         or a page index is out of range (all the request's
                         rows written as 0 / -inf, with or without splits);
                         entries of requests without a problem are not
                         written                                               */
  int num_splits;     /* 0 = auto, 1 = single pass, 2..64 = split-KV + merge    */
  void* workspace;    /* [device] >= va_workspace_bytes(), 256-byte aligned     */
  size_t workspace_bytes;
  int flags;          /* VA_FLAG_* below                                        */
  float kv_scale;     /* with VA_FLAG_KV_FP8_E4M3: the value of one cache unit
                         (finite, > 0); ignored otherwise                      */
} va_attn_args;

/* Run bf16 inputs on the CUDA-core FFMA kernel instead of the tensor-core
 * kernel (a second, independent GPU path for cross-checks). */
#define VA_FLAG_BF16_CUDA_CORES 1

/* Test hook for the bounded waits (bf16 tensor-core path only; rejected with
 * VA_ERR_INVALID_ARG elsewhere): the kernel issues no tensor-core work, so
 * every wait on tensor-core completion runs into its 1 s bound.  Each
 * request then comes back with req_status VA_ERR_CUDA, zero output and lse
 * -inf, va_device_timeouts() grows, and the context stays usable.  No copy
 * is in flight when the CTAs give up, so nothing lands after they exit. */
#define VA_FLAG_TEST_STALL_MMA 2

/* Test hook for the CUDA-core kernel's bounded staging wait (fp32 queries on
 * an fp32 cache only; rejected with VA_ERR_INVALID_ARG elsewhere): the kernel
 * arms each tile's staging barrier but issues no bulk copy, so the wait runs
 * into its 1 s bound.  Each request then comes back with req_status
 * VA_ERR_CUDA, zero output and lse -inf, va_device_timeouts() grows, and the
 * context stays usable.  No copy is in flight when the CTAs give up. */
#define VA_FLAG_TEST_STALL_COPIES 8

/* Latent cache kept as FP8 E4M3 codes, one byte per element, with one scale
 * for the whole cache: c_kv is uint8 [num_pages, 64, 512], k_pe uint8
 * [num_pages, 64, 64], and code x stands for kv_scale * value(x) in every
 * formula of va_verify_attn.  E4M3 is the OCP 8-bit floating point format
 * (sign, 4-bit exponent with bias 7, 3-bit mantissa; exponent field 0 is
 * subnormal; S.1111.111 is NaN; no infinities; largest magnitude 448).  The
 * cache takes half the bytes of a bf16 one; queries and outputs keep `dtype`
 * (fp32 or bf16).  The pages keep the cache in the model's dtype: this is an
 * addition.  bf16 queries run on the tensor-core kernel: a first kernel
 * widens the pages the batch reads into bf16 scratch pages in the workspace
 * (every E4M3 value is exactly a bf16 value; slots past kv_len become zeros),
 * and kv_scale is folded into the score scale and the output normalisation.
 * fp32 queries (or VA_FLAG_BF16_CUDA_CORES) run on the CUDA-core kernel,
 * which widens codes to fp32 as it stages them.  kv_scale must be finite and
 * > 0, else VA_ERR_INVALID_ARG; VA_FLAG_TEST_STALL_MMA is rejected with this
 * flag. */
#define VA_FLAG_KV_FP8_E4M3 4

/*
 * Workspace needed by va_verify_attn for these arguments (0 when none is
 * needed).  With S = the split count the call will use, the workspace holds,
 * each part starting on a 256-byte boundary:
 *   - for bf16 queries on the tensor cores: the requests' longest-first
 *     order, int32 [B] (written by the call itself; the longest requests are
 *     scheduled first so the launch does not end on one long request);
 *   - for S > 1: o_part float [S, B, T, H, 512], then lse_part float
 *     [S, B, T, H] (the layout va_merge reads), then int32 [B]: the splits'
 *     per-request status, zeroed and filled by the call itself;
 *   - for bf16 queries on the tensor cores with an FP8 cache: the widened
 *     cache, bf16 [B * max_pages, 64, 512] and [B * max_pages, 64, 64], and
 *     its page table int32 [B, max_pages].
 * Returns 0 on bad args.
 */
size_t va_workspace_bytes(const va_attn_args* args);

/* The split count va_verify_attn will use for these arguments (>= 1; for
 * the balanced CUDA-core plan below, the number of partials per row), or a
 * negative va_status on bad arguments. */
int va_num_splits(const va_attn_args* args);

/*
 * Tree-verify MLA-absorb attention (page "The Milestone Commit...", section
 * "The Context", item 2: masked softmax over the concatenated prefix and
 * tree tail, latent output, no host round-trips; section "How Decisions Were
 * Made", production notes: flash+merge for long prefixes).
 *
 * For row (b, t, h), with P = kv_len[b] - T, key j in [0, kv_len[b]) lives at
 * c_kv[page_table[b][j / 64]][j % 64] (and k_pe likewise); it is visible iff
 * j < P, or bit (j - P) of tree_mask[b][t] is set.
 *   s_j = scale * (q_nope . c_kv_j + q_pe . k_pe_j)
 *   out = sum_j softmax(s)_j c_kv_j      lse = ln sum_j exp(s_j)
 * A row whose own tree bit is clear (absent node) gets out = 0, lse = -inf.
 * With S > 1 splits, split s covers keys [e(s), e(s+1)): e(0) = 0,
 * e(S) = kv_len, and for 0 < s < S, e(s) = min(kv_len, 256 * floor((2 s kv_len
 * + 256 S) / (512 S))), i.e. s * kv_len / S rounded to the nearest multiple
 * of 256, ties up (splits may be empty when kv_len < 128 S); the partials go
 * to the workspace and va_merge combines them on the same stream.
 * Balanced plan: a call on the CUDA-core kernel with num_splits = 0 whose
 * (request, 32-row tile) segments are fewer than the device's SMs instead
 * cuts each segment's key range into 2 * max_pages 32-key tiles and divides
 * the tiles of all segments, in order, into equal contiguous ranges, one CTA
 * each (at least 4 tiles per CTA; none of this when that leaves no more CTAs
 * than segments).  Every CTA writes one partial per segment it touches, a
 * segment's unused slots are marked empty, and va_merge combines S = the
 * largest number of CTAs sharing a segment (<= VA_MAX_SPLITS) partials.  The
 * result is the same function of the inputs; only the fp32 rounding order
 * differs.  va_verify_attn_partials never uses this plan.
 * bf16 runs on tensor cores with fp32 accumulation; fp32, and any call with
 * an FP8 cache (VA_FLAG_KV_FP8_E4M3), on CUDA cores.
 * Requirements: page_size == 64, H >= 1, 1 <= T <= 65, 0 <= B <= VA_MAX_BATCH
 * (larger batches: VA_ERR_UNSUPPORTED; split them across calls).  Slots past
 * kv_len in a request's last page may hold any finite values (they are
 * multiplied by exact zeros; NaN or Inf there would propagate); with an FP8
 * cache they may hold any codes, NaN included (both FP8 routes replace them
 * by zeros before any product).
 */
int va_verify_attn(const va_attn_args* args, va_stream_t stream);

/*
 * Split-KV partials of some of the splits, without the merge: the per-GPU
 * step of sharding one long prefix across GPUs (the flash+merge production
 * note, page "The Milestone Commit...", section "How Decisions Were Made":
 * each GPU computes some of the flash-decode chunks, their partials are
 * gathered to one GPU, and va_merge combines them there).
 *
 *   args        as for va_verify_attn, with args->num_splits = S, 1 <= S <=
 *               64, given explicitly (0 is rejected: every participant must
 *               use the same partition); out and lse are not used (may be
 *               NULL).  The workspace must hold va_workspace_bytes() of the
 *               same arguments with num_splits = 1 (the request order, and
 *               the widened pages for bf16 queries with an FP8 cache).
 *   split_first, split_count
 *               the splits [split_first, split_first + split_count) of the
 *               S-way partition va_verify_attn defines; 0 <= split_first,
 *               1 <= split_count, split_first + split_count <= S
 *   o_part      [device] float [split_count, B, T, H, 512]  out: normalised
 *               partial outputs, 16-byte aligned
 *   lse_part    [device] float [split_count, B, T, H]  out: partial lse
 *               (-inf for a split with no visible key)
 * Partial c holds split split_first + c.  va_merge over all S partials gives
 * va_verify_attn's result (up to the rounding of a different association).
 */
int va_verify_attn_partials(const va_attn_args* args, int split_first, int split_count,
                            float* o_part, float* lse_part, va_stream_t stream);

/*
 * Merge of split-KV partials (the flash+merge production note, page "The
 * Milestone Commit...", section "How Decisions Were Made").
 *   o_part   [device] float [S, B, T, H, 512]  normalised partial outputs
 *   lse_part [device] float [S, B, T, H]       partial lse (-inf = empty)
 *   out      [device] out_dtype [B, T, H, 512]
 *   lse      [device] float [B, T, H]
 * lse = ln sum_c exp(lse_c); out = sum_c exp(lse_c - lse) o_c; a row whose
 * partials are all empty gets out = 0, lse = -inf.  1 <= S <= 64.
 */
int va_merge(const float* o_part, const float* lse_part, int S, int B, int T, int H,
             int out_dtype, void* out, float* lse, va_stream_t stream);

/* Size of the fixed device array va_verify_attn_noalloc keeps its split-KV
 * partials in (on every device that loads the library, until exit). */
#define VA_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * va_verify_attn without a caller-provided workspace.  The pages have no
 * counterpart of this call: it exists for callers that cannot allocate device
 * memory when they run the verify step -- a serving loop whose device memory
 * is planned once at start-up, or a latency-critical path where an
 * allocation, which may synchronise the device, is not acceptable.
 *
 * Same arguments, checks, split plan and results as va_verify_attn, except
 * that args->workspace / workspace_bytes are ignored: the split-KV partials
 * live in a fixed array of VA_NOALLOC_SCRATCH_BYTES inside the library.
 *   - Returns VA_ERR_UNSUPPORTED, before launching anything, when the
 *     workspace va_verify_attn would need (va_workspace_bytes) exceeds that:
 *     the partials, S * B * T * H * (512 + 1) floats, and for bf16 queries
 *     against an FP8 cache the widened pages, B * max_pages * 73,728 bytes
 *     plus the page table.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *   - The first call on a device looks up the array's device address (once
 *     per device, with that device current); make that first call before any
 *     stream capture.
 *   - Every call shares the array and leaves its contents behind; calls whose
 *     GPU work overlaps (for instance on two streams) race on it.
 */
int va_verify_attn_noalloc(const va_attn_args* args, va_stream_t stream);

/*
 * Diagnostic: number of bounded barrier waits inside the attention kernels
 * (the tensor-core kernel's pipeline barriers, the CUDA-core kernel's
 * bulk-copy staging of an fp32 cache) that expired on the current device
 * since the library was loaded (each expiry also flags its request with
 * VA_ERR_CUDA).  Synchronises the
 * device; returns 0xFFFFFFFF if the counter cannot be read.
 */
unsigned int va_device_timeouts(void);

#ifdef __cplusplus
}
#endif

#endif /* VERIFYATTN_H_ */
