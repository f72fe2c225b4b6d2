// Draft-tree kernels: best-first builder and ancestor (visibility) mask.
//
// Builder: page "The Milestone Commit: Cementing Phase 1 of a Custom CUDA
// Speculative Decoding Engine", section "The Context", item 1 (GPU best-first
// builder replacing the per-request CPU heap) and page "Strategic Pivots in
// CUDA Kernel Engineering...", section "Why This Message Was Written" (ties
// follow tuple comparison, fp64 accumulation).
// Mask: page "Strategic Pivots in CUDA Kernel Engineering...", section
// "The Message" (tree visibility mask from the builder).
#include "va_common.cuh"

namespace va {
namespace {

struct Cand {
  double s;  // score
  int p;     // parent node
  int r;     // rank within the parent's children
};

// Strict "a pops before b": higher score, then lower parent, then lower rank.
// (parent, rank) identifies a candidate, so this is a total order and any
// correct priority queue pops the same sequence.
__device__ __forceinline__ bool before(const Cand& a, const Cand& b) {
  if (a.s != b.s) return a.s > b.s;
  if (a.p != b.p) return a.p < b.p;
  return a.r < b.r;
}

// One thread per request; the frontier is a binary heap in local memory.
// It never holds more than T candidates (each pop adds at most two).
__global__ void build_tree_kernel(const double* __restrict__ lp, const int32_t* __restrict__ tok,
                                  int B, int L, int K, int budget, int32_t* __restrict__ parents,
                                  int32_t* __restrict__ tokens, int32_t* __restrict__ depth,
                                  int32_t* __restrict__ n_nodes) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const int T = budget + 1;
  const double* lpb = lp + (size_t)b * L * K;
  const int32_t* tkb = tok + (size_t)b * L * K;
  int32_t* pb = parents + (size_t)b * T;
  int32_t* tb = tokens + (size_t)b * T;
  int32_t* db = depth + (size_t)b * T;

  double nscore[VA_MAX_QLEN];
  int ndepth[VA_MAX_QLEN];
  Cand heap[VA_MAX_QLEN + 1];
  int hn = 0;

  for (int i = 0; i < T; ++i) { pb[i] = -1; tb[i] = -1; db[i] = -1; }
  db[0] = 0;
  nscore[0] = 0.0;
  ndepth[0] = 0;

  auto push = [&](Cand c) {
    int i = hn++;
    while (i > 0) {
      int up = (i - 1) >> 1;
      if (!before(c, heap[up])) break;
      heap[i] = heap[up];
      i = up;
    }
    heap[i] = c;
  };
  auto pop = [&]() {
    Cand top = heap[0];
    Cand last = heap[--hn];
    int i = 0;
    for (;;) {
      int l = 2 * i + 1;
      if (l >= hn) break;
      int c = (l + 1 < hn && before(heap[l + 1], heap[l])) ? l + 1 : l;
      if (!before(heap[c], last)) break;
      heap[i] = heap[c];
      i = c;
    }
    if (hn > 0) heap[i] = last;
    return top;
  };

  if (L >= 1 && K >= 1) push(Cand{nscore[0] + lpb[0], 0, 0});
  int n = 1;
  while (n < T && hn > 0) {
    Cand c = pop();
    const int node = n++;
    const int d = ndepth[c.p] + 1;  // depth of the new node, 1..L
    nscore[node] = c.s;
    ndepth[node] = d;
    pb[node] = c.p;
    db[node] = d;
    tb[node] = tkb[(d - 1) * K + c.r];
    if (c.r + 1 < K) push(Cand{nscore[c.p] + lpb[(d - 1) * K + c.r + 1], c.p, c.r + 1});
    if (d + 1 <= L) push(Cand{nscore[node] + lpb[d * K], node, 0});
  }
  n_nodes[b] = n;
}

// One block per request, one thread per node.  Each node walks its parent
// chain (strictly decreasing indices, so at most T steps), checking every
// link; any malformed link invalidates the whole request.
__global__ void tree_mask_kernel(const int32_t* __restrict__ parents, int T,
                                 uint64_t* __restrict__ mask, int32_t* __restrict__ status) {
  __shared__ int bad_any;
  const int b = blockIdx.x;
  const int i = threadIdx.x;
  const int W = (T + 63) >> 6;
  const int32_t* pb = parents + (size_t)b * T;
  if (i == 0) bad_any = 0;
  __syncthreads();

  uint64_t w0 = 0, w1 = 0;
  bool bad = false;
  if (i < T) {
    const int p = pb[i];
    bool present = true;
    if (i == 0) {
      bad = (p != -1);
    } else if (p == -1) {
      present = false;
    } else if (p < 0 || p >= i) {
      bad = true;
    }
    if (present && !bad) {
      int cur = i;
      for (int steps = 0; steps <= T; ++steps) {
        if (cur < 64) w0 |= 1ull << cur; else w1 |= 1ull << (cur - 64);
        if (cur == 0) break;
        const int pp = pb[cur];
        if (pp < 0 || pp >= cur) { bad = true; break; }  // absent or malformed ancestor
        cur = pp;
      }
    }
    if (bad) atomicOr(&bad_any, 1);
  }
  __syncthreads();
  if (i < T) {
    uint64_t* row = mask + ((size_t)b * T + i) * W;
    if (bad_any) { w0 = 0; w1 = 0; }
    row[0] = w0;
    if (W > 1) row[1] = w1;
  }
  if (i == 0 && status) status[b] = bad_any ? VA_ERR_INVALID_TREE : VA_OK;
}

// Greedy accept walk over the verified tree (page "The Milestone Commit...",
// section "The Context", item 3: next-token / next-sibling pointers).  One
// thread per request: link every node to its parent's child list (children
// in increasing index order), then from the root follow the child whose
// token equals the target's greedy next token.  Only links with
// 0 <= parent < index count.
__global__ void tree_accept_kernel(const int32_t* __restrict__ parents,
                                   const int32_t* __restrict__ tokens,
                                   const int32_t* __restrict__ target_next, int B, int T,
                                   int32_t* __restrict__ path, int32_t* __restrict__ accept_len,
                                   int32_t* __restrict__ next_token) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const int32_t* par = parents + (size_t)b * T;
  const int32_t* tok = tokens + (size_t)b * T;
  const int32_t* tgt = target_next + (size_t)b * T;
  int32_t* pb = path + (size_t)b * T;
  int8_t first_child[VA_MAX_QLEN], next_sib[VA_MAX_QLEN];
  for (int i = 0; i < T; ++i) { first_child[i] = -1; next_sib[i] = -1; pb[i] = -1; }
  for (int i = T - 1; i >= 1; --i) {
    const int p = par[i];
    if (p >= 0 && p < i) { next_sib[i] = first_child[p]; first_child[p] = (int8_t)i; }
  }
  int cur = 0, n = 0;
  pb[n++] = 0;
  for (;;) {
    const int want = tgt[cur];
    int c = first_child[cur];
    while (c >= 0 && tok[c] != want) c = next_sib[c];
    if (c < 0) break;
    cur = c;
    pb[n++] = cur;
  }
  accept_len[b] = n;
  next_token[b] = tgt[cur];
}

}  // namespace

cudaError_t launch_tree_accept(const int32_t* parents, const int32_t* tokens,
                               const int32_t* target_next, int B, int T, int32_t* path,
                               int32_t* accept_len, int32_t* next_token, cudaStream_t st) {
  if (B == 0) return cudaSuccess;
  tree_accept_kernel<<<(B + 63) / 64, 64, 0, st>>>(parents, tokens, target_next, B, T, path,
                                                    accept_len, next_token);
  return cudaGetLastError();
}

cudaError_t launch_build_tree(const double* lp, const int32_t* tok, int B, int L, int K,
                              int budget, int32_t* parents, int32_t* tokens, int32_t* depth,
                              int32_t* n_nodes, cudaStream_t st) {
  if (B == 0) return cudaSuccess;
  const int threads = 64;
  build_tree_kernel<<<(B + threads - 1) / threads, threads, 0, st>>>(
      lp, tok, B, L, K, budget, parents, tokens, depth, n_nodes);
  return cudaGetLastError();
}

cudaError_t launch_tree_mask(const int32_t* parents, int B, int T, uint64_t* mask,
                             int32_t* status, cudaStream_t st) {
  if (B == 0) return cudaSuccess;
  tree_mask_kernel<<<B, 96, 0, st>>>(parents, T, mask, status);
  return cudaGetLastError();
}

}  // namespace va
