// Oracle for DDTree tree-verify MLA attention -- TEST INFRASTRUCTURE ONLY.
//
// A plain, slow, single-threaded fp64 restatement of what the verify step
// computes.  Only the tests, the package's smoke check and the benchmark's
// CPU-baseline leg may load it; the CUDA library never links or calls it and
// the two share no code, headers or tables.
//
// Sources (web pages; section named in each function's comment):
//   [MC]  "The Milestone Commit: Cementing Phase 1 of a Custom CUDA
//          Speculative Decoding Engine"
//   [SP]  "Strategic Pivots in CUDA Kernel Engineering: Validating the DDTree
//          Tree Builder and Planning the Verify-Attn Kernel"
//
// Readings where the pages are silent (each is pinned by a CPU test):
//   * node i of the tree tail sits at key position P_b + i of the request's
//     key sequence (P_b = kv_len_b - T);
//   * q_nope arrives already absorbed into the 512-d latent space, V = c_kv,
//     output stays latent, scale = 1/sqrt(192) passed in by the caller;
//   * lse is the natural log of sum(exp(scaled score));
//   * a row whose own tree bit is clear is an absent (padding) node:
//     out = 0, lse = -inf;  an empty key set gives the same.
//
// Pins (tests/): brute-force softmax on tiny inputs, hand-worked 3-node
// trees, chain tree == causal attention, popcount(mask) == depth + 1,
// page-table permutation invariance, split+merge == unsplit, brute-force
// enumeration of the best-first tree on tiny (k, L); the FP8 E4M3 decoder
// against the format's closed-form values and against torch's float8_e4m3fn
// conversion of all 256 codes.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>

namespace {

constexpr double kNegInf = -std::numeric_limits<double>::infinity();

// One FP8 E4M3 code as a double, from the OCP 8-bit floating point format
// definition (OFP8, the E4M3 encoding): bit 7 sign, bits 6..3 exponent field
// E with bias 7, bits 2..0 mantissa M.  E = 0 is subnormal, M/8 * 2^-6; the
// other fields are normal, (1 + M/8) * 2^(E - 7); the one pattern E = 15,
// M = 7 is NaN (the format has no infinities, so its largest value is
// 1.75 * 2^8 = 448).  Every code widens to double exactly.
double decode_e4m3(uint8_t code) {
  const int sign = code >> 7;
  const int e = (code >> 3) & 15;
  const int m = code & 7;
  if (e == 15 && m == 7) return std::numeric_limits<double>::quiet_NaN();
  const double mag = e == 0 ? std::ldexp(static_cast<double>(m) / 8.0, -6)
                            : std::ldexp(1.0 + static_cast<double>(m) / 8.0, e - 7);
  return sign ? -mag : mag;
}

// Element fetch: dtype 0 = float32 storage, 1 = bf16 bit patterns, 2 = FP8
// E4M3 codes.  All widen to double exactly.
inline double fetch(const void* base, int64_t idx, int dtype) {
  if (dtype == 0) return static_cast<double>(static_cast<const float*>(base)[idx]);
  if (dtype == 2) return decode_e4m3(static_cast<const uint8_t*>(base)[idx]);
  uint32_t bits = static_cast<uint32_t>(static_cast<const uint16_t*>(base)[idx]) << 16;
  float f;
  std::memcpy(&f, &bits, sizeof f);
  return static_cast<double>(f);
}

struct Cand {
  double score;
  int parent;
  int depth;
  int rank;
};

// Best candidate first: larger score; equal scores -> smaller parent node
// index, then smaller rank (a lexicographic tuple order, [SP] "Why This
// Message Was Written": tie-breaking matched tuple comparison).
bool better(const Cand& a, const Cand& b) {
  if (a.score != b.score) return a.score > b.score;
  if (a.parent != b.parent) return a.parent < b.parent;
  return a.rank < b.rank;
}

}  // namespace

extern "C" {

// FP8 E4M3 codes -> doubles (decode_e4m3 above), for the format's pins.
void or_decode_e4m3(const uint8_t* codes, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = decode_e4m3(codes[i]);
}

// Best-first draft-tree builder ([MC] "The Context", item 1; [SP] "Why This
// Message Was Written").  lp/tok are [L][K]: row d holds the drafter's top-K
// log-probs (descending) and token ids for depth d + 1.  Node 0 is the root
// (depth 0, score 0, parent -1, token -1).  A node at depth d with rank r
// under parent p scores score[p] + lp[d-1][r].  The frontier starts with the
// root's best child; each popped candidate becomes the next node and offers
// its next sibling and its own best child.  Building stops at budget + 1
// nodes or when the frontier is empty (an underfull tree).  The frontier is a
// plain vector scanned linearly: slow and obviously correct.
// Returns the node count n; entries n..budget are set to parent -1,
// token -1, depth -1, rank -1, score -inf.
int or_build_tree(const double* lp, const int32_t* tok, int L, int K, int budget,
                  int32_t* parent, int32_t* token, int32_t* depth, int32_t* rank,
                  double* score) {
  const int T = budget + 1;
  for (int i = 0; i < T; ++i) {
    parent[i] = -1; token[i] = -1; depth[i] = -1; rank[i] = -1; score[i] = kNegInf;
  }
  parent[0] = -1; token[0] = -1; depth[0] = 0; rank[0] = 0; score[0] = 0.0;
  int n = 1;
  std::vector<Cand> frontier;
  if (L >= 1 && K >= 1) frontier.push_back({score[0] + lp[0], 0, 1, 0});
  while (n < T && !frontier.empty()) {
    size_t best = 0;
    for (size_t i = 1; i < frontier.size(); ++i)
      if (better(frontier[i], frontier[best])) best = i;
    Cand c = frontier[best];
    frontier.erase(frontier.begin() + static_cast<long>(best));
    const int node = n++;
    parent[node] = c.parent;
    depth[node] = c.depth;
    rank[node] = c.rank;
    score[node] = c.score;
    token[node] = tok[(c.depth - 1) * K + c.rank];
    if (c.rank + 1 < K)
      frontier.push_back({score[c.parent] + lp[(c.depth - 1) * K + c.rank + 1],
                          c.parent, c.depth, c.rank + 1});
    if (c.depth + 1 <= L)
      frontier.push_back({score[node] + lp[c.depth * K], node, c.depth + 1, 0});
  }
  return n;
}

// Tree visibility mask ([SP] "The Message": "a tree visibility mask from the
// builder").  Row t of request b gets bit i (word i / 64, bit i % 64) for
// every node i on the path from the root to t, t included.  parent[b][0]
// must be -1; for i >= 1, parent -1 marks an absent (padding) node whose row
// stays all-zero; otherwise 0 <= parent < i and the parent must be present.
// A request that breaks this gets status 1 and all-zero rows; else status 0.
void or_ancestor_mask(const int32_t* parents, int B, int T, uint64_t* mask,
                      int32_t* status) {
  const int W = (T + 63) / 64;
  for (int b = 0; b < B; ++b) {
    const int32_t* par = parents + static_cast<int64_t>(b) * T;
    uint64_t* mb = mask + static_cast<int64_t>(b) * T * W;
    std::memset(mb, 0, sizeof(uint64_t) * T * W);
    bool ok = (T >= 1) && par[0] == -1;
    std::vector<bool> present(T, false);
    if (ok) present[0] = true;
    for (int i = 1; ok && i < T; ++i) {
      if (par[i] == -1) continue;
      if (par[i] < 0 || par[i] >= i || !present[par[i]]) { ok = false; break; }
      present[i] = true;
    }
    status[b] = ok ? 0 : 1;
    if (!ok) continue;
    for (int t = 0; t < T; ++t) {
      if (!present[t]) continue;
      for (int i = t; i != -1; i = par[i]) mb[t * W + i / 64] |= (uint64_t{1} << (i % 64));
    }
  }
}

// Masked MLA-absorb attention for selected rows ([MC] "The Context", item 2:
// masked softmax over the concatenated prefix and tree tail, latent output;
// [MC] "Input Knowledge Required": MLA absorbed latent space).
//
// Row id r = (b*T + t)*H + h.  Keys of request b are positions j in
// [0, kv_len[b]); key j lives in physical page page_table[b][j / page_size],
// slot j % page_size.  With P = kv_len[b] - T, key j is visible to (b, t) iff
// j < P, or j >= P and bit (j - P) of mask[b][t] is set; only keys inside
// [key_lo[b], key_hi[b]) count (NULL bounds = whole range, for split chunks).
//   s_j = scale * (sum_d q_nope[d] c_kv_j[d] + sum_e q_pe[e] k_pe_j[e])
//   m = max s_j,  l = sum exp(s_j - m)
//   out = sum_j exp(s_j - m) / l * c_kv_j,   lse = m + ln l
// No visible key, or the row's own tree bit clear: out = 0, lse = -inf.
// dtype (queries): 0 = float32 inputs, 1 = bf16 bit patterns.  kv_dtype
// (c_kv, k_pe): the same codes, or 2 = FP8 E4M3 codes; a cached element is
// kv_scale times its stored value (the latent cache kept at 8 bits with one
// scale for the whole tensor; not a step the pages describe).  Every c_kv_j
// and k_pe_j above is that scaled value.  Outputs are float64.
void or_attention_rows(int B, int T, int H, int Dc, int Dr, double scale, int dtype,
                       int kv_dtype, double kv_scale, const void* q_nope, const void* q_pe, const void* c_kv,
                       const void* k_pe, int page_size, const int32_t* page_table,
                       int max_pages, const int32_t* kv_len, const uint64_t* mask,
                       const int32_t* key_lo, const int32_t* key_hi,
                       int n_rows, const int32_t* rows, double* out, double* lse) {
  const int W = (T + 63) / 64;
  std::vector<double> s;
  std::vector<int64_t> krow;
  for (int ri = 0; ri < n_rows; ++ri) {
    const int64_t r = rows ? rows[ri] : ri;
    const int h = static_cast<int>(r % H);
    const int t = static_cast<int>((r / H) % T);
    const int b = static_cast<int>(r / (static_cast<int64_t>(H) * T));
    double* o = out + static_cast<int64_t>(ri) * Dc;
    for (int d = 0; d < Dc; ++d) o[d] = 0.0;
    lse[ri] = kNegInf;

    const uint64_t* mrow = mask + (static_cast<int64_t>(b) * T + t) * W;
    if (((mrow[t / 64] >> (t % 64)) & 1u) == 0) continue;  // absent node

    const int kv = kv_len[b];
    const int P = kv - T;
    const int lo = key_lo ? key_lo[b] : 0;
    const int hi = key_hi ? key_hi[b] : kv;
    s.clear();
    krow.clear();
    for (int j = lo; j < hi; ++j) {
      if (j >= P) {
        const int i = j - P;
        if (((mrow[i / 64] >> (i % 64)) & 1u) == 0) continue;
      }
      const int64_t page = page_table[static_cast<int64_t>(b) * max_pages + j / page_size];
      const int64_t kr = page * page_size + j % page_size;
      double dot = 0.0;
      for (int d = 0; d < Dc; ++d)
        dot += fetch(q_nope, r * Dc + d, dtype) * (kv_scale * fetch(c_kv, kr * Dc + d, kv_dtype));
      for (int e = 0; e < Dr; ++e)
        dot += fetch(q_pe, r * Dr + e, dtype) * (kv_scale * fetch(k_pe, kr * Dr + e, kv_dtype));
      s.push_back(scale * dot);
      krow.push_back(kr);
    }
    if (s.empty()) continue;
    double m = s[0];
    for (double v : s) m = v > m ? v : m;
    double l = 0.0;
    for (double v : s) l += std::exp(v - m);
    for (size_t k = 0; k < s.size(); ++k) {
      const double w = std::exp(s[k] - m) / l;
      for (int d = 0; d < Dc; ++d) o[d] += w * (kv_scale * fetch(c_kv, krow[k] * Dc + d, kv_dtype));
    }
    lse[ri] = m + std::log(l);
  }
}

// Merge of split-KV partials (the flash+merge note of [MC] "How Decisions
// Were Made", production notes).  Partial c of a row holds its normalised
// output O_c and its lse_c.  lse = log sum_c exp(lse_c); out = sum_c
// exp(lse_c - lse) O_c.  Chunks with lse_c = -inf weigh nothing; a row with
// every chunk empty gets out = 0, lse = -inf.  Layout: o_part [S][rows][D],
// lse_part [S][rows].
void or_merge(const double* o_part, const double* lse_part, int S, int64_t rows, int D,
              double* out, double* lse) {
  for (int64_t r = 0; r < rows; ++r) {
    double m = kNegInf;
    for (int c = 0; c < S; ++c) m = lse_part[c * rows + r] > m ? lse_part[c * rows + r] : m;
    double* o = out + r * D;
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    if (m == kNegInf) { lse[r] = kNegInf; continue; }
    double z = 0.0;
    for (int c = 0; c < S; ++c) z += std::exp(lse_part[c * rows + r] - m);
    const double L = m + std::log(z);
    for (int c = 0; c < S; ++c) {
      const double lc = lse_part[c * rows + r];
      if (lc == kNegInf) continue;
      const double w = std::exp(lc - L);
      const double* oc = o_part + (c * rows + r) * D;
      for (int d = 0; d < D; ++d) o[d] += w * oc[d];
    }
    lse[r] = L;
  }
}

// Greedy tree accept ([MC] "The Context", item 3: follow the verified tree
// with next-token / next-sibling pointers to find the accepted tokens).  For
// request b, start at the root; while the target's greedy next token after
// the current node (target_next[b][cur]) equals the token of one of cur's
// children, move to that child (the lowest node index among equal tokens).
// Absent nodes (parent -1 for i >= 1) are never children.  Outputs: the
// accepted path path[b][0..n-1] (root first, rest -1), accept_len[b] = n
// (tokens committed this step: n - 1 draft tokens plus the target's token
// after the last accepted node), next_token[b] = target_next[b][last node].
void or_tree_accept(const int32_t* parents, const int32_t* tokens, const int32_t* target_next,
                    int B, int T, int32_t* path, int32_t* accept_len, int32_t* next_token) {
  for (int b = 0; b < B; ++b) {
    const int32_t* par = parents + static_cast<int64_t>(b) * T;
    const int32_t* tok = tokens + static_cast<int64_t>(b) * T;
    const int32_t* tgt = target_next + static_cast<int64_t>(b) * T;
    int32_t* pb = path + static_cast<int64_t>(b) * T;
    for (int i = 0; i < T; ++i) pb[i] = -1;
    int cur = 0, n = 0;
    pb[n++] = 0;
    for (;;) {
      int next = -1;
      for (int i = cur + 1; i < T; ++i)  // children carry larger indices than their parent
        if (par[i] == cur && tok[i] == tgt[cur]) { next = i; break; }
      if (next < 0) break;
      cur = next;
      pb[n++] = cur;
    }
    accept_len[b] = n;
    next_token[b] = tgt[cur];
  }
}

}  // extern "C"
