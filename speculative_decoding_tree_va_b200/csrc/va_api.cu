// C ABI of libverifyattn: argument checks, split planning, dispatch.
// Every entry point validates on the host and returns a va_status before
// launching anything; the caller owns all device memory.
#include <atomic>
#include <cfloat>
#include <cstdio>

#include "va_common.cuh"

namespace {

constexpr int kDefaultSms = 148;  // B200; used when no device can be queried
constexpr int kMaxDevices = 128;
std::atomic<int> g_sm_count[kMaxDevices];  // 0 = not looked up yet

// SM count of the current device (the split planner's wave size), looked up
// once per device.  Without a usable device (host-only use of the planner)
// it is the B200's 148; the runtime error that lookup leaves is cleared.
int sm_count() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    (void)cudaGetLastError();
    return kDefaultSms;
  }
  int n = g_sm_count[dev].load(std::memory_order_relaxed);
  if (n > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 2) {
    (void)cudaGetLastError();
    return kDefaultSms;
  }
  g_sm_count[dev].store(n, std::memory_order_relaxed);
  return n;
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }


// Host-side checks shared by va_verify_attn / va_workspace_bytes.  A
// partials-only call (va_verify_attn_partials) writes neither out nor lse.
int check_args(const va_attn_args* a, bool needs_out = true) {
  if (!a) return VA_ERR_INVALID_ARG;
  if (a->dtype != VA_F32 && a->dtype != VA_BF16) return VA_ERR_INVALID_ARG;
  if (a->B < 0 || a->H < 1 || a->T < 1 || a->T > VA_MAX_QLEN) return VA_ERR_INVALID_ARG;
  if (a->page_size != VA_PAGE_SIZE) return VA_ERR_UNSUPPORTED;
  if (a->B > VA_MAX_BATCH) return VA_ERR_UNSUPPORTED;  // the launches' request axis (grid y)
  if (a->num_splits < 0 || a->num_splits > VA_MAX_SPLITS) return VA_ERR_INVALID_ARG;
  if (a->flags & ~(VA_FLAG_BF16_CUDA_CORES | VA_FLAG_TEST_STALL_MMA | VA_FLAG_KV_FP8_E4M3 |
                   VA_FLAG_TEST_STALL_COPIES))
    return VA_ERR_INVALID_ARG;
  if ((a->flags & VA_FLAG_TEST_STALL_COPIES) &&
      (a->dtype != VA_F32 || (a->flags & (VA_FLAG_KV_FP8_E4M3 | VA_FLAG_TEST_STALL_MMA))))
    return VA_ERR_INVALID_ARG;  // only the bulk-staged fp32 cache has the hook
  if ((a->flags & VA_FLAG_TEST_STALL_MMA) &&
      (!va::uses_tensor_cores(*a) || (a->flags & VA_FLAG_KV_FP8_E4M3)))
    return VA_ERR_INVALID_ARG;  // only the tensor-core kernel on a bf16 cache has the hook
  if ((a->flags & VA_FLAG_KV_FP8_E4M3) && !(a->kv_scale > 0.f && a->kv_scale <= FLT_MAX))
    return VA_ERR_INVALID_ARG;  // NaN, zero, negative or infinite cache scale
  if (!(a->scale == a->scale)) return VA_ERR_INVALID_ARG;  // NaN scale
  if (a->B == 0) return VA_OK;
  if (a->num_pages < 1 || a->max_pages < 1) return VA_ERR_INVALID_ARG;
  if ((long long)a->num_pages * VA_PAGE_SIZE > 0x7fffffffLL) return VA_ERR_UNSUPPORTED;
  if (va::widens_fp8_cache(*a) && (long long)a->B * a->max_pages * VA_PAGE_SIZE > 0x7fffffffLL)
    return VA_ERR_UNSUPPORTED;  // the widened pages are indexed like a pool
  const void* need16[] = {a->q_nope, a->q_pe, a->c_kv, a->k_pe};
  for (const void* p : need16)
    if (!p || !aligned(p, 16)) return VA_ERR_INVALID_ARG;
  if (needs_out && (!a->out || !aligned(a->out, 16))) return VA_ERR_INVALID_ARG;
  if (!a->page_table || !aligned(a->page_table, 4)) return VA_ERR_INVALID_ARG;
  if (!a->kv_len || !aligned(a->kv_len, 4)) return VA_ERR_INVALID_ARG;
  if (!a->tree_mask || !aligned(a->tree_mask, 8)) return VA_ERR_INVALID_ARG;
  if (needs_out && (!a->lse || !aligned(a->lse, 4))) return VA_ERR_INVALID_ARG;
  if (a->req_status && !aligned(a->req_status, 4)) return VA_ERR_INVALID_ARG;
  return VA_OK;
}

// Split count: the caller's, or (num_splits == 0) the smallest power of two
// that fills >= 90% of the last wave, keeping >= 1024 keys per split.  The
// host does not see kv_len, so the planner uses the page-table capacity as
// the key count.  A CUDA-core call with fewer segments than SMs uses the
// balanced plan instead (va_common.cuh), and its count is the plan's slots.
int plan_splits(const va_attn_args* a) {
  if (a->num_splits > 0) return a->num_splits;
  if (a->B == 0) return 1;
  const va::Balance bal = va::plan_balance(*a, sm_count());
  if (bal.G) return bal.slots;
  const long long rows = (long long)a->T * a->H;
  long long units_per_split, slots;
  const int sms = sm_count();
  if (va::uses_tensor_cores(*a)) {
    units_per_split = (long long)a->B * ((rows + 127) / 128);  // CTA pairs
    slots = sms / 2;
  } else {
    units_per_split = (long long)a->B * ((rows + 31) / 32);
    slots = sms;
  }
  const long long keys = (long long)a->max_pages * VA_PAGE_SIZE;
  for (int S = 1; S <= VA_MAX_SPLITS; S *= 2) {
    if (S > 1 && keys / S < 1024) return S / 2;
    const long long units = units_per_split * S;
    const long long waves = (units + slots - 1) / slots;
    if (units * 10 >= waves * slots * 9) return S;
  }
  return VA_MAX_SPLITS;
}

}  // namespace

namespace va {

namespace {

// The attention launches of one call (after the FP8 widening pass and the
// request order, when they apply): splits sp of the partition, partials to
// o_part / lse_part (nullptr: a single split writing out / lse directly).
int launch_attention(const va_attn_args& a, SplitRange sp, const WorkspaceLayout& w, char* base,
                     float* o_part, float* lse_part, cudaStream_t st, const Balance& bal) {
  cudaError_t e;
  const int32_t* order = nullptr;
  if (uses_tensor_cores(a)) {
    int32_t* ord = reinterpret_cast<int32_t*>(base + w.order);
    e = launch_request_order(a.kv_len, a.B, ord, st);
    if (e != cudaSuccess) return VA_ERR_CUDA;
    order = ord;
  }
  if (widens_fp8_cache(a)) {
    // FP8 cache under bf16 queries: widen the pages the batch reads, then run
    // the tensor-core kernel on them with the cache scale folded into the
    // score scale and into the output normalisation.
    void* wc = base + w.w_ckv;
    void* wk = base + w.w_kpe;
    int32_t* wt = reinterpret_cast<int32_t*>(base + w.w_table);
    e = launch_kv_widen(a, wc, wk, wt, st);
    if (e != cudaSuccess) return VA_ERR_CUDA;
    va_attn_args b = a;
    b.c_kv = wc;
    b.k_pe = wk;
    b.page_table = wt;
    b.num_pages = a.B * a.max_pages;
    b.scale = a.scale * a.kv_scale;
    e = launch_attn_tc(b, sp, order, o_part, lse_part, st, a.kv_scale);
  } else if (uses_tensor_cores(a)) {
    e = launch_attn_tc(a, sp, order, o_part, lse_part, st, 1.f);
  } else {
    e = launch_attn_simt(a, sp, o_part, lse_part, st, bal);
  }
  if (e == cudaErrorNotSupported) return VA_ERR_UNSUPPORTED;
  if (e != cudaSuccess) return VA_ERR_CUDA;
  return VA_OK;
}

}  // namespace

int run_verify(const va_attn_args& a, int S, void* ws, cudaStream_t st) {
  const WorkspaceLayout w = workspace_layout(a, S);
  char* base = static_cast<char*>(ws);
  float* o_part = S > 1 ? reinterpret_cast<float*>(base + w.o_part) : nullptr;
  float* lse_part = S > 1 ? reinterpret_cast<float*>(base + w.lse_part) : nullptr;
  // the balanced plan is a function of the arguments and the device, so it is
  // the one the split count S came from
  const Balance bal = plan_balance(a, sm_count());
  if (bal.G && bal.slots != S) return VA_ERR_INVALID_ARG;
  if (S == 1) return launch_attention(a, SplitRange{1, 0, 1}, w, base, nullptr, nullptr, st, bal);
  // Split: a request flagged by one split (a bad page, an expired wait) must
  // come out empty although its other splits hold partials, so the splits
  // report into the call's own status array and the merge empties flagged
  // requests and passes their status on to the caller's array.
  int32_t* status = reinterpret_cast<int32_t*>(base + w.status);
  if (cudaMemsetAsync(status, 0, (size_t)a.B * sizeof(int32_t), st) != cudaSuccess)
    return VA_ERR_CUDA;
  va_attn_args as = a;
  as.req_status = status;
  const int r = launch_attention(as, SplitRange{S, 0, S}, w, base, o_part, lse_part, st, bal);
  if (r != VA_OK) return r;
  cudaError_t e = launch_merge(o_part, lse_part, S, (long long)a.B * a.T * a.H, a.dtype, a.out,
                               a.lse, st, status, a.T * a.H, a.req_status);
  return e == cudaSuccess ? VA_OK : VA_ERR_CUDA;
}

int run_partials(const va_attn_args& a, SplitRange sp, void* ws, float* o_part, float* lse_part,
                 cudaStream_t st) {
  const WorkspaceLayout w = workspace_layout(a, sp.S, false);
  return launch_attention(a, sp, w, static_cast<char*>(ws), o_part, lse_part, st, Balance{});
}

}  // namespace va

extern "C" {

int va_max_qlen(void) { return VA_MAX_QLEN; }

const char* va_status_string(int status) {
  switch (status) {
    case VA_OK: return "VA_OK";
    case VA_ERR_INVALID_ARG: return "VA_ERR_INVALID_ARG";
    case VA_ERR_UNSUPPORTED: return "VA_ERR_UNSUPPORTED";
    case VA_ERR_CUDA: return "VA_ERR_CUDA";
    case VA_ERR_INVALID_TREE: return "VA_ERR_INVALID_TREE";
    default: return "VA_ERR_UNKNOWN";
  }
}

int va_build_tree(const double* lp, const int32_t* tok, int B, int L, int K, int budget,
                  int32_t* parents, int32_t* tokens, int32_t* depth, int32_t* n_nodes,
                  va_stream_t stream) {
  if (B < 0 || L < 1 || L > VA_MAX_DEPTH || K < 1 || K > VA_MAX_TOPK || budget < 0 ||
      budget + 1 > VA_MAX_QLEN)
    return VA_ERR_INVALID_ARG;
  if (B == 0) return VA_OK;
  if (!lp || !tok || !parents || !tokens || !depth || !n_nodes) return VA_ERR_INVALID_ARG;
  if (!aligned(lp, 8)) return VA_ERR_INVALID_ARG;
  cudaError_t e = va::launch_build_tree(lp, tok, B, L, K, budget, parents, tokens, depth,
                                        n_nodes, (cudaStream_t)stream);
  return e == cudaSuccess ? VA_OK : VA_ERR_CUDA;
}

int va_build_tree_mask(const int32_t* parents, int B, int T, uint64_t* mask,
                       int32_t* tree_status, va_stream_t stream) {
  if (B < 0 || T < 1 || T > VA_MAX_QLEN) return VA_ERR_INVALID_ARG;
  if (B == 0) return VA_OK;
  if (!parents || !mask || !aligned(mask, 8)) return VA_ERR_INVALID_ARG;
  cudaError_t e = va::launch_tree_mask(parents, B, T, mask, tree_status, (cudaStream_t)stream);
  return e == cudaSuccess ? VA_OK : VA_ERR_CUDA;
}

int va_tree_accept(const int32_t* parents, const int32_t* tokens, const int32_t* target_next,
                   int B, int T, int32_t* path, int32_t* accept_len, int32_t* next_token,
                   va_stream_t stream) {
  if (B < 0 || T < 1 || T > VA_MAX_QLEN) return VA_ERR_INVALID_ARG;
  if (B == 0) return VA_OK;
  if (!parents || !tokens || !target_next || !path || !accept_len || !next_token)
    return VA_ERR_INVALID_ARG;
  cudaError_t e = va::launch_tree_accept(parents, tokens, target_next, B, T, path, accept_len,
                                         next_token, (cudaStream_t)stream);
  return e == cudaSuccess ? VA_OK : VA_ERR_CUDA;
}

int va_num_splits(const va_attn_args* args) {
  const int st = check_args(args);
  if (st != VA_OK) return -st;
  return plan_splits(args);
}

size_t va_workspace_bytes(const va_attn_args* args) {
  if (check_args(args) != VA_OK || args->B == 0) return 0;
  return va::workspace_layout(*args, plan_splits(args)).total;
}

int va_verify_attn(const va_attn_args* args, va_stream_t stream) {
  const int st = check_args(args);
  if (st != VA_OK) return st;
  if (args->B == 0) return VA_OK;
  const int S = plan_splits(args);
  const size_t need = va::workspace_layout(*args, S).total;
  if (need && (!args->workspace || !aligned(args->workspace, 256) || args->workspace_bytes < need))
    return VA_ERR_INVALID_ARG;
  return va::run_verify(*args, S, args->workspace, (cudaStream_t)stream);
}

int va_verify_attn_partials(const va_attn_args* args, int split_first, int split_count,
                            float* o_part, float* lse_part, va_stream_t stream) {
  const int st = check_args(args, false);
  if (st != VA_OK) return st;
  const int S = args->num_splits;
  if (S < 1) return VA_ERR_INVALID_ARG;  // the partition must be explicit
  if (split_first < 0 || split_count < 1 || split_first > S - split_count)
    return VA_ERR_INVALID_ARG;
  if (args->B == 0) return VA_OK;
  if (!o_part || !lse_part || !aligned(o_part, 16) || !aligned(lse_part, 4))
    return VA_ERR_INVALID_ARG;
  const size_t need = va::workspace_layout(*args, S, false).total;
  if (need && (!args->workspace || !aligned(args->workspace, 256) || args->workspace_bytes < need))
    return VA_ERR_INVALID_ARG;
  return va::run_partials(*args, va::SplitRange{S, split_first, split_count}, args->workspace,
                          o_part, lse_part, (cudaStream_t)stream);
}

int va_merge(const float* o_part, const float* lse_part, int S, int B, int T, int H,
             int out_dtype, void* out, float* lse, va_stream_t stream) {
  if (S < 1 || S > VA_MAX_SPLITS || B < 0 || T < 1 || T > VA_MAX_QLEN || H < 1)
    return VA_ERR_INVALID_ARG;
  if (out_dtype != VA_F32 && out_dtype != VA_BF16) return VA_ERR_INVALID_ARG;
  if (B == 0) return VA_OK;
  if (!o_part || !lse_part || !out || !lse) return VA_ERR_INVALID_ARG;
  if (!aligned(o_part, 16) || !aligned(out, 8) || !aligned(lse_part, 4) || !aligned(lse, 4))
    return VA_ERR_INVALID_ARG;
  cudaError_t e = va::launch_merge(o_part, lse_part, S, (long long)B * T * H, out_dtype, out,
                                   lse, (cudaStream_t)stream);
  return e == cudaSuccess ? VA_OK : VA_ERR_CUDA;
}

unsigned int va_device_timeouts(void) {
  const unsigned int a = va::tc_timeouts(), b = va::simt_timeouts();
  if (a == 0xFFFFFFFFu || b == 0xFFFFFFFFu) return 0xFFFFFFFFu;
  return a + b;
}

}  // extern "C"
