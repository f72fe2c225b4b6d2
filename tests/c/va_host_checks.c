/* Host-side use of libverifyattn from plain C99 (no GPU needed): status strings,
 * argument rejection before any launch, split planning.  Exit code 0 = all good. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "verifyattn.h"

#define CHECK(c) do { if (!(c)) { printf("failed: %s (line %d)\n", #c, __LINE__); return 1; } } while (0)

int main(void) {
  static char fake[64];  /* a non-null, 16-byte-aligned address; never dereferenced */
  void* p = (void*)(((uintptr_t)fake + 15) & ~(uintptr_t)15);
  va_attn_args a;
  memset(&a, 0, sizeof a);
  a.dtype = VA_BF16; a.B = 2; a.H = 64; a.T = 33; a.scale = 0.07f;
  a.q_nope = a.q_pe = a.c_kv = a.k_pe = p;
  a.page_table = (const int32_t*)p; a.kv_len = (const int32_t*)p;
  a.tree_mask = (const uint64_t*)p; a.out = p; a.lse = (float*)p;
  a.num_pages = 100; a.page_size = VA_PAGE_SIZE; a.max_pages = 50;

  CHECK(va_max_qlen() == VA_MAX_QLEN);
  CHECK(strcmp(va_status_string(VA_ERR_INVALID_TREE), "VA_ERR_INVALID_TREE") == 0);

  a.num_splits = 16;
  CHECK(va_num_splits(&a) == 16);
  CHECK(va_workspace_bytes(&a) > 0);
  CHECK(va_verify_attn(&a, 0) == VA_ERR_INVALID_ARG);   /* split without a workspace */
  a.num_splits = 1;
  CHECK(va_workspace_bytes(&a) == 256);   /* tensor cores: the request order, int32 [B] */
  a.dtype = VA_F32;
  CHECK(va_workspace_bytes(&a) == 0);     /* CUDA cores, one pass: nothing */
  a.dtype = VA_BF16;
  CHECK(va_verify_attn_partials(&a, 0, 2, (float*)p, (float*)p, 0) == VA_ERR_INVALID_ARG);

  a.T = VA_MAX_QLEN + 1;
  CHECK(va_verify_attn(&a, 0) == VA_ERR_INVALID_ARG);
  CHECK(va_num_splits(&a) == -VA_ERR_INVALID_ARG);
  a.T = 33;
  a.page_size = 32;
  CHECK(va_verify_attn(&a, 0) == VA_ERR_UNSUPPORTED);
  a.page_size = VA_PAGE_SIZE;
  CHECK(va_build_tree_mask(0, 1, VA_MAX_QLEN + 1, 0, 0, 0) == VA_ERR_INVALID_ARG);
  CHECK(va_tree_accept(0, 0, 0, 1, 0, 0, 0, 0, 0) == VA_ERR_INVALID_ARG);
  CHECK(va_merge(0, 0, 0, 1, 1, 1, VA_F32, 0, 0, 0) == VA_ERR_INVALID_ARG);

  /* FP8 cache: a finite, positive scale is required */
  a.flags = VA_FLAG_KV_FP8_E4M3;
  a.kv_scale = 0.0f;
  CHECK(va_num_splits(&a) == -VA_ERR_INVALID_ARG);
  a.kv_scale = -1.0f;
  CHECK(va_verify_attn(&a, 0) == VA_ERR_INVALID_ARG);
  a.kv_scale = 0.4375f;
  a.num_splits = 1;
  CHECK(va_num_splits(&a) == 1);
  CHECK(va_workspace_bytes(&a) > 0);   /* bf16 on tensor cores: the widened pages */
  a.dtype = VA_F32;
  CHECK(va_workspace_bytes(&a) == 0);  /* fp32 on CUDA cores widens while staging */
  a.dtype = VA_BF16;
  a.flags |= VA_FLAG_TEST_STALL_MMA;
  CHECK(va_num_splits(&a) == -VA_ERR_INVALID_ARG);
  a.flags = 0;
  printf("VA_NOALLOC_SCRATCH_BYTES=%lu\n", (unsigned long)VA_NOALLOC_SCRATCH_BYTES);
  printf("host checks ok\n");
  return 0;
}
