/* One greedy verify step through the C ABI from plain C99 with the CUDA runtime:
 * draft-tree mask, verify attention (split count left to the library), accept walk.
 *
 *   va_step <dir>
 *
 * <dir>/dims.txt holds "B T H num_pages max_pages"; the inputs are raw little-endian
 * files in <dir> (q_nope, q_pe, c_kv, k_pe as bf16 bit patterns; page_table, kv_len,
 * parents, tokens, target as int32).  Writes out.bin (bf16), lse.bin (float32),
 * path.bin, accept_len.bin, next_token.bin (int32) and returns 0 when every call
 * reports VA_OK. */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "verifyattn.h"

static char* dir;

static void* read_file(const char* name, size_t bytes) {
  char path[4096];
  snprintf(path, sizeof path, "%s/%s", dir, name);
  FILE* f = fopen(path, "rb");
  if (!f) { printf("cannot open %s\n", path); exit(2); }
  void* h = malloc(bytes ? bytes : 1);
  if (fread(h, 1, bytes, f) != bytes) { printf("short read %s\n", path); exit(2); }
  fclose(f);
  return h;
}
static void write_file(const char* name, const void* h, size_t bytes) {
  char path[4096];
  snprintf(path, sizeof path, "%s/%s", dir, name);
  FILE* f = fopen(path, "wb");
  if (!f || fwrite(h, 1, bytes, f) != bytes) { printf("cannot write %s\n", path); exit(2); }
  fclose(f);
}
static void* upload(const char* name, size_t bytes) {
  void* h = read_file(name, bytes);
  void* d = 0;
  if (cudaMalloc(&d, bytes) != cudaSuccess || cudaMemcpy(d, h, bytes, cudaMemcpyHostToDevice) != cudaSuccess) {
    printf("upload %s failed\n", name); exit(3);
  }
  free(h);
  return d;
}
static void* device(size_t bytes) {
  void* d = 0;
  if (cudaMalloc(&d, bytes) != cudaSuccess) { printf("cudaMalloc failed\n"); exit(3); }
  return d;
}
static void download(const char* name, const void* d, size_t bytes) {
  void* h = malloc(bytes);
  if (cudaMemcpy(h, d, bytes, cudaMemcpyDeviceToHost) != cudaSuccess) { printf("download failed\n"); exit(3); }
  write_file(name, h, bytes);
  free(h);
}

#define VA(call) do { int s_ = (call); if (s_ != VA_OK) { printf("%s -> %s\n", #call, va_status_string(s_)); return 1; } } while (0)

int main(int argc, char** argv) {
  if (argc != 2) { printf("usage: va_step <dir>\n"); return 2; }
  dir = argv[1];
  int B, T, H, num_pages, max_pages;
  {
    char path[4096];
    snprintf(path, sizeof path, "%s/dims.txt", dir);
    FILE* f = fopen(path, "r");
    if (!f || fscanf(f, "%d %d %d %d %d", &B, &T, &H, &num_pages, &max_pages) != 5) { printf("bad dims\n"); return 2; }
    fclose(f);
  }
  const size_t rows = (size_t)B * T * H, W = (size_t)(T + 63) / 64;
  void* q_nope = upload("q_nope.bin", rows * VA_D_LATENT * 2);
  void* q_pe = upload("q_pe.bin", rows * VA_D_ROPE * 2);
  void* c_kv = upload("c_kv.bin", (size_t)num_pages * VA_PAGE_SIZE * VA_D_LATENT * 2);
  void* k_pe = upload("k_pe.bin", (size_t)num_pages * VA_PAGE_SIZE * VA_D_ROPE * 2);
  int32_t* page_table = (int32_t*)upload("page_table.bin", (size_t)B * max_pages * 4);
  int32_t* kv_len = (int32_t*)upload("kv_len.bin", (size_t)B * 4);
  int32_t* parents = (int32_t*)upload("parents.bin", (size_t)B * T * 4);
  int32_t* tokens = (int32_t*)upload("tokens.bin", (size_t)B * T * 4);
  int32_t* target = (int32_t*)upload("target.bin", (size_t)B * T * 4);
  uint64_t* mask = (uint64_t*)device((size_t)B * T * W * 8);
  int32_t* tree_status = (int32_t*)device((size_t)B * 4);
  void* out = device(rows * VA_D_LATENT * 2);
  float* lse = (float*)device(rows * 4);
  int32_t* path = (int32_t*)device((size_t)B * T * 4);
  int32_t* accept_len = (int32_t*)device((size_t)B * 4);
  int32_t* next_token = (int32_t*)device((size_t)B * 4);

  cudaStream_t st;
  if (cudaStreamCreate(&st) != cudaSuccess) return 3;
  VA(va_build_tree_mask(parents, B, T, mask, tree_status, st));

  va_attn_args a;
  memset(&a, 0, sizeof a);
  a.dtype = VA_BF16; a.B = B; a.H = H; a.T = T; a.scale = 0.07216878364870322f;  /* 1/sqrt(192) */
  a.q_nope = q_nope; a.q_pe = q_pe; a.c_kv = c_kv; a.k_pe = k_pe;
  a.num_pages = num_pages; a.page_size = VA_PAGE_SIZE; a.page_table = page_table; a.max_pages = max_pages;
  a.kv_len = kv_len; a.tree_mask = mask; a.out = out; a.lse = lse;
  a.num_splits = 0;
  const size_t ws = va_workspace_bytes(&a);
  if (ws) { a.workspace = device(ws); a.workspace_bytes = ws; }
  VA(va_verify_attn(&a, st));
  VA(va_tree_accept(parents, tokens, target, B, T, path, accept_len, next_token, st));
  if (cudaStreamSynchronize(st) != cudaSuccess) { printf("stream failed\n"); return 3; }

  download("out.bin", out, rows * VA_D_LATENT * 2);
  download("lse.bin", lse, rows * 4);
  download("path.bin", path, (size_t)B * T * 4);
  download("accept_len.bin", accept_len, (size_t)B * 4);
  download("next_token.bin", next_token, (size_t)B * 4);
  printf("step ok: %d requests, %d splits\n", B, va_num_splits(&a));
  return 0;
}
