/*
 * Plain-C client of libdcpmla.so: one emulated DCP decode step (2 shards +
 * merge) through the C ABI, with device memory from the CUDA runtime and no
 * other framework.  Inputs are read from a binary file, outputs written to
 * another; tests/test_c_abi_gpu.py prepares the inputs and checks the
 * outputs against the CPU oracle.
 *
 * Input file (little-endian): int32 batch, heads, num_shards, max_blocks,
 * num_blocks, kv_dtype; float32 softmax_scale; int32 seq_lens[batch];
 * int32 block_tables[num_shards][batch][max_blocks]; uint16 q[batch][heads][576];
 * uint8 kv_cache[num_blocks][64][row bytes].
 * Output file: float32 out[batch][heads][512], float32 out_lse[batch][heads].
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include <cuda_runtime_api.h>

#include "dcpmla.h"

#define CHECK_CUDA(x) do { cudaError_t e_ = (x); if (e_ != cudaSuccess) { \
  fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_)); return 2; } } while (0)
#define CHECK_DCP(x) do { int r_ = (x); if (r_ != DCPMLA_OK) { \
  fprintf(stderr, "%s: %s\n", #x, dcpmla_error_string(r_)); return 3; } } while (0)

static void* read_block(FILE* f, size_t bytes) {
  void* p = malloc(bytes ? bytes : 1);
  if (p && bytes && fread(p, 1, bytes, f) != bytes) { free(p); return NULL; }
  return p;
}

int main(int argc, char** argv) {
  if (argc != 3) { fprintf(stderr, "usage: %s inputs.bin outputs.bin\n", argv[0]); return 1; }
  FILE* f = fopen(argv[1], "rb");
  if (!f) { perror(argv[1]); return 1; }
  int32_t hdr[6];
  float scale;
  if (fread(hdr, 4, 6, f) != 6 || fread(&scale, 4, 1, f) != 1) return 1;
  const int B = hdr[0], H = hdr[1], N = hdr[2], MB = hdr[3], NB = hdr[4], kvd = hdr[5];
  const size_t row = kvd == DCPMLA_KV_FP8 ? 656 : 1152;
  const size_t lens_b = (size_t)B * 4, tab_b = (size_t)N * B * MB * 4;
  const size_t q_b = (size_t)B * H * DCPMLA_HEAD_DIM * 2, kv_b = (size_t)NB * 64 * row;
  void* h_lens = read_block(f, lens_b);
  void* h_tab = read_block(f, tab_b);
  void* h_q = read_block(f, q_b);
  void* h_kv = read_block(f, kv_b);
  fclose(f);
  if (!h_lens || !h_tab || !h_q || !h_kv) { fprintf(stderr, "short input\n"); return 1; }

  void *d_lens, *d_tab, *d_q, *d_kv, *d_parts, *d_lses, *d_out, *d_lse, *d_ws;
  size_t ws_bytes = 0;
  CHECK_DCP(mla_decode_workspace_size(B, H, 0, 0, &ws_bytes));
  CHECK_CUDA(cudaMalloc(&d_lens, lens_b));
  CHECK_CUDA(cudaMalloc(&d_tab, tab_b));
  CHECK_CUDA(cudaMalloc(&d_q, q_b));
  CHECK_CUDA(cudaMalloc(&d_kv, kv_b));
  CHECK_CUDA(cudaMalloc(&d_parts, (size_t)N * B * H * 512 * 4));
  CHECK_CUDA(cudaMalloc(&d_lses, (size_t)N * B * H * 4));
  CHECK_CUDA(cudaMalloc(&d_out, (size_t)B * H * 512 * 4));
  CHECK_CUDA(cudaMalloc(&d_lse, (size_t)B * H * 4));
  CHECK_CUDA(cudaMalloc(&d_ws, ws_bytes));
  CHECK_CUDA(cudaMemset(d_ws, 0, ws_bytes));
  CHECK_CUDA(cudaMemcpy(d_lens, h_lens, lens_b, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(d_tab, h_tab, tab_b, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(d_q, h_q, q_b, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(d_kv, h_kv, kv_b, cudaMemcpyHostToDevice));

  for (int s = 0; s < N; ++s) {
    CHECK_DCP(mla_decode_partial(d_q, d_kv, kvd, NB, 64, (const int32_t*)d_tab + (size_t)s * B * MB,
                                 MB, (const int32_t*)d_lens, B, H, s, N, NULL, 0, scale,
                                 (float*)d_parts + (size_t)s * B * H * 512,
                                 (float*)d_lses + (size_t)s * B * H, d_ws, ws_bytes, 0,
                                 DCPMLA_IMPL_AUTO, NULL));
  }
  CHECK_DCP(dcp_merge((const float*)d_parts, (const float*)d_lses, N, B, H, (float*)d_out,
                      (float*)d_lse, NULL));
  CHECK_CUDA(cudaDeviceSynchronize());
  int32_t flags = 0;
  CHECK_CUDA(cudaMemcpy(&flags, d_ws, 4, cudaMemcpyDeviceToHost));
  if (flags != 0) { fprintf(stderr, "device flags 0x%x\n", flags); return 4; }

  float* h_out = (float*)malloc((size_t)B * H * 512 * 4);
  float* h_lse = (float*)malloc((size_t)B * H * 4);
  CHECK_CUDA(cudaMemcpy(h_out, d_out, (size_t)B * H * 512 * 4, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(h_lse, d_lse, (size_t)B * H * 4, cudaMemcpyDeviceToHost));
  FILE* o = fopen(argv[2], "wb");
  if (!o) { perror(argv[2]); return 1; }
  fwrite(h_out, 4, (size_t)B * H * 512, o);
  fwrite(h_lse, 4, (size_t)B * H, o);
  fclose(o);
  printf("ok\n");
  return 0;
}
