/*
 * A C caller of libkvzip without torch: the whole compression from host
 * buffers, staged with the CUDA runtime the way the header describes
 * (device pointers in every call, copies and calls on one stream).
 *
 *   c_abi_host_staging IN OUT
 *
 * IN  (little-endian): int64 B, G, d, n_c, n_chunks; double r; int64 n_in[n_chunks];
 *     then bf16 k_ctx [B][n_c][d], v [B][n_c][d], and per chunk q [B][G][n_in][d]
 *     followed by k_self [B][n_in][d].
 * OUT: int64 k; float scores [B][n_c]; int64 offsets [B + 1]; bf16 k_out [k][d],
 *     v_out [k][d]; int32 pos [k].
 *
 * Every input lives in page-locked host memory (cudaMallocHost) and goes up
 * with cudaMemcpyAsync; one device buffer pair is reused by every chunk, which
 * the stream order makes safe.  Exit status 0 on success; any CUDA or kvzip
 * error is printed and gives exit status 1.
 */
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "kvzip.h"

#define CUDA_OK(x)                                                               \
  do {                                                                           \
    cudaError_t e_ = (x);                                                        \
    if (e_ != cudaSuccess) {                                                     \
      fprintf(stderr, "%s:%d %s: %s\n", __FILE__, __LINE__, #x,                  \
              cudaGetErrorString(e_));                                           \
      exit(1);                                                                   \
    }                                                                            \
  } while (0)

#define KVZIP_OK_(x)                                                             \
  do {                                                                           \
    kvzip_status s_ = (x);                                                       \
    if (s_ != KVZIP_OK) {                                                        \
      fprintf(stderr, "%s:%d %s: %s\n", __FILE__, __LINE__, #x,                  \
              kvzip_status_string(s_));                                          \
      exit(1);                                                                   \
    }                                                                            \
  } while (0)

static void read_exact(FILE* f, void* dst, size_t bytes) {
  if (bytes && fread(dst, 1, bytes, f) != bytes) {
    fprintf(stderr, "short input file\n");
    exit(1);
  }
}

static void write_exact(FILE* f, const void* src, size_t bytes) {
  if (bytes && fwrite(src, 1, bytes, f) != bytes) {
    fprintf(stderr, "short write\n");
    exit(1);
  }
}

/* page-locked host buffer filled from the input file */
static void* pinned_from(FILE* f, size_t bytes) {
  void* p = NULL;
  CUDA_OK(cudaMallocHost(&p, bytes ? bytes : 1));
  read_exact(f, p, bytes);
  return p;
}

static void* dev_alloc(size_t bytes) {
  void* p = NULL;
  CUDA_OK(cudaMalloc(&p, bytes ? bytes : 256));
  return p;
}

int main(int argc, char** argv) {
  if (argc != 3) {
    fprintf(stderr, "usage: %s IN OUT\n", argv[0]);
    return 2;
  }
  FILE* in = fopen(argv[1], "rb");
  if (!in) {
    perror(argv[1]);
    return 1;
  }
  int64_t hdr[5];
  double r = 0.0;
  read_exact(in, hdr, sizeof hdr);
  read_exact(in, &r, sizeof r);
  const int64_t B = hdr[0], G = hdr[1], d = hdr[2], n_c = hdr[3], n_chunks = hdr[4];
  if (B <= 0 || G <= 0 || n_c <= 0 || n_chunks <= 0 || n_chunks > 4096) {
    fprintf(stderr, "bad header\n");
    return 1;
  }
  int64_t* n_in = (int64_t*)malloc(sizeof(int64_t) * (size_t)n_chunks);
  read_exact(in, n_in, sizeof(int64_t) * (size_t)n_chunks);
  int64_t max_n_in = 0;
  for (int64_t c = 0; c < n_chunks; ++c) max_n_in = n_in[c] > max_n_in ? n_in[c] : max_n_in;

  const size_t row = (size_t)d * 2; /* bytes of one bf16 row */
  const size_t kv_bytes = (size_t)B * (size_t)n_c * row;
  void* h_k = pinned_from(in, kv_bytes);
  void* h_v = pinned_from(in, kv_bytes);
  void** h_q = (void**)malloc(sizeof(void*) * (size_t)n_chunks);
  void** h_ks = (void**)malloc(sizeof(void*) * (size_t)n_chunks);
  for (int64_t c = 0; c < n_chunks; ++c) {
    h_q[c] = pinned_from(in, (size_t)B * (size_t)G * (size_t)n_in[c] * row);
    h_ks[c] = pinned_from(in, (size_t)B * (size_t)n_in[c] * row);
  }
  fclose(in);

  cudaStream_t st;
  CUDA_OK(cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking));
  const int64_t N = B * n_c;
  void* d_k = dev_alloc(kv_bytes);
  void* d_v = dev_alloc(kv_bytes);
  void* d_q = dev_alloc((size_t)B * (size_t)G * (size_t)max_n_in * row);
  void* d_ks = dev_alloc((size_t)B * (size_t)max_n_in * row);
  float* d_s = (float*)dev_alloc(sizeof(float) * (size_t)N);
  const size_t sws_bytes = kvzip_score_workspace_size((int)B, (int)G, (int)max_n_in);
  void* d_sws = dev_alloc(sws_bytes);
  CUDA_OK(cudaMemsetAsync(d_s, 0, sizeof(float) * (size_t)N, st));   /* scores start at 0 */
  CUDA_OK(cudaMemsetAsync(d_sws, 0, sws_bytes, st));                 /* status header */

  /* context keys and values up once; then each chunk's queries and self keys */
  CUDA_OK(cudaMemcpyAsync(d_k, h_k, kv_bytes, cudaMemcpyHostToDevice, st));
  CUDA_OK(cudaMemcpyAsync(d_v, h_v, kv_bytes, cudaMemcpyHostToDevice, st));
  for (int64_t c = 0; c < n_chunks; ++c) {
    CUDA_OK(cudaMemcpyAsync(d_q, h_q[c], (size_t)B * (size_t)G * (size_t)n_in[c] * row,
                            cudaMemcpyHostToDevice, st));
    CUDA_OK(cudaMemcpyAsync(d_ks, h_ks[c], (size_t)B * (size_t)n_in[c] * row,
                            cudaMemcpyHostToDevice, st));
    KVZIP_OK_(kvzip_score_chunk(KVZIP_BF16, d_q, d_k, d_ks, d_s, (int)B, (int)G, (int)n_in[c],
                                (int)n_c, (int)d, 0.0f, d_sws, sws_bytes, st));
  }

  /* global top-k selection, then per-head compaction */
  const int64_t k = kvzip_keep_count(r, N);
  uint8_t* d_keep = (uint8_t*)dev_alloc((size_t)N);
  int64_t* d_off = (int64_t*)dev_alloc(sizeof(int64_t) * (size_t)(B + 1));
  float* d_thr = (float*)dev_alloc(sizeof(float));
  const size_t selws_bytes = kvzip_select_workspace_size(N, B);
  void* d_selws = dev_alloc(selws_bytes);
  CUDA_OK(cudaMemsetAsync(d_selws, 0, selws_bytes, st));
  KVZIP_OK_(kvzip_select(d_s, N, k, B, d_keep, d_off, d_thr, d_selws, selws_bytes, st));
  void* d_ko = dev_alloc((size_t)k * row);
  void* d_vo = dev_alloc((size_t)k * row);
  int32_t* d_pos = (int32_t*)dev_alloc(sizeof(int32_t) * (size_t)k);
  const size_t cws_bytes = kvzip_compact_workspace_size(B, (int)n_c);
  void* d_cws = dev_alloc(cws_bytes);
  KVZIP_OK_(kvzip_compact(d_k, d_v, d_keep, d_off, B, (int)n_c, (int)d, d_ko, d_vo, d_pos, d_cws,
                          cws_bytes, st));
  /* the sticky status words of the scoring and selection workspaces */
  KVZIP_OK_(kvzip_workspace_status(d_sws, st));
  KVZIP_OK_(kvzip_workspace_status(d_selws, st));

  /* results back to page-locked host memory */
  float* h_s = NULL;
  int64_t* h_off = NULL;
  void *h_ko = NULL, *h_vo = NULL;
  int32_t* h_pos = NULL;
  CUDA_OK(cudaMallocHost((void**)&h_s, sizeof(float) * (size_t)N));
  CUDA_OK(cudaMallocHost((void**)&h_off, sizeof(int64_t) * (size_t)(B + 1)));
  CUDA_OK(cudaMallocHost(&h_ko, (size_t)k * row + 1));
  CUDA_OK(cudaMallocHost(&h_vo, (size_t)k * row + 1));
  CUDA_OK(cudaMallocHost((void**)&h_pos, sizeof(int32_t) * (size_t)k + 1));
  CUDA_OK(cudaMemcpyAsync(h_s, d_s, sizeof(float) * (size_t)N, cudaMemcpyDeviceToHost, st));
  CUDA_OK(cudaMemcpyAsync(h_off, d_off, sizeof(int64_t) * (size_t)(B + 1), cudaMemcpyDeviceToHost,
                          st));
  CUDA_OK(cudaMemcpyAsync(h_ko, d_ko, (size_t)k * row, cudaMemcpyDeviceToHost, st));
  CUDA_OK(cudaMemcpyAsync(h_vo, d_vo, (size_t)k * row, cudaMemcpyDeviceToHost, st));
  CUDA_OK(cudaMemcpyAsync(h_pos, d_pos, sizeof(int32_t) * (size_t)k, cudaMemcpyDeviceToHost, st));
  CUDA_OK(cudaStreamSynchronize(st));

  FILE* out = fopen(argv[2], "wb");
  if (!out) {
    perror(argv[2]);
    return 1;
  }
  write_exact(out, &k, sizeof k);
  write_exact(out, h_s, sizeof(float) * (size_t)N);
  write_exact(out, h_off, sizeof(int64_t) * (size_t)(B + 1));
  write_exact(out, h_ko, (size_t)k * row);
  write_exact(out, h_vo, (size_t)k * row);
  write_exact(out, h_pos, sizeof(int32_t) * (size_t)k);
  fclose(out);

  void* dev[] = {d_k, d_v, d_q, d_ks, d_s, d_sws, d_keep, d_off, d_thr, d_selws, d_ko, d_vo, d_pos,
                 d_cws};
  for (size_t i = 0; i < sizeof dev / sizeof dev[0]; ++i) CUDA_OK(cudaFree(dev[i]));
  void* host[] = {h_k, h_v, h_s, h_off, h_ko, h_vo, h_pos};
  for (size_t i = 0; i < sizeof host / sizeof host[0]; ++i) CUDA_OK(cudaFreeHost(host[i]));
  for (int64_t c = 0; c < n_chunks; ++c) {
    CUDA_OK(cudaFreeHost(h_q[c]));
    CUDA_OK(cudaFreeHost(h_ks[c]));
  }
  free(h_q);
  free(h_ks);
  free(n_in);
  CUDA_OK(cudaStreamDestroy(st));
  return 0;
}
