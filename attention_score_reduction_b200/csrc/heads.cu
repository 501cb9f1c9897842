// Head-level importance: the largest score of each (layer, head).
//
// The authors compute a context-independent head score as max_i S[:, :, i]
// over the sequence dimension of the L x H x n_c score tensor (OpenReview
// rebuttal, answer on how head-level scores were measured for the
// DuoAttention comparison).  Scores are >= 0, so their IEEE bits order like
// the values and the per-segment maxima combine with an integer atomicMax
// into an output zeroed first (0.0f is a lower bound of every score).
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "kvzip_internal.h"

namespace kvzip {

namespace {

constexpr int kHeadThreads = 256;
constexpr int64_t kHeadSeg = 16384;  // scores per block

__global__ void __launch_bounds__(kHeadThreads)
    head_max_kernel(const float* __restrict__ s, int64_t n_c, int64_t segs, uint32_t* out) {
  const int64_t h = blockIdx.x / segs, sg = blockIdx.x % segs;
  const int64_t j0 = sg * kHeadSeg;
  const int64_t j1 = (j0 + kHeadSeg < n_c) ? j0 + kHeadSeg : n_c;
  const float* base = s + h * n_c;
  uint32_t m = 0;
  for (int64_t j = j0 + threadIdx.x; j < j1; j += kHeadThreads) {
    const uint32_t u = __float_as_uint(__ldcs(base + j));
    m = u > m ? u : m;
  }
  m = __reduce_max_sync(0xffffffffu, m);
  __shared__ uint32_t red[kHeadThreads / 32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t t = 0;
    for (int w = 0; w < kHeadThreads / 32; ++w) t = red[w] > t ? red[w] : t;
    atomicMax(out + h, t);
  }
}

// Token-level scores: tok[j] = max over heads of scores[h][j] (blog post
// section 4.3.3, a position kept or evicted in every head at once).
__global__ void __launch_bounds__(256)
    token_max_kernel(const float* __restrict__ s, int64_t n_heads, int64_t n_c, float* tok) {
  for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < n_c;
       j += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float m = s[j];
    for (int64_t h = 1; h < n_heads; ++h) m = fmaxf(m, s[h * n_c + j]);
    tok[j] = m;
  }
}

// keep[h][j] = keep_pos[j] for every head; offsets[h] = h * (kept positions).
__global__ void __launch_bounds__(256)
    expand_keep_kernel(const uint8_t* __restrict__ keep_pos, const int64_t* __restrict__ pos_off,
                       int64_t n_heads, int64_t n_c, uint8_t* keep, int64_t* offsets) {
  const int64_t total = n_heads * n_c;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t i0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (int64_t i = i0; i < total; i += stride) keep[i] = keep_pos[i % n_c] ? 1 : 0;
  const int64_t kept = pos_off[1] - pos_off[0];
  for (int64_t h = i0; h <= n_heads; h += stride) offsets[h] = h * kept;
}

}  // namespace

cudaError_t launch_token_scores(const float* scores, int64_t n_heads, int64_t n_c, float* tok,
                                cudaStream_t s, int* launches) {
  const int64_t blocks = std::min<int64_t>((n_c + 255) / 256, 148 * 8);
  token_max_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(scores, n_heads, n_c, tok);
  if (launches) *launches += 1;
  return cudaGetLastError();
}

cudaError_t launch_expand_keep(const uint8_t* keep_pos, const int64_t* pos_off, int64_t n_heads,
                               int64_t n_c, uint8_t* keep, int64_t* offsets, cudaStream_t s,
                               int* launches) {
  const int64_t blocks = std::min<int64_t>((n_heads * n_c + 255) / 256, 148 * 8);
  expand_keep_kernel<<<static_cast<unsigned>(std::max<int64_t>(blocks, 1)), 256, 0, s>>>(
      keep_pos, pos_off, n_heads, n_c, keep, offsets);
  if (launches) *launches += 1;
  return cudaGetLastError();
}

cudaError_t launch_head_scores(const float* scores, int64_t n_heads, int64_t n_c, float* out,
                               cudaStream_t s, int* launches) {
  cudaError_t e = cudaMemsetAsync(out, 0, sizeof(float) * n_heads, s);
  if (e != cudaSuccess) return e;
  const int64_t segs = (n_c + kHeadSeg - 1) / kHeadSeg;
  head_max_kernel<<<static_cast<unsigned>(n_heads * segs), kHeadThreads, 0, s>>>(
      scores, n_c, segs, reinterpret_cast<uint32_t*>(out));
  if (launches) *launches += 1;
  return cudaGetLastError();
}

}  // namespace kvzip
