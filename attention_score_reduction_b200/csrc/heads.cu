// Head-level importance: the largest score of each (layer, head).
//
// The authors compute a context-independent head score as max_i S[:, :, i]
// over the sequence dimension of the L x H x n_c score tensor (OpenReview
// rebuttal, answer on how head-level scores were measured for the
// DuoAttention comparison).  Scores are >= 0, so the bits of |s| (mag: -0.0
// reads as 0.0) order like the values and the per-segment maxima combine with
// an integer atomicMax into an output zeroed first (0.0f is a lower bound of
// every score).
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
    const uint32_t u = mag(__float_as_uint(__ldcs(base + j)));
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

// Vector forms for n_c a multiple of 4 (every row then starts on 16 bytes).
// head_max_v: four 16-byte loads in flight per thread.
__global__ void __launch_bounds__(kHeadThreads)
    head_max_v(const float* __restrict__ s, int64_t n_c, int64_t segs, uint32_t* out) {
  const int64_t h = blockIdx.x / segs, sg = blockIdx.x % segs;
  const int64_t j0 = sg * kHeadSeg;
  const int64_t n4 = (((j0 + kHeadSeg < n_c) ? j0 + kHeadSeg : n_c) - j0) / 4;
  const uint4* b4 = reinterpret_cast<const uint4*>(s + h * n_c + j0);
  uint32_t m = 0;
  for (int64_t i = threadIdx.x; i < n4; i += 4 * kHeadThreads) {
    uint4 u[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)   // zeros never raise a maximum of scores >= 0
      u[q] = (i + q * kHeadThreads < n4) ? __ldcs(b4 + i + q * kHeadThreads) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      m = max(m, max(max(mag(u[q].x), mag(u[q].y)), max(mag(u[q].z), mag(u[q].w))));
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

// token_max_v: block (x, y) takes four positions per thread over a group of
// kTokHeads heads and merges its maxima into tok (zeroed first) with an integer
// atomicMax on the float bits (scores >= 0 order like their bits).
constexpr int kTokHeads = 16;
__global__ void __launch_bounds__(256)
    token_max_v(const float* __restrict__ s, int64_t n_heads, int64_t n_c, uint32_t* tok) {
  const int64_t j4 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (4 * j4 >= n_c) return;
  const int64_t h0 = static_cast<int64_t>(blockIdx.y) * kTokHeads;
  const int64_t h1 = (h0 + kTokHeads < n_heads) ? h0 + kTokHeads : n_heads;
  const uint4* p = reinterpret_cast<const uint4*>(s + h0 * n_c) + j4;
  const int64_t row4 = n_c / 4;
  uint4 m = make_uint4(0, 0, 0, 0);
#pragma unroll 4
  for (int64_t h = h0; h < h1; ++h, p += row4) {
    const uint4 u = __ldcs(p);
    m.x = max(m.x, mag(u.x));
    m.y = max(m.y, mag(u.y));
    m.z = max(m.z, mag(u.z));
    m.w = max(m.w, mag(u.w));
  }
  uint32_t* t = tok + 4 * j4;
  atomicMax(t + 0, m.x);
  atomicMax(t + 1, m.y);
  atomicMax(t + 2, m.z);
  atomicMax(t + 3, m.w);
}

// expand_keep_v: 16 mask bytes per thread (n_c a multiple of 16), the same
// position bytes written for kExpHeads heads; bytes normalised to 0 / 1.
constexpr int kExpHeads = 8;
__global__ void __launch_bounds__(256)
    expand_keep_v(const uint8_t* __restrict__ keep_pos, const int64_t* __restrict__ pos_off,
                  int64_t n_heads, int64_t n_c, uint8_t* keep, int64_t* offsets) {
  const int64_t j16 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (blockIdx.x == 0 && blockIdx.y == 0) {
    const int64_t kept = pos_off[1] - pos_off[0];
    for (int64_t h = threadIdx.x; h <= n_heads; h += blockDim.x) offsets[h] = h * kept;
  }
  if (16 * j16 >= n_c) return;
  uint4 u = reinterpret_cast<const uint4*>(keep_pos)[j16];
  uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int e = 0; e < 4; ++e)   // bit 0 of each byte = OR of that byte's bits
    w[e] = (w[e] | (w[e] >> 1) | (w[e] >> 2) | (w[e] >> 3) | (w[e] >> 4) | (w[e] >> 5) |
            (w[e] >> 6) | (w[e] >> 7)) & 0x01010101u;
  u = make_uint4(w[0], w[1], w[2], w[3]);
  const int64_t h0 = static_cast<int64_t>(blockIdx.y) * kExpHeads;
  const int64_t h1 = (h0 + kExpHeads < n_heads) ? h0 + kExpHeads : n_heads;
  for (int64_t h = h0; h < h1; ++h) __stcs(reinterpret_cast<uint4*>(keep + h * n_c) + j16, u);
}

}  // namespace

cudaError_t launch_token_scores(const float* scores, int64_t n_heads, int64_t n_c, float* tok,
                                cudaStream_t s, int* launches) {
  if (n_c % 4 == 0 && n_heads > 1 && reinterpret_cast<uintptr_t>(scores) % 16 == 0) {
    cudaError_t e = cudaMemsetAsync(tok, 0, sizeof(float) * n_c, s);
    if (e != cudaSuccess) return e;
    const dim3 grid(static_cast<unsigned>((n_c / 4 + 255) / 256),
                    static_cast<unsigned>((n_heads + kTokHeads - 1) / kTokHeads));
    token_max_v<<<grid, 256, 0, s>>>(scores, n_heads, n_c, reinterpret_cast<uint32_t*>(tok));
  } else {
    const int64_t blocks = std::min<int64_t>((n_c + 255) / 256, 148 * 8);
    token_max_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(scores, n_heads, n_c, tok);
  }
  if (launches) *launches += 1;
  return cudaGetLastError();
}

cudaError_t launch_expand_keep(const uint8_t* keep_pos, const int64_t* pos_off, int64_t n_heads,
                               int64_t n_c, uint8_t* keep, int64_t* offsets, cudaStream_t s,
                               int* launches) {
  if (n_c % 16 == 0 && reinterpret_cast<uintptr_t>(keep_pos) % 16 == 0 &&
      reinterpret_cast<uintptr_t>(keep) % 16 == 0) {
    const dim3 grid(static_cast<unsigned>((n_c / 16 + 255) / 256),
                    static_cast<unsigned>((n_heads + kExpHeads - 1) / kExpHeads));
    expand_keep_v<<<grid, 256, 0, s>>>(keep_pos, pos_off, n_heads, n_c, keep, offsets);
  } else {
    const int64_t blocks = std::min<int64_t>((n_heads * n_c + 255) / 256, 148 * 8);
    expand_keep_kernel<<<static_cast<unsigned>(std::max<int64_t>(blocks, 1)), 256, 0, s>>>(
        keep_pos, pos_off, n_heads, n_c, keep, offsets);
  }
  if (launches) *launches += 1;
  return cudaGetLastError();
}

cudaError_t launch_head_scores(const float* scores, int64_t n_heads, int64_t n_c, float* out,
                               cudaStream_t s, int* launches) {
  cudaError_t e = cudaMemsetAsync(out, 0, sizeof(float) * n_heads, s);
  if (e != cudaSuccess) return e;
  const int64_t segs = (n_c + kHeadSeg - 1) / kHeadSeg;
  if (n_c % 4 == 0 && reinterpret_cast<uintptr_t>(scores) % 16 == 0)
    head_max_v<<<static_cast<unsigned>(n_heads * segs), kHeadThreads, 0, s>>>(
        scores, n_c, segs, reinterpret_cast<uint32_t*>(out));
  else
    head_max_kernel<<<static_cast<unsigned>(n_heads * segs), kHeadThreads, 0, s>>>(
        scores, n_c, segs, reinterpret_cast<uint32_t*>(out));
  if (launches) *launches += 1;
  return cudaGetLastError();
}

}  // namespace kvzip
