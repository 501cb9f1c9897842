// Two-pass KVzip chunk scorer for fp32 Q / K on the CUDA cores.
//
// Same quantities as the tensor-core scorer (KVzip blog post, sections 4.3.1,
// 4.3.2, 4.5): pass 1 writes the base-2 log-sum-exp of every query row over
// the n_c context keys and its causal self keys; pass 2 takes, for every
// context key, the max over query rows of c*s - lse2 and merges 2^max into
// the running scores.  fp32 inputs are multiplied in fp32 (no bf16/tf32
// rounding of the operands).
//
// Tiling: a CTA holds 32 A rows in shared memory and streams 32-row B tiles;
// warp w owns A rows 4w..4w+3 and lane L owns row L of the B tile, so the
// per-row reductions are warp shuffles.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "kvzip_internal.h"

namespace kvzip {

constexpr int kSimtRows = 32;
constexpr int kSimtThreads = 256;

struct SimtParams {
  const float* q;       // [B][R][d]
  const float* k_ctx;   // [B][n_c][d]
  const float* k_self;  // [B][n_in][d]
  float* scores;
  float* lse2;
  int n_in, n_c, d, R, R_pad;
  float c;
  uint32_t* hist;       // null, or the round-1 histogram of the new scores (pass 2)
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Copy rows [row0, row0+32) of a [rows][d] matrix into sm[32][d+1], zero past `rows`.
__device__ __forceinline__ void load_tile(float* sm, const float* src, int row0, int rows, int d) {
  for (int e = threadIdx.x; e < kSimtRows * d; e += kSimtThreads) {
    const int r = e / d, t = e % d;
    sm[r * (d + 1) + t] = (row0 + r < rows) ? src[static_cast<size_t>(row0 + r) * d + t] : 0.f;
  }
}

__device__ __forceinline__ float dot_row(const float* a, const float* b, int d) {
  float acc0 = 0.f, acc1 = 0.f;
  int t = 0;
  for (; t + 1 < d; t += 2) {
    acc0 = fmaf(a[t], b[t], acc0);
    acc1 = fmaf(a[t + 1], b[t + 1], acc1);
  }
  if (t < d) acc0 = fmaf(a[t], b[t], acc0);
  return acc0 + acc1;
}

__global__ void __launch_bounds__(kSimtThreads)
    simt_lse_kernel(const SimtParams p) {
  extern __shared__ float sm[];
  const int d = p.d;
  float* As = sm;
  float* Bs = sm + kSimtRows * (d + 1);
  const int b = blockIdx.y;
  const int row0 = blockIdx.x * kSimtRows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (row0 >= p.R) {  // padding rows only: keep them out of the pass-2 maximum
    for (int r = threadIdx.x; r < kSimtRows; r += kSimtThreads)
      p.lse2[static_cast<size_t>(b) * p.R_pad + row0 + r] = INFINITY;
    return;
  }
  const float* qb = p.q + static_cast<size_t>(b) * p.R * d;
  load_tile(As, qb, row0, p.R, d);

  float m[4], l[4];
  int irow[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
    irow[r] = (row0 + warp * 4 + r) % p.n_in;
  }
  const int r_last = min(row0 + kSimtRows, p.R) - 1;
  const int i_max = (r_last / p.n_in != row0 / p.n_in) ? p.n_in - 1 : r_last % p.n_in;
  const int n_ctx_t = (p.n_c + kSimtRows - 1) / kSimtRows;
  const int n_t = n_ctx_t + (i_max + kSimtRows) / kSimtRows;
  for (int it = 0; it < n_t; ++it) {
    __syncthreads();
    const bool self = it >= n_ctx_t;
    const int key0 = self ? (it - n_ctx_t) * kSimtRows : it * kSimtRows;
    if (self)
      load_tile(Bs, p.k_self + static_cast<size_t>(b) * p.n_in * d, key0, p.n_in, d);
    else
      load_tile(Bs, p.k_ctx + static_cast<size_t>(b) * p.n_c * d, key0, p.n_c, d);
    __syncthreads();
    const int key = key0 + lane;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      float s = dot_row(As + (warp * 4 + r) * (d + 1), Bs + lane * (d + 1), d) * p.c;
      const bool vis = self ? (key <= irow[r]) : (key < p.n_c);
      s = vis ? s : -INFINITY;
      const float m_new = fmaxf(m[r], warp_max(s));
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float e = warp_sum(exp2f(s - m_use));
      l[r] = l[r] * exp2f(m[r] - m_use) + e;
      m[r] = m_new;
    }
  }
  if (lane < 4) {
    const int row = row0 + warp * 4 + lane;
    float mr = m[0], lr = l[0];
#pragma unroll
    for (int r = 1; r < 4; ++r)
      if (lane == r) {
        mr = m[r];
        lr = l[r];
      }
    if (row < p.R_pad)
      p.lse2[static_cast<size_t>(b) * p.R_pad + row] = (row < p.R) ? mr + log2f(lr) : INFINITY;
  }
}

__global__ void __launch_bounds__(kSimtThreads)
    simt_colmax_kernel(const SimtParams p) {
  extern __shared__ float sm[];
  const int d = p.d;
  float* As = sm;
  float* Bs = sm + kSimtRows * (d + 1);
  const int b = blockIdx.y;
  const int key0 = blockIdx.x * kSimtRows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  load_tile(As, p.k_ctx + static_cast<size_t>(b) * p.n_c * d, key0, p.n_c, d);
  const float* qb = p.q + static_cast<size_t>(b) * p.R * d;
  const float* L = p.lse2 + static_cast<size_t>(b) * p.R_pad;
  float best[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
  const int n_t = (p.R + kSimtRows - 1) / kSimtRows;
  for (int it = 0; it < n_t; ++it) {
    __syncthreads();
    load_tile(Bs, qb, it * kSimtRows, p.R, d);
    __syncthreads();
    const int row = it * kSimtRows + lane;
    const float lse = (row < p.R) ? L[row] : INFINITY;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float s = dot_row(As + (warp * 4 + r) * (d + 1), Bs + lane * (d + 1), d);
      best[r] = fmaxf(best[r], s * p.c - lse);
    }
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) best[r] = warp_max(best[r]);
  if (lane < 4) {
    const int key = key0 + warp * 4 + lane;
    float br = best[0];
#pragma unroll
    for (int r = 1; r < 4; ++r)
      if (lane == r) br = best[r];
    if (key < p.n_c) {
      float* dst = p.scores + static_cast<size_t>(b) * p.n_c + key;
      const float s_new = fmaxf(*dst, exp2f(br));
      *dst = s_new;
      if (p.hist)
        atomicAdd(p.hist + (mag(__float_as_uint(s_new)) >> kScoreHistShift), 1u);
    }
  }
}

cudaError_t launch_score_simt_f32(const ScoreArgs& a, cudaStream_t s, int* launches) {
  SimtParams p;
  p.q = static_cast<const float*>(a.q);
  p.k_ctx = static_cast<const float*>(a.k_ctx);
  p.k_self = static_cast<const float*>(a.k_self);
  p.scores = a.scores;
  p.lse2 = a.lse2;
  p.n_in = a.n_in;
  p.n_c = a.n_c;
  p.d = a.d;
  p.R = a.R;
  p.R_pad = a.R_pad;
  p.c = a.scale * 1.4426950408889634f;
  p.hist = a.score_hist;
  const size_t smem = 2 * kSimtRows * (a.d + 1) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(simt_lse_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(simt_colmax_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  // pass 1 covers every row of the padded lse buffer
  if (a.passes & 1) {
    dim3 g1(a.R_pad / kSimtRows, a.B);
    simt_lse_kernel<<<g1, kSimtThreads, smem, s>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (launches) *launches += 1;
  }
  if (a.passes & 2) {
    dim3 g2((a.n_c + kSimtRows - 1) / kSimtRows, a.B);
    simt_colmax_kernel<<<g2, kSimtThreads, smem, s>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (launches) *launches += 1;
  }
  return cudaSuccess;
}

}  // namespace kvzip
