// One decoding step of attention over the compressed, per-head variable-length
// KV cache that kvzip_compact produces.
//
// KVzip's payoff is cheaper decoding: attention reads only the kept KV pairs
// (rebuttal, decoding-efficiency table: latency and cache size fall with the
// kept ratio; scime.ai summary: about 2x lower FlashAttention decoding
// latency).  For KV head h with kept rows [offsets[h], offsets[h+1]) and its
// G query heads: o[h][g] = softmax(scale * K_h q[h][g]) V_h.
//
// The step is HBM-bound (every kept K and V row is read once), so it runs on
// the CUDA cores as split-K flash decoding: each CTA takes a contiguous slice
// of one head's rows and produces a partial (max, sum, weighted V) per query
// head; a second kernel merges the slices.  Inside a CTA, each warp handles
// 32-row batches:
//   A  lane = 1/32 of the head dimension: coalesced 256-byte row loads; each
//      lane forms partial dot products for 32 rows, and a butterfly
//      transpose-reduce (31 shuffles per query head) leaves lane r holding
//      row r's logit;
//   B  online softmax across the warp (max / sum by shuffles);
//   C  lane = 1/32 of the head dimension again: o += p_row * v_row with the
//      probabilities broadcast from shared memory.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "kvzip_internal.h"
#include "sm100_ptx.cuh"

namespace kvzip {

namespace {

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Butterfly transpose-reduce: v[i] holds this lane's partial for row i (32
// rows); on return lane r's v[0] is the warp-wide sum for row r.
__device__ __forceinline__ float transpose_reduce32(float (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool upper = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float send = upper ? v[i] : v[i + w];
      const float keep = upper ? v[i + w] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
    }
  }
  return v[0];
}

template <int D>
struct DecCfg {
  static constexpr int WARPS = (D == 128) ? 8 : 4;     // one 32-row batch in flight per warp
  static constexpr int THREADS = 32 * WARPS;
  static constexpr int ROW_BYTES = D * 2;
  static constexpr int BATCH_BYTES = 32 * ROW_BYTES;  // one K or V batch
  static constexpr int SMEM = WARPS * 2 * BATCH_BYTES + 1024;
};

// Bounded mbarrier wait; on timeout records the status and returns false.
__device__ __forceinline__ bool dec_wait(uint64_t* bar, uint32_t parity, uint32_t* status,
                                         uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) {
      atomicOr(status, kStatusTimeout);
      return false;
    }
  }
  return true;
}

// grid (S, n_heads); partial results per (head, split, g): ml = (max, sum) in
// the log2 domain, o = sum_j 2^(c s_j - max) v_j.  Each warp streams its
// 32-row batches of K and V into its own shared-memory slots with one bulk
// copy each (a head's kept rows are contiguous): K of the next batch loads
// while this batch's softmax and V phases run, V of the next batch while its
// logits are formed.
template <int D, int G>
__global__ void __launch_bounds__(DecCfg<D>::THREADS)
    decode_partial(const uint16_t* __restrict__ q, const uint16_t* __restrict__ kp,
                   const uint16_t* __restrict__ vp, const int64_t* __restrict__ offsets,
                   float c, int S, float2* __restrict__ ml_out, float* __restrict__ o_out,
                   uint32_t* status, uint64_t timeout_ns) {
  using Cfg = DecCfg<D>;
  constexpr int E = D / 32;              // head-dim elements per lane
  constexpr int WARPS = Cfg::WARPS;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* dsm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t kbar[WARPS], vbar[WARPS];
  __shared__ float p_s[WARPS][32][G];
  __shared__ float xm[WARPS][G], xl[WARPS][G];
  __shared__ float xo[WARPS][G][D];
  const int h = blockIdx.y, s = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t base = offsets[h];
  int64_t len = offsets[h + 1] - base;
  // the head's kept rows must lie inside the packed cache; otherwise read none
  if (!in_bounds(base >= 0 && len >= 0 && base + len <= offsets[gridDim.y])) len = 0;
  const int64_t r0 = base + len * s / S, r1 = base + len * (s + 1) / S;
  uint8_t* ks = dsm + warp * 2 * Cfg::BATCH_BYTES;
  uint8_t* vs = ks + Cfg::BATCH_BYTES;
  if (lane == 0) {
    mbar_init(&kbar[warp], 1);
    mbar_init(&vbar[warp], 1);
    fence_mbar_init();
  }
  __syncwarp();

  // this lane's slice of every query head, pre-scaled by c = scale * log2(e)
  float qv[G][E];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      const uint32_t w = reinterpret_cast<const uint32_t*>(
          q + (static_cast<size_t>(h) * G + g) * D)[(lane * E + e) / 2];
      qv[g][e] = bf16lo(w) * c;
      qv[g][e + 1] = bf16hi(w) * c;
    }
  float m[G], l[G], o[G][E];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) o[g][e] = 0.f;
  }

  auto rows_of = [&](int64_t rb) -> int { return static_cast<int>(r1 - rb < 32 ? r1 - rb : 32); };
  auto issue = [&](uint64_t* bar, uint8_t* dst, const uint16_t* src, int64_t rb) {
    const uint32_t bytes = static_cast<uint32_t>(rows_of(rb)) * Cfg::ROW_BYTES;
    mbar_arrive_expect_tx(bar, bytes);
    bulk_load(dst, src + static_cast<size_t>(rb) * D, bytes, bar);
  };
  const int64_t stride = static_cast<int64_t>(WARPS) * 32;
  int64_t rb = r0 + warp * 32;
  if (lane == 0 && rb < r1) {
    issue(&kbar[warp], ks, kp, rb);
    issue(&vbar[warp], vs, vp, rb);
  }
  bool ok = true;
  uint32_t ph = 0;
  for (; ok && rb < r1; rb += stride, ph ^= 1) {
    const int nrow = rows_of(rb);
    const int64_t nxt = rb + stride;
    // ---- A: logits of this batch's rows (lane r ends up with row r)
    ok = dec_wait(&kbar[warp], ph, status, timeout_ns);
    if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
    float sc[G];
#pragma unroll
    for (int g0 = 0; g0 < G; g0 += 2) {
      constexpr int kPair = 2;
      float part[kPair][32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        float kv[E];
        const uint8_t* row = ks + i * Cfg::ROW_BYTES + lane * E * 2;
        if (E == 4) {
          const uint2 w = *reinterpret_cast<const uint2*>(row);
          kv[0] = bf16lo(w.x); kv[1] = bf16hi(w.x); kv[2] = bf16lo(w.y); kv[3] = bf16hi(w.y);
        } else {
          const uint4 w = *reinterpret_cast<const uint4*>(row);
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) { kv[2 * k] = bf16lo(ws[k]); kv[2 * k + 1] = bf16hi(ws[k]); }
        }
#pragma unroll
        for (int gb = 0; gb < kPair; ++gb) {
          if (g0 + gb < G) {
            float a = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) a = fmaf(qv[g0 + gb][e], kv[e], a);
            part[gb][i] = a;   // rows past nrow hold stale bytes; masked below
          }
        }
      }
#pragma unroll
      for (int gb = 0; gb < kPair; ++gb)
        if (g0 + gb < G) sc[g0 + gb] = transpose_reduce32(part[gb]);
    }
    __syncwarp();
    if (lane == 0 && nxt < r1) issue(&kbar[warp], ks, kp, nxt);   // K slot is free again
    // ---- B: online softmax per query head
    float p[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float scg = (lane < nrow) ? sc[g] : -INFINITY;
      float mx = scg;
#pragma unroll
      for (int w = 16; w >= 1; w >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, w));
      const float m_new = fmaxf(m[g], mx);
      const float pr = exp2f(scg - m_new);
      float sum = pr;
#pragma unroll
      for (int w = 16; w >= 1; w >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, w);
      const float alpha = exp2f(m[g] - m_new);
      l[g] = l[g] * alpha + sum;
#pragma unroll
      for (int e = 0; e < E; ++e) o[g][e] *= alpha;
      m[g] = m_new;
      p[g] = pr;
    }
#pragma unroll
    for (int g = 0; g < G; ++g) p_s[warp][lane][g] = p[g];
    __syncwarp();
    // ---- C: o += p_row * v_row
    ok = dec_wait(&vbar[warp], ph, status, timeout_ns);
    if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
#pragma unroll 8
    for (int i = 0; i < nrow; ++i) {
      float vv[E];
      const uint8_t* row = vs + i * Cfg::ROW_BYTES + lane * E * 2;
      if (E == 4) {
        const uint2 w = *reinterpret_cast<const uint2*>(row);
        vv[0] = bf16lo(w.x); vv[1] = bf16hi(w.x); vv[2] = bf16lo(w.y); vv[3] = bf16hi(w.y);
      } else {
        const uint4 w = *reinterpret_cast<const uint4*>(row);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) { vv[2 * k] = bf16lo(ws[k]); vv[2 * k + 1] = bf16hi(ws[k]); }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float pg = p_s[warp][i][g];
#pragma unroll
        for (int e = 0; e < E; ++e) o[g][e] = fmaf(pg, vv[e], o[g][e]);
      }
    }
    __syncwarp();
    if (lane == 0 && nxt < r1) issue(&vbar[warp], vs, vp, nxt);   // V slot is free again
  }
  if (!ok && lane == 0) {
    // timed out: let this warp's copies in flight land before the CTA exits
    const uint64_t t0 = globaltimer_ns();
    while ((!mbar_try_wait(&kbar[warp], ph) || !mbar_try_wait(&vbar[warp], ph)) &&
           globaltimer_ns() - t0 < 1000000000ull) {
    }
  }
  __syncwarp();
  // ---- merge the warps of this CTA
#pragma unroll
  for (int g = 0; g < G; ++g) {
    if (lane == 0) {
      xm[warp][g] = m[g];
      xl[warp][g] = l[g];
    }
#pragma unroll
    for (int e = 0; e < E; ++e) xo[warp][g][lane * E + e] = o[g][e];
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < G * D; idx += Cfg::THREADS) {
    const int g = idx / D, t = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) M = fmaxf(M, xm[w][g]);
    float L = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < WARPS; ++w) {
        const float a = exp2f(xm[w][g] - M);
        L += xl[w][g] * a;
        O += xo[w][g][t] * a;
      }
    }
    const size_t slot = (static_cast<size_t>(h) * S + s) * G + g;
    o_out[slot * D + t] = O;
    if (t == 0) ml_out[slot] = make_float2(M, L);
  }
}

// out[h][g][:] = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s; zeros for an empty head.
template <int D>
__global__ void __launch_bounds__(D)
    decode_merge(const float2* __restrict__ ml, const float* __restrict__ o, int S, int G,
                 float* __restrict__ out) {
  const int h = blockIdx.x, g = blockIdx.y, t = threadIdx.x;
  float M = -INFINITY;
  for (int s = 0; s < S; ++s) M = fmaxf(M, ml[(static_cast<size_t>(h) * S + s) * G + g].x);
  float L = 0.f, O = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < S; ++s) {
      const size_t slot = (static_cast<size_t>(h) * S + s) * G + g;
      const float a = exp2f(ml[slot].x - M);
      L += ml[slot].y * a;
      O += o[slot * D + t] * a;
    }
  }
  out[(static_cast<size_t>(h) * G + g) * D + t] = (L > 0.f) ? O / L : 0.f;
}

template <int D, int G>
cudaError_t launch_decode_dg(const DecodeArgs& a, cudaStream_t st, int* launches) {
  using Cfg = DecCfg<D>;
  const int S = decode_splits(a.n_heads);
  uint32_t* status = static_cast<uint32_t*>(a.ws);
  float2* ml = reinterpret_cast<float2*>(static_cast<uint8_t*>(a.ws) + kDecodeWsHeader);
  float* o = reinterpret_cast<float*>(static_cast<uint8_t*>(a.ws) + kDecodeWsHeader +
                                      decode_ml_bytes(a.n_heads, a.G));
  cudaError_t e = cudaFuncSetAttribute(decode_partial<D, G>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
  if (e != cudaSuccess) return e;
  dim3 g1(S, static_cast<unsigned>(a.n_heads));
  decode_partial<D, G><<<g1, Cfg::THREADS, Cfg::SMEM, st>>>(
      static_cast<const uint16_t*>(a.q), static_cast<const uint16_t*>(a.k),
      static_cast<const uint16_t*>(a.v), a.offsets, a.scale * 1.4426950408889634f, S, ml, o,
      status, a.timeout_ns);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 g2(static_cast<unsigned>(a.n_heads), G);
  decode_merge<D><<<g2, D, 0, st>>>(ml, o, S, G, a.out);
  if (launches) *launches += 2;
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_decode_d(const DecodeArgs& a, cudaStream_t st, int* launches) {
  switch (a.G) {
    case 1: return launch_decode_dg<D, 1>(a, st, launches);
    case 2: return launch_decode_dg<D, 2>(a, st, launches);
    case 4: return launch_decode_dg<D, 4>(a, st, launches);
    case 5: return launch_decode_dg<D, 5>(a, st, launches);
    case 8: return launch_decode_dg<D, 8>(a, st, launches);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t bounds_flag_decode(unsigned int* out) { return take_bounds_flag(out); }

int decode_splits(int64_t n_heads) {
  // about two CTAs (one per SM at a time) per SM of a 148-SM B200 in total,
  // at most 64 slices per head
  const int64_t s = (296 + n_heads - 1) / n_heads;
  return static_cast<int>(s < 1 ? 1 : (s > 64 ? 64 : s));
}

size_t decode_ml_bytes(int64_t n_heads, int G) {
  const size_t b = static_cast<size_t>(n_heads) * decode_splits(n_heads) * G * sizeof(float2);
  return (b + 255) / 256 * 256;
}

size_t decode_ws_bytes(int64_t n_heads, int G, int d) {
  return kDecodeWsHeader + decode_ml_bytes(n_heads, G) +
         static_cast<size_t>(n_heads) * decode_splits(n_heads) * G * d * sizeof(float);
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s, int* launches) {
  if (a.d == 128) return launch_decode_d<128>(a, s, launches);
  if (a.d == 256) return launch_decode_d<256>(a, s, launches);
  return cudaErrorInvalidValue;
}

}  // namespace kvzip
