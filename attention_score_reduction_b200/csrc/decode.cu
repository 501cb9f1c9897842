// One decoding step of attention over the compressed, per-head variable-length
// KV cache that kvzip_compact produces.
//
// KVzip's payoff is cheaper decoding: attention reads only the kept KV pairs
// (rebuttal, decoding-efficiency table: latency and cache size fall with the
// kept ratio; scime.ai summary: about 2x lower FlashAttention decoding
// latency).  For KV head h with kept rows [offsets[h], offsets[h+1]) and its
// G query heads: o[h][g] = softmax(scale * K_h q[h][g]) V_h.
//
// The step is HBM-bound (every kept K and V row is read once), so it runs as
// split-K flash decoding: each CTA takes a contiguous slice of one head's rows
// and produces a partial (max, sum, weighted V) per query head; a second kernel
// merges the slices.  Inside a CTA, each warp streams 32-row batches of K and V
// through a ring of shared-memory slots (TMA tiles of 32 rows x 128 bytes with
// the 128-byte swizzle, so that ldmatrix reads eight rows of one column without
// bank conflicts) and forms both products with bf16 mma.sync fragments
// (m16n8k16, fp32 accumulation):
//   logits  S^T = Q K^T      M = query heads (G <= 8 of 16 used), N = 8 rows,
//                            K = 16 head-dim elements; Q stays in registers;
//   output  O^T += V^T P^T   M = 16 head-dim elements, N = query heads,
//                            K = 16 rows; V^T comes from ldmatrix.trans, and
//                            P^T is the logits' accumulator fragment itself,
//                            converted to bf16 as a high and a low part (two
//                            products), so the weights keep about 16 bits.
// With G query heads per row the logits are a G-column product: on the CUDA
// cores the dot products, bf16 unpacking and lane reductions took ~2,000
// instructions per 32-row batch and capped the kernel at ~0.64 of HBM
// bandwidth with issue 68% busy; as fragments they take a few hundred.  The
// tcgen05 path does not fit: its smallest MMA is 64 rows, and G <= 8 query
// heads would fill a few of them.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "kvzip_internal.h"
#include "sm100_ptx.cuh"
#include "tc_common.cuh"

namespace kvzip {

namespace {

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
// d += a * b on one m16n8k16 bf16 fragment, fp32 accumulators
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// two floats as bf16x2 (x in the low half), round to nearest even
__device__ __forceinline__ uint32_t pack_bf16(float x, float y) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(y), "f"(x));
  return r;
}

template <int D>
struct DecCfg {
  // 192 KB of batch slots per CTA (one CTA per SM).  At d = 128, six warps with
  // two slots each ran 5% faster than four with three or three with four: more
  // warps hide the per-batch latencies better than a deeper ring per warp.
  static constexpr int WARPS = (D == 128) ? 6 : 2;
  static constexpr int THREADS = 32 * WARPS;
  static constexpr int NSLOT = (D == 128) ? 2 : 3;     // batches in flight per warp
  static constexpr int BOXES = D / 64;                 // 128-byte column boxes per row
  static constexpr int BOX_BYTES = 32 * 128;           // one TMA tile: 32 rows x 64 elements
  static constexpr int TILE_BYTES = BOXES * BOX_BYTES; // one 32-row K or V batch
  static constexpr int SLOT_BYTES = 2 * TILE_BYTES;    // K then V
  static constexpr int SMEM = WARPS * NSLOT * SLOT_BYTES + 1024;   // + 1024-B alignment
};

// Byte offset of 16-byte column c of row r (0..31) in a swizzled batch tile:
// box c / 8, row r at 128 r, and the chunk index XORed with r mod 8.
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return static_cast<uint32_t>((c >> 3) * (32 * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

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
// the log2 domain, o = sum_j 2^(c s_j - max) v_j.  Warp w of a CTA takes
// batches w, w + WARPS, ... of the CTA's slice; batch n of a warp lands in
// slot n % NSLOT, and the copy of batch n + NSLOT is issued as soon as batch
// n has been read.
template <int D, int G>
__global__ void __launch_bounds__(DecCfg<D>::THREADS)
    decode_partial(const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap, const uint16_t* __restrict__ q,
                   int64_t n_rows, const int64_t* __restrict__ offsets, float c, int S,
                   float2* __restrict__ ml_out, float* __restrict__ o_out, uint32_t* status,
                   uint64_t timeout_ns) {
  using Cfg = DecCfg<D>;
  constexpr int WARPS = Cfg::WARPS;
  constexpr int NSLOT = Cfg::NSLOT;
  constexpr int KS = D / 16;             // k-steps of the logits; m-tiles of the output
  static_assert(G >= 1 && G <= 8, "query heads occupy rows 0..7 of the fragment");
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* dsm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t full[WARPS][NSLOT];
  __shared__ float xm[WARPS][G], xl[WARPS][G];
  __shared__ float xo[WARPS][G][D];
  const int h = blockIdx.y, s = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quad = lane >> 2, qp = lane & 3;   // fragment row group, column pair
  const int64_t base = offsets[h];
  int64_t len = offsets[h + 1] - base;
  // the head's kept rows must lie inside the packed cache; otherwise read none
  // (the debug build also records the failed check)
  const bool range_ok = base >= 0 && len >= 0 && base + len <= n_rows;
  if (!(in_bounds(range_ok) && range_ok)) len = 0;
  const int64_t r0 = base + len * s / S, r1 = base + len * (s + 1) / S;
  uint8_t* wsm = dsm + warp * NSLOT * Cfg::SLOT_BYTES;
  if (lane == 0) {
    for (int i = 0; i < NSLOT; ++i) mbar_init(&full[warp][i], 1);
    fence_mbar_init();
  }
  __syncwarp();

  // Q as the A operand: row = query head `quad` (zero for quad >= G), k = head
  // dimension.  a0 holds k = 16 ks + 2 qp (+1), a2 the same + 8; a1 and a3
  // (heads 8..15) are zero.
  uint32_t qa[KS][2];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    if (quad < G) {
      const uint32_t* qr = reinterpret_cast<const uint32_t*>(
          q + (static_cast<size_t>(h) * G + quad) * D + 16 * ks + 2 * qp);
      qa[ks][0] = qr[0];
      qa[ks][1] = qr[4];
    } else {
      qa[ks][0] = qa[ks][1] = 0u;
    }
  }
  // this lane's softmax state is head `quad`'s; its output accumulators are
  // O^T[16 mt + quad (+8)][2 qp (+1)]
  float m = -INFINITY, l = 0.f;
  float o[KS][4];
#pragma unroll
  for (int mt = 0; mt < KS; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[mt][e] = 0.f;

  const int64_t stride = static_cast<int64_t>(WARPS) * 32;
  const int64_t rb0 = r0 + warp * 32;
  const int nb = (rb0 < r1) ? static_cast<int>((r1 - rb0 + stride - 1) / stride) : 0;
  // copy batch n of this warp into slot n % NSLOT: whole 32-row tiles (rows
  // past n_rows arrive as zeros; rows past the slice are masked below)
  auto issue = [&](int n) {
    if (lane != 0) return;
    const int row = static_cast<int>(rb0 + n * stride);
    uint64_t* bar = &full[warp][n % NSLOT];
    uint8_t* kt_ = wsm + (n % NSLOT) * Cfg::SLOT_BYTES;
    mbar_arrive_expect_tx(bar, Cfg::SLOT_BYTES);
#pragma unroll
    for (int b = 0; b < Cfg::BOXES; ++b) {
      tma_load_3d(kt_ + b * Cfg::BOX_BYTES, &kmap, bar, 64 * b, row, 0);
      tma_load_3d(kt_ + Cfg::TILE_BYTES + b * Cfg::BOX_BYTES, &vmap, bar, 64 * b, row, 0);
    }
  };
#pragma unroll
  for (int n = 0; n < NSLOT; ++n)
    if (n < nb) issue(n);

  bool ok = true;
  int n = 0;
  for (; n < nb; ++n) {
    const int64_t rb = rb0 + n * stride;
    const int nrow = static_cast<int>(r1 - rb < 32 ? r1 - rb : 32);
    uint8_t* kt = wsm + (n % NSLOT) * Cfg::SLOT_BYTES;
    uint8_t* vt = kt + Cfg::TILE_BYTES;
    ok = dec_wait(&full[warp][n % NSLOT], (n / NSLOT) & 1, status, timeout_ns);
    if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
    if (nrow < 32) {
      // the last batch of the slice: rows past its end (other heads' rows)
      // take zeros, since their weight 0 times a non-finite value is NaN
      constexpr int W16 = D / 8;   // 16-byte columns per row
      for (int idx = lane; idx < (32 - nrow) * W16; idx += 32) {
        const int r = nrow + idx / W16, w = idx % W16;
        *reinterpret_cast<uint4*>(kt + swz(r, w)) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(vt + swz(r, w)) = make_uint4(0, 0, 0, 0);
      }
      __syncwarp();
    }
    // ---- logits: S^T[head][row] for rows 8 j + 2 qp (+1), j = 0..3
    float sacc[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[j][e] = 0.f;
    const uint32_t kt_u = smem_u32(kt);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int kk = 0; kk < KS / 2; ++kk) {
        // matrices: rows 8 j .. 8 j + 7, 16-byte columns 4 kk .. 4 kk + 3
        uint32_t b[4];
        ldsm_x4(kt_u + swz(8 * j + (lane & 7), 4 * kk + (lane >> 3)), b);
        mma16816(sacc[j], qa[2 * kk][0], 0u, qa[2 * kk][1], 0u, b[0], b[1]);
        mma16816(sacc[j], qa[2 * kk + 1][0], 0u, qa[2 * kk + 1][1], 0u, b[2], b[3]);
      }
    }
    // ---- online softmax for head `quad` (its 32 logits sit in the 4 lanes of the quad)
    float x[4][2];
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        x[j][e] = (8 * j + 2 * qp + e < nrow) ? sacc[j][e] * c : -INFINITY;
        mx = fmaxf(mx, x[j][e]);
      }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m, mx);   // finite: row 0 of a batch is always real
    const float alpha = exp2f(m - m_new);
    float sum = 0.f;
    uint32_t phi[4], plo[4];   // P^T as B fragments, high and low bf16 parts
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float p0 = exp2f(x[j][0] - m_new), p1 = exp2f(x[j][1] - m_new);
      sum += p0 + p1;
      phi[j] = pack_bf16(p0, p1);
      const float h0 = __uint_as_float(phi[j] << 16), h1 = __uint_as_float(phi[j] & 0xffff0000u);
      plo[j] = pack_bf16(p0 - h0, p1 - h1);
    }
    sum += __shfl_xor_sync(0xffffffffu, sum, 1);
    sum += __shfl_xor_sync(0xffffffffu, sum, 2);
    l = l * alpha + sum;
    m = m_new;
    // rescale the output columns this lane holds: heads 2 qp and 2 qp + 1
    const float a_lo = __shfl_sync(0xffffffffu, alpha, 8 * qp);
    const float a_hi = __shfl_sync(0xffffffffu, alpha, 8 * qp + 4);
#pragma unroll
    for (int mt = 0; mt < KS; ++mt) {
      o[mt][0] *= a_lo;
      o[mt][1] *= a_hi;
      o[mt][2] *= a_lo;
      o[mt][3] *= a_hi;
    }
    // ---- O^T += V^T P^T over the batch's two 16-row k-steps
    const uint32_t vt_u = smem_u32(vt);
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        // matrices (transposed): rows 16 kk + {0, 8} + 0..7, 16-byte columns 2 mt + {0, 1}
        const int mi = lane >> 3;
        uint32_t a[4];
        ldsm_x4_t(vt_u + swz(16 * kk + 8 * (mi >> 1) + (lane & 7), 2 * mt + (mi & 1)), a);
        mma16816(o[mt], a[0], a[1], a[2], a[3], phi[2 * kk], phi[2 * kk + 1]);
        mma16816(o[mt], a[0], a[1], a[2], a[3], plo[2 * kk], plo[2 * kk + 1]);
      }
    }
    __syncwarp();   // every lane is done with the slot
    if (n + NSLOT < nb) issue(n + NSLOT);
  }
  if (!ok && lane == 0) {
    // timed out: let this warp's copies in flight land before the CTA exits
    const uint64_t t0 = globaltimer_ns();
    for (int i = n; i < nb && i < n + NSLOT; ++i)
      while (!mbar_try_wait(&full[warp][i % NSLOT], (i / NSLOT) & 1) &&
             globaltimer_ns() - t0 < 1000000000ull) {
      }
  }
  __syncwarp();
  // ---- merge the warps of this CTA
  if (qp == 0 && quad < G) {
    xm[warp][quad] = m;
    xl[warp][quad] = l;
  }
#pragma unroll
  for (int mt = 0; mt < KS; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int g = 2 * qp + (e & 1), t = 16 * mt + quad + 8 * (e >> 1);
      if (g < G) xo[warp][g][t] = o[mt][e];
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
// Warp 0 forms the split weights 2^(m_s - M) (lanes over splits); then every
// thread sums its output column over the splits, four independent loads at a
// time.
template <int D>
__global__ void __launch_bounds__(D)
    decode_merge(const float2* __restrict__ ml, const float* __restrict__ o, int S, int G,
                 float* __restrict__ out) {
  constexpr int kMaxSplits = 64;
  __shared__ float wgt[kMaxSplits];
  __shared__ float l_all;
  const int h = blockIdx.x, g = blockIdx.y, t = threadIdx.x;
  const size_t slot0 = static_cast<size_t>(h) * S * G + g;   // split s at slot0 + s * G
  if (t < 32) {
    float2 v[2];
    float M = -INFINITY;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int sp = t + 32 * i;
      v[i] = (sp < S) ? ml[slot0 + static_cast<size_t>(sp) * G] : make_float2(-INFINITY, 0.f);
      M = fmaxf(M, v[i].x);
    }
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, w));
    float L = 0.f;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int sp = t + 32 * i;
      const float a = (M == -INFINITY) ? 0.f : exp2f(v[i].x - M);
      if (sp < S) wgt[sp] = a;
      L += v[i].y * a;
    }
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) L += __shfl_xor_sync(0xffffffffu, L, w);
    if (t == 0) l_all = L;
  }
  __syncthreads();
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  int sp = 0;
  for (; sp + 4 <= S; sp += 4) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      acc[i] = fmaf(o[(slot0 + static_cast<size_t>(sp + i) * G) * D + t], wgt[sp + i], acc[i]);
  }
  for (; sp < S; ++sp) acc[0] = fmaf(o[(slot0 + static_cast<size_t>(sp) * G) * D + t], wgt[sp], acc[0]);
  const float O = (acc[0] + acc[1]) + (acc[2] + acc[3]);
  const float L = l_all;
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
  // [n_rows][d] bf16 maps, 32-row x 64-element boxes with the 128-byte
  // swizzle; with nothing kept no map is built and no tile is loaded
  CUtensorMap kmap{}, vmap{};
  if (a.n_rows > 0 && (!make_map(&kmap, a.k, 1, static_cast<int>(a.n_rows), D, 32) ||
                       !make_map(&vmap, a.v, 1, static_cast<int>(a.n_rows), D, 32)))
    return cudaErrorInvalidValue;
  dim3 g1(S, static_cast<unsigned>(a.n_heads));
  decode_partial<D, G><<<g1, Cfg::THREADS, Cfg::SMEM, st>>>(
      kmap, vmap, static_cast<const uint16_t*>(a.q), a.n_rows, a.offsets,
      a.scale * 1.4426950408889634f, S, ml, o, status, a.timeout_ns);
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
