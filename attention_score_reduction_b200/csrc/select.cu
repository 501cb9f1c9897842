// Global top-k selection over all (layer, head, position) scores.
//
// KVzip evicts the lowest-scoring KV pairs once per context, ranking all
// L x H x n_c scores together so that head budgets follow the scores (scime.ai
// summary, "Approach" and the "Measured effects" row on non-uniform head
// budgets; rebuttal: S has shape L x H x n_c).  The kept set is the k largest
// scores; equal scores are taken lowest flat index first, so the mask is unique.
//
// Scores are finite and >= 0, so the bit patterns of |s| (mag: -0.0 reads as
// 0.0), read as uint32, sort like the values.  The threshold tau (the k-th
// largest such pattern) is found
// by a three-round radix select on 13 + 10 + 9 bits; every round is one
// histogram pass over HBM plus a one-block pick, all on the stream with no
// host round trip.  A mask pass then writes keep[f] and per-block kept counts;
// a one-block scan turns those into per-head offsets.  When more elements equal
// tau than are still needed, a counting pass and a scan give every block the
// number of equal elements before it, and ties are ranked in flat order.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "kvzip.h"
#include "kvzip_internal.h"

namespace kvzip {

namespace {

constexpr int kSelThreads = 256;
constexpr int kSelSeg = 8192;     // scores per block in the mask / tie passes
constexpr int kHistThreads = 512;
constexpr int kPickThreads = 1024;

struct SelState {
  uint32_t prefix;                // bits of tau fixed so far
  uint32_t tau;                   // final threshold bit pattern
  unsigned long long k_rem;       // rank still sought inside the current prefix class
  unsigned long long count_gt;    // elements strictly above the current prefix class
  unsigned long long n_eq;        // elements equal to tau
  unsigned long long take_eq;     // of those, how many are kept
  uint32_t keep_none;             // k == 0
  uint32_t pad[5];
};

struct SelWs {
  SelState* st;
  uint32_t* hist;     // 2048 + 2048 + 1024 bins
  uint32_t* blk_cnt;  // kept per mask block
  uint32_t* blk_eq;   // equal-to-tau per mask block, scanned in place
};

// Radix rounds of 13 + 10 + 9 bits: bins, shift of the digit, bits fixed before
// the round, histogram offset.  Scores in [0, 1] share few exponents, so the
// first round takes 5 mantissa bits along with sign and exponent to spread
// them over enough shared-memory bins to keep atomic contention low.
__host__ __device__ constexpr int hist_bins(int p) { return p == 0 ? 8192 : (p == 1 ? 1024 : 512); }
__host__ __device__ constexpr int hist_shift(int p) { return p == 0 ? 19 : (p == 1 ? 9 : 0); }
__host__ __device__ constexpr uint32_t hist_mask(int p) {
  return p == 0 ? 0u : (p == 1 ? 0xFFF80000u : 0xFFFFFE00u);
}
__host__ __device__ constexpr int hist_off(int p) { return p == 0 ? 0 : (p == 1 ? 8192 : 9216); }
constexpr int kHistTotal = 9728;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ __forceinline__ int64_t imin64(int64_t a, int64_t b) { return a < b ? a : b; }

int64_t segs_per_head(int64_t n_c) { return (n_c + kSelSeg - 1) / kSelSeg; }

// One block per selection problem (the whole array, or one head for uniform
// budgets): zero its histograms and set its state.
__global__ void sel_init(SelState* st, uint32_t* hist, unsigned long long k, float* threshold) {
  st += blockIdx.x;
  hist += static_cast<size_t>(blockIdx.x) * kHistTotal;
  for (int i = threadIdx.x; i < kHistTotal; i += blockDim.x) hist[i] = 0;
  if (threadIdx.x == 0) {
    if (k == 0 && threshold) *threshold = INFINITY;
    st->prefix = 0;
    st->tau = 0x7F800000u;  // +inf: nothing above it is finite
    st->k_rem = k;
    st->count_gt = 0;
    st->n_eq = 0;
    st->take_eq = 0;
    st->keep_none = (k == 0);
  }
}

// This block's share of one radix round's histogram into shared memory: the
// digit of every score whose higher bits equal `prefix`.
template <int PASS>
__device__ __forceinline__ void hist_count(const float* __restrict__ s, int64_t N, uint32_t prefix,
                                           bool vec, uint32_t* h) {
  constexpr int NB = hist_bins(PASS);
  constexpr int SH = hist_shift(PASS);
  constexpr uint32_t PM = hist_mask(PASS);
  // vector loads need 16-byte aligned problems (N a multiple of 4)
  const int64_t n4 = vec ? N / 4 : 0;
  const uint4* s4 = reinterpret_cast<const uint4*>(s);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  // two independent 16-byte loads in flight per thread
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += 2 * stride) {
    const bool in1 = i + stride < n4;
    const uint4 u0 = __ldcs(s4 + i);
    const uint4 u1 = in1 ? __ldcs(s4 + i + stride) : make_uint4(0, 0, 0, 0);
    const uint32_t w[8] = {mag(u0.x), mag(u0.y), mag(u0.z), mag(u0.w),
                           mag(u1.x), mag(u1.y), mag(u1.z), mag(u1.w)};
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if ((e < 4 || in1) && (w[e] & PM) == prefix) atomicAdd(&h[(w[e] >> SH) & (NB - 1)], 1u);
  }
  for (int64_t i = 4 * n4 + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < N;
       i += stride) {
    const uint32_t w = mag(__float_as_uint(s[i]));
    if ((w & PM) == prefix) atomicAdd(&h[(w >> SH) & (NB - 1)], 1u);
  }
}

// blockIdx.y selects the problem: elements [y * N, (y + 1) * N).
template <int PASS>
__global__ void __launch_bounds__(kHistThreads)
    sel_hist(const float* __restrict__ s, int64_t N, const SelState* st, uint32_t* hist) {
  constexpr int NB = hist_bins(PASS);
  __shared__ uint32_t h[NB];
  s += static_cast<size_t>(blockIdx.y) * N;
  st += blockIdx.y;
  hist += static_cast<size_t>(blockIdx.y) * kHistTotal;
  for (int i = threadIdx.x; i < NB; i += blockDim.x) h[i] = 0;
  __syncthreads();
  hist_count<PASS>(s, N, st->prefix, gridDim.y == 1 || N % 4 == 0, h);
  __syncthreads();
  for (int i = threadIdx.x; i < NB; i += blockDim.x)
    if (h[i]) atomicAdd(&hist[hist_off(PASS) + i], h[i]);
}

// Inclusive scan of one value per thread across a block of kPickThreads.
__device__ unsigned long long block_incl_scan(unsigned long long v, unsigned long long* sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) sm[warp] = v;
  __syncthreads();
  if (warp == 0) {
    unsigned long long w = (lane < static_cast<int>(blockDim.x >> 5)) ? sm[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    sm[lane] = w;
  }
  __syncthreads();
  const unsigned long long add = warp ? sm[warp - 1] : 0;
  __syncthreads();
  return v + add;
}

// Find the bin (counting from the top) of histogram h (NB bins of round PASS)
// that holds the k_rem-th largest element, and narrow the state to it.
template <int PASS, typename CountT>
__device__ void pick_impl(SelState* st, const CountT* h, float* threshold) {
  constexpr int NB = hist_bins(PASS);
  constexpr int PER = (NB + kPickThreads - 1) / kPickThreads;  // 8, 1 or 1 bins per thread
  __shared__ unsigned long long sm[32];
  __shared__ int found_bin;
  __shared__ unsigned long long found_above;
  if (st->keep_none) return;
  // thread t owns bins NB-1-PER*t ... NB-PER*(t+1) (descending)
  unsigned long long mine = 0;
  unsigned long long cnt[PER];
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int bin = NB - 1 - (PER * static_cast<int>(threadIdx.x) + j);
    cnt[j] = bin >= 0 ? static_cast<unsigned long long>(h[bin]) : 0ull;
    mine += cnt[j];
  }
  const unsigned long long incl = block_incl_scan(mine, sm);
  const unsigned long long excl = incl - mine;
  const unsigned long long k_rem = st->k_rem;
  if (threadIdx.x == 0) found_bin = -1;
  __syncthreads();
  if (excl < k_rem && k_rem <= incl) {
    unsigned long long above = excl;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      if (above + cnt[j] >= k_rem) {
        found_bin = NB - 1 - (PER * threadIdx.x + j);
        found_above = above;
        break;
      }
      above += cnt[j];
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && found_bin >= 0) {
    const uint32_t bin = static_cast<uint32_t>(found_bin);
    st->prefix |= bin << hist_shift(PASS);
    st->count_gt += found_above;
    st->k_rem = k_rem - found_above;
    if (PASS == 2) {
      st->tau = st->prefix;
      st->n_eq = static_cast<unsigned long long>(h[bin]);
      st->take_eq = st->k_rem;
      if (threshold) *threshold = __uint_as_float(st->prefix);
    }
  }
}

template <int PASS>
__global__ void __launch_bounds__(kPickThreads)
    sel_pick(SelState* st, const uint32_t* hist, float* threshold) {
  // one block per selection problem
  pick_impl<PASS>(st + blockIdx.x, hist + static_cast<size_t>(blockIdx.x) * kHistTotal +
                                        hist_off(PASS), threshold);
}

__device__ __forceinline__ uint32_t warp_excl_prefix(bool flag, uint32_t* total) {
  const uint32_t m = __ballot_sync(0xffffffffu, flag);
  *total = __popc(m);
  return __popc(m & ((1u << (threadIdx.x & 31)) - 1u));
}

// Count scores equal to tau per mask block (only when ties must be ranked).
__global__ void __launch_bounds__(kSelThreads)
    sel_eqcount(const float* __restrict__ s, int64_t n_c, int64_t segs, const SelState* st,
                uint32_t* blk_eq, int per_head) {
  const int64_t blk = blockIdx.x;
  const int64_t h = blk / segs, sg = blk % segs;
  if (per_head) st += h;
  if (st->keep_none || st->take_eq == st->n_eq) return;
  const int64_t j0 = sg * kSelSeg, j1 = imin64(j0 + kSelSeg, n_c);
  const float* base = s + h * n_c;
  const uint32_t tau = st->tau;
  uint32_t c = 0;
  for (int64_t j = j0 + threadIdx.x; j < j1; j += kSelThreads)
    c += (mag(__float_as_uint(base[j])) == tau);
  __shared__ uint32_t red[kSelThreads / 32];
  c = __reduce_add_sync(0xffffffffu, c);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t t = 0;
    for (int w = 0; w < kSelThreads / 32; ++w) t += red[w];
    blk_eq[blk] = t;
  }
}

// Vector forms of the two passes below for n_c a multiple of 4: each thread
// reads four consecutive scores with one 16-byte load (two loads in flight)
// and writes their four mask bytes with one 4-byte store.
__global__ void __launch_bounds__(kSelThreads)
    sel_eqcount_v(const float* __restrict__ s, int64_t n_c, int64_t segs, const SelState* st,
                  uint32_t* blk_eq, int per_head) {
  const int64_t blk = blockIdx.x;
  const int64_t h = blk / segs, sg = blk % segs;
  if (per_head) st += h;
  if (st->keep_none || st->take_eq == st->n_eq) return;
  const int64_t j0 = sg * kSelSeg, n4 = (imin64(j0 + kSelSeg, n_c) - j0) / 4;
  const uint4* b4 = reinterpret_cast<const uint4*>(s + h * n_c + j0);
  const uint32_t tau = st->tau;
  uint32_t c = 0;
  for (int64_t i = threadIdx.x; i < n4; i += 2 * kSelThreads) {
    const bool in1 = i + kSelThreads < n4;
    const uint4 u0 = __ldcs(b4 + i);
    const uint4 u1 = in1 ? __ldcs(b4 + i + kSelThreads) : make_uint4(0, 0, 0, 0);
    c += (mag(u0.x) == tau) + (mag(u0.y) == tau) + (mag(u0.z) == tau) + (mag(u0.w) == tau);
    if (in1)
      c += (mag(u1.x) == tau) + (mag(u1.y) == tau) + (mag(u1.z) == tau) + (mag(u1.w) == tau);
  }
  __shared__ uint32_t red[kSelThreads / 32];
  c = __reduce_add_sync(0xffffffffu, c);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t t = 0;
    for (int w = 0; w < kSelThreads / 32; ++w) t += red[w];
    blk_eq[blk] = t;
  }
}

__device__ __forceinline__ uint32_t mask4(uint4 u, uint32_t tau, bool eq_keeps) {
  const uint32_t w[4] = {mag(u.x), mag(u.y), mag(u.z), mag(u.w)};
  uint32_t m = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e)
    m |= static_cast<uint32_t>(w[e] > tau || (eq_keeps && w[e] == tau)) << (8 * e);
  return m;
}

__global__ void __launch_bounds__(kSelThreads)
    sel_mask_v(const float* __restrict__ s, int64_t n_c, int64_t segs, const SelState* st,
               const uint32_t* blk_eq_base, uint8_t* keep, uint32_t* blk_cnt, int per_head) {
  const int64_t blk = blockIdx.x;
  const int64_t h = blk / segs, sg = blk % segs;
  if (per_head) st += h;
  const int64_t j0 = sg * kSelSeg, n4 = (imin64(j0 + kSelSeg, n_c) - j0) / 4;
  const uint4* b4 = reinterpret_cast<const uint4*>(s + h * n_c + j0);
  uint32_t* k4 = reinterpret_cast<uint32_t*>(keep + h * n_c + j0);
  const bool none = st->keep_none != 0;
  const uint32_t tau = st->tau;
  const bool rank_ties = !none && st->take_eq != st->n_eq;
  const unsigned long long take_eq = st->take_eq;
  __shared__ uint32_t wsum[kSelThreads / 32];
  __shared__ uint32_t red[kSelThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t kept = 0;
  // mask words of this block stay inside head h's n_c bytes
  if (!in_bounds(j0 + 4 * n4 <= n_c)) return;
  if (none) {
    for (int64_t i = threadIdx.x; i < n4; i += kSelThreads) k4[i] = 0u;
  } else if (!rank_ties) {   // every score >= tau is kept
    for (int64_t i = threadIdx.x; i < n4; i += 2 * kSelThreads) {
      const bool in1 = i + kSelThreads < n4;
      const uint4 u0 = __ldcs(b4 + i);
      const uint4 u1 = in1 ? __ldcs(b4 + i + kSelThreads) : make_uint4(0, 0, 0, 0);
      const uint32_t m0 = mask4(u0, tau, true), m1 = in1 ? mask4(u1, tau, true) : 0u;
      k4[i] = m0;
      if (in1) k4[i + kSelThreads] = m1;
      kept += __popc(m0) + __popc(m1);   // one set bit per kept byte
    }
  } else {                   // rank the scores equal to tau in flat order
    unsigned long long tie_before = blk_eq_base[blk];
    for (int64_t ib = 0; ib < n4; ib += kSelThreads) {
      const int64_t i = ib + threadIdx.x;
      const bool in = i < n4;
      const uint4 u = in ? __ldcs(b4 + i) : make_uint4(0, 0, 0, 0);
      const uint32_t w[4] = {mag(u.x), mag(u.y), mag(u.z), mag(u.w)};
      uint32_t c_eq = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) c_eq += (in && w[e] == tau);
      uint32_t incl = c_eq;   // inclusive scan over the warp's lanes (flat order)
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      if (lane == 31) wsum[warp] = incl;
      __syncthreads();
      uint32_t before = 0, total = 0;
      for (int ww = 0; ww < kSelThreads / 32; ++ww) {
        before += (ww < warp) ? wsum[ww] : 0;
        total += wsum[ww];
      }
      unsigned long long rank = tie_before + before + incl - c_eq;
      uint32_t m = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool eq = in && w[e] == tau;
        const bool k = (in && w[e] > tau) || (eq && rank < take_eq);
        rank += eq;
        m |= static_cast<uint32_t>(k) << (8 * e);
      }
      if (in) k4[i] = m;
      kept += __popc(m);
      tie_before += total;
      __syncthreads();
    }
  }
  kept = __reduce_add_sync(0xffffffffu, kept);
  if (lane == 0) red[warp] = kept;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t t = 0;
    for (int ww = 0; ww < kSelThreads / 32; ++ww) t += red[ww];
    blk_cnt[blk] = t;
  }
}

// Exclusive scan of per-block values, in place, one block.
__global__ void __launch_bounds__(kPickThreads)
    sel_scan_blocks(uint32_t* v, int64_t n, const SelState* st, int only_if_ties) {
  // one block per selection problem: values [x * n, (x + 1) * n)
  v += static_cast<size_t>(blockIdx.x) * n;
  st += blockIdx.x;
  if (only_if_ties && (st->keep_none || st->take_eq == st->n_eq)) return;
  __shared__ unsigned long long sm[32];
  __shared__ unsigned long long carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int64_t base = 0; base < n; base += kPickThreads) {
    const int64_t i = base + threadIdx.x;
    const unsigned long long x = (i < n) ? v[i] : 0;
    const unsigned long long incl = block_incl_scan(x, sm);
    const unsigned long long c0 = carry;
    if (i < n) v[i] = static_cast<uint32_t>(c0 + incl - x);
    __syncthreads();
    if (threadIdx.x == kPickThreads - 1) carry = c0 + incl;
    __syncthreads();
  }
}

// keep[f] and kept count per block.
__global__ void __launch_bounds__(kSelThreads)
    sel_mask(const float* __restrict__ s, int64_t n_c, int64_t segs, const SelState* st,
             const uint32_t* blk_eq_base, uint8_t* keep, uint32_t* blk_cnt, int per_head) {
  const int64_t blk = blockIdx.x;
  const int64_t h = blk / segs, sg = blk % segs;
  if (per_head) st += h;
  const int64_t j0 = sg * kSelSeg, j1 = imin64(j0 + kSelSeg, n_c);
  const float* base = s + h * n_c;
  uint8_t* kb = keep + h * n_c;
  const bool none = st->keep_none != 0;
  const uint32_t tau = st->tau;
  const bool rank_ties = !none && st->take_eq != st->n_eq;
  const unsigned long long take_eq = st->take_eq;
  __shared__ uint32_t wsum[kSelThreads / 32];
  __shared__ uint32_t red[kSelThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned long long tie_before = rank_ties ? blk_eq_base[blk] : 0;
  uint32_t kept = 0;
  for (int64_t jb = j0; jb < j1; jb += kSelThreads) {
    const int64_t j = jb + threadIdx.x;
    const bool in = j < j1;
    const uint32_t u = in ? mag(__float_as_uint(base[j])) : 0u;
    bool k = in && !none && u > tau;
    const bool eq = in && !none && u == tau;
    if (!rank_ties) {
      k = k || eq;
    } else {
      // rank of this tie among all ties in flat order
      uint32_t wt;
      const uint32_t pre = warp_excl_prefix(eq, &wt);
      if (lane == 0) wsum[warp] = wt;
      __syncthreads();
      uint32_t before = 0, total = 0;
      for (int w = 0; w < kSelThreads / 32; ++w) {
        before += (w < warp) ? wsum[w] : 0;
        total += wsum[w];
      }
      k = k || (eq && tie_before + before + pre < take_eq);
      tie_before += total;
      __syncthreads();
    }
    if (in && in_bounds(j < n_c)) kb[j] = k ? 1 : 0;
    kept += k;
  }
  kept = __reduce_add_sync(0xffffffffu, kept);
  if (lane == 0) red[warp] = kept;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t t = 0;
    for (int w = 0; w < kSelThreads / 32; ++w) t += red[w];
    blk_cnt[blk] = t;
  }
}

// offsets[h] = kept in heads < h, from per-block counts (one block).
__global__ void __launch_bounds__(kPickThreads)
    sel_offsets(const uint32_t* blk_cnt, int64_t n_heads, int64_t segs, int64_t* offsets) {
  __shared__ unsigned long long sm[32];
  __shared__ unsigned long long carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int64_t base = 0; base < n_heads; base += kPickThreads) {
    const int64_t h = base + threadIdx.x;
    unsigned long long c = 0;
    if (h < n_heads)
      for (int64_t sg = 0; sg < segs; ++sg) c += blk_cnt[h * segs + sg];
    const unsigned long long incl = block_incl_scan(c, sm);
    const unsigned long long c0 = carry;
    if (h < n_heads) offsets[h] = static_cast<int64_t>(c0 + incl - c);
    __syncthreads();
    if (threadIdx.x == kPickThreads - 1) carry = c0 + incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) offsets[n_heads] = static_cast<int64_t>(carry);
}

SelWs carve(void* ws, int64_t nblk) {
  uint8_t* p = static_cast<uint8_t*>(ws);
  SelWs w;
  w.st = reinterpret_cast<SelState*>(p);
  p += 256;
  w.hist = reinterpret_cast<uint32_t*>(p);
  p += align_up(kHistTotal * 4, 256);
  w.blk_cnt = reinterpret_cast<uint32_t*>(p);
  p += align_up(static_cast<size_t>(nblk) * 4, 256);
  w.blk_eq = reinterpret_cast<uint32_t*>(p);
  return w;
}

}  // namespace

size_t select_multipass_ws_bytes(int64_t N, int64_t n_heads) {
  const int64_t n_c = n_heads > 0 ? N / n_heads : 0;
  const int64_t nblk = n_heads * segs_per_head(n_c);
  return 256 + align_up(kHistTotal * 4, 256) + 2 * align_up(static_cast<size_t>(nblk) * 4, 256);
}

// The vector passes need every head's scores on 16 bytes and its mask bytes on 4.
static bool use_vec(const SelectArgs& a) {
  return a.n_c % 4 == 0 && reinterpret_cast<uintptr_t>(a.scores) % 16 == 0 &&
         reinterpret_cast<uintptr_t>(a.keep) % 4 == 0;
}

cudaError_t launch_select_multipass(const SelectArgs& a, cudaStream_t s, int* launches) {
  const bool vec = use_vec(a);
  const int64_t segs = segs_per_head(a.n_c);
  const int64_t nblk = a.n_heads * segs;
  SelWs w = carve(a.ws, nblk);
  int n = 0;
  sel_init<<<1, 1024, 0, s>>>(w.st, w.hist, static_cast<unsigned long long>(a.k), a.threshold);
  ++n;
  if (a.k > 0) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (a.N / 4 + kHistThreads - 1) / kHistThreads;
    const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(want, 4LL * sms)));
    sel_hist<0><<<grid, kHistThreads, 0, s>>>(a.scores, a.N, w.st, w.hist);
    sel_pick<0><<<1, kPickThreads, 0, s>>>(w.st, w.hist, a.threshold);
    sel_hist<1><<<grid, kHistThreads, 0, s>>>(a.scores, a.N, w.st, w.hist);
    sel_pick<1><<<1, kPickThreads, 0, s>>>(w.st, w.hist, a.threshold);
    sel_hist<2><<<grid, kHistThreads, 0, s>>>(a.scores, a.N, w.st, w.hist);
    sel_pick<2><<<1, kPickThreads, 0, s>>>(w.st, w.hist, a.threshold);
    if (vec)
      sel_eqcount_v<<<static_cast<unsigned>(nblk), kSelThreads, 0, s>>>(a.scores, a.n_c, segs,
                                                                       w.st, w.blk_eq, 0);
    else
      sel_eqcount<<<static_cast<unsigned>(nblk), kSelThreads, 0, s>>>(a.scores, a.n_c, segs,
                                                                     w.st, w.blk_eq, 0);
    sel_scan_blocks<<<1, kPickThreads, 0, s>>>(w.blk_eq, nblk, w.st, 1);
    n += 8;
  }
  if (vec)
    sel_mask_v<<<static_cast<unsigned>(nblk), kSelThreads, 0, s>>>(a.scores, a.n_c, segs, w.st,
                                                                  w.blk_eq, a.keep, w.blk_cnt, 0);
  else
    sel_mask<<<static_cast<unsigned>(nblk), kSelThreads, 0, s>>>(a.scores, a.n_c, segs, w.st,
                                                                w.blk_eq, a.keep, w.blk_cnt, 0);
  sel_offsets<<<1, kPickThreads, 0, s>>>(w.blk_cnt, a.n_heads, segs, a.offsets);
  n += 2;
  if (launches) *launches += n;
  return cudaGetLastError();
}

// No scores at all: every head keeps nothing and the threshold is +inf.  One
// block writes the outputs so that the call stays asynchronous.
__global__ void sel_empty(int64_t* offsets, int64_t n_heads, float* threshold) {
  for (int64_t i = threadIdx.x; i <= n_heads; i += blockDim.x) offsets[i] = 0;
  if (threadIdx.x == 0 && threshold) *threshold = INFINITY;
}

cudaError_t launch_select_empty(int64_t* offsets, int64_t n_heads, float* threshold,
                                cudaStream_t s, int* launches) {
  sel_empty<<<1, 256, 0, s>>>(offsets, n_heads, threshold);
  if (launches) *launches += 1;
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Sharded selection: one context's heads split across ranks (one process per
// GPU).  Each rank holds a contiguous run of heads, in rank order, so the flat
// order of the whole context is rank order, then local order.  The radix
// rounds need the histogram of all ranks: each rank counts its own scores into
// 64-bit bins, the caller sums the bins over ranks (an all-reduce) and every
// rank picks the same bin from the sum.  After the last round every rank knows
// tau and how many scores equal to tau are kept; the caller gathers each
// rank's count of scores equal to tau, and a rank keeps its ties whose global
// flat-order rank (ties on earlier ranks, then its own in flat order) is below
// that number.

namespace {

template <int PASS>
__global__ void __launch_bounds__(kHistThreads)
    shard_hist(const float* __restrict__ s, int64_t N, const SelState* st,
               unsigned long long* out) {
  constexpr int NB = hist_bins(PASS);
  __shared__ uint32_t h[NB];
  for (int i = threadIdx.x; i < NB; i += blockDim.x) h[i] = 0;
  __syncthreads();
  const bool vec = reinterpret_cast<uintptr_t>(s) % 16 == 0;   // 16-byte loads when aligned
  if (!st->keep_none) hist_count<PASS>(s, N, st->prefix, vec, h);
  __syncthreads();
  for (int i = threadIdx.x; i < NB; i += blockDim.x)
    if (h[i]) atomicAdd(out + i, static_cast<unsigned long long>(h[i]));
}

template <int PASS>
__global__ void __launch_bounds__(kPickThreads)
    shard_pick(SelState* st, const long long* hist, float* threshold) {
  pick_impl<PASS>(st, hist, threshold);
}

// Scores equal to tau on this rank.
__global__ void __launch_bounds__(kSelThreads)
    shard_ties(const float* __restrict__ s, int64_t N, const SelState* st,
               unsigned long long* n_ties) {
  if (st->keep_none) return;
  const uint32_t tau = st->tau;
  uint32_t c = 0;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < N;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    c += (mag(__float_as_uint(s[i])) == tau);
  c = __reduce_add_sync(0xffffffffu, c);
  if ((threadIdx.x & 31) == 0 && c) atomicAdd(n_ties, static_cast<unsigned long long>(c));
}

// Turn the global tie quota into this rank's: ties on earlier ranks come first.
__global__ void shard_localize(SelState* st, const long long* tie_counts, int rank) {
  if (threadIdx.x != 0 || st->keep_none) return;
  unsigned long long before = 0;
  for (int r = 0; r < rank; ++r) before += static_cast<unsigned long long>(tie_counts[r]);
  const unsigned long long mine = static_cast<unsigned long long>(tie_counts[rank]);
  const unsigned long long quota = st->take_eq;
  const unsigned long long left = quota > before ? quota - before : 0ull;
  st->n_eq = mine;
  st->take_eq = left < mine ? left : mine;
}

int hist_grid(int64_t N) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (N / 4 + kHistThreads - 1) / kHistThreads;
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(want, 4LL * sms)));
}

}  // namespace

cudaError_t bounds_flag_select(unsigned int* out) { return take_bounds_flag(out); }

int shard_bins(int round) { return (round >= 0 && round <= 2) ? hist_bins(round) : 0; }

cudaError_t launch_shard_begin(void* ws, int64_t k, cudaStream_t s, int* launches) {
  SelWs w = carve(ws, 0);
  sel_init<<<1, 1024, 0, s>>>(w.st, w.hist, static_cast<unsigned long long>(k), nullptr);
  if (launches) *launches += 1;
  return cudaGetLastError();
}

cudaError_t launch_shard_hist(const float* scores, int64_t N, int round, long long* hist,
                              void* ws, cudaStream_t s, int* launches) {
  SelWs w = carve(ws, 0);
  cudaError_t e = cudaMemsetAsync(hist, 0, sizeof(long long) * hist_bins(round), s);
  if (e != cudaSuccess) return e;
  const int grid = hist_grid(N);
  auto* out = reinterpret_cast<unsigned long long*>(hist);
  if (round == 0) shard_hist<0><<<grid, kHistThreads, 0, s>>>(scores, N, w.st, out);
  if (round == 1) shard_hist<1><<<grid, kHistThreads, 0, s>>>(scores, N, w.st, out);
  if (round == 2) shard_hist<2><<<grid, kHistThreads, 0, s>>>(scores, N, w.st, out);
  if (launches) *launches += 1;
  return cudaGetLastError();
}

cudaError_t launch_shard_pick(const long long* hist, int round, float* threshold, void* ws,
                              cudaStream_t s, int* launches) {
  SelWs w = carve(ws, 0);
  if (round == 0) shard_pick<0><<<1, kPickThreads, 0, s>>>(w.st, hist, threshold);
  if (round == 1) shard_pick<1><<<1, kPickThreads, 0, s>>>(w.st, hist, threshold);
  if (round == 2) shard_pick<2><<<1, kPickThreads, 0, s>>>(w.st, hist, threshold);
  if (launches) *launches += 1;
  return cudaGetLastError();
}

cudaError_t launch_shard_ties(const float* scores, int64_t N, long long* n_ties, void* ws,
                              cudaStream_t s, int* launches) {
  SelWs w = carve(ws, 0);
  cudaError_t e = cudaMemsetAsync(n_ties, 0, sizeof(long long), s);
  if (e != cudaSuccess) return e;
  const int grid = hist_grid(N);
  shard_ties<<<grid, kSelThreads, 0, s>>>(scores, N, w.st,
                                          reinterpret_cast<unsigned long long*>(n_ties));
  if (launches) *launches += 1;
  return cudaGetLastError();
}

cudaError_t launch_shard_mask(const SelectArgs& a, const long long* tie_counts, int rank,
                              cudaStream_t s, int* launches) {
  const bool vec = use_vec(a);
  const int64_t segs = segs_per_head(a.n_c);
  const int64_t nblk = a.n_heads * segs;
  SelWs w = carve(a.ws, nblk);
  shard_localize<<<1, 32, 0, s>>>(w.st, tie_counts, rank);
  if (vec)
    sel_eqcount_v<<<static_cast<unsigned>(nblk), kSelThreads, 0, s>>>(a.scores, a.n_c, segs,
                                                                     w.st, w.blk_eq, 0);
  else
    sel_eqcount<<<static_cast<unsigned>(nblk), kSelThreads, 0, s>>>(a.scores, a.n_c, segs, w.st,
                                                                   w.blk_eq, 0);
  sel_scan_blocks<<<1, kPickThreads, 0, s>>>(w.blk_eq, nblk, w.st, 1);
  if (vec)
    sel_mask_v<<<static_cast<unsigned>(nblk), kSelThreads, 0, s>>>(a.scores, a.n_c, segs, w.st,
                                                                  w.blk_eq, a.keep, w.blk_cnt, 0);
  else
    sel_mask<<<static_cast<unsigned>(nblk), kSelThreads, 0, s>>>(a.scores, a.n_c, segs, w.st,
                                                                w.blk_eq, a.keep, w.blk_cnt, 0);
  sel_offsets<<<1, kPickThreads, 0, s>>>(w.blk_cnt, a.n_heads, segs, a.offsets);
  if (launches) *launches += 5;
  return cudaGetLastError();
}

}  // namespace kvzip

// ---------------------------------------------------------------------------
// Allocation-free selection: kvzip_select_noalloc.
//
// Some callers cannot hand the library a workspace: code that runs inside a
// host process whose device memory is owned by someone else's pool (a plugin
// in a serving engine that has reserved the GPU's memory up front), or a
// latency-critical loop that may not call cudaMalloc because it can block and
// synchronise the device.  For them the selection scratch lives in this
// file-scope array instead; every GPU that loads the library holds it until
// the process exits.  Its contents survive between calls: the selection
// kernels re-initialise the state and histograms at the start of every call,
// and every per-block count is written before it is read.  All calls on one
// device share the array, so calls that overlap on the GPU (different
// streams, no ordering) race and give wrong masks.
namespace kvzip {
namespace {

constexpr size_t kSelectStaticBytes = size_t{1} << 20;  // 1 MiB
__device__ __align__(256) uint8_t g_select_scratch[kSelectStaticBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_select_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up with
// that device current.  Outside stream capture it is looked up on every call
// (cheap), so a context torn down and re-created (cudaDeviceReset) gets its new
// address; while `stream` is capturing, the address cached by an earlier call
// on this device is used, because the lookup may have to load the module.
cudaError_t static_scratch(cudaStream_t stream, void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(stream, &cap);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_select_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  } else if (!g_scratch_ptr[dev]) {
    return cudaErrorStreamCaptureUnsupported;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace kvzip

extern "C" kvzip_status kvzip_select_noalloc(const float* scores, int64_t N, int64_t k,
                                             int64_t n_heads, uint8_t* keep, int64_t* offsets,
                                             float* threshold, void* stream) {
  if (N <= 0 || n_heads <= 0 || k < 0 || k > N) return KVZIP_ERR_INVALID_ARG;
  if (N % n_heads != 0 || N >= (int64_t{1} << 31)) return KVZIP_ERR_INVALID_ARG;
  if (!scores || !keep || !offsets) return KVZIP_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(scores) & 15) || (reinterpret_cast<uintptr_t>(offsets) & 7) ||
      (threshold && (reinterpret_cast<uintptr_t>(threshold) & 3)))
    return KVZIP_ERR_INVALID_ARG;
  // Larger problems need more scratch than the static array holds.
  if (kvzip::select_multipass_ws_bytes(N, n_heads) > kvzip::kSelectStaticBytes)
    return KVZIP_ERR_UNSUPPORTED;
  void* ws = nullptr;
  if (kvzip::static_scratch(static_cast<cudaStream_t>(stream), &ws) != cudaSuccess)
    return KVZIP_ERR_CUDA;
  kvzip::SelectArgs a;
  a.scores = scores;
  a.N = N;
  a.k = k;
  a.n_heads = n_heads;
  a.n_c = N / n_heads;
  a.keep = keep;
  a.offsets = offsets;
  a.threshold = threshold;
  a.ws = ws;
  a.ws_bytes = kvzip::kSelectStaticBytes;
  int launches = 0;
  const cudaError_t e =
      kvzip::launch_select_multipass(a, static_cast<cudaStream_t>(stream), &launches);
  if (e != cudaSuccess) return KVZIP_ERR_CUDA;
  kvzip::note_launches(launches);
  return KVZIP_OK;
}
