// Global top-k selection in one cooperative launch, reading the scores twice.
//
// Same result as the multi-launch radix selection in select.cu (the k largest
// of all L x H x n_c scores, equal scores taken lowest flat index first; scime.ai
// summary "Approach" and "Measured effects" on non-uniform head budgets;
// rebuttal: S has shape L x H x n_c), with fewer passes over HBM:
//
//   A  every block histograms the top 13 bits of the scores in its contiguous
//      range (read 1); grid barrier.
//   B  every block finds, from the merged histogram, the bin b1 that holds the
//      k-th largest score (the same answer in every block).
//   C  every block reads its range again (read 2) and writes the final mask
//      byte of every score outside bin b1 (kept iff its bin is above b1).  The
//      flat indices of the scores inside bin b1 (the candidates) are appended,
//      in flat order, to the block's own segment of a candidate buffer, and
//      their next 10 bits are histogrammed; grid barrier.
//   D  bin b2 of round 2, then a histogram of the last 9 bits over the
//      candidates that match b1 b2 (gathered by index); grid barrier.
//   E  bin b3 gives the threshold tau exactly.  If fewer scores equal to tau
//      are kept than exist, every block counts its candidates equal to tau and,
//      after a barrier, sums the counts of the blocks before it: the flat-order
//      rank of its first tie.
//   F  every block sets the mask of its kept candidates; grid barrier.
//   G  block 0 turns the per-head kept counts into offsets and writes tau.
//
// Per-head kept counts are accumulated on the way (C and F) by run-length
// counting per thread: a thread's scores are visited in increasing flat order,
// so its head only changes at head boundaries.
//
// The blocks wait on one another, so the kernel is launched cooperatively (all
// blocks resident).  Every grid-barrier wait is bounded: on timeout the block
// records KVZIP_ERR_TIMEOUT in the workspace status word, raises an abort flag
// that releases the other blocks, and the kernel returns with an incomplete
// mask.
#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "kvzip.h"
#include "kvzip_internal.h"
#include "sm100_ptx.cuh"

namespace kvzip {
namespace {

constexpr int kThr = 512;                // threads per block
constexpr int kTile = kThr * 4;          // scores per block tile (4 per thread, 16-byte loads)
constexpr int kMaxBlocks = 1024;
constexpr int kBins1 = 8192, kBins2 = 1024, kBins3 = 512;
constexpr int kShift1 = 19, kShift2 = 9;  // digit of round 1: bits 31..19, round 2: 18..9, round 3: 8..0

// Workspace layout (bytes).  [kOffSync, zero_end) is zeroed by the host before
// every launch; the rest is written before it is read.
constexpr size_t kOffStatus = 0;          // sticky status word (kvzip_workspace_status)
constexpr size_t kOffSync = 256;          // grid-barrier counters (Sync), zeroed per launch
constexpr int kBarGroups = 16;            // first-level barrier counters
constexpr size_t kLine = 128;             // one counter per 128-byte line
constexpr size_t kOffH1 = kOffSync + (kBarGroups + 2) * kLine;
constexpr size_t kOffH2 = kOffH1 + kBins1 * 4;
constexpr size_t kOffH3 = kOffH2 + kBins2 * 4;
constexpr size_t kOffHeads = kOffH3 + kBins3 * 4;

__host__ __device__ size_t up256(size_t x) { return (x + 255) / 256 * 256; }

struct Layout {
  size_t zero_end;    // end of the region zeroed before each launch
  size_t off_blk;     // blk_cand[kMaxBlocks], blk_tie[kMaxBlocks]
  size_t off_cand;    // candidate flat indices, one segment per block
  size_t total;
};

// Candidate capacity: every block's segment holds its whole range (ranges are
// multiples of 4 scores), so the buffer never overflows.
__host__ __device__ Layout layout(int64_t N, int64_t n_heads) {
  Layout L;
  L.zero_end = up256(kOffHeads + static_cast<size_t>(n_heads) * 4);
  L.off_blk = L.zero_end;
  L.off_cand = L.off_blk + up256(2 * kMaxBlocks * 4);
  L.total = L.off_cand + up256((static_cast<size_t>(N) + 4 * kMaxBlocks) * 4);
  return L;
}

struct Params {
  const float* s;
  uint32_t N, n_c, n_heads;
  uint64_t k;
  uint8_t* keep;
  int64_t* offsets;
  float* threshold;
  uint8_t* ws;
  uint32_t* cand;        // base of the candidate buffer
  uint32_t seg;          // scores per block range (multiple of 4)
  uint64_t timeout_ns;
  int vec;               // scores 16-byte aligned: 16-byte loads
  int vec_keep;          // keep 4-byte aligned: 4-byte mask stores
  int test_stall;        // test hook: block 0 never reaches a barrier, so the others time out
};

// Grid-barrier words, each on its own 128-byte line: kBarGroups first-level
// arrival counters, the second-level counter, then the generation and abort
// flag.  Arrivals on one address serialise in L2 (and cross between the two
// dies for half of the SMs), so the blocks first arrive in kBarGroups groups
// (block b in group b % kBarGroups) and only each group's last block arrives
// on the second level.
struct Sync {
  unsigned int group[kBarGroups][kLine / 4];
  unsigned int top[kLine / 4];
  unsigned int gen;
  unsigned int abort;
};

// Grid barrier with a bounded wait.  Returns false if this block must stop
// (a wait timed out here or elsewhere).
__device__ bool grid_barrier(Sync* sy, uint32_t* status, uint64_t timeout_ns) {
  __shared__ int ok_s;
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile unsigned int* vgen = &sy->gen;
    volatile unsigned int* vabort = &sy->abort;
    const unsigned int g = *vgen;
    __threadfence();
    int ok = 1;
    const unsigned int n_groups = min(gridDim.x, static_cast<unsigned int>(kBarGroups));
    const unsigned int grp = blockIdx.x % n_groups;
    const unsigned int grp_size = (gridDim.x - grp + n_groups - 1) / n_groups;
    bool last = false;
    if (atomicAdd(&sy->group[grp][0], 1u) == grp_size - 1) {
      atomicExch(&sy->group[grp][0], 0u);
      __threadfence();
      last = atomicAdd(&sy->top[0], 1u) == n_groups - 1;
    }
    if (last) {
      atomicExch(&sy->top[0], 0u);
      __threadfence();
      atomicAdd(&sy->gen, 1u);
    } else {
      const uint64_t t0 = globaltimer_ns();
      while (*vgen == g) {
        if (*vabort) {
          ok = 0;
          break;
        }
        if (globaltimer_ns() - t0 > timeout_ns) {
          atomicOr(status, kStatusTimeout);
          atomicExch(&sy->abort, 1u);
          ok = 0;
          break;
        }
        __nanosleep(64);
      }
    }
    __threadfence();
    ok_s = ok && !*vabort;
  }
  __syncthreads();
  return ok_s != 0;
}

// Block-wide exclusive scan of one 32-bit value per thread (kThr threads).
// `tmp` holds kThr/32 words; returns the exclusive prefix and the block total.
__device__ __forceinline__ uint32_t block_excl(uint32_t v, uint32_t* tmp, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  if (lane == 31) tmp[warp] = inc;
  __syncthreads();
  uint32_t before = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kThr / 32; ++w) {
    const uint32_t t = tmp[w];
    before += (w < warp) ? t : 0u;
    tot += t;
  }
  __syncthreads();
  *total = tot;
  return before + inc - v;
}

// The same for two words per thread in one pass (one pair of barriers).
__device__ __forceinline__ void block_excl2(uint32_t v0, uint32_t v1, uint32_t* tmp,
                                            uint32_t* ex0, uint32_t* ex1, uint32_t* tot0,
                                            uint32_t* tot1) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t a = v0, b = v1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t na = __shfl_up_sync(0xffffffffu, a, o);
    const uint32_t nb = __shfl_up_sync(0xffffffffu, b, o);
    if (lane >= o) {
      a += na;
      b += nb;
    }
  }
  if (lane == 31) {
    tmp[warp] = a;
    tmp[kThr / 32 + warp] = b;
  }
  __syncthreads();
  uint32_t ba = 0, bb = 0, ta = 0, tb = 0;
#pragma unroll
  for (int w = 0; w < kThr / 32; ++w) {
    const uint32_t xa = tmp[w], xb = tmp[kThr / 32 + w];
    ba += (w < warp) ? xa : 0u;
    bb += (w < warp) ? xb : 0u;
    ta += xa;
    tb += xb;
  }
  __syncthreads();
  *ex0 = ba + a - v0;
  *ex1 = bb + b - v1;
  *tot0 = ta;
  *tot1 = tb;
}

// Round-1 histogram of the top 13 bits of the scores [lo, hi) of s (indices
// relative to s) into shared memory: four 16-byte loads in flight per thread.
__device__ __forceinline__ void hist_top(const float* __restrict__ s, uint32_t lo, uint32_t hi,
                                         bool vec, uint32_t* h1) {
  const uint4* s4 = reinterpret_cast<const uint4*>(s);
  const uint32_t* su = reinterpret_cast<const uint32_t*>(s);
  for (uint32_t g0 = lo; g0 < hi; g0 += 4 * kTile) {
    const uint32_t i0 = g0 + 4 * threadIdx.x;
    if (vec && i0 + 3 * kTile + 3 < hi) {
      uint4 a[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) a[q] = __ldg(s4 + (i0 + q * kTile) / 4);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        atomicAdd(&h1[a[q].x >> kShift1], 1u);
        atomicAdd(&h1[a[q].y >> kShift1], 1u);
        atomicAdd(&h1[a[q].z >> kShift1], 1u);
        atomicAdd(&h1[a[q].w >> kShift1], 1u);
      }
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t f = i0 + q * kTile + e;
          if (f < hi) atomicAdd(&h1[__ldg(su + f) >> kShift1], 1u);
        }
    }
  }
}

// Second pass over the scores [lo, hi) of s, four tiles of kTile per step
// (four 16-byte loads in flight per thread): the final mask byte of every
// score outside bin b1 (kept iff its bin is above b1; 0 for candidates, set
// later), the candidates' indices appended to seg in index order (positions
// from one block scan of packed per-tile counts), their round-2 digits
// histogrammed into h2, and on_kept(f) for every kept score (in increasing f
// per thread).  Indices are relative to s; returns the block's candidate count.
template <class OnKept>
__device__ uint32_t mask_pass(const float* __restrict__ s, uint32_t lo, uint32_t hi, uint32_t b1,
                              bool none, bool vec, bool vec_keep, uint8_t* keep, uint32_t* seg,
                              uint32_t seg_cap, uint32_t* h2, uint32_t* tmp, OnKept on_kept) {
  const uint4* s4 = reinterpret_cast<const uint4*>(s);
  const uint32_t* su = reinterpret_cast<const uint32_t*>(s);
  uint32_t n_cand = 0;   // block-uniform
  for (uint32_t g0 = lo; g0 < hi; g0 += 4 * kTile) {
    const uint32_t ib = g0 + 4 * threadIdx.x;   // this thread's first score of tile 0
    uint4 a[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {               // four loads in flight
      const uint32_t i0 = ib + q * kTile;
      if (vec && i0 + 3 < hi) {
        a[q] = __ldcs(s4 + i0 / 4);
      } else {
        a[q].x = (i0 + 0 < hi) ? __ldcs(su + i0 + 0) : 0u;
        a[q].y = (i0 + 1 < hi) ? __ldcs(su + i0 + 1) : 0u;
        a[q].z = (i0 + 2 < hi) ? __ldcs(su + i0 + 2) : 0u;
        a[q].w = (i0 + 3 < hi) ? __ldcs(su + i0 + 3) : 0u;
      }
    }
    // classify tile by tile; only the candidate bits stay live across the scan
    uint32_t cm = 0;   // bit 4q + e: score e of tile q is a candidate
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t i0 = ib + q * kTile;
      const uint32_t w[4] = {a[q].x, a[q].y, a[q].z, a[q].w};
      uint32_t km = 0, word = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t d = w[e] >> kShift1;
        const bool in = i0 + e < hi && !none;
        const bool k1 = in && d > b1, c1 = in && d == b1;
        km |= static_cast<uint32_t>(k1) << e;
        word |= static_cast<uint32_t>(k1) << (8 * e);
        if (c1) {
          cm |= 1u << (4 * q + e);
          atomicAdd(&h2[(w[e] >> kShift2) & (kBins2 - 1)], 1u);
        }
      }
      if (vec_keep && i0 + 3 < hi) {
        *reinterpret_cast<uint32_t*>(keep + i0) = word;   // 0 for candidates, set later
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (i0 + e < hi) keep[i0 + e] = static_cast<uint8_t>((km >> e) & 1u);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if ((km >> e) & 1u) on_kept(i0 + e);
    }
    // candidate positions: counts of tiles 0/1 and 2/3 packed in 16-bit halves
    // (a tile has at most kTile = 2048 candidates, so the halves never carry)
    const uint32_t c0 = __popc(cm & 0xFu), c1 = __popc(cm & 0xF0u), c2 = __popc(cm & 0xF00u),
                   c3 = __popc(cm & 0xF000u);
    uint32_t ex01, ex23, t01, t23;
    block_excl2(c0 | (c1 << 16), c2 | (c3 << 16), tmp, &ex01, &ex23, &t01, &t23);
    if (cm) {
      const uint32_t b0 = n_cand, bq1 = b0 + (t01 & 0xFFFFu), bq2 = bq1 + (t01 >> 16),
                     bq3 = bq2 + (t23 & 0xFFFFu);
      const uint32_t pos[4] = {b0 + (ex01 & 0xFFFFu), bq1 + (ex01 >> 16), bq2 + (ex23 & 0xFFFFu),
                               bq3 + (ex23 >> 16)};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t x = pos[q];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if ((cm >> (4 * q + e)) & 1u) {
            if (in_bounds(x < seg_cap)) seg[x] = ib + q * kTile + e;
            ++x;
          }
      }
    }
    n_cand += (t01 & 0xFFFFu) + (t01 >> 16) + (t23 & 0xFFFFu) + (t23 >> 16);
  }
  return n_cand;
}

// The bin (scanning from the top) that holds the k_rem-th largest element of a
// histogram with NB bins (in global memory, merged by other blocks, or in this
// block's shared memory); every thread gets the answer.
template <int NB, bool SHARED = false>
__device__ void pick_bin(const uint32_t* h, uint64_t k_rem, int* bin_out, uint64_t* above_out) {
  constexpr int PER = NB / kThr;          // 16, 2 or 1 bins per thread
  __shared__ unsigned long long wsum[kThr / 32];
  __shared__ int bin_s;
  __shared__ unsigned long long above_s;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t c[PER];
  unsigned long long mine = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) {      // thread t owns bins NB-1-PER*t ... descending
    const int bin = NB - 1 - (PER * threadIdx.x + j);
    c[j] = SHARED ? h[bin] : __ldcg(h + bin);
    mine += c[j];
  }
  unsigned long long inc = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  if (lane == 31) wsum[warp] = inc;
  if (threadIdx.x == 0) bin_s = -1;
  __syncthreads();
  unsigned long long base = 0;
  for (int w = 0; w < warp; ++w) base += wsum[w];
  const unsigned long long excl = base + inc - mine, incl = base + inc;
  if (excl < k_rem && k_rem <= incl) {
    unsigned long long above = excl;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      if (above + c[j] >= k_rem) {
        bin_s = NB - 1 - (PER * threadIdx.x + j);
        above_s = above;
        break;
      }
      above += c[j];
    }
  }
  __syncthreads();
  *bin_out = bin_s;
  *above_out = above_s;
  __syncthreads();
}

// Per-head kept counts.  A thread visits its kept scores in increasing flat
// order, so it adds up a run for one head and only flushes when its index
// crosses into another head.  Flushes go to a shared-memory window of
// kHeadWin heads starting at the block's first head (a block's range covers
// a few heads unless heads are very short), and the block adds the window to
// the global counts once at the end; heads past the window go to global
// memory directly.
constexpr int kHeadWin = 64;
struct HeadCounter {
  uint32_t h = 0, end = 0, cnt = 0;
  uint32_t h_lo, n_c, n_heads;
  uint32_t* win;      // shared [kHeadWin]
  uint32_t* heads;    // global [n_heads]
  __device__ HeadCounter(uint32_t h_lo_, uint32_t n_c_, uint32_t n_heads_, uint32_t* win_,
                         uint32_t* heads_)
      : h_lo(h_lo_), n_c(n_c_), n_heads(n_heads_), win(win_), heads(heads_) {}
  __device__ __forceinline__ void add(uint32_t f) {
    if (f >= end) {
      flush();
      h = f / n_c;
      end = (h + 1) * n_c;
    }
    ++cnt;
  }
  __device__ __forceinline__ void flush() {
    if (!cnt) return;
    if (h - h_lo < static_cast<uint32_t>(kHeadWin))
      atomicAdd(win + (h - h_lo), cnt);
    else if (in_bounds(h < n_heads))
      atomicAdd(heads + h, cnt);
    cnt = 0;
  }
};

__global__ void __launch_bounds__(kThr, 2)
    select_fused_kernel(const Params p) {
  __shared__ uint32_t h1[kBins1];       // round-1 histogram (32 KB), reused by later rounds
  __shared__ uint32_t h2[kBins2];
  __shared__ uint32_t tmp[2 * (kThr / 32)];
  __shared__ uint32_t win[kHeadWin];

  uint32_t* status = reinterpret_cast<uint32_t*>(p.ws + kOffStatus);
  Sync* sy = reinterpret_cast<Sync*>(p.ws + kOffSync);
  uint32_t* g1 = reinterpret_cast<uint32_t*>(p.ws + kOffH1);
  uint32_t* g2 = reinterpret_cast<uint32_t*>(p.ws + kOffH2);
  uint32_t* g3 = reinterpret_cast<uint32_t*>(p.ws + kOffH3);
  uint32_t* heads = reinterpret_cast<uint32_t*>(p.ws + kOffHeads);
  const Layout Lw = layout(p.N, p.n_heads);
  uint32_t* blk_cand = reinterpret_cast<uint32_t*>(p.ws + Lw.off_blk);
  uint32_t* blk_tie = blk_cand + kMaxBlocks;

  const uint32_t lo = blockIdx.x * p.seg;
  const uint32_t hi = min(lo + p.seg, p.N);
  uint32_t* seg = p.cand + static_cast<size_t>(blockIdx.x) * p.seg;
  const uint32_t* su = reinterpret_cast<const uint32_t*>(p.s);
  const bool none = p.k == 0;
  if (p.test_stall && blockIdx.x == 0) return;
  for (int i = threadIdx.x; i < kHeadWin; i += kThr) win[i] = 0;

  // ------------------------------------------------------------ A: round-1 histogram
  if (!none) {
    for (int i = threadIdx.x; i < kBins1; i += kThr) h1[i] = 0;
    __syncthreads();
    hist_top(p.s, lo, hi, p.vec != 0, h1);
    __syncthreads();
    for (int i = threadIdx.x; i < kBins1; i += kThr)
      if (h1[i]) atomicAdd(g1 + i, h1[i]);
  }
  if (!grid_barrier(sy, status, p.timeout_ns)) return;

  // ------------------------------------------------------------ B: bin of round 1
  int b1 = -1;
  uint64_t k_rem = p.k;
  if (!none) {
    uint64_t above;
    pick_bin<kBins1>(g1, k_rem, &b1, &above);
    k_rem -= above;
  }

  // ------------------------------------------------------------ C: mask, candidates, round-2 histogram
  for (int i = threadIdx.x; i < kBins2; i += kThr) h2[i] = 0;
  __syncthreads();
  const uint32_t ub1 = static_cast<uint32_t>(b1);
  HeadCounter hc(lo / p.n_c, p.n_c, p.n_heads, win, heads);
  const uint32_t n_cand =
      mask_pass(p.s, lo, hi, ub1, none, p.vec != 0, p.vec_keep != 0, p.keep, seg, hi - lo,
                h2, tmp, [&](uint32_t f) { hc.add(f); });
  hc.flush();
  __syncthreads();
  for (int i = threadIdx.x; i < kBins2; i += kThr)
    if (h2[i]) atomicAdd(g2 + i, h2[i]);
  if (threadIdx.x == 0) blk_cand[blockIdx.x] = n_cand;
  if (!grid_barrier(sy, status, p.timeout_ns)) return;

  uint32_t tau = 0x7F800000u;
  uint64_t take_eq = 0;
  bool rank_ties = false;
  uint64_t tie_base = 0;
  if (!none) {
    // ---------------------------------------------------------- D: round 2, round-3 histogram
    int b2;
    uint64_t above;
    pick_bin<kBins2>(g2, k_rem, &b2, &above);
    k_rem -= above;
    const uint32_t pre2 = (ub1 << kShift1) | (static_cast<uint32_t>(b2) << kShift2);
    uint32_t* h3 = h1;   // reuse
    for (int i = threadIdx.x; i < kBins3; i += kThr) h3[i] = 0;
    __syncthreads();
    for (uint32_t j = threadIdx.x; j < n_cand; j += kThr) {
      const uint32_t w = __ldg(su + seg[j]);
      if ((w >> kShift2) == (pre2 >> kShift2)) atomicAdd(&h3[w & (kBins3 - 1)], 1u);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kBins3; i += kThr)
      if (h3[i]) atomicAdd(g3 + i, h3[i]);
    if (!grid_barrier(sy, status, p.timeout_ns)) return;

    // ---------------------------------------------------------- E: threshold, tie ranks
    int b3;
    pick_bin<kBins3>(g3, k_rem, &b3, &above);
    k_rem -= above;
    tau = pre2 | static_cast<uint32_t>(b3);
    take_eq = k_rem;                                   // scores equal to tau that are kept
    const uint64_t n_eq = __ldcg(g3 + b3);
    rank_ties = take_eq < n_eq;                        // the same decision in every block
    HeadCounter hf(lo / p.n_c, p.n_c, p.n_heads, win, heads);
    if (!rank_ties) {
      // ---------------------------------------------------------- F: kept candidates
      for (uint32_t j = threadIdx.x; j < n_cand; j += kThr) {
        const uint32_t f = seg[j];
        if (__ldg(su + f) >= tau && in_bounds(f >= lo && f < hi)) {
          p.keep[f] = 1;
          hf.add(f);
        }
      }
    } else {
      // Ties straddle the threshold: rank them in flat order.  Each thread takes a
      // contiguous run of the block's candidates (which are in flat order), so one
      // block scan of per-thread tie counts and one scan over the blocks give
      // every tie its global rank.
      const uint32_t run = (n_cand + kThr - 1) / kThr;
      const uint32_t j0 = min(threadIdx.x * run, n_cand), j1 = min(j0 + run, n_cand);
      uint32_t c = 0;
      for (uint32_t j = j0; j < j1; ++j) c += (__ldg(su + seg[j]) == tau);
      uint32_t tot;
      const uint32_t mine_before = block_excl(c, tmp, &tot);
      if (threadIdx.x == 0) blk_tie[blockIdx.x] = tot;
      if (!grid_barrier(sy, status, p.timeout_ns)) return;
      uint32_t part = 0;
      for (uint32_t b = threadIdx.x; b < blockIdx.x; b += kThr) part += __ldcg(blk_tie + b);
      block_excl(part, tmp, &tot);
      tie_base = tot;
      // ---------------------------------------------------------- F: kept candidates
      uint64_t rank = tie_base + mine_before;
      for (uint32_t j = j0; j < j1; ++j) {
        const uint32_t f = seg[j];
        const uint32_t w = __ldg(su + f);
        bool kp = w > tau;
        if (w == tau) kp = rank++ < take_eq;
        if (kp && in_bounds(f >= lo && f < hi)) {
          p.keep[f] = 1;
          hf.add(f);
        }
      }
    }
    hf.flush();
  }
  __syncthreads();
  {
    const uint32_t h_lo = lo / p.n_c;   // the block's share of the per-head counts
    for (int i = threadIdx.x; i < kHeadWin; i += kThr)
      if (win[i] && in_bounds(h_lo + i < p.n_heads)) atomicAdd(heads + h_lo + i, win[i]);
  }
  if (!grid_barrier(sy, status, p.timeout_ns)) return;

  // ------------------------------------------------------------ G: offsets, threshold
  if (blockIdx.x != 0) return;
  unsigned long long carry = 0;
  for (uint32_t base = 0; base < p.n_heads; base += kThr) {
    const uint32_t hh = base + threadIdx.x;
    const uint32_t c = hh < p.n_heads ? __ldcg(heads + hh) : 0u;
    uint32_t tot;
    const uint32_t ex = block_excl(c, tmp, &tot);
    if (hh < p.n_heads) p.offsets[hh] = static_cast<int64_t>(carry + ex);
    carry += tot;
  }
  if (threadIdx.x == 0) {
    p.offsets[p.n_heads] = static_cast<int64_t>(carry);
    if (p.threshold) *p.threshold = none ? INFINITY : __uint_as_float(tau);
  }
}

// Uniform head budgets (scime.ai summary, "Measured effects": the weaker
// alternative to the global ranking): keep the k largest scores inside every
// head, lowest position first among equal scores.  One block per head runs the
// same phases as select_fused_kernel on its own n_c scores with block-level
// synchronisation only: histogram (read 1), bin of round 1, final mask bytes
// and candidates in position order (read 2), rounds 2 and 3 and the tie ranks
// on the candidates, then the kept candidates.  offsets[h] = h * k.
__global__ void __launch_bounds__(kThr, 2)
    select_per_head_kernel(const float* __restrict__ s, uint32_t n_c, uint32_t n_heads,
                           uint32_t k, uint8_t* keep, int64_t* offsets, uint32_t* cand,
                           int vec, int vec_keep) {
  __shared__ uint32_t h1[kBins1];
  __shared__ uint32_t h2[kBins2];
  __shared__ uint32_t tmp[2 * (kThr / 32)];
  const uint32_t head = blockIdx.x;
  const size_t lo = static_cast<size_t>(head) * n_c;
  const float* sh = s + lo;
  uint8_t* kh = keep + lo;
  uint32_t* seg = cand + lo;
  const uint32_t* su = reinterpret_cast<const uint32_t*>(sh);
  const bool none = k == 0;
  // rows of this head start on 16 bytes only when n_c is a multiple of 4
  const bool v4 = vec && (n_c % 4 == 0);
  const bool k4 = vec_keep && (n_c % 4 == 0);
  if (threadIdx.x == 0) {
    offsets[head] = static_cast<int64_t>(head) * k;
    if (head == n_heads - 1) offsets[n_heads] = static_cast<int64_t>(n_heads) * k;
  }

  int b1 = -1;
  uint64_t k_rem = k;
  if (!none) {
    for (int i = threadIdx.x; i < kBins1; i += kThr) h1[i] = 0;
    __syncthreads();
    hist_top(sh, 0, n_c, v4, h1);
    __syncthreads();
    uint64_t above;
    pick_bin<kBins1, true>(h1, k_rem, &b1, &above);
    k_rem -= above;
  }
  const uint32_t ub1 = static_cast<uint32_t>(b1);
  for (int i = threadIdx.x; i < kBins2; i += kThr) h2[i] = 0;
  __syncthreads();
  const uint32_t n_cand = mask_pass(sh, 0, n_c, ub1, none, v4, k4, kh, seg, n_c, h2, tmp,
                                    [](uint32_t) {});
  __syncthreads();
  if (none) return;
  int b2;
  uint64_t above;
  pick_bin<kBins2, true>(h2, k_rem, &b2, &above);
  k_rem -= above;
  const uint32_t pre2 = (ub1 << kShift1) | (static_cast<uint32_t>(b2) << kShift2);
  uint32_t* h3 = h1;
  for (int i = threadIdx.x; i < kBins3; i += kThr) h3[i] = 0;
  __syncthreads();
  for (uint32_t j = threadIdx.x; j < n_cand; j += kThr) {
    const uint32_t w = __ldg(su + seg[j]);
    if ((w >> kShift2) == (pre2 >> kShift2)) atomicAdd(&h3[w & (kBins3 - 1)], 1u);
  }
  __syncthreads();
  int b3;
  pick_bin<kBins3, true>(h3, k_rem, &b3, &above);
  k_rem -= above;
  const uint32_t tau = pre2 | static_cast<uint32_t>(b3);
  const uint64_t take_eq = k_rem;
  const bool rank_ties = take_eq < h3[b3];
  if (!rank_ties) {
    for (uint32_t j = threadIdx.x; j < n_cand; j += kThr) {
      const uint32_t f = seg[j];
      if (__ldg(su + f) >= tau && in_bounds(f < n_c)) kh[f] = 1;
    }
    return;
  }
  // ties straddle the threshold: contiguous runs of candidates per thread, one
  // block scan of the per-thread tie counts gives each tie its rank in position order
  const uint32_t run = (n_cand + kThr - 1) / kThr;
  const uint32_t j0 = min(threadIdx.x * run, n_cand), j1 = min(j0 + run, n_cand);
  uint32_t c = 0;
  for (uint32_t j = j0; j < j1; ++j) c += (__ldg(su + seg[j]) == tau);
  uint32_t tot;
  uint64_t rank = block_excl(c, tmp, &tot);
  for (uint32_t j = j0; j < j1; ++j) {
    const uint32_t f = seg[j];
    const uint32_t w = __ldg(su + f);
    bool kp = w > tau;
    if (w == tau) kp = rank++ < take_eq;
    if (kp && in_bounds(f < n_c)) kh[f] = 1;
  }
}

std::mutex g_coop_mu;
int g_coop_blocks[64] = {};   // co-resident blocks per device (0 = not yet queried)

cudaError_t coop_capacity(int* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_coop_mu);
  if (!g_coop_blocks[dev]) {
    int sms = 0, per_sm = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, select_fused_kernel, kThr, 0);
    if (e != cudaSuccess) return e;
    g_coop_blocks[dev] = std::max(1, std::min(kMaxBlocks, sms * per_sm));
  }
  *out = g_coop_blocks[dev];
  return cudaSuccess;
}

}  // namespace

size_t select_fused_ws_bytes(int64_t N, int64_t n_heads) { return layout(N, n_heads).total; }

size_t select_per_head_ws_bytes(int64_t n_heads, int64_t n_c) {
  return up256(static_cast<size_t>(n_heads) * static_cast<size_t>(n_c) * 4);
}

cudaError_t launch_select_per_head(const SelectArgs& a, cudaStream_t s, int* launches) {
  select_per_head_kernel<<<static_cast<unsigned>(a.n_heads), kThr, 0, s>>>(
      a.scores, static_cast<uint32_t>(a.n_c), static_cast<uint32_t>(a.n_heads),
      static_cast<uint32_t>(a.k), a.keep, a.offsets, static_cast<uint32_t*>(a.ws),
      reinterpret_cast<uintptr_t>(a.scores) % 16 == 0 ? 1 : 0,
      reinterpret_cast<uintptr_t>(a.keep) % 4 == 0 ? 1 : 0);
  if (launches) *launches += 1;
  return cudaGetLastError();
}

cudaError_t bounds_flag_select_fused(unsigned int* out) { return take_bounds_flag(out); }

cudaError_t launch_select_fused(const SelectArgs& a, uint64_t timeout_ns, int test_stall,
                                cudaStream_t s, int* launches) {
  int cap = 0;
  cudaError_t e = coop_capacity(&cap);
  if (e != cudaSuccess) return e;
  const int64_t N = a.N;
  // Blocks: enough to fill the GPU, but no block with less than one tile.
  const int64_t want = (N + kTile - 1) / kTile;
  const int P = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(cap, want)));
  int64_t seg = (N + P - 1) / P;
  seg = (seg + 3) / 4 * 4;
  const int P_used = static_cast<int>((N + seg - 1) / seg);
  const Layout L = layout(N, a.n_heads);
  uint8_t* ws = static_cast<uint8_t*>(a.ws);
  e = cudaMemsetAsync(ws + kOffSync, 0, L.zero_end - kOffSync, s);
  if (e != cudaSuccess) return e;
  Params p;
  p.s = a.scores;
  p.N = static_cast<uint32_t>(N);
  p.n_c = static_cast<uint32_t>(a.n_c);
  p.n_heads = static_cast<uint32_t>(a.n_heads);
  p.k = static_cast<uint64_t>(a.k);
  p.keep = a.keep;
  p.offsets = a.offsets;
  p.threshold = a.threshold;
  p.ws = ws;
  p.cand = reinterpret_cast<uint32_t*>(ws + L.off_cand);
  p.seg = static_cast<uint32_t>(seg);
  p.timeout_ns = timeout_ns;
  p.vec = reinterpret_cast<uintptr_t>(a.scores) % 16 == 0 ? 1 : 0;   // ranges start on 4 scores
  p.vec_keep = reinterpret_cast<uintptr_t>(a.keep) % 4 == 0 ? 1 : 0;
  p.test_stall = test_stall;
  void* args[] = {&p};
  e = cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(select_fused_kernel),
                                  dim3(P_used), dim3(kThr), args, 0, s);
  if (e != cudaSuccess) return e;
  if (launches) *launches += 1;
  return cudaSuccess;
}

}  // namespace kvzip
