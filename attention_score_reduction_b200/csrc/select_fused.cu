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
//      byte of every score outside bin b1 (kept iff its bin is above b1).  Each
//      warp owns a contiguous slice of the block's range and appends the
//      scores inside bin b1 (the candidates), as (flat index, bits of |s|)
//      pairs in flat order, to its own segment of a candidate buffer, placed
//      by a warp scan (no block barrier in the streaming loop); their next 10
//      bits are histogrammed; grid barrier.
//   D  bin b2 of round 2, then a histogram of the last 9 bits over the
//      candidates that match b1 b2 (coalesced reads of the pairs); each block
//      also stores its own round-3 histogram; grid barrier.
//   E  bin b3 gives the threshold tau exactly.  If fewer scores equal to tau
//      are kept than exist, the ties are ranked in flat order: the blocks'
//      stored histograms give the ties before this block, a per-warp count
//      the ties before this warp, and a ballot walk the rest.
//   F  every block sets the mask of its kept candidates; grid barrier.
//   G  block 0 turns the per-head kept counts into offsets and writes tau.
//
// Given the round-1 histogram (kvzip_select_hist; the last chunk's pass 2
// counts it while writing the final scores), A and its barrier are skipped and
// the scores are read once.  After C every block checks the histogram against
// what C counted (the candidates in b1 and the scores kept above it); on a
// mismatch nothing is kept and the status word records it.
//
// Scores are ordered by the bits of |s| (mag): the value order for s >= 0,
// with -0.0 equal to 0.0.
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
constexpr int kWarps = kThr / 32;
constexpr int kTile = kThr * 4;          // scores per block tile (4 per thread, 16-byte loads)
constexpr int kWarpStep = 4 * 128;       // scores per warp step of the mask pass (4 loads of 512 B)
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
constexpr size_t kOffKeptC = kOffH3 + kBins3 * 4;   // scores the mask pass keeps (one word)
constexpr size_t kOffHeads = kOffKeptC + 256;

__host__ __device__ size_t up256(size_t x) { return (x + 255) / 256 * 256; }

struct Layout {
  size_t zero_end;    // end of the region zeroed before each launch
  size_t off_h3blk;   // every block's round-3 histogram [blocks][kBins3]
  size_t off_cand;    // candidate (flat index, score bits) pairs
  size_t total;
};

// The most blocks a launch over N scores uses (no block gets less than a tile).
__host__ __device__ int64_t max_blocks(int64_t N) {
  const int64_t b = (N + kTile - 1) / kTile;
  return b < 1 ? 1 : (b > kMaxBlocks ? kMaxBlocks : b);
}

// Candidate capacity: the pair of score f lives at cand[f] at most (a warp's
// segment starts at its slice's first flat index and holds the whole slice),
// so the buffer never overflows.
__host__ __device__ Layout layout(int64_t N, int64_t n_heads) {
  Layout L;
  L.zero_end = up256(kOffHeads + static_cast<size_t>(n_heads) * 4);
  L.off_h3blk = L.zero_end;
  L.off_cand = L.off_h3blk + up256(static_cast<size_t>(max_blocks(N)) * kBins3 * 4);
  L.total = L.off_cand + up256(static_cast<size_t>(N) * 8);
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
  uint2* cand;           // base of the candidate buffer
  uint32_t seg;          // scores per block range (multiple of 128)
  uint64_t timeout_ns;
  int vec;               // scores 16-byte aligned: 16-byte loads
  int vec_keep;          // keep 4-byte aligned: 4-byte mask stores
  int test_stall;        // test hook: block 0 never reaches a barrier, so the others time out
  const uint32_t* hist_in;   // round-1 histogram of the scores (phase A is skipped), or null
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

// |x| - t on the FMA pipe, IEEE subnormals kept: negative iff |x| < t (for t
// finite or +inf and x not NaN; a NaN gives a positive NaN).
__device__ __forceinline__ float abs_minus(uint32_t x, float t) {
  float r;
  asm("{\n\t.reg .f32 a;\n\tabs.f32 a, %1;\n\tsub.rn.f32 %0, a, %2;\n\t}"
      : "=f"(r)
      : "f"(__uint_as_float(x)), "f"(t));
  return r;
}

// Byte e = 0xFF if the e-th argument's sign bit is set, else 0x00 (byte
// permutes with sign replication, then one merge).
__device__ __forceinline__ uint32_t sign_bytes4(float a, float b, float c, float d) {
  uint32_t lo, hi, r;
  asm("prmt.b32 %0, %1, %2, 0x00FB;" : "=r"(lo) : "r"(__float_as_uint(a)), "r"(__float_as_uint(b)));
  asm("prmt.b32 %0, %1, %2, 0xFB00;" : "=r"(hi) : "r"(__float_as_uint(c)), "r"(__float_as_uint(d)));
  asm("prmt.b32 %0, %1, %2, 0x7610;" : "=r"(r) : "r"(lo), "r"(hi));
  return r;
}

// Four 16-byte loads issued back to back from one statement, so all four are
// in flight before the first is used: scores p[0..3], p[128..131],
// p[256..259], p[384..387] (512-byte steps; ld.global.cs, evict first) or,
// for ld4_nc_tile, four block tiles apart (read-only path).
__device__ __forceinline__ void ld4_cs(const uint4* p, uint4 (&a)[4]) {
  asm volatile(
      "{\n\t"
      "ld.global.cs.v4.u32 {%0,%1,%2,%3}, [%16];\n\t"
      "ld.global.cs.v4.u32 {%4,%5,%6,%7}, [%16+512];\n\t"
      "ld.global.cs.v4.u32 {%8,%9,%10,%11}, [%16+1024];\n\t"
      "ld.global.cs.v4.u32 {%12,%13,%14,%15}, [%16+1536];\n\t}"
      : "=r"(a[0].x), "=r"(a[0].y), "=r"(a[0].z), "=r"(a[0].w), "=r"(a[1].x), "=r"(a[1].y),
        "=r"(a[1].z), "=r"(a[1].w), "=r"(a[2].x), "=r"(a[2].y), "=r"(a[2].z), "=r"(a[2].w),
        "=r"(a[3].x), "=r"(a[3].y), "=r"(a[3].z), "=r"(a[3].w)
      : "l"(p)
      : "memory");
}
static_assert(kTile * 4 == 8192, "ld4_nc_tile's four loads are one block tile (8192 bytes) apart");
__device__ __forceinline__ void ld4_nc_tile(const uint4* p, uint4 (&a)[4]) {
  asm volatile(
      "{\n\t"
      "ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%16];\n\t"
      "ld.global.nc.v4.u32 {%4,%5,%6,%7}, [%16+8192];\n\t"
      "ld.global.nc.v4.u32 {%8,%9,%10,%11}, [%16+16384];\n\t"
      "ld.global.nc.v4.u32 {%12,%13,%14,%15}, [%16+24576];\n\t}"
      : "=r"(a[0].x), "=r"(a[0].y), "=r"(a[0].z), "=r"(a[0].w), "=r"(a[1].x), "=r"(a[1].y),
        "=r"(a[1].z), "=r"(a[1].w), "=r"(a[2].x), "=r"(a[2].y), "=r"(a[2].z), "=r"(a[2].w),
        "=r"(a[3].x), "=r"(a[3].y), "=r"(a[3].z), "=r"(a[3].w)
      : "l"(p)
      : "memory");
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
      ld4_nc_tile(s4 + i0 / 4, a);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        atomicAdd(&h1[mag(a[q].x) >> kShift1], 1u);
        atomicAdd(&h1[mag(a[q].y) >> kShift1], 1u);
        atomicAdd(&h1[mag(a[q].z) >> kShift1], 1u);
        atomicAdd(&h1[mag(a[q].w) >> kShift1], 1u);
      }
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t f = i0 + q * kTile + e;
          if (f < hi) atomicAdd(&h1[mag(__ldg(su + f)) >> kShift1], 1u);
        }
    }
  }
}

// A warp's slice of the block range [lo, hi): 16 slices of equal length, each
// a multiple of 32 scores (so slices start on 16 bytes when lo does).
__device__ __forceinline__ void warp_slice(uint32_t lo, uint32_t hi, uint32_t* wl, uint32_t* wh) {
  const uint32_t len = ((hi - lo + kWarps - 1) / kWarps + 31) & ~31u;
  *wl = min(lo + (threadIdx.x >> 5) * len, hi);
  *wh = min(*wl + len, hi);
}

// Round-1 decision per score, from w = mag(bits): kept iff w > lim (its
// 13-bit bin is above b1); a candidate iff w - base < width (its bin is b1).
// With k = 0 nothing is kept or a candidate.  When the first value of bin
// b1 + 1 is finite or +inf (fast), the same decisions come from float
// subtractions on the FMA pipe: kept iff |s| >= t_keep, below bin b1 iff
// |s| < t_base.  For |s| not NaN this is the bit order; a NaN's bits lie above
// +inf and its difference is a positive NaN, so it counts as kept either way.
struct Round1 {
  uint32_t lim, base, width;
  bool fast;
  float t_keep, t_base;
  __device__ Round1(int b1, bool none) {
    const uint32_t b = static_cast<uint32_t>(b1);
    lim = none ? 0xFFFFFFFFu : ((b << kShift1) | ((1u << kShift1) - 1));
    base = none ? 0u : (b << kShift1);
    width = none ? 0u : (1u << kShift1);
    fast = !none && b + 1 <= (0x7F800000u >> kShift1);
    t_keep = __uint_as_float(fast ? (b + 1) << kShift1 : 0u);
    t_base = __uint_as_float(fast ? b << kShift1 : 0u);
  }
};

// Second pass over a warp's slice [wl, wh) of s, 512 scores per step (four
// 16-byte loads in flight per lane): the final mask byte of every score
// outside bin b1 (0 for candidates, set later), the candidates appended as
// (flat index, mag bits) pairs to seg in flat order (positions from one warp
// scan of per-load counts packed in bytes; each lane then walks its own
// candidate bits), their round-2 digits histogrammed into h2, and each step's
// kept scores passed to cnt.add_step and added to *kept.  Each group of four scores gets its
// decisions as byte masks: on the fast path four float subtractions and the
// sign bytes of their results, otherwise integer compares.  Returns the
// warp's candidate count.
template <class Counter>
__device__ uint32_t mask_pass(const float* __restrict__ s, uint32_t wl, uint32_t wh,
                              const Round1 r1, bool vec, bool vec_keep, uint8_t* keep,
                              uint2* seg, uint32_t* h2, Counter& cnt, uint32_t* kept) {
  const uint4* s4 = reinterpret_cast<const uint4*>(s);
  const uint32_t* su = reinterpret_cast<const uint32_t*>(s);
  const uint32_t lane = threadIdx.x & 31;
  uint32_t n_w = 0;   // warp-uniform
  for (uint32_t g0 = wl; g0 < wh; g0 += kWarpStep) {
    const uint32_t ib = g0 + 4 * lane;   // this lane's first score of load 0
    const bool full = g0 + kWarpStep <= wh;   // warp-uniform
    uint4 a[4];
    if (vec && full) {
      ld4_cs(s4 + ib / 4, a);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t i0 = ib + q * 128;
        if (vec && i0 + 3 < wh) {
          a[q] = __ldcs(s4 + i0 / 4);
        } else {
          a[q].x = (i0 + 0 < wh) ? __ldcs(su + i0 + 0) : 0u;
          a[q].y = (i0 + 1 < wh) ? __ldcs(su + i0 + 1) : 0u;
          a[q].z = (i0 + 2 < wh) ? __ldcs(su + i0 + 2) : 0u;
          a[q].w = (i0 + 3 < wh) ? __ldcs(su + i0 + 3) : 0u;
        }
      }
    }
    uint32_t cw[4], kws[4];   // candidate and kept byte masks per load
    uint32_t any = 0, kacc = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t i0 = ib + q * 128;
      uint32_t kw, c;
      if (r1.fast) {
        const uint32_t nk = sign_bytes4(abs_minus(a[q].x, r1.t_keep), abs_minus(a[q].y, r1.t_keep),
                                        abs_minus(a[q].z, r1.t_keep), abs_minus(a[q].w, r1.t_keep));
        const uint32_t nb = sign_bytes4(abs_minus(a[q].x, r1.t_base), abs_minus(a[q].y, r1.t_base),
                                        abs_minus(a[q].z, r1.t_base), abs_minus(a[q].w, r1.t_base));
        kw = ~nk & 0x01010101u;        // not below bin b1 + 1
        c = nk & ~nb & 0x01010101u;    // below bin b1 + 1, not below bin b1
      } else {
        const uint32_t w[4] = {mag(a[q].x), mag(a[q].y), mag(a[q].z), mag(a[q].w)};
        uint32_t km = 0, cq = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          km |= static_cast<uint32_t>(w[e] > r1.lim) << e;
          cq |= static_cast<uint32_t>(w[e] - r1.base < r1.width) << e;
        }
        // bit e to byte e (the shifted copies do not overlap, so no carries)
        kw = (km * 0x00204081u) & 0x01010101u;
        c = (cq * 0x00204081u) & 0x01010101u;
      }
      const uint32_t n_in = full ? 4u : (i0 < wh ? min(wh - i0, 4u) : 0u);
      if (!full) {
        const uint32_t bm = n_in == 4 ? ~0u : (1u << (8 * n_in)) - 1u;
        kw &= bm;
        c &= bm;
      }
      if (vec_keep && n_in == 4) {
        *reinterpret_cast<uint32_t*>(keep + i0) = kw;
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (e < static_cast<int>(n_in)) keep[i0 + e] = static_cast<uint8_t>((kw >> (8 * e)) & 1u);
      }
      if (c) {
        const uint32_t w[4] = {a[q].x, a[q].y, a[q].z, a[q].w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if ((c >> (8 * e)) & 1u) atomicAdd(&h2[(mag(w[e]) >> kShift2) & (kBins2 - 1)], 1u);
      }
      kws[q] = kw;
      kacc += kw;               // bytes <= 4: no carries
      cw[q] = c;
      any |= c;
    }
    const uint32_t n_kept = (kacc * 0x01010101u) >> 24;
    *kept += n_kept;
    cnt.add_step(g0, min(g0 + kWarpStep, wh), ib, kws, n_kept);
    if (__any_sync(0xffffffffu, any != 0)) {
      // candidates per load, one byte each; <= 128 per warp, so the scan's bytes never carry
      const uint32_t packed = __popc(cw[0]) | (__popc(cw[1]) << 8) | (__popc(cw[2]) << 16) |
                              (__popc(cw[3]) << 24);
      uint32_t inc = packed;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= static_cast<uint32_t>(o)) inc += n;
      }
      const uint32_t tot = __shfl_sync(0xffffffffu, inc, 31), ex = inc - packed;
      const uint32_t t0 = tot & 0xFFu, t1 = (tot >> 8) & 0xFFu, t2 = (tot >> 16) & 0xFFu,
                     t3 = tot >> 24;
      // this lane's candidates as bits 4q + e, written in that (flat) order
      uint32_t m = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) m |= ((cw[q] * 0x01020408u) >> 24 & 0xFu) << (4 * q);
      uint32_t prev_q = 0, x = n_w + (ex & 0xFFu);
      while (m) {
        const uint32_t b = __ffs(m) - 1;
        m &= m - 1;
        const uint32_t q = b >> 2;
        if (q != prev_q) {   // first candidate of a later load: its base position
          x = n_w + (q > 0 ? t0 : 0u) + (q > 1 ? t1 : 0u) + (q > 2 ? t2 : 0u) +
              ((ex >> (8 * q)) & 0xFFu);
          prev_q = q;
        }
        const uint32_t e = b & 3u;
        const uint32_t wq = q == 0 ? (e == 0 ? a[0].x : e == 1 ? a[0].y : e == 2 ? a[0].z : a[0].w)
                          : q == 1 ? (e == 0 ? a[1].x : e == 1 ? a[1].y : e == 2 ? a[1].z : a[1].w)
                          : q == 2 ? (e == 0 ? a[2].x : e == 1 ? a[2].y : e == 2 ? a[2].z : a[2].w)
                                   : (e == 0 ? a[3].x : e == 1 ? a[3].y : e == 2 ? a[3].z : a[3].w);
        if (in_bounds(x < wh - wl)) seg[x] = make_uint2(ib + q * 128 + e, mag(wq));
        ++x;
      }
      n_w += t0 + t1 + t2 + t3;
    }
  }
  return n_w;
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
  if (threadIdx.x == 0) {
    bin_s = -1;   // k_rem beyond the histogram's total
    above_s = 0;
  }
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
  // One mask-pass step of a lane: scores i + 128 q + e (q, e < 4) with kept
  // bytes kw[q] (byte e = 1 if kept), n_kept of them; all in [lo, hi).
  __device__ __forceinline__ void add_step(uint32_t lo, uint32_t hi, uint32_t i,
                                           const uint32_t (&kw)[4], uint32_t n_kept) {
    if (lo >= h * n_c && hi <= end) {   // the whole step lies in the current head
      cnt += n_kept;
      return;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if ((kw[q] >> (8 * e)) & 1u) add(i + 128 * q + e);
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

struct NoCounter {
  __device__ __forceinline__ void add_step(uint32_t, uint32_t, uint32_t, const uint32_t (&)[4],
                                           uint32_t) {}
};

__global__ void __launch_bounds__(kThr, 2)
    select_fused_kernel(const Params p) {
  __shared__ uint32_t h1[kBins1];       // round-1 histogram (32 KB), reused by later rounds
  __shared__ uint32_t h2[kBins2];
  __shared__ uint32_t tmp[2 * (kThr / 32)];
  __shared__ uint32_t win[kHeadWin];
  __shared__ uint32_t wtie[kWarps];

  uint32_t* status = reinterpret_cast<uint32_t*>(p.ws + kOffStatus);
  Sync* sy = reinterpret_cast<Sync*>(p.ws + kOffSync);
  uint32_t* g1 = reinterpret_cast<uint32_t*>(p.ws + kOffH1);
  uint32_t* g2 = reinterpret_cast<uint32_t*>(p.ws + kOffH2);
  uint32_t* g3 = reinterpret_cast<uint32_t*>(p.ws + kOffH3);
  uint32_t* heads = reinterpret_cast<uint32_t*>(p.ws + kOffHeads);
  const Layout Lw = layout(p.N, p.n_heads);
  uint32_t* h3blk = reinterpret_cast<uint32_t*>(p.ws + Lw.off_h3blk);

  const uint32_t lo = blockIdx.x * p.seg;
  const uint32_t hi = min(lo + p.seg, p.N);
  uint32_t wl, wh;
  warp_slice(lo, hi, &wl, &wh);
  uint2* wseg = p.cand + wl;   // this warp's candidate pairs
  const uint32_t lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool none = p.k == 0;
  if (p.test_stall && blockIdx.x == 0) return;
  for (int i = threadIdx.x; i < kHeadWin; i += kThr) win[i] = 0;

  // With a given round-1 histogram the first read and its barrier are skipped;
  // the histogram is checked against the scores after the mask pass.
  const bool given = p.hist_in != nullptr && !none;

  // ------------------------------------------------------------ A: round-1 histogram
  if (!none && !given) {
    for (int i = threadIdx.x; i < kBins1; i += kThr) h1[i] = 0;
    __syncthreads();
    hist_top(p.s, lo, hi, p.vec != 0, h1);
    __syncthreads();
    for (int i = threadIdx.x; i < kBins1; i += kThr)
      if (h1[i]) atomicAdd(g1 + i, h1[i]);
  }
  if (!given && !grid_barrier(sy, status, p.timeout_ns)) return;

  // ------------------------------------------------------------ B: bin of round 1
  int b1 = -1;
  uint64_t k_rem = p.k, above1 = 0;
  if (!none) {
    pick_bin<kBins1>(given ? p.hist_in : g1, k_rem, &b1, &above1);
    k_rem -= above1;
  }

  // ------------------------------------------------------------ C: mask, candidates, round-2 histogram
  for (int i = threadIdx.x; i < kBins2; i += kThr) h2[i] = 0;
  __syncthreads();
  const uint32_t ub1 = static_cast<uint32_t>(b1);
  HeadCounter hc(lo / p.n_c, p.n_c, p.n_heads, win, heads);
  uint32_t kept_c = 0;
  const uint32_t n_w = mask_pass(p.s, wl, wh, Round1(b1, none), p.vec != 0, p.vec_keep != 0,
                                 p.keep, wseg, h2, hc, &kept_c);
  hc.flush();
  if (given) {   // scores this block kept in the mask pass
    uint32_t tot;
    block_excl(kept_c, tmp, &tot);
    if (threadIdx.x == 0 && tot) atomicAdd(reinterpret_cast<uint32_t*>(p.ws + kOffKeptC), tot);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kBins2; i += kThr)
    if (h2[i]) atomicAdd(g2 + i, h2[i]);
  if (!grid_barrier(sy, status, p.timeout_ns)) return;

  // A given histogram must agree with the scores above and inside bin b1; if it
  // does, b1 and k_rem are what phase A would have found.  Otherwise nothing is
  // kept: every block clears its mask bytes and block 0 writes empty offsets.
  bool mismatch = false;
  if (given) {
    uint32_t c = 0, tot;
    for (int i = threadIdx.x; i < kBins2; i += kThr) c += __ldcg(g2 + i);
    block_excl(c, tmp, &tot);
    const uint32_t kept_tot = __ldcg(reinterpret_cast<const uint32_t*>(p.ws + kOffKeptC));
    // (a histogram with fewer than k scores has no bin b1 at all)
    mismatch = b1 < 0 || tot != __ldcg(p.hist_in + b1) || kept_tot != above1;
    if (mismatch) {
      if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(status, kStatusHistMismatch);
      for (uint32_t f = lo + threadIdx.x; f < hi; f += kThr) p.keep[f] = 0;
    }
  }

  uint32_t tau = 0x7F800000u;
  uint64_t take_eq = 0;
  bool rank_ties = false;
  if (!none && !mismatch) {
    // ---------------------------------------------------------- D: round 2, round-3 histogram
    int b2;
    uint64_t above;
    pick_bin<kBins2>(g2, k_rem, &b2, &above);
    k_rem -= above;
    const uint32_t pre2 = (ub1 << kShift1) | (static_cast<uint32_t>(b2) << kShift2);
    uint32_t* h3 = h1;   // reuse
    for (int i = threadIdx.x; i < kBins3; i += kThr) h3[i] = 0;
    __syncthreads();
    for (uint32_t j = lane; j < n_w; j += 32) {
      const uint32_t w = wseg[j].y;
      if ((w >> kShift2) == (pre2 >> kShift2)) atomicAdd(&h3[w & (kBins3 - 1)], 1u);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kBins3; i += kThr) {   // kept for the tie ranks of E
      h3blk[static_cast<size_t>(blockIdx.x) * kBins3 + i] = h3[i];
      if (h3[i]) atomicAdd(g3 + i, h3[i]);
    }
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
      for (uint32_t j = lane; j < n_w; j += 32) {
        const uint2 c = wseg[j];
        if (c.y >= tau && in_bounds(c.x >= lo && c.x < hi)) {
          p.keep[c.x] = 1;
          hf.add(c.x);
        }
      }
    } else {
      // Ties straddle the threshold: rank them in flat order.  Ties in earlier
      // blocks come from their stored round-3 histograms (bin b3 holds exactly
      // the scores equal to tau), ties in earlier warps from per-warp counts,
      // and a ballot walk over the warp's pairs ranks the rest.
      uint32_t part = 0;
      for (uint32_t b = threadIdx.x; b < blockIdx.x; b += kThr)
        part += __ldcg(h3blk + static_cast<size_t>(b) * kBins3 + b3);
      uint32_t tot;
      block_excl(part, tmp, &tot);
      uint32_t c = 0;
      for (uint32_t j = lane; j < n_w; j += 32) c += (wseg[j].y == tau);
      c = __reduce_add_sync(0xffffffffu, c);
      if (lane == 0) wtie[warp] = c;
      __syncthreads();
      uint64_t rank = tot;
      for (uint32_t v = 0; v < warp; ++v) rank += wtie[v];
      // ---------------------------------------------------------- F: kept candidates
      const uint32_t lt = (1u << lane) - 1u;
      for (uint32_t j0 = 0; j0 < n_w; j0 += 32) {
        const uint32_t j = j0 + lane;
        const bool valid = j < n_w;
        const uint2 e = valid ? wseg[j] : make_uint2(0u, 0u);
        const bool tie = valid && e.y == tau;
        const uint32_t m = __ballot_sync(0xffffffffu, tie);
        const bool kp = valid && (e.y > tau || (tie && rank + __popc(m & lt) < take_eq));
        rank += __popc(m);
        if (kp && in_bounds(e.x >= lo && e.x < hi)) {
          p.keep[e.x] = 1;
          hf.add(e.x);
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
    const uint32_t c = hh < p.n_heads && !mismatch ? __ldcg(heads + hh) : 0u;
    uint32_t tot;
    const uint32_t ex = block_excl(c, tmp, &tot);
    if (hh < p.n_heads) p.offsets[hh] = static_cast<int64_t>(carry + ex);
    carry += tot;
  }
  if (threadIdx.x == 0) {
    p.offsets[p.n_heads] = static_cast<int64_t>(carry);
    if (p.threshold) *p.threshold = none || mismatch ? INFINITY : __uint_as_float(tau);
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
                           uint32_t k, uint8_t* keep, int64_t* offsets, uint2* cand, int vec,
                           int vec_keep) {
  __shared__ uint32_t h1[kBins1];
  __shared__ uint32_t h2[kBins2];
  __shared__ uint32_t wtie[kWarps];
  const uint32_t head = blockIdx.x;
  const size_t lo = static_cast<size_t>(head) * n_c;
  const float* sh = s + lo;
  uint8_t* kh = keep + lo;
  const uint32_t lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t wl, wh;
  warp_slice(0, n_c, &wl, &wh);
  uint2* wseg = cand + lo + wl;   // this warp's candidate pairs (indices within the head)
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
  NoCounter nc;
  uint32_t kept_unused = 0;
  const uint32_t n_w =
      mask_pass(sh, wl, wh, Round1(b1, none), v4, k4, kh, wseg, h2, nc, &kept_unused);
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
  for (uint32_t j = lane; j < n_w; j += 32) {
    const uint32_t w = wseg[j].y;
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
    for (uint32_t j = lane; j < n_w; j += 32) {
      const uint2 c = wseg[j];
      if (c.y >= tau && in_bounds(c.x < n_c)) kh[c.x] = 1;
    }
    return;
  }
  // ties straddle the threshold: per-warp tie counts give each warp the rank
  // of its first tie in position order, and a ballot walk ranks the rest
  uint32_t c = 0;
  for (uint32_t j = lane; j < n_w; j += 32) c += (wseg[j].y == tau);
  c = __reduce_add_sync(0xffffffffu, c);
  if (lane == 0) wtie[warp] = c;
  __syncthreads();
  uint64_t rank = 0;
  for (uint32_t v = 0; v < warp; ++v) rank += wtie[v];
  const uint32_t lt = (1u << lane) - 1u;
  for (uint32_t j0 = 0; j0 < n_w; j0 += 32) {
    const uint32_t j = j0 + lane;
    const bool valid = j < n_w;
    const uint2 e = valid ? wseg[j] : make_uint2(0u, 0u);
    const bool tie = valid && e.y == tau;
    const uint32_t m = __ballot_sync(0xffffffffu, tie);
    const bool kp = valid && (e.y > tau || (tie && rank + __popc(m & lt) < take_eq));
    rank += __popc(m);
    if (kp && in_bounds(e.x < n_c)) kh[e.x] = 1;
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
  return up256(static_cast<size_t>(n_heads) * static_cast<size_t>(n_c) * 8);
}

cudaError_t launch_select_per_head(const SelectArgs& a, cudaStream_t s, int* launches) {
  select_per_head_kernel<<<static_cast<unsigned>(a.n_heads), kThr, 0, s>>>(
      a.scores, static_cast<uint32_t>(a.n_c), static_cast<uint32_t>(a.n_heads),
      static_cast<uint32_t>(a.k), a.keep, a.offsets, static_cast<uint2*>(a.ws),
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
  const int P = static_cast<int>(std::min<int64_t>(cap, max_blocks(N)));
  int64_t seg = (N + P - 1) / P;
  seg = (seg + 127) / 128 * 128;   // ranges start on 512 bytes
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
  p.cand = reinterpret_cast<uint2*>(ws + L.off_cand);
  p.seg = static_cast<uint32_t>(seg);
  p.timeout_ns = timeout_ns;
  p.vec = reinterpret_cast<uintptr_t>(a.scores) % 16 == 0 ? 1 : 0;   // ranges start on 4 scores
  p.vec_keep = reinterpret_cast<uintptr_t>(a.keep) % 4 == 0 ? 1 : 0;
  p.test_stall = test_stall;
  p.hist_in = a.hist_in;
  void* args[] = {&p};
  e = cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(select_fused_kernel),
                                  dim3(P_used), dim3(kThr), args, 0, s);
  if (e != cudaSuccess) return e;
  if (launches) *launches += 1;
  return cudaSuccess;
}

}  // namespace kvzip
