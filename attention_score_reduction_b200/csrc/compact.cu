// Per-head stream compaction of the kept K/V rows.
//
// After global selection, KVzip keeps a variable number of KV pairs in every
// head (blog post section 4.1, step 5: evict by score; scime.ai summary:
// non-uniform head budgets).  The kept rows of head h, positions ascending,
// land at k_out[offsets[h] + t], v_out[...] and pos_out[...].  The rebuttal's
// decoding table (KV size 32.7 -> 26.2 -> 19.6 -> 13.1 -> 6.5 GB at kept
// ratio 1 -> 0.2) is exactly this: only kept rows are stored.
//
// Three launches: count kept rows per segment of kCmpSeg rows, scan the counts
// into per-segment output bases (within each head, from offsets[h]), then copy.
// The copy is HBM-bound: every kept row is read once and written once with
// 16-byte vector accesses (a half warp per 256-byte row at d = 128, a full warp
// per 512-byte row at d = 256); evicted rows are never read.
#include <cuda_runtime.h>

#include <climits>
#include <cstdint>

#include "kvzip_internal.h"

namespace kvzip {

namespace {

constexpr int kCmpThreads = 256;
constexpr int kCmpSeg = 4096;          // rows per block
constexpr int kScanThreads = 1024;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ __forceinline__ int64_t imin64(int64_t a, int64_t b) { return a < b ? a : b; }
int64_t cmp_segs(int n_c) { return (static_cast<int64_t>(n_c) + kCmpSeg - 1) / kCmpSeg; }

__global__ void __launch_bounds__(kCmpThreads)
    cmp_count(const uint8_t* __restrict__ keep, int n_c, int64_t segs, uint32_t* blk_cnt) {
  const int64_t blk = blockIdx.x;
  const int64_t h = blk / segs, sg = blk % segs;
  const int64_t j0 = sg * kCmpSeg, j1 = imin64(j0 + kCmpSeg, static_cast<int64_t>(n_c));
  const uint8_t* kb = keep + h * n_c;
  uint32_t c = 0;
  for (int64_t j = j0 + threadIdx.x; j < j1; j += kCmpThreads) c += (kb[j] != 0);
  c = __reduce_add_sync(0xffffffffu, c);
  __shared__ uint32_t red[kCmpThreads / 32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t t = 0;
    for (int w = 0; w < kCmpThreads / 32; ++w) t += red[w];
    blk_cnt[blk] = t;
  }
}

// blk_base[h*segs + s] = offsets[h] + kept rows of head h in segments < s.
__global__ void __launch_bounds__(kScanThreads)
    cmp_scan(const uint32_t* blk_cnt, const int64_t* offsets, int64_t n_heads, int64_t segs,
             int64_t* blk_base) {
  for (int64_t h = threadIdx.x; h < n_heads; h += kScanThreads) {
    int64_t acc = offsets[h];
    for (int64_t sg = 0; sg < segs; ++sg) {
      blk_base[h * segs + sg] = acc;
      acc += blk_cnt[h * segs + sg];
    }
  }
}

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void st_stream(uint4* p, const uint4& v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

// LPR = 16-byte lanes per row (16 for d = 128, 32 for d = 256).
template <int LPR>
__global__ void __launch_bounds__(kCmpThreads)
    cmp_copy(const uint4* __restrict__ k, const uint4* __restrict__ v,
             const uint8_t* __restrict__ keep, const int64_t* __restrict__ offsets,
             const int64_t* __restrict__ blk_base, int n_c, int64_t segs, int64_t n_heads,
             uint4* k_out, uint4* v_out, int32_t* pos_out) {
  constexpr int ROWS_PER_PASS = kCmpThreads / LPR;     // rows copied per block step
  __shared__ int list[kCmpThreads];
  __shared__ uint32_t wsum[kCmpThreads / 32];
  const int64_t blk = blockIdx.x;
  const int64_t h = blk / segs, sg = blk % segs;
  const int64_t j0 = sg * kCmpSeg, j1 = imin64(j0 + kCmpSeg, static_cast<int64_t>(n_c));
  // Rows past the head's declared range are never written; with no output
  // buffers (nothing kept) no row is written at all.
  const int64_t head_end = k_out ? imin64(offsets[h + 1], offsets[n_heads]) : INT64_MIN;
  const uint8_t* kb = keep + h * n_c;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int64_t out = blk_base[blk];
  const int sub = threadIdx.x / LPR;                    // which row of the pass
  const int col = threadIdx.x % LPR;                    // which 16-byte lane of the row
  for (int64_t jb = j0; jb < j1; jb += kCmpThreads) {
    const int64_t j = jb + threadIdx.x;
    const bool kept = (j < j1) && kb[j] != 0;
    const uint32_t m = __ballot_sync(0xffffffffu, kept);
    if (lane == 0) wsum[warp] = __popc(m);
    __syncthreads();
    uint32_t before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kCmpThreads / 32; ++w) {
      before += (w < warp) ? wsum[w] : 0;
      total += wsum[w];
    }
    const uint32_t rank = before + __popc(m & ((1u << lane) - 1u));
    if (kept) {
      list[rank] = static_cast<int>(j);
      if (pos_out && out + rank < head_end && in_bounds(out + rank >= 0))
        pos_out[out + rank] = static_cast<int32_t>(j);
    }
    __syncthreads();
    // copy the `total` kept rows of this group; ROWS_PER_PASS rows per step
#pragma unroll 4
    for (uint32_t r = sub; r < total; r += ROWS_PER_PASS) {
      const int64_t o = out + r;
      if (o >= head_end) break;
      // destination row inside the packed output, source row inside head h
      if (!in_bounds(o >= 0 && h < n_heads && list[r] >= j0 && list[r] < j1)) continue;
      const int64_t src = (h * n_c + list[r]) * LPR + col;
      const uint4 kv = ld_stream(k + src);
      const uint4 vv = ld_stream(v + src);
      st_stream(k_out + o * LPR + col, kv);
      st_stream(v_out + o * LPR + col, vv);
    }
    out += total;
    __syncthreads();
  }
}

}  // namespace

cudaError_t bounds_flag_compact(unsigned int* out) { return take_bounds_flag(out); }

size_t compact_ws_bytes(int64_t n_heads, int n_c) {
  const int64_t nblk = n_heads * cmp_segs(n_c);
  return align_up(static_cast<size_t>(nblk) * 4, 256) + align_up(static_cast<size_t>(nblk) * 8, 256);
}

cudaError_t launch_compact(const CompactArgs& a, cudaStream_t s, int* launches) {
  const int64_t segs = cmp_segs(a.n_c);
  const int64_t nblk = a.n_heads * segs;
  uint8_t* p = static_cast<uint8_t*>(a.ws);
  uint32_t* blk_cnt = reinterpret_cast<uint32_t*>(p);
  int64_t* blk_base = reinterpret_cast<int64_t*>(p + align_up(static_cast<size_t>(nblk) * 4, 256));
  cmp_count<<<static_cast<unsigned>(nblk), kCmpThreads, 0, s>>>(a.keep, a.n_c, segs, blk_cnt);
  cmp_scan<<<1, kScanThreads, 0, s>>>(blk_cnt, a.offsets, a.n_heads, segs, blk_base);
  const uint4* k = static_cast<const uint4*>(a.k);
  const uint4* v = static_cast<const uint4*>(a.v);
  uint4* ko = static_cast<uint4*>(a.k_out);
  uint4* vo = static_cast<uint4*>(a.v_out);
  if (a.d == 128)
    cmp_copy<16><<<static_cast<unsigned>(nblk), kCmpThreads, 0, s>>>(
        k, v, a.keep, a.offsets, blk_base, a.n_c, segs, a.n_heads, ko, vo, a.pos_out);
  else
    cmp_copy<32><<<static_cast<unsigned>(nblk), kCmpThreads, 0, s>>>(
        k, v, a.keep, a.offsets, blk_base, a.n_c, segs, a.n_heads, ko, vo, a.pos_out);
  if (launches) *launches += 3;
  return cudaGetLastError();
}

}  // namespace kvzip
