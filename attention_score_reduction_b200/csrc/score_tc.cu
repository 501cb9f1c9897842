// Two-pass KVzip chunk scorer on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// What is computed (KVzip blog post, sections 4.3.1, 4.3.2 and 4.5): for each
// (layer, head) unit b and query row rho = g*n_in + i of the chunk,
//   P[rho][j] = softmax over { s_rho,j : j < n_c } U { s'_rho,j' : j' <= i }
// with s = scale * q . k_ctx[j] and s' = scale * q . k_self[j'], and
//   scores[b][j] = max(scores[b][j], max_rho P[rho][j]),  j < n_c.
//
// Pass 1 (LSE): A = 128-row query tiles, B stream = context key tiles then the
//   chunk's causal self-key tiles.  TMEM lane = query row, so each softmax
//   thread owns one row and keeps an online max / sum in registers.  It writes
//   lse2[rho] = log2 sum_j 2^(c * s_rho,j),  c = scale * log2(e).
// Pass 2 (column max): A = 128-key context tiles, B stream = query row tiles.
//   TMEM lane = key, so the max over query rows is a per-thread running max of
//   c * s - lse2[rho]; exp is monotone, so one exp2 per key at the end:
//   p_j = 2^(max_rho (c s_rho,j - lse2[rho])).
//
// One skeleton serves both passes: warp 0 issues TMA loads (A tiles once, then
// a STAGES-deep ring of B tiles), warp 1 allocates TMEM and issues tcgen05.mma
// from one thread, warps 2..9 are two 128-thread epilogue groups, one per A
// tile, each reading its own double-buffered fp32 accumulator from TMEM.
// Every wait is bounded; on timeout the CTA records KVZIP_ERR_TIMEOUT in the
// status word, drains its in-flight copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "kvzip_internal.h"
#include "sm100_ptx.cuh"

namespace kvzip {

template <int D>
struct TcCfg;
template <>
struct TcCfg<128> {
  static constexpr int BN = 128;     // rows per B tile (N of the MMA)
  static constexpr int STAGES = 4;   // B ring depth
};
template <>
struct TcCfg<256> {
  static constexpr int BN = 64;
  static constexpr int STAGES = 3;
};

constexpr int kThreads = 320;        // 10 warps
constexpr int kBM = 128;             // rows per A tile (M of the MMA)
constexpr int kATiles = 2;           // A tiles per CTA
constexpr uint64_t kDrainTimeoutNs = 1000000000ull;
// Pass 1: out of every 8 pairs of exponentials, this many are evaluated by
// polynomial on the FMA pipe instead of the MUFU unit (16 ex2 per clock per SM,
// half the tensor core's 32 logits per clock at d = 128).
#ifndef KVZIP_POLY_PAIRS
#define KVZIP_POLY_PAIRS 0
#endif
constexpr int kPolyPairs = KVZIP_POLY_PAIRS;

template <int D>
struct TcLayout {
  static constexpr int BN = TcCfg<D>::BN;
  static constexpr int STAGES = TcCfg<D>::STAGES;
  static constexpr int KB = D / 64;                      // 128-byte K blocks per row
  static constexpr int A_KB_BYTES = kBM * 128;           // one K block of an A tile
  static constexpr int A_BYTES = KB * A_KB_BYTES;
  static constexpr int B_KB_BYTES = BN * 128;
  static constexpr int B_BYTES = KB * B_KB_BYTES;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + kATiles * A_BYTES;
  static constexpr int L_BYTES = BN * 4;                // pass 2: lse2 of one B tile
  static constexpr int OFF_L = OFF_B + STAGES * B_BYTES;
  static constexpr int OFF_BAR = OFF_L + STAGES * L_BYTES;
  // barriers: a_full, b_full[S], b_empty[S], s_full[2][2], s_empty[2][2], mma_done, l_empty[S]
  static constexpr int N_BARS = 1 + 2 * STAGES + 8 + 1 + STAGES;
  static constexpr int OFF_MISC = OFF_BAR + 8 * N_BARS;  // tmem base, abort flag
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = BYTES + 1024;        // slack for 1024-B alignment
  static constexpr int TMEM_COLS = kATiles * 2 * BN;     // 2 buffers per A tile
  static_assert(TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM allocation must be a power of 2");
  static_assert(SMEM_ALLOC <= 232448, "exceeds 227 KB of shared memory");
};

struct Ctl {
  volatile int* abort_flag;
  uint32_t* status;
  uint64_t timeout_ns;
};

// One thread waits; bounded by the timeout and by the CTA abort flag.
__device__ __forceinline__ bool wait_one(uint64_t* bar, uint32_t parity, const Ctl& ctl) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 16; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*ctl.abort_flag) return false;
    if (globaltimer_ns() - t0 > ctl.timeout_ns) {
      *ctl.abort_flag = 1;
      atomicOr(ctl.status, kStatusTimeout);
      return false;
    }
  }
}

// A whole warp waits; the outcome is warp-uniform so that the .sync.aligned
// tcgen05 instructions after it stay convergent.
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, const Ctl& ctl) {
  const int lane = threadIdx.x & 31;
  uint64_t t0 = 0;
#pragma unroll 1
  for (uint32_t it = 0;; ++it) {
    const bool ok = mbar_try_wait(bar, parity);
    if (__all_sync(0xffffffffu, ok)) return true;
    if ((it & 15u) == 15u) {
      int stop = 0;
      if (lane == 0) {
        const uint64_t now = globaltimer_ns();
        if (it == 15u) t0 = now;
        if (*ctl.abort_flag) {
          stop = 1;
        } else if (it != 15u && now - t0 > ctl.timeout_ns) {
          *ctl.abort_flag = 1;
          atomicOr(ctl.status, kStatusTimeout);
          stop = 1;
        }
      }
      if (__shfl_sync(0xffffffffu, stop, 0)) return false;
    }
  }
}

// Drain wait: ignores the abort flag, bounded by a fixed limit.
__device__ __forceinline__ void wait_drain(uint64_t* bar, uint32_t parity, uint32_t* status) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kDrainTimeoutNs) {
      atomicOr(status, kStatusTimeout);
      return;
    }
  }
}

// The whole BN-column accumulator row of this thread in one TMEM round trip.
__device__ __forceinline__ void tmem_ld_tile(uint32_t taddr, float (&v)[128]) { tmem_ld128(taddr, v); }
__device__ __forceinline__ void tmem_ld_tile(uint32_t taddr, float (&v)[64]) { tmem_ld64(taddr, v); }

struct TcParams {
  float* scores;
  float* lse2;
  uint32_t* status;
  int G, n_in, n_c, R, R_pad;
  float c;            // scale * log2(e)
  uint64_t timeout_ns;
  int test_stall;     // test hook: the loader issues no copies, so every wait runs out
};

template <int D, bool PASS2>
__global__ void __launch_bounds__(kThreads, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap amap,
                    const __grid_constant__ CUtensorMap bmap0,
                    const __grid_constant__ CUtensorMap bmap1, const TcParams p) {
  using Lay = TcLayout<D>;
  constexpr int BN = Lay::BN;
  constexpr int STAGES = Lay::STAGES;
  constexpr int KB = Lay::KB;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::OFF_BAR);
  uint64_t* a_full = bars;
  uint64_t* b_full = bars + 1;
  uint64_t* b_empty = bars + 1 + STAGES;
  uint64_t* s_full = bars + 1 + 2 * STAGES;        // [t*2 + buf]
  uint64_t* s_empty = bars + 1 + 2 * STAGES + 4;   // [t*2 + buf]
  uint64_t* mma_done = bars + 1 + 2 * STAGES + 8;
  uint64_t* l_empty = bars + 2 + 2 * STAGES + 8;    // pass 2: lse2 stage free again
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(smem + Lay::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int a_row0 = blockIdx.x * (kATiles * kBM);

  // ---- per-CTA work description
  const int a_extent = PASS2 ? p.n_c : p.R;                 // rows of the A operand
  const int nA = min(kATiles, (a_extent - a_row0 + kBM - 1) / kBM);
  const int n_kt_ctx = PASS2 ? 0 : (p.n_c + BN - 1) / BN;
  int n_b;
  if (PASS2) {
    n_b = (p.R + BN - 1) / BN;
  } else {
    const int r_last = min(a_row0 + kATiles * kBM, p.R) - 1;
    const int i_max = (r_last / p.n_in != a_row0 / p.n_in) ? p.n_in - 1 : r_last % p.n_in;
    n_b = n_kt_ctx + (i_max + 1 + BN - 1) / BN;
  }

  if (threadIdx.x == 0) {
    mbar_init(a_full, 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], kBM);
    }
    mbar_init(mma_done, 1);
    // every thread of every active epilogue group releases each lse2 stage
    for (int s = 0; s < STAGES; ++s) mbar_init(&l_empty[s], nA * kBM);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_slot, Lay::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_base_slot;
  const Ctl ctl{abort_flag, p.status, p.timeout_ns};

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&amap);
      tma_prefetch_desc(&bmap0);
      if (!PASS2) tma_prefetch_desc(&bmap1);
      const bool stall = p.test_stall != 0;
      if (!stall) {
        mbar_arrive_expect_tx(a_full, nA * Lay::A_BYTES);
        for (int t = 0; t < nA; ++t)
          for (int kb = 0; kb < KB; ++kb)
            tma_load_3d(smem + Lay::OFF_A + t * Lay::A_BYTES + kb * Lay::A_KB_BYTES, &amap,
                        a_full, kb * 64, a_row0 + t * kBM, b);
      }
      int issued = 0;
#pragma unroll 1
      for (int it = 0; !stall && it < n_b; ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!wait_one(&b_empty[s], ph ^ 1, ctl)) break;
        if (PASS2 && !wait_one(&l_empty[s], ph ^ 1, ctl)) break;
        mbar_arrive_expect_tx(&b_full[s], Lay::B_BYTES + (PASS2 ? Lay::L_BYTES : 0));
        const void* map = &bmap0;
        int row = it * BN;
        if (!PASS2 && it >= n_kt_ctx) {
          map = &bmap1;
          row = (it - n_kt_ctx) * BN;
        }
        uint8_t* dst = smem + Lay::OFF_B + s * Lay::B_BYTES;
        for (int kb = 0; kb < KB; ++kb)
          tma_load_3d(dst + kb * Lay::B_KB_BYTES, map, &b_full[s], kb * 64, row, b);
        if (PASS2)  // the row normalisers of this query tile ride on the same barrier
          bulk_load(smem + Lay::OFF_L + s * Lay::L_BYTES,
                    p.lse2 + static_cast<size_t>(b) * p.R_pad + row, Lay::L_BYTES, &b_full[s]);
        issued = it + 1;
      }
      // Drain: every copy this CTA started must land before shared memory is released.
      if (!stall) wait_drain(a_full, 0, p.status);
      for (int s = 0; s < STAGES && s < issued; ++s) {
        const int last = s + ((issued - 1 - s) / STAGES) * STAGES;
        wait_drain(&b_full[s], (last / STAGES) & 1, p.status);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN);
      const uint32_t a_base = smem_u32(smem + Lay::OFF_A);
      const uint32_t b_base = smem_u32(smem + Lay::OFF_B);
      bool ok = wait_one(a_full, 0, ctl);
      tc_fence_after();
#pragma unroll 1
      for (int it = 0; ok && it < n_b; ++it) {
        const int s = it % STAGES;
        if (!wait_one(&b_full[s], (it / STAGES) & 1, ctl)) break;
        tc_fence_after();
        const int buf = it & 1;
        const uint32_t sph = (it >> 1) & 1;
        for (int t = 0; t < nA; ++t) {
          if (!wait_one(&s_empty[t * 2 + buf], sph ^ 1, ctl)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + (t * 2 + buf) * BN;
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) {
            const uint64_t ad = sdesc_sw128(a_base + t * Lay::A_BYTES + kb * Lay::A_KB_BYTES);
            const uint64_t bd = sdesc_sw128(b_base + s * Lay::B_BYTES + kb * Lay::B_KB_BYTES);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16_ss(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0);
          }
          umma_commit(&s_full[t * 2 + buf]);
        }
        if (!ok) break;
        umma_commit(&b_empty[s]);
      }
      // Drain: all MMAs issued by this thread complete before TMEM is freed.
      umma_commit(mma_done);
      wait_drain(mma_done, 0, p.status);
    }
    __syncwarp();
  } else {
    // ================================================================ epilogue groups
    const int t = (warp - 2) >> 2;          // A tile served by this group
    const int quarter = warp & 3;           // TMEM lanes 32*quarter .. +31
    const int lrow = quarter * 32 + lane;   // row of the A tile
    const int arow = a_row0 + t * kBM + lrow;
    const float c = p.c;
    if (t < nA) {
      if (!PASS2) {
        // ---------------- pass 1: online log-sum-exp over the row
        const int i_row = arow % p.n_in;
        float m = -INFINITY, l = 0.f;
#pragma unroll 1
        for (int it = 0; it < n_b; ++it) {
          const int buf = it & 1;
          if (!wait_warp(&s_full[t * 2 + buf], (it >> 1) & 1, ctl)) break;
          tc_fence_after();
          float v[BN];
          const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                 (t * 2 + buf) * BN;
          tmem_ld_tile(taddr, v);
          tc_fence_before();
          mbar_arrive(&s_empty[t * 2 + buf]);
          // masks: ragged context tail, causal self keys
          if (it < n_kt_ctx) {
            const int lim = p.n_c - it * BN;
            if (lim < BN) {
#pragma unroll
              for (int j = 0; j < BN; ++j)
                if (j >= lim) v[j] = -INFINITY;
            }
          } else {
            const int lim = i_row - (it - n_kt_ctx) * BN;   // self key j' visible iff j' <= i
#pragma unroll
            for (int j = 0; j < BN; ++j)
              if (j > lim) v[j] = -INFINITY;
          }
          float mx0 = v[0], mx1 = v[1];
#pragma unroll
          for (int j = 2; j + 3 < BN; j += 4) {
            mx0 = fmax3(mx0, v[j], v[j + 1]);
            mx1 = fmax3(mx1, v[j + 2], v[j + 3]);
          }
          mx0 = fmax3(mx0, mx1, fmaxf(v[BN - 2], v[BN - 1]));
          const float m_new = fmaxf(m, mx0 * c);
          const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
          // x = c*s - m in packed pairs; of every 8 pairs, kPolyPairs take 2^x on
          // the FMA pipe and the rest on the MUFU unit, so both pipes share the work.
          const float2 c2 = make_float2(c, c);
          const float2 nm2 = make_float2(-m_use, -m_use);
          float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
          for (int j = 0; j < BN; j += 16) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float2 x = ffma2(make_float2(v[j + 2 * q], v[j + 2 * q + 1]), c2, nm2);
              float2 e;
              if (q < kPolyPairs) {
                e = exp2_poly2(x);
              } else {
                e.x = ex2_approx(x.x);
                e.y = ex2_approx(x.y);
              }
              if (q & 1)
                acc1 = fadd2(acc1, e);
              else
                acc0 = fadd2(acc0, e);
            }
          }
          l = fmaf(l, ex2_approx(m - m_use), (acc0.x + acc0.y) + (acc1.x + acc1.y));
          m = m_new;
        }
        if (!*abort_flag && arow < p.R_pad)
          p.lse2[static_cast<size_t>(b) * p.R_pad + arow] =
              (arow < p.R) ? m + lg2_approx(l) : INFINITY;
      } else {
        // ---------------- pass 2: running max over query rows of c*s - lse2
        float best = -INFINITY;
#pragma unroll 1
        for (int it = 0; it < n_b; ++it) {
          const int buf = it & 1;
          const int st = it % STAGES;
          // The stage's lse2 bytes landed with b_full; the stage cannot be refilled
          // before this group releases l_empty, so this phase is still the latest.
          if (!wait_warp(&b_full[st], (it / STAGES) & 1, ctl)) break;
          if (!wait_warp(&s_full[t * 2 + buf], (it >> 1) & 1, ctl)) break;
          tc_fence_after();
          float v[BN];
          const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                 (t * 2 + buf) * BN;
          tmem_ld_tile(taddr, v);
          tc_fence_before();
          mbar_arrive(&s_empty[t * 2 + buf]);
          const float4* L4 = reinterpret_cast<const float4*>(smem + Lay::OFF_L + st * Lay::L_BYTES);
          float b0 = best, b1 = -INFINITY;
#pragma unroll
          for (int j = 0; j < BN; j += 4) {
            const float4 L = L4[j / 4];   // same address in every lane: broadcast
            b0 = fmax3(b0, fmaf(v[j + 0], c, -L.x), fmaf(v[j + 1], c, -L.y));
            b1 = fmax3(b1, fmaf(v[j + 2], c, -L.z), fmaf(v[j + 3], c, -L.w));
          }
          best = fmaxf(b0, b1);
          mbar_arrive(&l_empty[st]);
        }
        if (!*abort_flag && arow < p.n_c) {
          float* dst = p.scores + static_cast<size_t>(b) * p.n_c + arow;
          *dst = fmaxf(*dst, ex2_approx(best));
        }
      }
    } else if (!PASS2) {
      // A tile beyond the query rows: pad the log-sum-exp buffer with +inf so
      // that padded columns never win the pass-2 maximum.
      if (arow < p.R_pad) p.lse2[static_cast<size_t>(b) * p.R_pad + arow] = INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Lay::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 3-D bf16 map over [units][rows][d], box = 64 elements x box_rows x 1, 128-B swizzle.
static bool make_map(CUtensorMap* m, const void* base, int units, int rows, int d, int box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(units)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(rows) * static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D>
static cudaError_t launch_tc(const ScoreArgs& a, cudaStream_t s, int* launches) {
  using Lay = TcLayout<D>;
  // The shared-memory limit is a per-device function attribute; set it each call.
  cudaError_t e = cudaFuncSetAttribute(score_tc_kernel<D, false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Lay::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(score_tc_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           Lay::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  CUtensorMap qmap, kmap, smap;
  if (!make_map(&qmap, a.q, a.B, a.R, D, kBM) ||  // A box for pass 1
      !make_map(&kmap, a.k_ctx, a.B, a.n_c, D, Lay::BN) ||
      !make_map(&smap, a.k_self, a.B, a.n_in, D, Lay::BN))
    return cudaErrorInvalidValue;
  TcParams p;
  p.scores = a.scores;
  p.lse2 = a.lse2;
  p.status = a.status;
  p.G = a.G;
  p.n_in = a.n_in;
  p.n_c = a.n_c;
  p.R = a.R;
  p.R_pad = a.R_pad;
  p.c = a.scale * 1.4426950408889634f;
  p.timeout_ns = a.timeout_ns;
  p.test_stall = a.test_stall;

  if (a.passes & 1) {
    dim3 g1((a.R + kATiles * kBM - 1) / (kATiles * kBM), a.B);
    score_tc_kernel<D, false><<<g1, kThreads, Lay::SMEM_ALLOC, s>>>(qmap, kmap, smap, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (launches) *launches += 1;
  }
  if (!(a.passes & 2)) return cudaSuccess;

  // pass 2: A = context key tiles (box 128 rows), B = query row tiles (box BN rows)
  CUtensorMap kmapA, qmapB;
  if (!make_map(&kmapA, a.k_ctx, a.B, a.n_c, D, kBM) ||
      !make_map(&qmapB, a.q, a.B, a.R, D, Lay::BN))
    return cudaErrorInvalidValue;
  dim3 g2((a.n_c + kATiles * kBM - 1) / (kATiles * kBM), a.B);
  score_tc_kernel<D, true><<<g2, kThreads, Lay::SMEM_ALLOC, s>>>(kmapA, qmapB, qmapB, p);
  e = cudaGetLastError();
  if (e == cudaSuccess && launches) *launches += 1;
  return e;
}

cudaError_t launch_score_tc(const ScoreArgs& a, cudaStream_t s, int* launches) {
  if (a.d == 128) return launch_tc<128>(a, s, launches);
  if (a.d == 256) return launch_tc<256>(a, s, launches);
  return cudaErrorInvalidValue;
}

}  // namespace kvzip
