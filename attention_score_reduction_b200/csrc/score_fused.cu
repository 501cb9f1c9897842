// Chunk-pipelined KVzip scorer: pass 1 (row log-sum-exp) of chunk c and pass 2
// (column max) of chunk c-1 in ONE persistent kernel, one CTA per SM.
//
// What is computed is exactly the two passes of score_tc.cu (KVzip blog post,
// sections 4.3.1, 4.3.2 and 4.5):
//   pass 1: lse2[rho] = log2 sum_j 2^(c * s_rho,j) over the n_c context keys and
//           the chunk's causal self keys (c = scale * log2(e));
//   pass 2: scores[b][j] = max(scores[b][j], 2^(max_rho (c * s_rho,j - lse2[rho]))).
// Pass 2 of a chunk needs that chunk's pass 1 to be complete, but pass 1 of the
// NEXT chunk does not depend on it, so the two can share the SM.  They are
// limited by different units: pass 1 by the exponentials (MUFU ex2 plus the
// polynomial share on the FMA pipe) with the tensor pipe half idle, pass 2 by
// the tensor pipe with MUFU idle.  Each CTA therefore runs two independent
// warp-specialised slots over one 512-column TMEM allocation:
//   slot 1 (pass 1 of chunk c):   A = 128 query rows in shared memory (TMA),
//                                 B = 64-key context / self-key tiles, 3-deep ring,
//                                 four 64-column accumulators, four epilogue groups;
//   slot 2 (pass 2 of chunk c-1): A = 128 context keys in shared memory (TMA,
//                                 double-buffered), B = 96-row query tiles plus
//                                 their lse2 values, 3-deep ring, two 96-column
//                                 accumulators, two epilogue groups.
// Warps: 0 slot-1 loader, 1 slot-1 MMA issuer (and TMEM owner), 2 slot-2 loader,
// 3 slot-2 MMA issuer, 4..19 slot-1 epilogue, 20..27 slot-2 epilogue.
// Work items are (unit, 128-row tile) for slot 1 and (unit, 128-key tile) for
// slot 2, dealt round-robin over the CTAs; the two slots advance independently.
// Both slots take both MMA operands from shared memory: tensor memory holds only
// accumulators, written by the MMAs and read back with tcgen05.ld.  (With the
// pass-1 A tile kept in tensor memory and rewritten by tcgen05.st at each item,
// pass-2 accumulators running beside it came out wrong now and then on B200.)
// Every wait is bounded; on timeout the CTA records KVZIP_ERR_TIMEOUT, all
// slots stop at their next item boundary, drain their copies and MMAs, and the
// CTA frees TMEM and returns.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "kvzip_internal.h"
#include "sm100_ptx.cuh"
#include "tc_common.cuh"

namespace kvzip {
namespace fused {

constexpr int D = 128;
constexpr int KB = D / 64;        // 128-byte K blocks per row
constexpr int BM = 128;           // A rows (M of both MMAs)
constexpr int BN1 = 64;           // pass-1 B tile: keys
constexpr int BN2 = 96;           // pass-2 B tile: query rows
constexpr int S1 = 3;             // pass-1 ring depth
constexpr int S2 = 3;             // pass-2 ring depth
constexpr int NG1 = 4;            // pass-1 epilogue groups (= accumulators)
constexpr int NG2 = 2;            // pass-2 epilogue groups (= accumulators)
constexpr int CH = 32;            // accumulator columns per TMEM load
constexpr int kCtlWarps = 4;
constexpr int kThreads = 32 * (kCtlWarps + 4 * NG1 + 4 * NG2);   // 896
constexpr int kPoly = 2;          // of every 8 exponential pairs, on the FMA pipe

// shared memory
constexpr int B1_KB = BN1 * 128;
constexpr int B1_BYTES = KB * B1_KB;
constexpr int A1_KB = BM * 128;
constexpr int A1_BYTES = KB * A1_KB;
constexpr int A2_KB = BM * 128;
constexpr int A2_BYTES = KB * A2_KB;
constexpr int B2_KB = BN2 * 128;
constexpr int B2_BYTES = KB * B2_KB;
constexpr int L2_BYTES = BN2 * 4;
constexpr int OFF_B1 = 0;
constexpr int OFF_A1 = OFF_B1 + S1 * B1_BYTES;
constexpr int OFF_A2 = OFF_A1 + A1_BYTES;
constexpr int OFF_B2 = OFF_A2 + 2 * A2_BYTES;
constexpr int OFF_L2 = OFF_B2 + S2 * B2_BYTES;
constexpr int OFF_BAR = OFF_L2 + S2 * L2_BYTES;
// barrier indices
constexpr int BAR_FULL1 = 0;
constexpr int BAR_EMPTY1 = BAR_FULL1 + S1;
constexpr int BAR_A1_FULL = BAR_EMPTY1 + S1;
constexpr int BAR_A1_EMPTY = BAR_A1_FULL + 1;
constexpr int BAR_SF1 = BAR_A1_EMPTY + 1;
constexpr int BAR_SE1 = BAR_SF1 + NG1;
constexpr int BAR_FULL2 = BAR_SE1 + NG1;
constexpr int BAR_EMPTY2 = BAR_FULL2 + S2;
constexpr int BAR_LEMPTY2 = BAR_EMPTY2 + S2;
constexpr int BAR_A2_FULL = BAR_LEMPTY2 + S2;
constexpr int BAR_A2_EMPTY = BAR_A2_FULL + 2;
constexpr int BAR_SF2 = BAR_A2_EMPTY + 2;
constexpr int BAR_SE2 = BAR_SF2 + NG2;
constexpr int BAR_DONE1 = BAR_SE2 + NG2;
constexpr int BAR_DONE2 = BAR_DONE1 + 1;
constexpr int N_BARS = BAR_DONE2 + 1;
constexpr int OFF_X1 = (OFF_BAR + 8 * N_BARS + 15) & ~15;   // pass-1 merge: [2][NG1-1][BM] float2
constexpr int OFF_X2 = OFF_X1 + 2 * (NG1 - 1) * BM * 8;     // pass-2 merge: [2][BM] float
constexpr int OFF_MISC = OFF_X2 + 2 * BM * 4;               // tmem base, abort flag
constexpr int BYTES = OFF_MISC + 16;
constexpr int SMEM_ALLOC = BYTES + 1024;
// tensor memory columns
constexpr int ACC1_COL = 0;                      // NG1 accumulators of BN1 columns
constexpr int ACC2_COL = ACC1_COL + NG1 * BN1;   // NG2 accumulators of BN2 columns
constexpr int TMEM_COLS = 512;
static_assert(ACC2_COL + NG2 * BN2 <= TMEM_COLS, "TMEM over-committed");
static_assert(SMEM_ALLOC <= 232448, "exceeds 227 KB of shared memory");
static_assert(B1_KB % 1024 == 0 && A1_KB % 1024 == 0 && A2_KB % 1024 == 0 &&
                  B2_KB % 1024 == 0,
              "swizzle atoms must stay 1024-B aligned");
static_assert(BN1 % CH == 0 && BN2 % CH == 0, "tile not a multiple of the TMEM load");

struct Params {
  // pass 1 (chunk c): queries and the row log-sum-exp it writes
  float* lse_out;         // [B][R_pad1]
  int n_in1, R1, R_pad1, n_rt1, items1;
  // pass 2 (chunk c-1): the row log-sum-exp it reads
  const float* lse_in;    // [B][R_pad2]
  int R2, R_pad2, n_kt2, items2;
  float* scores;          // [B][n_c]
  uint32_t* status;
  int n_c;
  float c;                // scale * log2(e)
  uint64_t timeout_ns;
  int test_stall;         // test hook: the loaders issue no copies, so every wait runs out
};

__device__ __forceinline__ int p1_tiles(const Params& p, int rt) {
  const int r0 = rt * BM;
  const int r_last = min(r0 + BM, p.R1) - 1;
  const int i_max = (r_last / p.n_in1 != r0 / p.n_in1) ? p.n_in1 - 1 : r_last % p.n_in1;
  return (p.n_c + BN1 - 1) / BN1 + (i_max + 1 + BN1 - 1) / BN1;
}

// Online base-2 log-sum-exp of CH scaled logits c * v into (m, l).
__device__ __forceinline__ void online_lse(const float (&v)[CH], float c, float& m, float& l) {
  float mx[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) mx[k] = fmaxf(v[2 * k], v[2 * k + 1]);
#pragma unroll
  for (int j = 16; j < CH; j += 16) {
#pragma unroll
    for (int k = 0; k < 8; ++k) mx[k] = fmax3(mx[k], v[j + 2 * k], v[j + 2 * k + 1]);
  }
  const float mxa = fmax3(mx[0], mx[1], mx[2]), mxb = fmax3(mx[3], mx[4], mx[5]);
  const float m_new = fmaxf(m, fmax3(mxa, mxb, fmaxf(mx[6], mx[7])) * c);
  const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
  const float2 c2 = make_float2(c, c);
  const float2 nm2 = make_float2(-m_use, -m_use);
  float2 acc[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.f, 0.f);
#pragma unroll
  for (int j = 0; j < CH; j += 16) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float2 x = ffma2(make_float2(v[j + 2 * q], v[j + 2 * q + 1]), c2, nm2);
      float2 e;
      if (q < kPoly) {
        e = exp2_poly2(x);
      } else {
        e.x = ex2_approx(x.x);
        e.y = ex2_approx(x.y);
      }
      acc[q & 3] = fadd2(acc[q & 3], e);
    }
  }
  const float2 s4 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
  l = fmaf(l, ex2_approx(m - m_use), s4.x + s4.y);
  m = m_new;
}

__global__ void __launch_bounds__(kThreads, 1)
    score_fused_kernel(const __grid_constant__ CUtensorMap kmap,   // K_ctx, box 64 x 64 rows
                       const __grid_constant__ CUtensorMap smap,   // K_self of chunk c, box 64 x 64
                       const __grid_constant__ CUtensorMap q1map,  // Q of chunk c, box 64 x 64
                       const __grid_constant__ CUtensorMap qmap,   // Q of chunk c-1, box 64 x 96
                       const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S1; ++s) {
      mbar_init(&bars[BAR_FULL1 + s], 1);
      mbar_init(&bars[BAR_EMPTY1 + s], 1);
    }
    mbar_init(&bars[BAR_A1_FULL], 1);
    mbar_init(&bars[BAR_A1_EMPTY], 1);
    for (int g = 0; g < NG1; ++g) {
      mbar_init(&bars[BAR_SF1 + g], 1);
      mbar_init(&bars[BAR_SE1 + g], BM);
    }
    for (int s = 0; s < S2; ++s) {
      mbar_init(&bars[BAR_FULL2 + s], 1);
      mbar_init(&bars[BAR_EMPTY2 + s], 1);
      mbar_init(&bars[BAR_LEMPTY2 + s], BM);   // the one group that drains the tile
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[BAR_A2_FULL + i], 1);
      mbar_init(&bars[BAR_A2_EMPTY + i], 1);
    }
    for (int g = 0; g < NG2; ++g) {
      mbar_init(&bars[BAR_SF2 + g], 1);
      mbar_init(&bars[BAR_SE2 + g], BM);
    }
    mbar_init(&bars[BAR_DONE1], 1);
    mbar_init(&bars[BAR_DONE2], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_base_slot;
  const Ctl ctl{abort_flag, p.status, p.timeout_ns};
  const bool stall = p.test_stall != 0;
  const int n_kt_ctx = (p.n_c + BN1 - 1) / BN1;
  const int nb2 = (p.R2 + BN2 - 1) / BN2;

  if (warp == 0) {
    // ============================================================ pass-1 loader
    if (lane == 0) {
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&smap);
      tma_prefetch_desc(&q1map);
      uint32_t T = 0, k = 0;
      bool ok = !stall;
#pragma unroll 1
      for (int item = blockIdx.x; ok && item < p.items1; item += gridDim.x, ++k) {
        const int b = item / p.n_rt1, rt = item % p.n_rt1;
        const int nb = p1_tiles(p, rt);
        // the item's 128 query rows (rows past R1 read as zeros)
        if (!wait_one(&bars[BAR_A1_EMPTY], (k & 1) ^ 1, ctl)) break;
        mbar_arrive_expect_tx(&bars[BAR_A1_FULL], A1_BYTES);
#pragma unroll
        for (int kb = 0; kb < KB; ++kb)
#pragma unroll
          for (int h = 0; h < BM / 64; ++h)
            tma_load_3d(smem + OFF_A1 + kb * A1_KB + h * 64 * 128, &q1map, &bars[BAR_A1_FULL],
                        kb * 64, rt * BM + h * 64, b);
#pragma unroll 1
        for (int it = 0; it < nb; ++it) {
          const int s = T % S1;
          if (!wait_one(&bars[BAR_EMPTY1 + s], ((T / S1) & 1) ^ 1, ctl)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars[BAR_FULL1 + s], B1_BYTES);
          const bool ctx = it < n_kt_ctx;
          const void* map = ctx ? static_cast<const void*>(&kmap) : static_cast<const void*>(&smap);
          const int row = (ctx ? it : it - n_kt_ctx) * BN1;
          uint8_t* dst = smem + OFF_B1 + s * B1_BYTES;
#pragma unroll
          for (int kb = 0; kb < KB; ++kb)
            tma_load_3d(dst + kb * B1_KB, map, &bars[BAR_FULL1 + s], kb * 64, row, b);
          ++T;
        }
      }
      // every copy issued lands before shared memory is released
      for (uint32_t s = 0; s < S1 && s < T; ++s) {
        const uint32_t last = s + ((T - 1 - s) / S1) * S1;
        wait_drain(&bars[BAR_FULL1 + s], (last / S1) & 1, p.status);
      }
      if (k > 0) wait_drain(&bars[BAR_A1_FULL], (k - 1) & 1, p.status);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================================================ pass-1 MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN1);
      const uint32_t b_base = smem_u32(smem + OFF_B1);
      const uint32_t a_base = smem_u32(smem + OFF_A1);
      uint32_t T = 0, k = 0;
      bool ok = true;
#pragma unroll 1
      for (int item = blockIdx.x; ok && item < p.items1; item += gridDim.x, ++k) {
        const int nb = p1_tiles(p, item % p.n_rt1);
        if (!wait_one(&bars[BAR_A1_FULL], k & 1, ctl)) break;
        tc_fence_after();
#pragma unroll 1
        for (int it = 0; it < nb; ++it, ++T) {
          const int s = T % S1;
          const int g = T % NG1;
          if (!wait_one(&bars[BAR_FULL1 + s], (T / S1) & 1, ctl) ||
              !wait_one(&bars[BAR_SE1 + g], ((T / NG1) & 1) ^ 1, ctl)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + ACC1_COL + g * BN1;
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) {
            const uint64_t ad = sdesc_sw128(a_base + kb * A1_KB);
            const uint64_t bd = sdesc_sw128(b_base + s * B1_BYTES + kb * B1_KB);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16_ss(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0);
          }
          umma_commit(&bars[BAR_SF1 + g]);
          umma_commit(&bars[BAR_EMPTY1 + s]);
        }
        umma_commit(&bars[BAR_A1_EMPTY]);   // A tile free once this item's MMAs are done
      }
      umma_commit(&bars[BAR_DONE1]);
      wait_drain(&bars[BAR_DONE1], 0, p.status);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ============================================================ pass-2 loader
    if (lane == 0) {
      tma_prefetch_desc(&qmap);
      uint32_t T = 0, k = 0;
      bool ok = !stall;
#pragma unroll 1
      for (int item = blockIdx.x; ok && item < p.items2; item += gridDim.x, ++k) {
        const int b = item / p.n_kt2, kt = item % p.n_kt2;
        const int buf = k & 1;
        if (!wait_one(&bars[BAR_A2_EMPTY + buf], ((k >> 1) & 1) ^ 1, ctl)) break;
        mbar_arrive_expect_tx(&bars[BAR_A2_FULL + buf], A2_BYTES);
        uint8_t* adst = smem + OFF_A2 + buf * A2_BYTES;
#pragma unroll
        for (int kb = 0; kb < KB; ++kb)
#pragma unroll
          for (int h = 0; h < BM / 64; ++h)
            tma_load_3d(adst + kb * A2_KB + h * 64 * 128, &kmap, &bars[BAR_A2_FULL + buf],
                        kb * 64, kt * BM + h * 64, b);
#pragma unroll 1
        for (int it = 0; it < nb2; ++it, ++T) {
          const int s = T % S2;
          const uint32_t ph = ((T / S2) & 1) ^ 1;
          if (!wait_one(&bars[BAR_EMPTY2 + s], ph, ctl) ||
              !wait_one(&bars[BAR_LEMPTY2 + s], ph, ctl)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars[BAR_FULL2 + s], B2_BYTES + L2_BYTES);
          uint8_t* dst = smem + OFF_B2 + s * B2_BYTES;
#pragma unroll
          for (int kb = 0; kb < KB; ++kb)
            tma_load_3d(dst + kb * B2_KB, &qmap, &bars[BAR_FULL2 + s], kb * 64, it * BN2, b);
          bulk_load(smem + OFF_L2 + s * L2_BYTES,
                    p.lse_in + static_cast<size_t>(b) * p.R_pad2 + it * BN2, L2_BYTES,
                    &bars[BAR_FULL2 + s]);
        }
      }
      for (uint32_t s = 0; s < S2 && s < T; ++s) {
        const uint32_t last = s + ((T - 1 - s) / S2) * S2;
        wait_drain(&bars[BAR_FULL2 + s], (last / S2) & 1, p.status);
      }
      // k counts the A tiles requested (the last one may have been issued
      // before the loop stopped)
      for (uint32_t i = 0; i < 2 && i < k; ++i) {
        const uint32_t last = i + ((k - 1 - i) / 2) * 2;
        wait_drain(&bars[BAR_A2_FULL + i], (last >> 1) & 1, p.status);
      }
    }
    __syncwarp();
  } else if (warp == 3) {
    // ============================================================ pass-2 MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN2);
      const uint32_t a_base = smem_u32(smem + OFF_A2);
      const uint32_t b_base = smem_u32(smem + OFF_B2);
      uint32_t T = 0, k = 0;
      bool ok = true;
#pragma unroll 1
      for (int item = blockIdx.x; ok && item < p.items2; item += gridDim.x, ++k) {
        const int buf = k & 1;
        if (!wait_one(&bars[BAR_A2_FULL + buf], (k >> 1) & 1, ctl)) break;
        tc_fence_after();
#pragma unroll 1
        for (int it = 0; it < nb2; ++it, ++T) {
          const int s = T % S2;
          const int g = T % NG2;
          if (!wait_one(&bars[BAR_FULL2 + s], (T / S2) & 1, ctl) ||
              !wait_one(&bars[BAR_SE2 + g], ((T / NG2) & 1) ^ 1, ctl)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + ACC2_COL + g * BN2;
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) {
            const uint64_t ad = sdesc_sw128(a_base + buf * A2_BYTES + kb * A2_KB);
            const uint64_t bd = sdesc_sw128(b_base + s * B2_BYTES + kb * B2_KB);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16_ss(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0);
          }
          umma_commit(&bars[BAR_SF2 + g]);
          umma_commit(&bars[BAR_EMPTY2 + s]);
        }
        umma_commit(&bars[BAR_A2_EMPTY + buf]);
      }
      umma_commit(&bars[BAR_DONE2]);
      wait_drain(&bars[BAR_DONE2], 0, p.status);
    }
    __syncwarp();
  } else if (warp < kCtlWarps + 4 * NG1) {
    // ============================================================ pass-1 epilogue
    const int g = (warp - kCtlWarps) >> 2;
    const int quarter = warp & 3;            // TMEM lanes 32*quarter .. +31
    const int lrow = quarter * 32 + lane;    // row within the A tile
    const uint32_t acc =
        tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + ACC1_COL + g * BN1;
    float2* xchg = reinterpret_cast<float2*>(smem + OFF_X1);
    const float c = p.c;
    uint32_t T = 0, k = 0;
#pragma unroll 1
    for (int item = blockIdx.x; item < p.items1; item += gridDim.x, ++k) {
      const int b = item / p.n_rt1, rt = item % p.n_rt1;
      const int nb = p1_tiles(p, rt);
      const int row = rt * BM + lrow;
      const int i_row = row % p.n_in1;
      float m = -INFINITY, l = 0.f;
#pragma unroll 1
      for (int it = (g - static_cast<int>(T % NG1) + NG1) % NG1; it < nb; it += NG1) {
        const uint32_t Tt = T + it;
        if (!wait_warp(&bars[BAR_SF1 + g], (Tt / NG1) & 1, ctl)) break;
        tc_fence_after();
#pragma unroll
        for (int ch = 0; ch < BN1; ch += CH) {
          float v[CH];
          tmem_ld32(acc + ch, v);
          if (ch + CH == BN1) {   // whole accumulator read: hand it back
            tc_fence_before();
            mbar_arrive(&bars[BAR_SE1 + g]);
          }
          if (it < n_kt_ctx) {   // ragged context tail
            const int lim = p.n_c - it * BN1 - ch;
            if (lim < CH) {
#pragma unroll
              for (int j = 0; j < CH; ++j)
                if (j >= lim) v[j] = -INFINITY;
            }
          } else {                // causal self keys: visible iff j' <= i
            const int lim = i_row - (it - n_kt_ctx) * BN1 - ch;
#pragma unroll
            for (int j = 0; j < CH; ++j)
              if (j > lim) v[j] = -INFINITY;
          }
          online_lse(v, c, m, l);
        }
      }
      T += nb;
      float2* xb = xchg + (k & 1) * (NG1 - 1) * BM;
      if (g > 0) xb[(g - 1) * BM + lrow] = make_float2(m, l);
      const bool stop = bar_red_or(1, 4 * NG1 * 32, *abort_flag != 0);
      if (stop) break;
      if (g == 0) {
        float M = m;
#pragma unroll
        for (int o = 0; o < NG1 - 1; ++o) M = fmaxf(M, xb[o * BM + lrow].x);
        float lse = -INFINITY;
        if (M != -INFINITY) {
          float lt = l * ex2_approx(m - M);
#pragma unroll
          for (int o = 0; o < NG1 - 1; ++o) {
            const float2 ml = xb[o * BM + lrow];
            lt += ml.y * ex2_approx(ml.x - M);
          }
          lse = M + lg2_approx(lt);
        }
        float* dst = p.lse_out + static_cast<size_t>(b) * p.R_pad1;
        if (row < p.R_pad1) dst[row] = (row < p.R1) ? lse : INFINITY;
        // rows past the last tile are padding too: never win a pass-2 maximum
        if (rt == p.n_rt1 - 1)
          for (int r = p.n_rt1 * BM + lrow; r < p.R_pad1; r += BM) dst[r] = INFINITY;
      }
    }
  } else {
    // ============================================================ pass-2 epilogue
    const int g = (warp - kCtlWarps - 4 * NG1) >> 2;
    const int quarter = warp & 3;
    const int lrow = quarter * 32 + lane;    // key within the A tile
    const uint32_t acc =
        tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + ACC2_COL + g * BN2;
    float* xchg = reinterpret_cast<float*>(smem + OFF_X2);
    const float c = p.c;
    uint32_t T = 0, k = 0;
#pragma unroll 1
    for (int item = blockIdx.x; item < p.items2; item += gridDim.x, ++k) {
      const int b = item / p.n_kt2, kt = item % p.n_kt2;
      const int key = kt * BM + lrow;
      float* dst = p.scores + static_cast<size_t>(b) * p.n_c + key;
      float s_old = 0.f;
      if (g == 0 && key < p.n_c) s_old = *dst;   // issued early; used after the merge
      float best = -INFINITY;
#pragma unroll 1
      for (int it = (g - static_cast<int>(T % NG2) + NG2) % NG2; it < nb2; it += NG2) {
        const uint32_t Tt = T + it;
        const int st = Tt % S2;
        // The stage's lse2 bytes landed with its full barrier; the stage cannot be
        // refilled before this group releases it, so this phase is still current.
        if (!wait_warp(&bars[BAR_FULL2 + st], (Tt / S2) & 1, ctl)) break;
        if (!wait_warp(&bars[BAR_SF2 + g], (Tt / NG2) & 1, ctl)) break;
        tc_fence_after();
        const float4* L4 = reinterpret_cast<const float4*>(smem + OFF_L2 + st * L2_BYTES);
#pragma unroll
        for (int ch = 0; ch < BN2; ch += CH) {
          float v[CH];
          tmem_ld32(acc + ch, v);
          if (ch + CH == BN2) {
            tc_fence_before();
            mbar_arrive(&bars[BAR_SE2 + g]);
          }
          float b0 = best, b1 = -INFINITY;
#pragma unroll
          for (int j = 0; j < CH; j += 4) {
            const float4 L = L4[(ch + j) / 4];   // same address in every lane: broadcast
            b0 = fmax3(b0, fmaf(v[j + 0], c, -L.x), fmaf(v[j + 1], c, -L.y));
            b1 = fmax3(b1, fmaf(v[j + 2], c, -L.z), fmaf(v[j + 3], c, -L.w));
          }
          best = fmaxf(b0, b1);
        }
        mbar_arrive(&bars[BAR_LEMPTY2 + st]);
      }
      T += nb2;
      float* xb = xchg + (k & 1) * BM;
      if (g == 1) xb[lrow] = best;
      const bool stop = bar_red_or(2, 4 * NG2 * 32, *abort_flag != 0);
      if (stop) break;
      if (g == 0 && key < p.n_c) *dst = fmaxf(s_old, ex2_approx(fmaxf(best, xb[lrow])));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace fused

cudaError_t launch_score_fused(const FusedArgs& a, cudaStream_t s, int* launches) {
  using namespace fused;
  if (a.d != D) return cudaErrorInvalidValue;
  const bool has1 = a.q1 != nullptr, has2 = a.q2 != nullptr;
  if (!has1 && !has2) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(score_fused_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  int dev = 0, n_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;

  Params p{};
  p.scores = a.scores;
  p.status = a.status;
  p.n_c = a.n_c;
  p.c = a.scale * 1.4426950408889634f;
  p.timeout_ns = a.timeout_ns;
  p.test_stall = a.test_stall;
  CUtensorMap kmap, smap, q1map, qmap;
  if (!make_map(&kmap, a.k_ctx, a.B, a.n_c, D, 64)) return cudaErrorInvalidValue;
  smap = kmap;
  q1map = kmap;
  qmap = kmap;
  if (has1) {
    p.lse_out = a.lse_out;
    p.n_in1 = a.n_in1;
    p.R1 = a.G * a.n_in1;
    p.R_pad1 = a.R_pad1;
    p.n_rt1 = (p.R1 + BM - 1) / BM;
    p.items1 = a.B * p.n_rt1;
    if (!make_map(&smap, a.k_self1, a.B, a.n_in1, D, 64) ||
        !make_map(&q1map, a.q1, a.B, p.R1, D, 64))
      return cudaErrorInvalidValue;
  } else {
    p.n_in1 = 1;
    p.n_rt1 = 1;
  }
  if (has2) {
    p.lse_in = a.lse_in;
    p.R2 = a.G * a.n_in2;
    p.R_pad2 = a.R_pad2;
    p.n_kt2 = (a.n_c + BM - 1) / BM;
    p.items2 = a.B * p.n_kt2;
    if (!make_map(&qmap, a.q2, a.B, p.R2, D, BN2)) return cudaErrorInvalidValue;
  } else {
    p.n_kt2 = 1;
  }
  const int grid = std::max(1, std::min(n_sm, std::max(p.items1, p.items2)));
  score_fused_kernel<<<grid, kThreads, SMEM_ALLOC, s>>>(kmap, smap, q1map, qmap, p);
  e = cudaGetLastError();
  if (e == cudaSuccess && launches) *launches += 1;
  return e;
}

}  // namespace kvzip
