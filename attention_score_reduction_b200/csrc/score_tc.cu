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
// One skeleton serves both passes.  The A tiles of a CTA never change.  Where
// TMEM has room (pass 1, and d = 256) they live in tensor memory: each epilogue
// thread copies its own row there once, before any MMA (tcgen05.st), and every
// MMA reads A from TMEM and only B from shared memory.  Pass 2 at d = 128 uses
// wider B tiles instead (N = 128, a quarter fewer tiles, each with its own
// barrier waits and commits; measured 62 against 66 ms per 128K chunk): the four
// 128-column accumulators fill TMEM, so its A tiles are loaded by TMA into
// shared memory and the MMAs read both operands there (tile sizes in TcCfg).
//   warp 0      : TMA producer: the A tiles when they live in shared memory, then
//                 a STAGES-deep ring of B tiles (+ pass-2 lse2 tiles)
//   warps 1, 2  : one MMA-issuing thread each, for A tile 0 and A tile 1 (warp 1
//                 also allocates TMEM).  tcgen05.mma issue stalls until the
//                 previous MMA is nearly done, so one thread's barrier waits and
//                 fences between batches idle the tensor pipe (measured: 113
//                 instead of 64 cycles per 128x128x16 MMA); with two issuers one
//                 feeds the pipe while the other waits.
//   warps 3..18 : four 128-thread epilogue groups, one per (A tile, accumulator
//                 buffer); with A in TMEM the even group of each A tile first
//                 copies the A rows there.  A group drains its BN-column
//                 accumulator in CH-column TMEM loads, so the tile's B tiles
//                 alternate between two groups (four epilogue warps per
//                 scheduler: the epilogue math is latency-bound with two).
// Work items are (unit, 256-row block of A).  Pass 2 with A in shared memory
// runs one persistent CTA per SM over the items: the B ring and the barrier
// phases run on from item to item, the next item's A tiles are prefetched into
// L2 and loaded once the issuers release the current ones.  Elsewhere each CTA
// takes one item.
// TMEM map (512 columns): the A tiles when they live there (D/2 columns each),
// then the (tile, buffer) accumulators.
// Every wait is bounded; on timeout the CTA records KVZIP_ERR_TIMEOUT in the
// status word, drains its in-flight copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "kvzip_internal.h"
#include "sm100_ptx.cuh"
#include "tc_common.cuh"

namespace kvzip {

// Tile configuration per head dimension and pass.
template <int D, bool PASS2>
struct TcCfg;
template <>
struct TcCfg<128, false> {           // pass 1 at d = 128
  static constexpr int BN = 96;      // rows per B tile (N of the MMA)
  static constexpr int STAGES = 6;   // B ring depth
  static constexpr bool A_SMEM = false;  // A tiles in TMEM (tcgen05.st once per CTA)
  static constexpr int CH = 48;          // accumulator columns per TMEM load
};
template <>
struct TcCfg<128, true> {            // pass 2 at d = 128
  static constexpr int BN = 128;
  static constexpr int STAGES = 4;
  static constexpr bool A_SMEM = true;   // A tiles in shared memory (TMA): TMEM holds 4 x 128
  static constexpr int CH = 32;          // accumulator columns
};
template <bool PASS2>
struct TcCfg<256, PASS2> {
  static constexpr int BN = 64;
  static constexpr int STAGES = 5;
  static constexpr bool A_SMEM = false;
  static constexpr int CH = 32;
};

constexpr int kEpiThreads = 512;     // four 128-thread epilogue groups
constexpr int kThreads = 32 * (1 + 2) + kEpiThreads;   // producer, 2 MMA issuers, epilogue
constexpr int kBM = 128;             // rows per A tile (M of the MMA)
constexpr int kATiles = 2;           // A tiles per CTA
// Pass 1: out of every 8 pairs of exponentials, this many are evaluated by
// polynomial on the FMA pipe instead of the MUFU unit (16 ex2 per clock per SM,
// half the tensor core's 32 logits per clock at d = 128).
#ifndef KVZIP_POLY_PAIRS
#define KVZIP_POLY_PAIRS 2
#endif
constexpr int kPolyPairs = KVZIP_POLY_PAIRS;

template <int D, bool PASS2>
struct TcLayout {
  using Cfg = TcCfg<D, PASS2>;
  static constexpr int BN = Cfg::BN;
  static constexpr int STAGES = Cfg::STAGES;
  static constexpr int KB = D / 64;                      // 128-byte K blocks per row
  static constexpr bool A_SMEM = Cfg::A_SMEM;
  static constexpr int B_KB_BYTES = BN * 128;
  static constexpr int B_BYTES = KB * B_KB_BYTES;
  static constexpr int L_BYTES = BN * 4;                 // pass 2: lse2 of one B tile
  static constexpr int A_KB_BYTES = kBM * 128;
  static constexpr int A_TILE_BYTES = KB * A_KB_BYTES;   // one A tile in shared memory
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + (A_SMEM ? kATiles * A_TILE_BYTES : 0);
  static constexpr int OFF_L = OFF_B + STAGES * B_BYTES;
  static constexpr int OFF_BAR = OFF_L + STAGES * L_BYTES;
  // barriers: a_full, b_full[S], b_empty[S], s_full[2][2], s_empty[2][2], mma_done, l_empty[S],
  // a_empty
  static constexpr int N_BARS = 1 + 2 * STAGES + 8 + 1 + STAGES + 1;
  static constexpr int OFF_XCHG = OFF_BAR + 8 * N_BARS;  // parity merge, float2 per row, 2 items
  static constexpr int OFF_MISC = OFF_XCHG + 2 * kATiles * kBM * 8;  // tmem base, abort flag
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int CH = Cfg::CH;                     // accumulator columns per TMEM load
  static constexpr int SMEM_ALLOC = BYTES + 1024;        // slack for 1024-B alignment
  static constexpr int A_COLS = A_SMEM ? 0 : D / 2;      // TMEM columns of one A tile
  static constexpr int ACC0 = kATiles * A_COLS;          // first accumulator column
  static constexpr int TMEM_COLS = 512;
  static_assert(ACC0 + kATiles * 2 * BN <= TMEM_COLS, "TMEM over-committed");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "invalid MMA N");
  static_assert(SMEM_ALLOC <= 232448, "exceeds 227 KB of shared memory");
  static_assert((B_KB_BYTES % 1024) == 0 && (A_KB_BYTES % 1024) == 0,
                "swizzle atoms must stay 1024-B aligned");
  static_assert(BN % CH == 0, "tile not a multiple of the TMEM load");
  static_assert(!A_SMEM || BN == kBM, "A tiles are loaded with the B maps' box height");
  // Pass 2 copies whole BN-row tiles of lse2 up to the padded row count, and
  // pass 1 pads it in steps of its CTA height: both must divide the pad.
  static_assert(kRowPad % BN == 0 && kRowPad % (kATiles * kBM) == 0,
                "row pad of the log-sum-exp buffer must divide by every tile height");
};

struct TcParams {
  const uint16_t* a_ptr;   // A operand rows: q ([B][R][d]) in pass 1, k_ctx ([B][n_c][d]) in pass 2
  float* scores;
  float* lse2;
  uint32_t* status;
  int B, G, n_in, n_c, R, R_pad;
  float c;            // scale * log2(e)
  uint64_t timeout_ns;
  int test_stall;     // test hook: the loader issues no copies, so every wait runs out
  uint32_t* hist;     // pass 2 (maxima) only, or null: round-1 histogram of the new scores
};

// SUM (pass 2 only): column sums of the probabilities instead of maxima (the
// rebuttal's average-aggregation ablation; sum and average rank identically).
template <int D, bool PASS2, bool SUM = false>
__global__ void __launch_bounds__(kThreads, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap bmap0,
                    const __grid_constant__ CUtensorMap bmap1,
                    const __grid_constant__ CUtensorMap amap,   // A rows, box kBM (A_SMEM only)
                    const TcParams p) {
  using Lay = TcLayout<D, PASS2>;
  constexpr int BN = Lay::BN;
  constexpr int STAGES = Lay::STAGES;
  constexpr int KB = Lay::KB;
  constexpr int CH = Lay::CH;

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
  uint64_t* a_empty = bars + 2 + 3 * STAGES + 8;    // an item's A tiles free again
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(smem + Lay::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work items: item w is unit w / items_x, A rows (w % items_x) * 256 ...
  // On the ordinary grid (items_x, B) each CTA takes one item; on a persistent
  // grid (pass 2 with A in shared memory, every item with two A tiles) a CTA
  // takes items blockIdx.x, blockIdx.x + gridDim.x, ... and its pipelines run on
  // across them: stages, buffers and barrier phases follow the CTA's running
  // count of B tiles, and the A tiles of the next item are loaded as soon as
  // the MMAs of the previous one are done with them.
  const int a_extent = PASS2 ? p.n_c : p.R;                 // rows of the A operand
  const int items_x = (a_extent + kATiles * kBM - 1) / (kATiles * kBM);
  const int n_items = items_x * p.B;
  const int w_first = blockIdx.y * gridDim.x + blockIdx.x;
  const int w_step = gridDim.x * gridDim.y;
  // with A in TMEM a CTA always has one item (its A rows are stored once), and
  // the item loops below reduce to their body
  const int w_end = Lay::A_SMEM ? n_items : w_first + 1;
  auto next_item = [&](int w) { return Lay::A_SMEM ? w + w_step : w_end; };
  const int n_kt_ctx = PASS2 ? 0 : (p.n_c + BN - 1) / BN;
  struct Item {
    int b, ix, a_row0, nA, n_b;
  };
  auto item_at = [&](int w) {
    Item it;
    it.b = w / items_x;
    it.ix = w % items_x;
    it.a_row0 = it.ix * (kATiles * kBM);
    it.nA = min(kATiles, (a_extent - it.a_row0 + kBM - 1) / kBM);
    if (PASS2) {
      it.n_b = (p.R + BN - 1) / BN;
    } else {
      const int r_last = min(it.a_row0 + kATiles * kBM, p.R) - 1;
      const int i_max =
          (r_last / p.n_in != it.a_row0 / p.n_in) ? p.n_in - 1 : r_last % p.n_in;
      it.n_b = n_kt_ctx + (i_max + 1 + BN - 1) / BN;
    }
    return it;
  };
  // barrier counts follow the first item; a CTA with several items has two A
  // tiles in every one of them
  const int nA = item_at(w_first).nA;

  if (threadIdx.x == 0) {
    // A in TMEM: every thread of every active group stores its row; A in shared
    // memory: one TMA transaction
    mbar_init(a_full, Lay::A_SMEM ? 1 : nA * kBM);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], nA);   // one commit per active MMA issuer
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], kBM);
    }
    mbar_init(mma_done, nA);
    // every thread of every active epilogue group releases each lse2 stage
    for (int s = 0; s < STAGES; ++s) mbar_init(&l_empty[s], nA * kBM);
    mbar_init(a_empty, nA);         // the issuers are done with an item's A tiles
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
      tma_prefetch_desc(&bmap0);
      if (!PASS2) tma_prefetch_desc(&bmap1);
      if (Lay::A_SMEM) tma_prefetch_desc(&amap);
      const bool stall = p.test_stall != 0;
      uint32_t g = 0;      // B tiles issued by this CTA
      int a_loads = 0;     // A loads issued by this CTA
      bool ok = !stall;
      int k = 0;
#pragma unroll 1
      for (int w = w_first; ok && w < w_end; w = next_item(w), ++k) {
        const Item itm = item_at(w);
        // the item's A tiles (rows past the operand read as zeros): on a CTA's
        // first item before its B tiles; later, after the item's first B tiles,
        // once the issuers have released the previous item's
        const int a_at = (k == 0) ? 0 : min(STAGES, itm.n_b - 1);
        if (Lay::A_SMEM && next_item(w) < w_end) {
          // the next item's A tiles into L2 now, so that their load between the
          // two items comes from L2 rather than HBM
          const Item nxt = item_at(next_item(w));
          for (int t = 0; t < nxt.nA; ++t)
            for (int kb = 0; kb < KB; ++kb)
              tma_prefetch_l2_3d(&amap, kb * 64, nxt.a_row0 + t * kBM, nxt.b);
        }
#pragma unroll 1
        for (int it = 0; it < itm.n_b; ++it, ++g) {
          if (Lay::A_SMEM && it == a_at) {
            if (k > 0 && !wait_one(a_empty, (k - 1) & 1, ctl)) { ok = false; break; }
            mbar_arrive_expect_tx(a_full, itm.nA * Lay::A_TILE_BYTES);
            for (int t = 0; t < itm.nA; ++t)
              for (int kb = 0; kb < KB; ++kb)
                tma_load_3d(smem + Lay::OFF_A + t * Lay::A_TILE_BYTES + kb * Lay::A_KB_BYTES,
                            &amap, a_full, kb * 64, itm.a_row0 + t * kBM, itm.b);
            ++a_loads;
          }
          const int s = g % STAGES;
          const uint32_t ph = (g / STAGES) & 1;
          if (!wait_one(&b_empty[s], ph ^ 1, ctl)) { ok = false; break; }
          if (PASS2 && !wait_one(&l_empty[s], ph ^ 1, ctl)) { ok = false; break; }
          const void* map = &bmap0;
          int row = it * BN;
          if (!PASS2 && it >= n_kt_ctx) {
            map = &bmap1;
            row = (it - n_kt_ctx) * BN;
          }
          // pass 2: the tile's BN normalisers must lie inside the unit's padded rows
          const uint32_t l_bytes = (PASS2 && in_bounds(row + BN <= p.R_pad)) ? Lay::L_BYTES : 0u;
          mbar_arrive_expect_tx(&b_full[s], Lay::B_BYTES + l_bytes);
          uint8_t* dst = smem + Lay::OFF_B + s * Lay::B_BYTES;
          for (int kb = 0; kb < KB; ++kb)
            tma_load_3d(dst + kb * Lay::B_KB_BYTES, map, &b_full[s], kb * 64, row, itm.b);
          if (l_bytes)  // the row normalisers of this query tile ride on the same barrier
            bulk_load(smem + Lay::OFF_L + s * Lay::L_BYTES,
                      p.lse2 + static_cast<size_t>(itm.b) * p.R_pad + row, l_bytes, &b_full[s]);
        }
      }
      // Drain: every copy this CTA started must land before shared memory is released.
      const uint32_t issued = g;
      for (uint32_t s = 0; s < STAGES && s < issued; ++s) {
        const uint32_t last = s + ((issued - 1 - s) / STAGES) * STAGES;
        wait_drain(&b_full[s], (last / STAGES) & 1, p.status);
      }
      if (Lay::A_SMEM && a_loads > 0) wait_drain(a_full, (a_loads - 1) & 1, p.status);
    }
    __syncwarp();
  } else if (warp <= kATiles) {
    // ================================================================ MMA issuers
    const int t = warp - 1;                 // A tile (and epilogue group) of this issuer
    if (lane == 0 && t < nA) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN);
      const uint32_t b_base = smem_u32(smem + Lay::OFF_B);
      const uint32_t a_tmem = tmem_base + t * Lay::A_COLS;
      const uint32_t a_sbase = smem_u32(smem + Lay::OFF_A + t * Lay::A_TILE_BYTES);
      uint32_t g = 0;      // B tiles consumed by this CTA
      bool ok = true;
      int k = 0;
#pragma unroll 1
      for (int w = w_first; ok && w < w_end; w = next_item(w), ++k) {
        const int n_b = item_at(w).n_b;
        if (!wait_one(a_full, k & 1, ctl)) break;
        tc_fence_after();
#pragma unroll 1
        for (int it = 0; it < n_b; ++it, ++g) {
          const int s = g % STAGES;
          const int buf = g & 1;
          if (!wait_one(&b_full[s], (g / STAGES) & 1, ctl)) { ok = false; break; }
          if (!wait_one(&s_empty[t * 2 + buf], ((g >> 1) & 1) ^ 1, ctl)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + Lay::ACC0 + (t * 2 + buf) * BN;
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) {
            const uint64_t bd = sdesc_sw128(b_base + s * Lay::B_BYTES + kb * Lay::B_KB_BYTES);
            if (Lay::A_SMEM) {
              const uint64_t ad = sdesc_sw128(a_sbase + kb * Lay::A_KB_BYTES);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)   // K = 16 per MMA: 32 B of each row
                umma_bf16_ss(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0);
            } else {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)   // K = 16 per MMA: 8 TMEM columns of A, 32 B of B
                umma_bf16_ts(d_tmem, a_tmem + (kb * 4 + kk) * 8, bd + 2 * kk, idesc,
                             (kb | kk) != 0);
            }
          }
          umma_commit(&s_full[t * 2 + buf]);
          umma_commit(&b_empty[s]);
        }
        if (ok) umma_commit(a_empty);   // this item's A tile is free once its MMAs finish
      }
      // Drain: all MMAs issued by this thread complete before TMEM is freed.
      umma_commit(mma_done);
      wait_drain(mma_done, 0, p.status);
    }
    __syncwarp();
  } else {
    // ================================================================ epilogue groups
    // Group g = (A tile t, parity par): drains accumulator buffer (t, par), i.e.
    // the B tiles of A tile t whose running index has parity par.  Four groups
    // of four warps give each scheduler four epilogue warps to hide MUFU / TMEM
    // latency.
    const int g_ep = (warp - 1 - kATiles) >> 2;
    const int t = g_ep >> 1, par = g_ep & 1;
    const int quarter = warp & 3;           // TMEM lanes 32*quarter .. +31
    const int lrow = quarter * 32 + lane;   // row of the A tile
    const float c = p.c;
    const uint32_t acc_lane = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                              Lay::ACC0 + (t * 2 + par) * BN;
    uint32_t g0 = 0;     // B tiles of the CTA's earlier items
    int k = 0;
#pragma unroll 1
    for (int w = w_first; w < w_end; w = next_item(w), ++k) {
      const Item itm = item_at(w);
      const int b = itm.b, n_b = itm.n_b;
      const int arow = itm.a_row0 + t * kBM + lrow;
      // the parity merge slot alternates between items
      float2* xchg = reinterpret_cast<float2*>(smem + Lay::OFF_XCHG) +
                     (k & 1) * (kATiles * kBM) + t * kBM + lrow;
      const int it0 = par ^ static_cast<int>(g0 & 1);   // first tile of this buffer
      if (t < itm.nA) {
        if (!Lay::A_SMEM && par == 0) {
          // ---- this thread's A row into its TMEM lane (zeros past the operand's rows)
          const uint4* src = reinterpret_cast<const uint4*>(
              p.a_ptr + (static_cast<size_t>(b) * a_extent + arow) * D);
          const bool in = arow < a_extent;
          const uint32_t a_lane = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                  t * Lay::A_COLS;
#pragma unroll
          for (int h = 0; h < D / 128; ++h) {   // 64 columns (128 bf16) per store
            uint32_t wv[64];
#pragma unroll
            for (int v4 = 0; v4 < 16; ++v4) {
              const uint4 x = in ? __ldg(src + h * 16 + v4) : make_uint4(0, 0, 0, 0);
              wv[4 * v4 + 0] = x.x;
              wv[4 * v4 + 1] = x.y;
              wv[4 * v4 + 2] = x.z;
              wv[4 * v4 + 3] = x.w;
            }
            tmem_st64(a_lane + h * 64, wv);
          }
          tc_fence_before();
          mbar_arrive(a_full);
        }
        bool stop;
        if (!PASS2) {
          // ---------------- pass 1: online log-sum-exp over the row (this parity's tiles)
          const int i_row = arow % p.n_in;
          float m = -INFINITY, l = 0.f;
#pragma unroll 1
          for (int it = it0; it < n_b; it += 2) {
            const uint32_t gt = g0 + it;
            if (!wait_warp(&s_full[t * 2 + par], (gt >> 1) & 1, ctl)) break;
            tc_fence_after();
#pragma unroll 1
            for (int ch = 0; ch < BN; ch += CH) {
              float v[CH];
              tmem_ld_tile(acc_lane + ch, v);
              if (ch + CH == BN) {           // whole accumulator read: hand it back
                tc_fence_before();
                mbar_arrive(&s_empty[t * 2 + par]);
              }
              // masks: ragged context tail, causal self keys
              if (it < n_kt_ctx) {
                const int lim = p.n_c - it * BN - ch;
                if (lim < CH) {
#pragma unroll
                  for (int j = 0; j < CH; ++j)
                    if (j >= lim) v[j] = -INFINITY;
                }
              } else {
                const int lim = i_row - (it - n_kt_ctx) * BN - ch;   // visible iff j' <= i
#pragma unroll
                for (int j = 0; j < CH; ++j)
                  if (j > lim) v[j] = -INFINITY;
              }
              // chunk maximum, 8 independent chains
              float mx[8];
#pragma unroll
              for (int q = 0; q < 8; ++q) mx[q] = fmaxf(v[2 * q], v[2 * q + 1]);
#pragma unroll
              for (int j = 16; j < CH; j += 16) {
#pragma unroll
                for (int q = 0; q < 8; ++q) mx[q] = fmax3(mx[q], v[j + 2 * q], v[j + 2 * q + 1]);
              }
              const float mxa = fmax3(mx[0], mx[1], mx[2]), mxb = fmax3(mx[3], mx[4], mx[5]);
              const float m_new = fmaxf(m, fmax3(mxa, mxb, fmaxf(mx[6], mx[7])) * c);
              const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
              // x = c*s - m in packed pairs; of every 8 pairs, kPolyPairs take 2^x on
              // the FMA pipe and the rest on the MUFU unit.
              const float2 c2 = make_float2(c, c);
              const float2 nm2 = make_float2(-m_use, -m_use);
              float2 acc[4];
#pragma unroll
              for (int q = 0; q < 4; ++q) acc[q] = make_float2(0.f, 0.f);
#pragma unroll
              for (int j = 0; j < CH; j += 16) {
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
                  acc[q & 3] = fadd2(acc[q & 3], e);
                }
              }
              const float2 s4 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
              l = fmaf(l, ex2_approx(m - m_use), s4.x + s4.y);
              m = m_new;
            }
          }
          // merge the two parities' (m, l) of this row; parity 0 writes lse2.  The
          // barrier's OR gives both groups the same view of the abort flag.
          if (par == 1) *xchg = make_float2(m, l);
          stop = named_barrier_or(1 + t, 2 * kBM, *abort_flag != 0);
          if (par == 0 && !stop && arow < p.R_pad) {
            const float2 o = *xchg;
            const float M = fmaxf(m, o.x);
            float lse;
            if (M == -INFINITY) {
              lse = -INFINITY;
            } else {
              const float lt = l * ex2_approx(m - M) + o.y * ex2_approx(o.x - M);
              lse = M + lg2_approx(lt);
            }
            p.lse2[static_cast<size_t>(b) * p.R_pad + arow] = (arow < p.R) ? lse : INFINITY;
          }
        } else {
          // ---------------- pass 2: running max over query rows of c*s - lse2
          // (or, for SUM, the running sum of 2^(c*s - lse2))
          float best = SUM ? 0.f : -INFINITY;
#pragma unroll 1
          for (int it = it0; it < n_b; it += 2) {
            const uint32_t gt = g0 + it;
            const int st = gt % STAGES;
            // The stage's lse2 bytes landed with b_full; the stage cannot be refilled
            // before this group releases l_empty, so this phase is still the latest.
            if (!wait_warp(&b_full[st], (gt / STAGES) & 1, ctl)) break;
            if (!wait_warp(&s_full[t * 2 + par], (gt >> 1) & 1, ctl)) break;
            tc_fence_after();
            const float4* L4 =
                reinterpret_cast<const float4*>(smem + Lay::OFF_L + st * Lay::L_BYTES);
#pragma unroll 1
            for (int ch = 0; ch < BN; ch += CH) {
              float v[CH];
              tmem_ld_tile(acc_lane + ch, v);
              if (ch + CH == BN) {
                tc_fence_before();
                mbar_arrive(&s_empty[t * 2 + par]);
              }
              if (SUM) {
                float a0 = 0.f, a1 = 0.f;
#pragma unroll
                for (int j = 0; j < CH; j += 4) {
                  const float4 L = L4[(ch + j) / 4];
                  a0 += ex2_approx(fmaf(v[j + 0], c, -L.x)) + ex2_approx(fmaf(v[j + 1], c, -L.y));
                  a1 += ex2_approx(fmaf(v[j + 2], c, -L.z)) + ex2_approx(fmaf(v[j + 3], c, -L.w));
                }
                best += a0 + a1;
              } else {
                // min over rows of lse2 - c*s (packed pairs), i.e. minus the running max
                const float2 nc2 = make_float2(-c, -c);
                float w0 = -best, w1 = INFINITY;
#pragma unroll
                for (int j = 0; j < CH; j += 4) {
                  const float4 L = L4[(ch + j) / 4];   // same address in every lane: broadcast
                  const float2 x01 =
                      ffma2(make_float2(v[j + 0], v[j + 1]), nc2, make_float2(L.x, L.y));
                  const float2 x23 =
                      ffma2(make_float2(v[j + 2], v[j + 3]), nc2, make_float2(L.z, L.w));
                  w0 = fmin3(w0, x01.x, x01.y);
                  w1 = fmin3(w1, x23.x, x23.y);
                }
                best = -fminf(w0, w1);
              }
            }
            mbar_arrive(&l_empty[st]);
          }
          if (par == 1) xchg->x = best;
          stop = named_barrier_or(1 + t, 2 * kBM, *abort_flag != 0);
          if (par == 0 && !stop && arow < p.n_c && in_bounds(b < p.B)) {
            float* dst = p.scores + static_cast<size_t>(b) * p.n_c + arow;
            if (SUM) {
              *dst += best + xchg->x;
            } else {
              const float s_new = fmaxf(*dst, ex2_approx(fmaxf(best, xchg->x)));
              *dst = s_new;
              if (p.hist) score_hist_add(p.hist, s_new);
            }
          }
        }
        if (stop) break;
      } else if (!PASS2 && par == 0) {
        // A tile beyond the query rows: pad the log-sum-exp buffer with +inf so
        // that padded columns never win the pass-2 maximum.
        if (arow < p.R_pad) p.lse2[static_cast<size_t>(b) * p.R_pad + arow] = INFINITY;
      }
      if (!PASS2 && itm.ix == items_x - 1) {
        // Pass 2 reads whole BN-row tiles of lse2, up to the padded row count:
        // rows past the last A block are padding too.
        for (int r = items_x * kATiles * kBM + (threadIdx.x - 32 * (1 + kATiles)); r < p.R_pad;
             r += kEpiThreads)
          p.lse2[static_cast<size_t>(b) * p.R_pad + r] = INFINITY;
      }
      g0 += n_b;
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

cudaError_t bounds_flag_score(unsigned int* out) { return take_bounds_flag(out); }

template <int D>
static cudaError_t launch_tc(const ScoreArgs& a, cudaStream_t s, int* launches) {
  using L1 = TcLayout<D, false>;
  using L2 = TcLayout<D, true>;
  // The shared-memory limit is a per-device function attribute; set it each call.
  cudaError_t e = cudaFuncSetAttribute(score_tc_kernel<D, false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       L1::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(score_tc_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           L2::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(score_tc_kernel<D, true, true>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, L2::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  TcParams p;
  p.a_ptr = static_cast<const uint16_t*>(a.q);
  p.scores = a.scores;
  p.lse2 = a.lse2;
  p.status = a.status;
  p.B = a.B;
  p.G = a.G;
  p.n_in = a.n_in;
  p.n_c = a.n_c;
  p.R = a.R;
  p.R_pad = a.R_pad;
  p.c = a.scale * 1.4426950408889634f;
  p.timeout_ns = a.timeout_ns;
  p.test_stall = a.test_stall;
  p.hist = nullptr;

  // Maps of box height BN (per pass).  With A in shared memory (BN = kBM) a map
  // of the A operand serves the A tiles; with A in TMEM its rows are copied from
  // global memory by the epilogue threads and the A map is not read.
  if (a.passes & 1) {
    CUtensorMap kmap, smap;
    if (!make_map(&kmap, a.k_ctx, a.B, a.n_c, D, L1::BN) ||
        !make_map(&smap, a.k_self, a.B, a.n_in, D, L1::BN))
      return cudaErrorInvalidValue;
    dim3 g1((a.R + kATiles * kBM - 1) / (kATiles * kBM), a.B);
    score_tc_kernel<D, false><<<g1, kThreads, L1::SMEM_ALLOC, s>>>(kmap, smap, kmap, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (launches) *launches += 1;
  }
  if (!(a.passes & 2)) return cudaSuccess;

  // pass 2: A = context key tiles, B = query row tiles
  CUtensorMap kmap2, qmap2;
  if (!make_map(&kmap2, a.k_ctx, a.B, a.n_c, D, L2::BN) ||
      !make_map(&qmap2, a.q, a.B, a.R, D, L2::BN))
    return cudaErrorInvalidValue;
  p.a_ptr = static_cast<const uint16_t*>(a.k_ctx);
  p.hist = a.sum_aggregation ? nullptr : a.score_hist;
  const int items_x = (a.n_c + kATiles * kBM - 1) / (kATiles * kBM);
  dim3 g2(items_x, a.B);
  // With A tiles in shared memory and two of them in every item (n_c a multiple
  // of 256, or a last block of more than 128 keys), one persistent CTA per SM
  // works through the items in turn: the per-CTA start (barriers, TMEM, the A
  // load, the pipeline fill) and end (drain, exit) were ~5.5 us of a ~70 us CTA.
  const int tail = a.n_c % (kATiles * kBM);
  if (L2::A_SMEM && (tail == 0 || tail > kBM)) {
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int64_t n_items = static_cast<int64_t>(items_x) * a.B;
    g2 = dim3(static_cast<unsigned>(std::min<int64_t>(n_items, sms)), 1);
  }
  if (a.sum_aggregation)
    score_tc_kernel<D, true, true><<<g2, kThreads, L2::SMEM_ALLOC, s>>>(qmap2, qmap2, kmap2, p);
  else
    score_tc_kernel<D, true><<<g2, kThreads, L2::SMEM_ALLOC, s>>>(qmap2, qmap2, kmap2, p);
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
