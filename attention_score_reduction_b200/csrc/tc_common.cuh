// Pieces shared by the tensor-core scorer kernels: bounded mbarrier waits with
// a CTA-wide abort flag, whole-row TMEM loads, and the host-side TMA map encoder.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kvzip_internal.h"
#include "sm100_ptx.cuh"

namespace kvzip {

constexpr uint64_t kDrainTimeoutNs = 1000000000ull;

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
__device__ __forceinline__ void tmem_ld_tile(uint32_t taddr, float (&v)[96]) { tmem_ld96(taddr, v); }
__device__ __forceinline__ void tmem_ld_tile(uint32_t taddr, float (&v)[64]) { tmem_ld64(taddr, v); }
__device__ __forceinline__ void tmem_ld_tile(uint32_t taddr, float (&v)[48]) { tmem_ld48(taddr, v); }
__device__ __forceinline__ void tmem_ld_tile(uint32_t taddr, float (&v)[32]) { tmem_ld32(taddr, v); }

// ------------------------------------------------------------------ host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn get_encode_fn() {
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
inline bool make_map(CUtensorMap* m, const void* base, int units, int rows, int d, int box_rows) {
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

}  // namespace kvzip
