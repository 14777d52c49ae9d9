// Pieces shared by the tcgen05 kernels: smem/instruction descriptors, bounded
// waits with a CTA-wide abort flag, and host-side tensor-map helpers.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"

namespace monarch {

constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s per wait
constexpr int kSmemBudget = 227 * 1024 - 1024;   // dynamic smem incl. 1 KB alignment slack

// ---------------------------------------------------------------- descriptors
// tcgen05 shared-memory matrix descriptor, K-major, given swizzle code
// (2 = 128B, 6 = 32B) and stride between 8-row groups (bytes).
__device__ __forceinline__ uint64_t make_sdesc(uint32_t saddr, uint32_t sbo_bytes, uint32_t swz) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)1 << 16;                              // leading byte offset (unused, K-major swizzled)
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFF) << 32;    // stride byte offset
  d |= (uint64_t)1 << 46;                              // descriptor version (sm_100)
  d |= (uint64_t)swz << 61;                            // layout / swizzle type
  return d;
}

// Same with an explicit leading byte offset (MN-major swizzled layouts: the byte distance
// between consecutive 64-element M/N blocks).
__device__ __forceinline__ uint64_t make_sdesc_lbo(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                                   uint32_t swz) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)swz << 61;
  return d;
}

// Instruction descriptor: kind::f16, A = B = bf16, D = fp32, both K-major.
__host__ __device__ constexpr uint32_t make_idesc(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// Wait for the phase of `bar` with the given parity.  Gives up (returns false)
// when another thread of the CTA has set *abort_flag, or after kWaitLimitNs, in
// which case it sets *abort_flag and records kStatusTimeout in the device status.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, int* abort_flag,
                                              int* status) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  while (true) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*(volatile int*)abort_flag) return false;
    if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) {
      *(volatile int*)abort_flag = 1;
      atomicExch(status, kStatusTimeout);
      return false;
    }
  }
}

// Wait for the MMA issuer's final commit (every MMA of this CTA has completed).  A wait that runs
// out records the timeout like wait_or_abort does, so the host sees MONARCH_ERR_TIMEOUT instead of
// an incomplete result with status OK.
__device__ __forceinline__ void wait_mma_done(uint64_t* bar, int* abort_flag, int* status) {
  if (!ptx::mbar_wait_bounded(bar, 0, kWaitLimitNs)) {
    *(volatile int*)abort_flag = 1;
    atomicExch(status, kStatusTimeout);
  }
}

// Warp-uniform version: lane 0 waits, the outcome is broadcast to the warp.
__device__ __forceinline__ bool warp_wait_or_abort(int lane, uint64_t* bar, uint32_t parity,
                                                   int* abort_flag, int* status) {
  bool r = true;
  if (lane == 0) r = wait_or_abort(bar, parity, abort_flag, status);
  return __shfl_sync(0xffffffffu, r ? 1 : 0, 0) != 0;
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  }
  return fn;
}

// 2-D bf16 tensor map over a row-major (outer x inner) matrix.
inline bool make_map_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                        uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  EncodeTiledFn enc = get_encode();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 tensor map: dims[0] contiguous; strides (bytes) of dims 1 and 2 may be in any order.
inline bool make_map_3d(CUtensorMap* m, const void* base, const uint64_t dims[3], const uint64_t strides[2],
                        const uint32_t box[3], CUtensorMapSwizzle swz) {
  EncodeTiledFn enc = get_encode();
  if (enc == nullptr) return false;
  cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
  cuuint64_t st[2] = {strides[0], strides[1]};
  cuuint32_t b[3] = {box[0], box[1], box[2]};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), d, st, b, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

}  // namespace monarch
