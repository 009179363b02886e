// tc_common.cuh -- small device helpers shared by the tensor-core kernels.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "carve_internal.cuh"
#include "sm100_ptx.cuh"

namespace carve {
namespace tc {

__device__ __forceinline__ float ldbf(const uint8_t* p) {
  return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
}
__device__ __forceinline__ void stbf(uint8_t* p, float x) {
  *reinterpret_cast<__nv_bfloat16*>(p) = __float2bfloat16_rn(x);
}
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float sigm(float x) {
  return __fdividef(1.0f, 1.0f + __expf(-x));
}
__device__ __forceinline__ void bar_named(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// 8 fp32 values -> one 16-byte chunk of bf16 at `p`.
__device__ __forceinline__ void st_chunk(uint8_t* p, const float* x) {
  uint4 u;
  u.x = pack2(x[0], x[1]);
  u.y = pack2(x[2], x[3]);
  u.z = pack2(x[4], x[5]);
  u.w = pack2(x[6], x[7]);
  *reinterpret_cast<uint4*>(p) = u;
}

constexpr long long kSpinCycles = 1LL << 31;  // ~1 s before a wait gives up

// Bounded wait on an mbarrier phase.  On expiry: record CARVE_ERR_TIMEOUT
// and the wait site in the workspace header, raise the CTA abort flag and
// return (the caller keeps its barrier sequence; the block loop exits at
// its next check of the flag).
__device__ __forceinline__ void wait_bar(uint64_t* bar, uint32_t parity,
                                         uint32_t where,
                                         volatile uint32_t* abort_flag,
                                         WsHeader* hdr) {
  const long long t0 = clock64();
  while (!*abort_flag) {
    if (ptx::mbar_try_wait(bar, parity)) return;
    if (clock64() - t0 > kSpinCycles) {
      atomicExch(&hdr->status, (uint32_t)CARVE_ERR_TIMEOUT);
      hdr->where = where;
      *abort_flag = 1;
    }
  }
}

}  // namespace tc
}  // namespace carve
