// Device helpers shared by the routing kernels (sm_100a).
//
// Bounded waits: every spin in this library polls %globaltimer and gives up
// after a limit, recording MOE_ERR_DEVICE_TIMEOUT in the status word that
// starts each workspace, so a wait that cannot complete returns instead of
// hanging the GPU.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "moe_route.h"

namespace moe {

constexpr long long kDefaultTimeoutNs = 1000LL * 1000 * 1000;  // 1 s; a healthy wait takes microseconds

// Header at the start of every workspace that has device-side waits.
struct WsHeader {
  int32_t status;              // MOE_OK or a MOE_ERR_DEVICE_* code
  uint32_t ticket;             // last-block-done counter (reductions)
  uint32_t pad[14];            // keeps the header 64 bytes
};
static_assert(sizeof(WsHeader) == 64, "workspace header is 64 bytes");

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void record_timeout(WsHeader* h) {
  atomicCAS(&h->status, MOE_OK, MOE_ERR_DEVICE_TIMEOUT);
}

__device__ __forceinline__ void record_bounds(WsHeader* h) {
  atomicCAS(&h->status, MOE_OK, MOE_ERR_DEVICE_BOUNDS);
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// ---- ordered keys: float -> uint32 whose unsigned order is the float order ----
__device__ __forceinline__ uint32_t ordered_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Packed (key, expert) for a max-reduction: larger key wins, then lower expert.
__device__ __forceinline__ unsigned long long pack_key(float f, int e) {
  return ((unsigned long long)ordered_key(f) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)e);
}
__device__ __forceinline__ int packed_expert(unsigned long long p) {
  return (int)(0xFFFFFFFFu - (uint32_t)(p & 0xFFFFFFFFull));
}

__device__ __forceinline__ unsigned long long shfl_xor_u64(unsigned mask, unsigned long long v, int off) {
  uint32_t lo = (uint32_t)v, hi = (uint32_t)(v >> 32);
  lo = __shfl_xor_sync(mask, lo, off);
  hi = __shfl_xor_sync(mask, hi, off);
  return ((unsigned long long)hi << 32) | lo;
}

// a / b rounded to nearest even, given y = 1/b rounded to nearest (one IEEE
// division shared by every a over the same b).  q0 = a*y is within 1.5 ulp of
// a/b; the correction q1 = q0 + (a - b*q0)*y (two fused multiply-adds) is
// within half an ulp plus a tiny fraction of one, so q1 is a faithful
// quotient, the remainder a - b*q1 is exact, and q1 + (a - b*q1)*y rounded to
// nearest is the correctly rounded quotient (Markstein, "Computation of
// elementary functions on the IBM RISC System/6000 processor", IBM J. Res.
// Dev. 34(1), 1990).  Away from underflow only: callers keep a >= 2^-60 and
// 2^-20 <= b <= 2^20 (positive), and take the IEEE division otherwise.
__device__ __forceinline__ float div_rn_by_recip(float a, float b, float y) {
  const float q0 = a * y;
  const float q1 = fmaf(fmaf(-q0, b, a), y, q0);
  return fmaf(fmaf(-q1, b, a), y, q1);
}
constexpr float kDivMinNum = 0x1p-60f;  // div_rn_by_recip's range: a >= kDivMinNum,
constexpr float kDivMinDen = 0x1p-20f;  // kDivMinDen <= b <= kDivMaxDen
constexpr float kDivMaxDen = 0x1p20f;

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(((uint32_t)b) << 16);
}

__device__ __forceinline__ float load_as_f32(const void* p, int dtype, size_t i) {
  if (dtype == MOE_BF16) return bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(p)[i]);
  return reinterpret_cast<const float*>(p)[i];
}

__device__ __forceinline__ void store_from_f32(void* p, int dtype, size_t i, float v) {
  if (dtype == MOE_BF16)
    reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<float*>(p)[i] = v;
}

// ---- mbarrier + 1-D bulk copy (TMA engine) ----
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Bounded wait for the phase with the given parity; false on timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, long long timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if ((long long)(globaltimer_ns() - t0) > timeout_ns) return false;
  }
  return true;
}

// Global -> shared bulk copy of `bytes` (multiple of 16, both addresses
// 16-byte aligned) completing on `bar`.  No multicast.
__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gmem_src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

__host__ __device__ constexpr int ceil_div(int a, int b) { return (a + b - 1) / b; }
// ---- programmatic dependent launch ----
// At kernel entry: let the next grid in the stream be scheduled (its blocks
// start as this grid's blocks retire), then wait until the previous grid has
// completed and its writes are visible; no global memory is touched before.
// Both are no-ops for a launch without the attribute.
__device__ __forceinline__ void pdl_entry() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Launch with programmatic stream serialization allowed (plain launch if the
// attribute is refused).
template <typename... Params, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e != cudaSuccess) {
    cudaGetLastError();
    cfg.numAttrs = 0;
    e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  }
  return e;
}


}  // namespace moe
