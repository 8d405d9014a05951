// PTX wrappers shared by the warp-specialised kernels (tensor-core FFN and
// decode FFN): shared-memory mbarriers, TMA tile loads, elected issue, the
// async-proxy fence, and the bounded wait every pipeline wait goes through.
// Host side: the driver's tensor-map encoder and the SM count.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace moe {
namespace tma {

constexpr uint64_t WAIT_NS = 2000000000ull;  // a pipeline wait gives up after about two seconds

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t *b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint64_t *b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t *b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes) : "memory");
}
// TMA tile loads (no multicast): completion counted in bytes on `bar`.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *tm, int c0, int c1, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *tm, int c0, int c1, int c2, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}
// One lane of a converged warp (the lowest), chosen by elect.sync: the
// issue idiom for tcgen05 and TMA instructions, whose operands then stay in
// uniform registers.
__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n .reg .b32 r;\n .reg .pred p;\n elect.sync r|p, 0xffffffff;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(pred));
  return pred != 0;
}
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Bounded wait on phase `parity` of `bar`: false (and *abort set, and the
// error word flagged) after WAIT_NS, or as soon as another role set *abort
// unless `drain` is set (a drain wait only gives up on its own time limit, so
// resources are never released under work still in flight). %globaltimer is
// read only every 256 polls (the first time after 256): a wait that ends
// soon never pays for the timer read.
static __device__ __noinline__ bool wait_bounded(int32_t *abort, uint64_t *bar, uint32_t parity, int32_t *err,
                                                 bool drain = false) {
  uint64_t t0 = 0;
  for (uint32_t spin = 1;; ++spin) {
    if (mbar_try(bar, parity)) return true;
    if ((spin & 255) == 0) {
      if (!drain && *(volatile int32_t *)abort) return false;
      const uint64_t now = globaltimer();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > WAIT_NS) {
        atomicExch(abort, 1);
        flag_error(err, MOE_DEVERR_TIMEOUT);
        return false;
      }
    }
  }
}

}  // namespace tma

// Host: number of SMs of the current device (cached per device), and
// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library; nullptr if unavailable).
int sm_count();
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

}  // namespace moe
