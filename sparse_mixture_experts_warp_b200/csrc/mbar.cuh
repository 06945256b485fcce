// mbarrier and bulk-copy helpers shared by the kernels that stage operands in shared memory
// (inline PTX, sm_100a).  Every wait is bounded by %globaltimer: a wait that gives up records
// an error code in the library's device error word and raises the CTA's abort flag, so a lost
// arrival ends the kernel with MOE_ERR_TIMEOUT instead of hanging the GPU.
#pragma once

#include <stdint.h>

namespace moe {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// kCluster: acquire at cluster scope, for barriers that the peer CTA of a pair arrives on.
template <bool kCluster = false>
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  if (kCluster)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
  return ok != 0;
}
// Bounded wait for the phase of parity `parity` to complete.  Returns false when it gave up:
// on its time limit (which records `code` and raises the CTA's abort flag) or, when
// honor_abort, as soon as another role has aborted.  Drain waits pass honor_abort = false so
// that they keep waiting (bounded) for work already in flight.
template <bool kCluster = false>
__device__ __noinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                       int* err, int code, uint64_t limit,
                                       bool honor_abort = true) {
  if (mbar_try_wait<kCluster>(bar, parity)) return true;
  const uint64_t t0 = gtimer();
  while (!mbar_try_wait<kCluster>(bar, parity)) {
    if (honor_abort && *abort_flag) return false;
    if (gtimer() - t0 > limit) {
      *abort_flag = 1;
      atomicCAS(err, 0, code);
      return false;
    }
  }
  return true;
}

// Untiled bulk copy global -> shared (both 16-byte aligned, bytes a multiple of 16), counted on
// the mbarrier's transaction count.  Source: this GPU's memory only.
__device__ __forceinline__ void bulk_load(void* dst_smem, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst_smem)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

}  // namespace moe
