// Untiled bulk copies and bulk async-groups (the copy engine behind TMA),
// as inline PTX: row copies of the gather and the TMA stores of the weight
// gradients use them.
#pragma once

#include "common.cuh"

namespace moe {

// Untiled bulk copies (the copy engine behind TMA).  Addresses 16-byte
// aligned, sizes a multiple of 16 bytes.
// global -> this CTA's shared memory, completing `bytes` on `bar`
__device__ __forceinline__ void bulk_load_1d(void* smem_dst, const void* gsrc, uint32_t bytes,
                                             uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"((uint64_t)gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// shared memory -> global, tracked by the thread's bulk async-group
__device__ __forceinline__ void bulk_store_1d(void* gdst, const void* smem_src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"((uint64_t)gdst),
               "r"(smem_u32(smem_src)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// at most N of this thread's bulk groups still reading shared memory
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_group_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

}  // namespace moe
