// Internal helpers shared by the library's CUDA sources: status reporting,
// launch checks, and thin inline-PTX wrappers for the sm_100a features the
// kernels use (mbarrier, bulk/tensor copies, tcgen05).  Nothing here is part
// of the C ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/qgemm.h"

namespace qg {

// ---------------------------------------------------------------------------
// Device status word (one per device, defined in api.cu).  Kernels record the
// first error they meet with atomicCAS; the host reads it via
// qg_device_status().
// ---------------------------------------------------------------------------
int* status_word();  // device address of this device's status word, or NULL

__device__ __forceinline__ void record_error(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Bounded waits: a spin that has not completed after this many polls (each
// poll of try_wait suspends for up to a hardware time limit) gives up, records
// QG_ERR_TIMEOUT and lets the kernel finish.  Generous: a healthy pipeline
// completes in far fewer.
constexpr uint32_t kSpinLimit = 1u << 20;

inline int launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? QG_OK : QG_ERR_CUDA;
}

int num_sms();  // multiprocessor count of the current device (cached)

inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ inline int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ inline int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }
inline int64_t round_up(int64_t a, int64_t b) { return cdiv(a, b) * b; }

// ---------------------------------------------------------------------------
// Shared-memory addresses and mbarriers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of `bar` to complete, at most `limit` polls.
// Returns false (after recording QG_ERR_TIMEOUT) if it never completed.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* status,
                                          uint32_t limit = kSpinLimit) {
  for (uint32_t i = 0; i < limit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
  }
  record_error(status, QG_ERR_TIMEOUT);
  return false;
}

// Non-blocking variant for single-thread roles (TMA producer, MMA issuer):
// polls with mbarrier.test_wait, so the thread reacts as soon as the phase
// completes instead of after a suspension; bounded like mbar_wait.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_poll(uint64_t* bar, uint32_t parity, int* status,
                                          uint32_t limit = kSpinLimit) {
  for (uint32_t i = 0; i < (limit << 4); ++i) {
    if (mbar_test(bar, parity)) return true;
  }
  record_error(status, QG_ERR_TIMEOUT);
  return false;
}

// Test hook (qg_test_arm_stall): which kernel family the next launch should
// stall, consumed by that launch.  Kernels given a stall skip one pipeline
// stage and wait with kStallSpinLimit polls, so their bounded waits run out
// quickly.
enum StallTarget { kStallNone = 0, kStallInt8Gemm = 1, kStallA8W4TC = 2 };
bool take_stall(int target);  // true once after qg_test_arm_stall(target)
constexpr uint32_t kStallSpinLimit = 1u << 12;

// ---------------------------------------------------------------------------
// Bulk copies (TMA engine)
// ---------------------------------------------------------------------------
// Non-tensor bulk copy global -> shared, completing `bytes` on `bar`.
// Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst_smem)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// 2-D tiled tensor load (no multicast) into shared memory.
__device__ __forceinline__ void tma_load_2d(void* dst_smem, const void* tmap, int32_t x, int32_t y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cta.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst_smem)),
      "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// Generic-proxy writes to shared memory made visible to the async proxy
// (tensor-core reads of operands written by ordinary stores).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Integer dot products
// ---------------------------------------------------------------------------
// sum_b a.u8[b] * b.s8[b] + c  (a unsigned bytes, b signed bytes)
__device__ __forceinline__ int dp4a_us(uint32_t a, int b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

}  // namespace qg
