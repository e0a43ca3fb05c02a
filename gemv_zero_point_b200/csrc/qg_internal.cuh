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
// Dynamic activation quantization (MNN BatchAsyDynamicQuant / BatchSym-
// DynamicQuant; ONNX QuantizeLinear rounding, half to even).  All float32,
// one IEEE rounding per operation, no contraction.
//   asymmetric: rmin = min(0, min x), rmax = max(0, max x),
//     scale = (rmax-rmin)/255 (1 if 0), inv = 1/scale,
//     zp = clamp(rne(-128 - rmin*inv), -128, 127), q = clamp(rne(x*inv)+zp)
//   symmetric: amax = max|x|, scale = amax/127, inv = 127/amax (both 1 when
//     amax is 0), zp = 0, q = clamp(rne(x*inv), -127, 127)
// ---------------------------------------------------------------------------
struct RowQuant {
  float scale, inv;
  int zp;
};

__device__ __forceinline__ RowQuant row_quant_params(float rmin, float rmax) {
  RowQuant r;
  float s = __fdiv_rn(__fsub_rn(rmax, rmin), 255.0f);
  if (s == 0.0f) s = 1.0f;
  r.scale = s;
  r.inv = __fdiv_rn(1.0f, s);
  float t = __fsub_rn(-128.0f, __fmul_rn(rmin, r.inv));
  int z = __float2int_rn(t);
  r.zp = min(max(z, -128), 127);
  return r;
}

__device__ __forceinline__ int quant_one(float x, const RowQuant& r) {
  int v = __float2int_rn(__fmul_rn(x, r.inv)) + r.zp;
  return min(max(v, -128), 127);
}

__device__ __forceinline__ RowQuant row_quant_params_sym(float amax) {
  RowQuant r;
  r.scale = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 127.0f);
  r.inv = amax == 0.0f ? 1.0f : __fdiv_rn(127.0f, amax);
  r.zp = 0;
  return r;
}

__device__ __forceinline__ int quant_one_sym(float x, const RowQuant& r) {
  return min(max(__float2int_rn(__fmul_rn(x, r.inv)), -127), 127);
}

// ---------------------------------------------------------------------------
// One call of the tensor-core A8W4 path (a8w4_tc.cu).  Activation rows are
// plain rows x[M][ldx], or (conv) the unrolled rows of an NHWC image.  mode
// 0: per-row asymmetric, 1: per-32-block asymmetric, 2: per-row symmetric
// quantization; wzero selects asymmetric weights (f32 zeros [N][K/32]).
// ---------------------------------------------------------------------------
struct A8W4TcCall {
  int64_t M;
  int N, K;
  const float* x;
  int64_t ldx;
  bool conv;
  int H, W, Cin, KH, KW, sh, sw, ph, pw, OH, OW;
  int mode;
  const void* packed;
  bool scale_bf16;
  const float* wzero;
  const float* bias;
  float lo, hi;
  float* y;
  int64_t ldy;
  int8_t* q_out;
  float* scale_out;
  int32_t* zp_out;
};
bool a8w4_tc_supported(int64_t M, int N, int K);
size_t a8w4_tc_workspace_bytes(int64_t M, int N, int K);
int launch_a8w4_tc_call(const A8W4TcCall& c, void* ws, size_t ws_bytes, cudaStream_t st);

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
