// Allocation-free variant of the A8W4 linear (qgemm_a8w4_f32_noalloc).
//
// Some callers cannot hand this library a workspace: a plugin running inside
// a host framework that owns the device allocator and exposes none to it, or
// a latency-critical serving loop that must not call cudaMalloc after
// start-up (cudaMalloc may synchronise the device and stall every stream).
// For them this entry point keeps its scratch — the per-row int8 activations
// with their scales and zero-points — in a fixed array in device global
// memory that the library declares itself.  Every GPU that loads the library
// holds that array (kScratchBytes) until the process exits.
//
// The arithmetic is that of qgemm_a8w4_f32, and the results agree with it
// within the A8W4 tolerance.  M == 1 runs the same fused GEMV (its scratch
// lives in shared memory, so the array is not touched).  M > 1 always runs
// the CUDA-core GEMM on activations quantized into the array, where the
// workspace entry point may take the tensor-core kernel instead; the two
// combine the same exact group dots in a different float order.
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "qg_internal.cuh"

namespace qg {

int launch_quantize_rows(int M, int K, const float* x, int64_t ldx, int8_t* q, int64_t ldq,
                         float* scale, int32_t* zp, cudaStream_t st);
int launch_a8w4_gemv(int N, int K, const float* x, const void* packed, const float* bias,
                     float lo, float hi, float* y, int8_t* q_out, float* scale_out,
                     int32_t* zp_out, bool scale_bf16, cudaStream_t st);
int launch_a8w4_gemm_simt(int M, int N, int K, const int8_t* q, const float* sA,
                          const int32_t* zA, const void* packed, const float* bias, float lo,
                          float hi, float* y, int64_t ldy, bool scale_bf16, cudaStream_t st);
int device_setup_status();

namespace {

// Limits of the fixed scratch: M*K int8 activation codes (4 MiB) and one
// f32 scale plus one int32 zero-point per row (up to 8192 rows).
constexpr size_t kMaxCodes = size_t(4) << 20;
constexpr int kMaxRows = 8192;
constexpr size_t kScaleOff = kMaxCodes;
constexpr size_t kZpOff = kScaleOff + size_t(kMaxRows) * 4;
constexpr size_t kScratchBytes = kZpOff + size_t(kMaxRows) * 4;
constexpr int kFusedGemvMaxK = 65536;  // same dispatch rule as qgemm_a8w4_f32
constexpr int kSimtMaxK = 25600;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kScratchBytes];

// The host-side name g_noalloc_scratch is only a stand-in for the symbol; the
// kernels need its device address, looked up once per device (with that
// device current) and published with release/acquire ordering, so a thread
// that sees the pointer also sees the completed lookup.
constexpr int kMaxDevices = 64;
std::atomic<uint8_t*> g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu;

int scratch_for_current_device(uint8_t** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QG_ERR_NO_DEVICE;
  uint8_t* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (!p) {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
    if (!p) {
      void* sym = nullptr;
      cudaError_t e = cudaGetSymbolAddress(&sym, g_noalloc_scratch);
      if (e != cudaSuccess || !sym) {
        cudaGetLastError();
        return QG_ERR_CUDA;
      }
      p = static_cast<uint8_t*>(sym);
      g_scratch_ptr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return QG_OK;
}

}  // namespace
}  // namespace qg

using namespace qg;

extern "C" int qgemm_a8w4_f32_noalloc(int M, int N, int K, const float* x, int64_t ldx,
                                      const void* packed_w, const float* bias, float clamp_min,
                                      float clamp_max, float* y, int64_t ldy, void* stream) {
  if (M < 0 || N <= 0 || K <= 0 || ldx < K || ldy < N) return QG_ERR_INVALID_ARG;
  if (K % 32) return QG_ERR_UNSUPPORTED;
  if (!(clamp_min <= clamp_max)) return QG_ERR_INVALID_ARG;
  if (M == 0) return QG_OK;
  if (!x || !packed_w || !y) return QG_ERR_INVALID_ARG;
  if (((uintptr_t)packed_w & 15) != 0) return QG_ERR_MISALIGNED;
  if (((uintptr_t)x & 3) || ((uintptr_t)y & 3) || (bias && ((uintptr_t)bias & 3)))
    return QG_ERR_MISALIGNED;
  int rc = device_setup_status();
  if (rc != QG_OK) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  if (M == 1 && K <= kFusedGemvMaxK)  // the fused GEMV keeps its scratch in shared memory
    return launch_a8w4_gemv(N, K, x, packed_w, bias, clamp_min, clamp_max, y, nullptr, nullptr,
                            nullptr, false, st);
  if (K > kSimtMaxK) return QG_ERR_UNSUPPORTED;
  if (M > kMaxRows || (size_t)M * (size_t)K > kMaxCodes) return QG_ERR_WORKSPACE;
  uint8_t* s = nullptr;
  rc = scratch_for_current_device(&s);
  if (rc != QG_OK) return rc;
  // Every byte read below is written first by the quantization kernel in the
  // same stream order, so no clearing is needed between calls.
  int8_t* q = (int8_t*)s;
  float* sA = (float*)(s + kScaleOff);
  int32_t* zA = (int32_t*)(s + kZpOff);
  rc = launch_quantize_rows(M, K, x, ldx, q, K, sA, zA, st);
  if (rc != QG_OK) return rc;
  return launch_a8w4_gemm_simt(M, N, K, q, sA, zA, packed_w, bias, clamp_min, clamp_max, y, ldy,
                               false, st);
}
