// C ABI entry points: argument checks, workspace layout, dispatch to the
// kernels, status codes and the per-device status word.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "qg_internal.cuh"

namespace qg {

// ---- kernels implemented in the other translation units ----
int launch_quantize_rows(int M, int K, const float* x, int64_t ldx, int8_t* q, int64_t ldq,
                         float* scale, int32_t* zp, cudaStream_t st);
int launch_pack_w4(int N, int K, const int8_t* w, int64_t ldw, const float* sw, void* packed,
                   bool scale_bf16, cudaStream_t st);
int launch_a8w4_gemv(int N, int K, const float* x, const void* packed, const float* bias,
                     float lo, float hi, float* y, int8_t* q_out, float* scale_out,
                     int32_t* zp_out, bool scale_bf16, cudaStream_t st);
int launch_a8w4_gemm_simt(int M, int N, int K, const int8_t* q, const float* sA,
                          const int32_t* zA, const void* packed, const float* bias, float lo,
                          float hi, float* y, int64_t ldy, bool scale_bf16, cudaStream_t st);
int launch_a8w4_gemv_actblock(int N, int K, const float* x, const void* packed, const float* bias,
                              float lo, float hi, float* y, int8_t* q_out, float* scale_out,
                              int32_t* zp_out, cudaStream_t st);
int launch_a8w4_gemv_asym(int N, int K, const float* x, const void* packed, const float* bias,
                          float lo, float hi, float* y, int8_t* q_out, float* scale_out,
                          int32_t* zp_out, cudaStream_t st);
int launch_quantize_rows_sym(int M, int K, const float* x, int64_t ldx, int8_t* q, int64_t ldq,
                             float* scale, int32_t* zp, cudaStream_t st);
int launch_im2col_quantize(int Nb, int H, int W, int Cin, int KH, int KW, int sh, int sw, int ph,
                           int pw, const float* x, bool symmetric, int8_t* q, float* scale,
                           int32_t* zp, cudaStream_t st);
int setup_a8w4_gemv();
int setup_a8w4_gemm_simt();
int i8gemm_setup();
int a8w4_tc_setup();

int i8gemm_pack_b(int K, int N, const int8_t* B, int64_t ldb, void* packed, cudaStream_t st);
size_t i8gemm_pack_b_bytes(int K, int N);
size_t i8gemm_packed_workspace_bytes(int M, int K);
int i8gemm_run_packed(int M, int N, int K, const int8_t* A, int64_t lda, const void* packed_b,
                      int8_t* C, int64_t ldc, const qg_requant_t& rq, int32_t* acc_out,
                      int64_t ld_acc, void* ws, size_t ws_bytes, cudaStream_t st);
size_t conv_pack_w_bytes(int Cout, int K);
int conv_pack_w(int Cout, int K, const int8_t* w, void* packed, cudaStream_t st);
int conv_run_packed(int Nb, int H, int W, int Cin, int Cout, int KH, int KW, int sh, int sw,
                    int ph, int pw, const int8_t* x, const void* packed_w, int8_t* y,
                    const qg_requant_t& rq, int32_t* acc_out, cudaStream_t st);
size_t conv_workspace_bytes(int Nb, int H, int W, int Cin, int Cout, int KH, int KW, int sh,
                            int sw, int ph, int pw);
int conv_run(int Nb, int H, int W, int Cin, int Cout, int KH, int KW, int sh, int sw, int ph,
             int pw, const int8_t* x, const int8_t* w, int8_t* y, const qg_requant_t& rq,
             int32_t* acc_out, void* ws, size_t ws_bytes, cudaStream_t st);

// ---- per-device state ----
static __device__ int g_status_word;

namespace {
constexpr int kMaxDevices = 64;
struct DeviceState {
  bool ready = false;
  int sms = 0;
  int* status = nullptr;
  int setup_rc = QG_OK;
};
DeviceState g_dev[kMaxDevices];
std::mutex g_mu;

DeviceState* current_state() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  DeviceState& s = g_dev[dev];
  if (s.ready) return &s;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!s.ready) {
    int major = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&s.sms, cudaDevAttrMultiProcessorCount, dev);
    void* p = nullptr;
    if (major != 10 || cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) {
      cudaGetLastError();
      s.setup_rc = QG_ERR_NO_DEVICE;
    } else {
      s.status = static_cast<int*>(p);
      int rc = setup_a8w4_gemv();
      if (rc == QG_OK) rc = setup_a8w4_gemm_simt();
      if (rc == QG_OK) rc = i8gemm_setup();
      if (rc == QG_OK) rc = a8w4_tc_setup();
      s.setup_rc = rc;
    }
    s.ready = true;
  }
  return &s;
}
}  // namespace

int* status_word() {
  DeviceState* s = current_state();
  return s ? s->status : nullptr;
}

int num_sms() {
  DeviceState* s = current_state();
  return (s && s->sms > 0) ? s->sms : 148;
}

static int device_ready() {
  DeviceState* s = current_state();
  if (!s) return QG_ERR_NO_DEVICE;
  return s->setup_rc;
}

// Per-device set-up status for entry points defined in other files.
int device_setup_status() { return device_ready(); }

// One-shot stall armed by qg_test_arm_stall: the next launch of the named
// kernel family takes it (and only that launch).
static std::atomic<int> g_stall_armed{kStallNone};

bool take_stall(int target) {
  int expected = target;
  return target != kStallNone && g_stall_armed.compare_exchange_strong(expected, kStallNone);
}

}  // namespace qg

using namespace qg;

// ---------------------------------------------------------------------------
// Status helpers
// ---------------------------------------------------------------------------
extern "C" const char* qg_status_string(int status) {
  switch (status) {
    case QG_OK: return "QG_OK";
    case QG_ERR_INVALID_ARG: return "QG_ERR_INVALID_ARG: invalid argument";
    case QG_ERR_MISALIGNED: return "QG_ERR_MISALIGNED: pointer alignment not met";
    case QG_ERR_OVERFLOW_BOUND: return "QG_ERR_OVERFLOW_BOUND: K*65025 + |bias| exceeds INT32_MAX";
    case QG_ERR_UNSUPPORTED: return "QG_ERR_UNSUPPORTED: parameters not supported";
    case QG_ERR_CUDA: return "QG_ERR_CUDA: CUDA runtime or launch error";
    case QG_ERR_TIMEOUT: return "QG_ERR_TIMEOUT: a bounded device-side wait ran out";
    case QG_ERR_WORKSPACE: return "QG_ERR_WORKSPACE: workspace missing or too small";
    case QG_ERR_NO_DEVICE: return "QG_ERR_NO_DEVICE: no sm_100 device is current";
    default: return "QG_ERR_UNKNOWN";
  }
}

extern "C" int qg_version(void) { return QG_API_VERSION; }

extern "C" int qg_device_status(int reset) {
  int rc = device_ready();
  if (rc != QG_OK) return rc;
  if (cudaDeviceSynchronize() != cudaSuccess) return QG_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, status_word(), sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return QG_ERR_CUDA;
  if (reset && v != 0) {
    if (cudaMemset(status_word(), 0, sizeof(int)) != cudaSuccess) return QG_ERR_CUDA;
  }
  return v;
}

extern "C" int qg_test_arm_stall(int which) {
  if (which != kStallNone && which != kStallInt8Gemm && which != kStallA8W4TC)
    return QG_ERR_INVALID_ARG;
  g_stall_armed.store(which);
  return QG_OK;
}

extern "C" int qg_requant_params(double ratio, int32_t* m0, int32_t* shift) {
  if (!m0 || !shift) return QG_ERR_INVALID_ARG;
  if (!(ratio > 0.0 && ratio < 1.0) || !isfinite(ratio)) return QG_ERR_UNSUPPORTED;
  int e = 0;
  double f = frexp(ratio, &e);           // ratio = f * 2^e, f in [0.5, 1)
  int64_t q = (int64_t)floor(f * 2147483648.0 + 0.5);  // f*2^31 is exact
  if (q == (int64_t)1 << 31) {
    q >>= 1;
    e += 1;
  }
  const int s = -e;
  if (s < 0 || s > 31) return QG_ERR_UNSUPPORTED;
  *m0 = (int32_t)q;
  *shift = s;
  return QG_OK;
}

// ---------------------------------------------------------------------------
// Argument checks shared by the INT8 entry points
// ---------------------------------------------------------------------------
static bool aligned(const void* p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

static int check_requant(const qg_requant_t* rq, int K) {
  if (!rq) return QG_ERR_INVALID_ARG;
  if (rq->a_zero_point < -128 || rq->a_zero_point > 127) return QG_ERR_INVALID_ARG;
  if (rq->b_zero_point < -128 || rq->b_zero_point > 127) return QG_ERR_INVALID_ARG;
  if (rq->out_zero_point < -128 || rq->out_zero_point > 127) return QG_ERR_INVALID_ARG;
  if (rq->clamp_min < -128 || rq->clamp_max > 127 || rq->clamp_min > rq->clamp_max)
    return QG_ERR_INVALID_ARG;
  if (rq->per_channel) {
    if (!rq->multiplier || !rq->shift) return QG_ERR_INVALID_ARG;
  } else {
    if (rq->multiplier0 < 0 || rq->shift0 < 0 || rq->shift0 > 31) return QG_ERR_INVALID_ARG;
  }
  if (rq->bias && rq->bias_abs_max < 0) return QG_ERR_INVALID_ARG;
  // [QG] section 4: K*65025 + |bias| must fit INT32
  const int64_t bound = (int64_t)K * 65025 + (rq->bias ? (int64_t)rq->bias_abs_max : 0);
  if (bound > (int64_t)INT32_MAX) return QG_ERR_OVERFLOW_BOUND;
  return QG_OK;
}

// ---------------------------------------------------------------------------
// INT8 GEMM
// ---------------------------------------------------------------------------
extern "C" size_t qgemm_pack_b_s8_bytes(int K, int N) {
  if (K <= 0 || N <= 0) return 0;
  return i8gemm_pack_b_bytes(K, N);
}

extern "C" int qgemm_pack_b_s8(int K, int N, const int8_t* B, int64_t ldb, void* packed_b,
                               size_t packed_bytes, void* stream) {
  if (K <= 0 || N <= 0 || !B || !packed_b || ldb < N) return QG_ERR_INVALID_ARG;
  if (!aligned(packed_b, 128)) return QG_ERR_MISALIGNED;
  if (packed_bytes < i8gemm_pack_b_bytes(K, N)) return QG_ERR_WORKSPACE;
  int rc = device_ready();
  if (rc != QG_OK) return rc;
  return i8gemm_pack_b(K, N, B, ldb, packed_b, (cudaStream_t)stream);
}

extern "C" size_t qgemm_s8s8_packed_workspace_bytes(int M, int K) {
  if (M <= 0 || K <= 0) return 0;
  return i8gemm_packed_workspace_bytes(M, K);
}

extern "C" size_t qgemm_s8s8_workspace_bytes(int M, int N, int K) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  return round_up(i8gemm_pack_b_bytes(K, N), 256) + i8gemm_packed_workspace_bytes(M, K);
}

static int check_gemm_args(int M, int N, int K, const int8_t* A, int64_t lda, int8_t* C,
                           int64_t ldc, const qg_requant_t* rq, int32_t* acc_out,
                           int64_t ld_acc) {
  if (M < 0 || N <= 0 || K <= 0) return QG_ERR_INVALID_ARG;
  if (M > 0 && (!A || !C)) return QG_ERR_INVALID_ARG;
  if (lda < K || ldc < N) return QG_ERR_INVALID_ARG;
  if (acc_out && ld_acc < N) return QG_ERR_INVALID_ARG;
  if (acc_out && !aligned(acc_out, 4)) return QG_ERR_MISALIGNED;
  return check_requant(rq, K);
}

extern "C" int qgemm_s8s8_requant_packed(int M, int N, int K, const int8_t* A, int64_t lda,
                                         const void* packed_b, int8_t* C, int64_t ldc,
                                         const qg_requant_t* rq, int32_t* acc_out,
                                         int64_t ld_acc, void* workspace,
                                         size_t workspace_bytes, void* stream) {
  int rc = check_gemm_args(M, N, K, A, lda, C, ldc, rq, acc_out, ld_acc);
  if (rc != QG_OK) return rc;
  if (!packed_b) return QG_ERR_INVALID_ARG;
  if (!aligned(packed_b, 128)) return QG_ERR_MISALIGNED;
  if (workspace && !aligned(workspace, 256)) return QG_ERR_MISALIGNED;
  if (M == 0) return QG_OK;
  rc = device_ready();
  if (rc != QG_OK) return rc;
  return i8gemm_run_packed(M, N, K, A, lda, packed_b, C, ldc, *rq, acc_out, ld_acc, workspace,
                           workspace_bytes, (cudaStream_t)stream);
}

extern "C" int qgemm_s8s8_requant(int M, int N, int K, const int8_t* A, int64_t lda,
                                  const int8_t* B, int64_t ldb, int8_t* C, int64_t ldc,
                                  const qg_requant_t* rq, int32_t* acc_out, int64_t ld_acc,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_gemm_args(M, N, K, A, lda, C, ldc, rq, acc_out, ld_acc);
  if (rc != QG_OK) return rc;
  if (!B || ldb < N) return QG_ERR_INVALID_ARG;
  if (M == 0) return QG_OK;
  if (!workspace) return QG_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return QG_ERR_MISALIGNED;
  const size_t pb = round_up(i8gemm_pack_b_bytes(K, N), 256);
  if (workspace_bytes < pb + i8gemm_packed_workspace_bytes(M, K)) return QG_ERR_WORKSPACE;
  rc = device_ready();
  if (rc != QG_OK) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  rc = i8gemm_pack_b(K, N, B, ldb, workspace, st);
  if (rc != QG_OK) return rc;
  return i8gemm_run_packed(M, N, K, A, lda, workspace, C, ldc, *rq, acc_out, ld_acc,
                           (char*)workspace + pb, workspace_bytes - pb, st);
}

// ---------------------------------------------------------------------------
// INT8 convolution
// ---------------------------------------------------------------------------
extern "C" size_t qconv2d_s8_workspace_bytes(int Nb, int H, int W, int Cin, int Cout, int KH,
                                             int KW, int stride_h, int stride_w, int pad_h,
                                             int pad_w) {
  if (Nb <= 0 || H <= 0 || W <= 0 || Cin <= 0 || Cout <= 0 || KH <= 0 || KW <= 0 ||
      stride_h <= 0 || stride_w <= 0 || pad_h < 0 || pad_w < 0)
    return 0;
  return conv_workspace_bytes(Nb, H, W, Cin, Cout, KH, KW, stride_h, stride_w, pad_h, pad_w);
}

// Checks shared by both conv entry points (everything but the weights).
static int conv_args(int Nb, int H, int W, int Cin, int Cout, int KH, int KW, int stride_h,
                     int stride_w, int pad_h, int pad_w, const int8_t* x, const int8_t* y,
                     const qg_requant_t* rq, int32_t* acc_out) {
  if (Nb <= 0 || H <= 0 || W <= 0 || Cin <= 0 || Cout <= 0 || KH <= 0 || KW <= 0 ||
      stride_h <= 0 || stride_w <= 0 || pad_h < 0 || pad_w < 0)
    return QG_ERR_INVALID_ARG;
  if (!x || !y) return QG_ERR_INVALID_ARG;
  if (H + 2 * pad_h < KH || W + 2 * pad_w < KW) return QG_ERR_INVALID_ARG;
  if (pad_h >= KH || pad_w >= KW) return QG_ERR_UNSUPPORTED;
  const int64_t K = (int64_t)KH * KW * Cin;
  if (K > INT32_MAX) return QG_ERR_INVALID_ARG;
  const int64_t M = (int64_t)Nb * ((H + 2 * pad_h - KH) / stride_h + 1) *
                    ((W + 2 * pad_w - KW) / stride_w + 1);
  if (M > INT32_MAX) return QG_ERR_UNSUPPORTED;
  int rc = check_requant(rq, (int)K);
  if (rc != QG_OK) return rc;
  if (rq->b_zero_point != 0) return QG_ERR_UNSUPPORTED;
  if (acc_out && !aligned(acc_out, 4)) return QG_ERR_MISALIGNED;
  return QG_OK;
}

extern "C" size_t qconv2d_s8_pack_w_bytes(int Cout, int KH, int KW, int Cin) {
  if (Cout <= 0 || KH <= 0 || KW <= 0 || Cin <= 0) return 0;
  const int64_t K = (int64_t)KH * KW * Cin;
  if (K > INT32_MAX) return 0;
  return conv_pack_w_bytes(Cout, (int)K);
}

extern "C" int qconv2d_s8_pack_w(int Cout, int KH, int KW, int Cin, const int8_t* w,
                                 void* packed_w, size_t packed_bytes, void* stream) {
  if (Cout <= 0 || KH <= 0 || KW <= 0 || Cin <= 0 || !w || !packed_w) return QG_ERR_INVALID_ARG;
  const int64_t K = (int64_t)KH * KW * Cin;
  if (K > INT32_MAX) return QG_ERR_INVALID_ARG;
  if (!aligned(packed_w, 128)) return QG_ERR_MISALIGNED;
  if (packed_bytes < conv_pack_w_bytes(Cout, (int)K)) return QG_ERR_WORKSPACE;
  int rc = device_ready();
  if (rc != QG_OK) return rc;
  return conv_pack_w(Cout, (int)K, w, packed_w, (cudaStream_t)stream);
}

extern "C" int qconv2d_s8_im2col_packed(int Nb, int H, int W, int Cin, int Cout, int KH, int KW,
                                        int stride_h, int stride_w, int pad_h, int pad_w,
                                        const int8_t* x, const void* packed_w, int8_t* y,
                                        const qg_requant_t* rq, int32_t* acc_out, void* stream) {
  int rc = conv_args(Nb, H, W, Cin, Cout, KH, KW, stride_h, stride_w, pad_h, pad_w, x, y, rq,
                     acc_out);
  if (rc != QG_OK) return rc;
  if (!packed_w) return QG_ERR_INVALID_ARG;
  if (!aligned(packed_w, 128)) return QG_ERR_MISALIGNED;
  rc = device_ready();
  if (rc != QG_OK) return rc;
  return conv_run_packed(Nb, H, W, Cin, Cout, KH, KW, stride_h, stride_w, pad_h, pad_w, x,
                         packed_w, y, *rq, acc_out, (cudaStream_t)stream);
}

extern "C" int qconv2d_s8_im2col(int Nb, int H, int W, int Cin, int Cout, int KH, int KW,
                                 int stride_h, int stride_w, int pad_h, int pad_w,
                                 const int8_t* x, const int8_t* w, int8_t* y,
                                 const qg_requant_t* rq, int32_t* acc_out, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  if (!w) return QG_ERR_INVALID_ARG;
  int rc = conv_args(Nb, H, W, Cin, Cout, KH, KW, stride_h, stride_w, pad_h, pad_w, x, y, rq,
                     acc_out);
  if (rc != QG_OK) return rc;
  if (workspace && !aligned(workspace, 256)) return QG_ERR_MISALIGNED;
  const size_t need =
      conv_workspace_bytes(Nb, H, W, Cin, Cout, KH, KW, stride_h, stride_w, pad_h, pad_w);
  if (need && (!workspace || workspace_bytes < need)) return QG_ERR_WORKSPACE;
  rc = device_ready();
  if (rc != QG_OK) return rc;
  return conv_run(Nb, H, W, Cin, Cout, KH, KW, stride_h, stride_w, pad_h, pad_w, x, w, y, *rq,
                  acc_out, workspace, workspace_bytes, (cudaStream_t)stream);
}

// ---------------------------------------------------------------------------
// Dynamic activation quantization, W4 pack, A8W4 linear
// ---------------------------------------------------------------------------
extern "C" int quantize_rows_a8(int M, int K, const float* x, int64_t ldx, int8_t* q,
                                int64_t ldq, float* scale, int32_t* zero_point, void* stream) {
  if (M < 0 || K <= 0 || ldx < K || ldq < K) return QG_ERR_INVALID_ARG;
  if (M == 0) return QG_OK;
  if (!x || !q || !scale || !zero_point) return QG_ERR_INVALID_ARG;
  if (!aligned(x, 4) || !aligned(scale, 4) || !aligned(zero_point, 4)) return QG_ERR_MISALIGNED;
  int rc = device_ready();
  if (rc != QG_OK) return rc;
  return launch_quantize_rows(M, K, x, ldx, q, ldq, scale, zero_point, (cudaStream_t)stream);
}

extern "C" size_t pack_w4_g32_bytes(int N, int K) {
  if (N <= 0 || K <= 0 || K % 32) return 0;
  return (size_t)N * (K / 2) + (size_t)N * (K / 32) * 4;
}

extern "C" size_t pack_w4_g32_bf16_bytes(int N, int K) {
  if (N <= 0 || K <= 0 || K % 32) return 0;
  return (size_t)N * (K / 2) + (size_t)N * (K / 32) * 2;
}

static int pack_w4(int N, int K, const int8_t* w, int64_t ldw, const float* group_scales,
                   void* packed, size_t packed_bytes, bool scale_bf16, void* stream) {
  if (N <= 0 || K <= 0 || ldw < K || !w || !group_scales || !packed) return QG_ERR_INVALID_ARG;
  if (K % 32) return QG_ERR_UNSUPPORTED;
  if (!aligned(packed, 16) || !aligned(group_scales, 4)) return QG_ERR_MISALIGNED;
  const size_t need = scale_bf16 ? pack_w4_g32_bf16_bytes(N, K) : pack_w4_g32_bytes(N, K);
  if (packed_bytes < need) return QG_ERR_WORKSPACE;
  int rc = device_ready();
  if (rc != QG_OK) return rc;
  return launch_pack_w4(N, K, w, ldw, group_scales, packed, scale_bf16, (cudaStream_t)stream);
}

extern "C" int pack_w4_g32(int N, int K, const int8_t* w, int64_t ldw, const float* group_scales,
                           void* packed, size_t packed_bytes, void* stream) {
  return pack_w4(N, K, w, ldw, group_scales, packed, packed_bytes, false, stream);
}

extern "C" int pack_w4_g32_bf16(int N, int K, const int8_t* w, int64_t ldw,
                                const float* group_scales, void* packed, size_t packed_bytes,
                                void* stream) {
  return pack_w4(N, K, w, ldw, group_scales, packed, packed_bytes, true, stream);
}

static const int kFusedGemvMaxK = 65536;   // activations held in shared memory
static const int kSimtMaxK = 25600;        // 8 rows of activations in shared memory

static size_t a8w4_ws_layout(int M, int K, size_t* off_scale, size_t* off_zp) {
  const size_t q = round_up((int64_t)M * K, 256);
  const size_t s = round_up((int64_t)M * 4, 256);
  if (off_scale) *off_scale = q;
  if (off_zp) *off_zp = q + s;
  return q + s + round_up((int64_t)M * 4, 256);
}

// Workspace of an M > 1 A8W4 call, for every variant (per-row or per-block
// activations, symmetric or asymmetric weights): the tensor-core layout
// where that path applies, else the CUDA-core one.
extern "C" size_t qgemm_a8w4_workspace_bytes(int M, int N, int K) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  if (M == 1 && K <= kFusedGemvMaxK) return 0;
  if (a8w4_tc_supported(M, N, K)) return a8w4_tc_workspace_bytes(M, N, K);
  return a8w4_ws_layout(M, K, nullptr, nullptr);
}

// Fields of the tensor-core call shared by the plain-row entry points.
static A8W4TcCall tc_rows(int M, int N, int K, const float* x, int64_t ldx, const void* packed_w,
                          const float* bias, float lo, float hi, float* y, int64_t ldy,
                          int8_t* q_out, float* scale_out, int32_t* zp_out) {
  A8W4TcCall c{};
  c.M = M; c.N = N; c.K = K; c.x = x; c.ldx = ldx; c.conv = false;
  c.packed = packed_w; c.bias = bias; c.lo = lo; c.hi = hi; c.y = y; c.ldy = ldy;
  c.q_out = q_out; c.scale_out = scale_out; c.zp_out = zp_out;
  return c;
}

static int a8w4_linear(int M, int N, int K, const float* x, int64_t ldx, const void* packed_w,
                       const float* bias, float clamp_min, float clamp_max, float* y,
                       int64_t ldy, int8_t* q_out, float* scale_out, int32_t* zp_out,
                       void* workspace, size_t workspace_bytes, bool sbf, void* stream) {
  if (M < 0 || N <= 0 || K <= 0 || ldx < K || ldy < N) return QG_ERR_INVALID_ARG;
  if (K % 32) return QG_ERR_UNSUPPORTED;
  if (!(clamp_min <= clamp_max)) return QG_ERR_INVALID_ARG;  // also rejects NaN
  if (M == 0) return QG_OK;
  if (!x || !packed_w || !y) return QG_ERR_INVALID_ARG;
  if (!aligned(packed_w, 16)) return QG_ERR_MISALIGNED;
  if (!aligned(x, 4) || !aligned(y, 4) || (bias && !aligned(bias, 4))) return QG_ERR_MISALIGNED;
  if ((scale_out && !aligned(scale_out, 4)) || (zp_out && !aligned(zp_out, 4)))
    return QG_ERR_MISALIGNED;
  int rc = device_ready();
  if (rc != QG_OK) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  if (M == 1 && K <= kFusedGemvMaxK)
    return launch_a8w4_gemv(N, K, x, packed_w, bias, clamp_min, clamp_max, y, q_out, scale_out,
                            zp_out, sbf, st);
  if (a8w4_tc_supported(M, N, K)) {
    if (!workspace) return QG_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return QG_ERR_MISALIGNED;
    A8W4TcCall c = tc_rows(M, N, K, x, ldx, packed_w, bias, clamp_min, clamp_max, y, ldy, q_out,
                           scale_out, zp_out);
    c.mode = 0;
    c.scale_bf16 = sbf;
    return launch_a8w4_tc_call(c, workspace, workspace_bytes, st);
  }
  if (K > kSimtMaxK) return QG_ERR_UNSUPPORTED;
  size_t off_s = 0, off_z = 0;
  const size_t need = a8w4_ws_layout(M, K, &off_s, &off_z);
  if (!workspace || workspace_bytes < need) return QG_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return QG_ERR_MISALIGNED;
  int8_t* q = (int8_t*)workspace;
  float* sA = (float*)((char*)workspace + off_s);
  int32_t* zA = (int32_t*)((char*)workspace + off_z);
  rc = launch_quantize_rows(M, K, x, ldx, q, K, sA, zA, st);
  if (rc != QG_OK) return rc;
  if (q_out && cudaMemcpyAsync(q_out, q, (size_t)M * K, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return QG_ERR_CUDA;
  if (scale_out &&
      cudaMemcpyAsync(scale_out, sA, (size_t)M * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return QG_ERR_CUDA;
  if (zp_out && cudaMemcpyAsync(zp_out, zA, (size_t)M * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return QG_ERR_CUDA;
  return launch_a8w4_gemm_simt(M, N, K, q, sA, zA, packed_w, bias, clamp_min, clamp_max, y, ldy,
                               sbf, st);
}

extern "C" int qgemm_a8w4_f32(int M, int N, int K, const float* x, int64_t ldx,
                              const void* packed_w, const float* bias, float clamp_min,
                              float clamp_max, float* y, int64_t ldy, int8_t* q_out,
                              float* scale_out, int32_t* zp_out, void* workspace,
                              size_t workspace_bytes, void* stream) {
  return a8w4_linear(M, N, K, x, ldx, packed_w, bias, clamp_min, clamp_max, y, ldy, q_out,
                     scale_out, zp_out, workspace, workspace_bytes, false, stream);
}

extern "C" int qgemm_a8w4_f32_bf16s(int M, int N, int K, const float* x, int64_t ldx,
                                    const void* packed_w, const float* bias, float clamp_min,
                                    float clamp_max, float* y, int64_t ldy, int8_t* q_out,
                                    float* scale_out, int32_t* zp_out, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  return a8w4_linear(M, N, K, x, ldx, packed_w, bias, clamp_min, clamp_max, y, ldy, q_out,
                     scale_out, zp_out, workspace, workspace_bytes, true, stream);
}

// Checks shared by the per-block-activation and asymmetric-weight variants,
// all made on the host before any device work: QG_OK when the call can run.
static int a8w4_variant_args(int M, int N, int K, const float* x, int64_t ldx,
                             const void* packed_w, const float* bias, float clamp_min,
                             float clamp_max, float* y, int64_t ldy, float* scale_out,
                             int32_t* zp_out, void* workspace, size_t workspace_bytes) {
  if (M < 0 || N <= 0 || K <= 0 || ldx < K || ldy < N) return QG_ERR_INVALID_ARG;
  if (K % 32) return QG_ERR_UNSUPPORTED;
  if (!(clamp_min <= clamp_max)) return QG_ERR_INVALID_ARG;  // also rejects NaN
  if (M == 0) return QG_OK;
  if (!x || !packed_w || !y) return QG_ERR_INVALID_ARG;
  if (!aligned(packed_w, 16)) return QG_ERR_MISALIGNED;
  if (!aligned(x, 4) || !aligned(y, 4) || (bias && !aligned(bias, 4))) return QG_ERR_MISALIGNED;
  if ((scale_out && !aligned(scale_out, 4)) || (zp_out && !aligned(zp_out, 4)))
    return QG_ERR_MISALIGNED;
  if (M == 1) {  // the fused GEMV: no workspace
    if (K % 128 || K > 8192 || !aligned(x, 16)) return QG_ERR_UNSUPPORTED;
  } else {       // the tensor-core path
    if (!a8w4_tc_supported(M, N, K)) return QG_ERR_UNSUPPORTED;
    if (!workspace || workspace_bytes < a8w4_tc_workspace_bytes(M, N, K)) return QG_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return QG_ERR_MISALIGNED;
  }
  return device_ready();
}

extern "C" int qgemm_a8w4_f32_actblock(int M, int N, int K, const float* x, int64_t ldx,
                                       const void* packed_w, const float* bias,
                                       float clamp_min, float clamp_max, float* y,
                                       int64_t ldy, int8_t* q_out, float* scale_out,
                                       int32_t* zp_out, void* workspace, size_t workspace_bytes,
                                       void* stream) {
  int rc = a8w4_variant_args(M, N, K, x, ldx, packed_w, bias, clamp_min, clamp_max, y, ldy,
                             scale_out, zp_out, workspace, workspace_bytes);
  if (rc != QG_OK || M == 0) return rc;
  if (M == 1)
    return launch_a8w4_gemv_actblock(N, K, x, packed_w, bias, clamp_min, clamp_max, y, q_out,
                                     scale_out, zp_out, (cudaStream_t)stream);
  A8W4TcCall c = tc_rows(M, N, K, x, ldx, packed_w, bias, clamp_min, clamp_max, y, ldy, q_out,
                         scale_out, zp_out);
  c.mode = 1;
  return launch_a8w4_tc_call(c, workspace, workspace_bytes, (cudaStream_t)stream);
}

extern "C" size_t pack_w4_g32_asym_bytes(int N, int K) {
  if (N <= 0 || K <= 0 || K % 32) return 0;
  return pack_w4_g32_bytes(N, K) + (size_t)N * (K / 32) * 4;
}

extern "C" int pack_w4_g32_asym(int N, int K, const int8_t* w, int64_t ldw,
                                const float* group_scales, const float* group_zeros,
                                void* packed, size_t packed_bytes, void* stream) {
  if (N <= 0 || K <= 0 || ldw < K || !w || !group_scales || !group_zeros || !packed)
    return QG_ERR_INVALID_ARG;
  if (K % 32) return QG_ERR_UNSUPPORTED;
  if (!aligned(packed, 16) || !aligned(group_scales, 4) || !aligned(group_zeros, 4))
    return QG_ERR_MISALIGNED;
  if (packed_bytes < pack_w4_g32_asym_bytes(N, K)) return QG_ERR_WORKSPACE;
  int rc = pack_w4(N, K, w, ldw, group_scales, packed, packed_bytes, false, stream);
  if (rc != QG_OK) return rc;
  // the zeros follow the scales as given (f32, [N][K/32])
  if (cudaMemcpyAsync((char*)packed + pack_w4_g32_bytes(N, K), group_zeros,
                      (size_t)N * (K / 32) * 4, cudaMemcpyDeviceToDevice,
                      (cudaStream_t)stream) != cudaSuccess)
    return QG_ERR_CUDA;
  return QG_OK;
}

extern "C" int qgemm_a8w4_f32_asym(int M, int N, int K, const float* x, int64_t ldx,
                                   const void* packed_w, const float* bias, float clamp_min,
                                   float clamp_max, float* y, int64_t ldy, int8_t* q_out,
                                   float* scale_out, int32_t* zp_out, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  int rc = a8w4_variant_args(M, N, K, x, ldx, packed_w, bias, clamp_min, clamp_max, y, ldy,
                             scale_out, zp_out, workspace, workspace_bytes);
  if (rc != QG_OK || M == 0) return rc;
  if (M == 1)
    return launch_a8w4_gemv_asym(N, K, x, packed_w, bias, clamp_min, clamp_max, y, q_out,
                                 scale_out, zp_out, (cudaStream_t)stream);
  A8W4TcCall c = tc_rows(M, N, K, x, ldx, packed_w, bias, clamp_min, clamp_max, y, ldy, q_out,
                         scale_out, zp_out);
  c.mode = 0;
  c.wzero = (const float*)((const uint8_t*)packed_w + pack_w4_g32_bytes(N, K));
  return launch_a8w4_tc_call(c, workspace, workspace_bytes, (cudaStream_t)stream);
}

// ---------------------------------------------------------------------------
// Symmetric row quantization; float-input convolution with dynamic int8
// activations and int4 weights
// ---------------------------------------------------------------------------
extern "C" int quantize_rows_a8_sym(int M, int K, const float* x, int64_t ldx, int8_t* q,
                                    int64_t ldq, float* scale, void* stream) {
  if (M < 0 || K <= 0 || ldx < K || ldq < K) return QG_ERR_INVALID_ARG;
  if (M == 0) return QG_OK;
  if (!x || !q || !scale) return QG_ERR_INVALID_ARG;
  if (!aligned(x, 4) || !aligned(scale, 4)) return QG_ERR_MISALIGNED;
  int rc = device_ready();
  if (rc != QG_OK) return rc;
  return launch_quantize_rows_sym(M, K, x, ldx, q, ldq, scale, nullptr, (cudaStream_t)stream);
}

// The conv's contraction runs on the tensor-core A8W4 kernel when K % 64 == 0
// (and K <= 8192); otherwise on the CUDA-core A8W4 kernel: 8 unrolled rows
// per CTA row of the grid (at most 65535 of them) and 8*K bytes of shared
// memory.
static const int64_t kDynConvMaxRows = 65535 * 8;
static const int64_t kDynConvMaxRowsTc = (int64_t)1 << 30;

// Unrolled-matrix shape of a float-input conv: QG_OK with P rows of K, or
// the status the call returns; *tc tells which kernel takes it.
static int dynconv_shape(int Nb, int H, int W, int Cin, int Cout, int KH, int KW, int sh, int sw,
                         int ph, int pw, int64_t* P, int* K, bool* tc) {
  if (Nb <= 0 || H <= 0 || W <= 0 || Cin <= 0 || Cout <= 0 || KH <= 0 || KW <= 0 || sh <= 0 ||
      sw <= 0 || ph < 0 || pw < 0)
    return QG_ERR_INVALID_ARG;
  if ((int64_t)H + 2 * (int64_t)ph < KH || (int64_t)W + 2 * (int64_t)pw < KW)
    return QG_ERR_INVALID_ARG;
  const int64_t k = (int64_t)KH * KW * Cin;
  if (k % 32 || k > INT32_MAX) return QG_ERR_UNSUPPORTED;
  const int64_t OH = ((int64_t)H + 2 * (int64_t)ph - KH) / sh + 1;
  const int64_t OW = ((int64_t)W + 2 * (int64_t)pw - KW) / sw + 1;
  const int64_t p = (int64_t)Nb * OH * OW;
  *tc = p >= 2 && p <= kDynConvMaxRowsTc && a8w4_tc_supported(p, Cout, (int)k);
  if (!*tc && (k > kSimtMaxK || p > kDynConvMaxRows)) return QG_ERR_UNSUPPORTED;
  *P = p;
  *K = (int)k;
  return QG_OK;
}

extern "C" size_t qconv2d_f32_dyn_a8w4_workspace_bytes(int Nb, int H, int W, int Cin, int Cout,
                                                       int KH, int KW, int stride_h,
                                                       int stride_w, int pad_h, int pad_w) {
  int64_t P = 0;
  int K = 0;
  bool tc = false;
  if (dynconv_shape(Nb, H, W, Cin, Cout, KH, KW, stride_h, stride_w, pad_h, pad_w, &P, &K, &tc) !=
      QG_OK)
    return 0;
  return tc ? a8w4_tc_workspace_bytes(P, Cout, K) : a8w4_ws_layout((int)P, K, nullptr, nullptr);
}

extern "C" int qconv2d_f32_dyn_a8w4(int Nb, int H, int W, int Cin, int Cout, int KH, int KW,
                                    int stride_h, int stride_w, int pad_h, int pad_w,
                                    const float* x, const void* packed_w, const float* bias,
                                    float clamp_min, float clamp_max, int symmetric, float* y,
                                    int8_t* q_out, float* scale_out, int32_t* zp_out,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  int64_t P = 0;
  int K = 0;
  bool tc = false;
  int rc = dynconv_shape(Nb, H, W, Cin, Cout, KH, KW, stride_h, stride_w, pad_h, pad_w, &P, &K,
                         &tc);
  if (rc != QG_OK) return rc;
  if (symmetric != 0 && symmetric != 1) return QG_ERR_INVALID_ARG;
  if (!(clamp_min <= clamp_max)) return QG_ERR_INVALID_ARG;  // also rejects NaN
  if (!x || !packed_w || !y) return QG_ERR_INVALID_ARG;
  if (!aligned(packed_w, 16)) return QG_ERR_MISALIGNED;
  if (!aligned(x, 4) || !aligned(y, 4) || (bias && !aligned(bias, 4))) return QG_ERR_MISALIGNED;
  if ((scale_out && !aligned(scale_out, 4)) || (zp_out && !aligned(zp_out, 4)))
    return QG_ERR_MISALIGNED;
  if (tc) {
    if (!workspace) return QG_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return QG_ERR_MISALIGNED;
    rc = device_ready();
    if (rc != QG_OK) return rc;
    const int OH = (int)(((int64_t)H + 2 * (int64_t)pad_h - KH) / stride_h + 1);
    const int OW = (int)(((int64_t)W + 2 * (int64_t)pad_w - KW) / stride_w + 1);
    A8W4TcCall c{};
    c.M = P; c.N = Cout; c.K = K; c.x = x; c.ldx = 0; c.conv = true;
    c.H = H; c.W = W; c.Cin = Cin; c.KH = KH; c.KW = KW; c.sh = stride_h; c.sw = stride_w;
    c.ph = pad_h; c.pw = pad_w; c.OH = OH; c.OW = OW;
    c.mode = symmetric ? 2 : 0;
    c.packed = packed_w; c.bias = bias; c.lo = clamp_min; c.hi = clamp_max;
    c.y = y; c.ldy = Cout; c.q_out = q_out; c.scale_out = scale_out; c.zp_out = zp_out;
    return launch_a8w4_tc_call(c, workspace, workspace_bytes, (cudaStream_t)stream);
  }
  size_t off_s = 0, off_z = 0;
  const size_t need = a8w4_ws_layout((int)P, K, &off_s, &off_z);
  if (!workspace || workspace_bytes < need) return QG_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return QG_ERR_MISALIGNED;
  rc = device_ready();
  if (rc != QG_OK) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  int8_t* q = (int8_t*)workspace;
  float* sA = (float*)((char*)workspace + off_s);
  int32_t* zA = (int32_t*)((char*)workspace + off_z);
  rc = launch_im2col_quantize(Nb, H, W, Cin, KH, KW, stride_h, stride_w, pad_h, pad_w, x,
                              symmetric != 0, q, sA, zA, st);
  if (rc != QG_OK) return rc;
  if (q_out && cudaMemcpyAsync(q_out, q, (size_t)P * K, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return QG_ERR_CUDA;
  if (scale_out &&
      cudaMemcpyAsync(scale_out, sA, (size_t)P * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return QG_ERR_CUDA;
  if (zp_out && cudaMemcpyAsync(zp_out, zA, (size_t)P * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return QG_ERR_CUDA;
  return launch_a8w4_gemm_simt((int)P, Cout, K, q, sA, zA, packed_w, bias, clamp_min, clamp_max, y,
                               Cout, false, st);
}
