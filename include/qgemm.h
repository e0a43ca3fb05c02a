/*
 * qgemm.h — C ABI of the B200 (sm_100a) quantized integer matmul library.
 *
 * Operations (sources cited by page title and section):
 *   [QG]  xidianedu, "量化 GEMM：数值契约、SRAM、DMA 与结果验证" (quantized GEMM:
 *         numeric contract, SRAM, DMA and result verification), sections 1-5.
 *   [MNN] MNN source/backend/cpu/compute/ConvInt8TiledExecutor.cpp
 *         (initializeConvInt8QuantInfo, reorderWeight, _computeReorderQuantInfo,
 *          BatchAsyDynamicQuant, BatchSymDynamicQuant, the low-memory float
 *          im2col path, tileSplitFunction / QuanPostTreatParameters).
 *   [KAI] pytorch/ao PR #997, "Kleidi 4b blockwise gemv prototype"
 *         (matmul_clamp_f32_qai8dxp_qsi4c32p micro-kernels and their wrapper).
 *
 * Conventions shared by every entry point
 *   - Pointers to tensors are DEVICE pointers unless a parameter says "host".
 *     The caller owns and allocates every buffer; no entry point allocates
 *     device memory.  Scratch space is passed as `workspace`, sized by the
 *     matching *_workspace_bytes() query (0 means none is needed).
 *   - Strides (ld*) count ELEMENTS, not bytes ([QG] section 5: row-major
 *     A at base_A + (m*lda + k)*elem_bytes).  Logical sizes may be smaller
 *     than physical ones (lda >= K, ...; [QG] section 2).  Inputs and outputs
 *     must not alias.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  The return value reports argument checks and launch
 *     errors.  Kernels are launched as programmatic dependents of the work
 *     before them on the stream: they may start while it is still running
 *     and wait for it on the device before they read activations or
 *     workspace or write any output.  Before that wait they may read the
 *     call's packed weights, scales and bias, so a kernel that signals its
 *     dependents early (griddepcontrol.launch_dependents) must not write
 *     those buffers for the call that follows it.  Errors found on the device (a bounded wait that ran out, an
 *     int4 weight out of range) are recorded in a per-device status word that
 *     qg_device_status() reads after the work has finished.
 *   - Every entry point returns QG_OK (0) or a negative qg_status.  It never
 *     aborts the process and never traps on the GPU.
 */
#ifndef QGEMM_H_
#define QGEMM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QG_API_VERSION 2

typedef enum {
  QG_OK = 0,
  QG_ERR_INVALID_ARG = -1,     /* bad size, NULL pointer, stride < logical size, bad clamp */
  QG_ERR_MISALIGNED = -2,      /* pointer alignment the operation requires is not met */
  QG_ERR_OVERFLOW_BOUND = -3,  /* K*65025 + |bias| > INT32_MAX ([QG] section 4) */
  QG_ERR_UNSUPPORTED = -4,     /* valid but not implemented (e.g. K % 32 != 0 for A8W4) */
  QG_ERR_CUDA = -5,            /* a CUDA runtime call or kernel launch failed */
  QG_ERR_TIMEOUT = -6,         /* a bounded device-side wait ran out (device status) */
  QG_ERR_WORKSPACE = -7,       /* workspace missing or smaller than the query says */
  QG_ERR_NO_DEVICE = -8        /* no sm_100 device is current */
} qg_status;

/* Human-readable name of a status code.  Never NULL. */
const char* qg_status_string(int status);

/* QG_API_VERSION of the built library. */
int qg_version(void);

/*
 * Per-device error word.  Synchronises the current device, then returns
 * QG_OK or the first qg_status a kernel recorded since the last reset; with
 * reset != 0 the word is cleared afterwards.  Returns QG_ERR_CUDA if the
 * synchronisation itself fails.
 */
int qg_device_status(int reset);

/*
 * Test hook for the bounded waits; the pages have no counterpart.  Every
 * pipeline wait in the tensor-core kernels gives up after a poll limit,
 * records QG_ERR_TIMEOUT in the device status word and lets the kernel
 * return (it first waits for its own copies and MMAs in flight and frees its
 * tensor memory), so a stalled pipeline never hangs the GPU.  This arms one
 * stall for the next launch of a kernel family, so that path can be
 * exercised on purpose: that launch skips one pipeline stage (nothing is
 * issued for it, so no copy is left in flight) and waits with a short poll
 * limit.  The call itself still returns QG_OK; qg_device_status() then
 * reports QG_ERR_TIMEOUT, the call's outputs are unspecified, and the next
 * call runs normally.
 *   which: 1 = INT8 GEMM one-CTA kernel (a call with K > 128 and M <= 128, or
 *              M <= 256 when its 128 x 256 tiles fit in one wave of SMs),
 *          2 = A8W4 tensor-core kernel (an M > 1 call that takes it),
 *          0 = disarm.
 * Returns QG_OK, or QG_ERR_INVALID_ARG for another value.  Not for
 * production use: one process-wide flag, taken by whichever thread launches
 * that kernel family next.
 */
int qg_test_arm_stall(int which);

/* ------------------------------------------------------------------------
 * Requantization parameters of the affine INT8 contract.
 *
 * [QG] section 1: real = scale * (q - zero_point); the int32 bias lives in
 * the accumulator scale sA*sB[n]; the ratio sA*sB[n]/sO is applied as an
 * integer multiplier and shift.  [MNN] initializeConvInt8QuantInfo /
 * QuanPostTreatParameters: output zero-point, clamp [clamp_min, clamp_max],
 * fused ReLU expressed as clamp_min = out_zero_point.
 *
 * For every output element the library computes, exactly:
 *   acc = sum_{k<K} (A[m,k]-a_zero_point)*(B[k,n]-b_zero_point) + bias[n]
 *   y   = clamp(out_zero_point + rne(acc * M0 / 2^(31+shift)),
 *               clamp_min, clamp_max)
 * where rne rounds half to even on the exact 64-bit product and M0/shift are
 * multiplier0/shift0 (per_channel == 0) or multiplier[n]/shift[n].
 * ------------------------------------------------------------------------ */
typedef struct {
  int32_t a_zero_point;       /* za in [-128,127]; also the conv pad value */
  int32_t b_zero_point;       /* zb in [-128,127]; 0 for symmetric weights */
  const int32_t* bias;        /* device int32 [N], or NULL for no bias */
  int32_t bias_abs_max;       /* host bound on |bias[n]| (>= 0) for the overflow check */
  int32_t per_channel;        /* 0: multiplier0/shift0; 1: multiplier[N]/shift[N] */
  int32_t multiplier0;        /* M0 in [2^30, 2^31) when per_channel == 0 */
  int32_t shift0;             /* right shift in [0, 31] when per_channel == 0 */
  const int32_t* multiplier;  /* device int32 [N] when per_channel == 1 */
  const int32_t* shift;       /* device int32 [N] when per_channel == 1 */
  int32_t out_zero_point;     /* zo in [-128,127] */
  int32_t clamp_min;          /* int8 range, clamp_min <= clamp_max */
  int32_t clamp_max;
} qg_requant_t;

/*
 * Host helper: ratio = sA*sB/sO (0 < ratio < 1) -> (M0, shift) with
 * ratio ~= M0 * 2^-(31+shift).  frexp(ratio) = f*2^e, M0 = round(f*2^31)
 * (ties away from zero; 2^31 -> 2^30 and e+1), shift = -e.
 * QG_ERR_UNSUPPORTED if ratio is outside (0,1) or shift would exceed 31;
 * QG_ERR_INVALID_ARG for NULL outputs.
 */
int qg_requant_params(double ratio, int32_t* m0, int32_t* shift);

/* ------------------------------------------------------------------------
 * Affine INT8 GEMM with fused zero-point correction, bias, requant, clamp.
 * [QG] sections 1 (contract), 2 (padding is real zero, logical vs physical
 * shape), 4 (INT32 accumulator kept across all K blocks, requant once after
 * the last block, overflow bound K*65025 + |bias|).
 *
 *   A: int8 row-major [M][lda], lda >= K.      B: int8 row-major [K][ldb], ldb >= N.
 *   C: int8 row-major [M][ldc], ldc >= N (written).
 *   acc_out: optional int32 row-major [M][ld_acc] (ld_acc >= N) receiving the
 *            pre-requant accumulator including bias; NULL to skip.
 *   rq: host pointer to the parameters above.
 * Rejects (QG_ERR_OVERFLOW_BOUND) any call with K*65025 + bias_abs_max
 * above INT32_MAX.  M, N, K >= 1.  Any alignment of A, B, C is accepted.
 * ------------------------------------------------------------------------ */
size_t qgemm_s8s8_workspace_bytes(int M, int N, int K);
int qgemm_s8s8_requant(int M, int N, int K,
                       const int8_t* A, int64_t lda,
                       const int8_t* B, int64_t ldb,
                       int8_t* C, int64_t ldc,
                       const qg_requant_t* rq,
                       int32_t* acc_out, int64_t ld_acc,
                       void* workspace, size_t workspace_bytes,
                       void* stream);

/*
 * Weight-stationary variant: B is packed once by qgemm_pack_b_s8 ([MNN]
 * reorderWeight: weights reordered once at load, with per-column kernel
 * sums) and reused.  The packed buffer is opaque; its size comes from
 * qgemm_pack_b_s8_bytes and it must be 128-byte aligned.  The pack stores no
 * zero-point: rq->b_zero_point is applied at GEMM time.  workspace is needed
 * only when A's rows are not 16-byte aligned or b_zero_point != 0.
 */
size_t qgemm_pack_b_s8_bytes(int K, int N);
int qgemm_pack_b_s8(int K, int N, const int8_t* B, int64_t ldb,
                    void* packed_b, size_t packed_bytes, void* stream);
size_t qgemm_s8s8_packed_workspace_bytes(int M, int K);
int qgemm_s8s8_requant_packed(int M, int N, int K,
                              const int8_t* A, int64_t lda,
                              const void* packed_b,
                              int8_t* C, int64_t ldc,
                              const qg_requant_t* rq,
                              int32_t* acc_out, int64_t ld_acc,
                              void* workspace, size_t workspace_bytes,
                              void* stream);

/* ------------------------------------------------------------------------
 * INT8 convolution as an implicit-im2col GEMM.  [MNN] tileSplitFunction: the
 * unrolled input holds the input zero-point where a tap falls in the
 * padding; [QG] section 2: padding must stand for real zero.  No im2col
 * buffer exists: the tensor-core kernel's producer gathers each row of the
 * virtual unrolled matrix straight from x into its shared-memory tile.
 *
 *   x: int8 NHWC [Nb][H][W][Cin]      w: int8 [Cout][KH][KW][Cin] (zw = 0)
 *   y: int8 NHWC [Nb][OH][OW][Cout], OH = (H+2*pad_h-KH)/stride_h + 1 (same for W)
 *   acc_out: optional int32 NHWC [Nb][OH][OW][Cout].
 * GEMM view: M = Nb*OH*OW, N = Cout, K = KH*KW*Cin; pad value =
 * rq->a_zero_point; rq->b_zero_point must be 0.  Per-Cout requant via
 * rq->per_channel.  Fused ReLU: rq->clamp_min = rq->out_zero_point.
 * pad_h < KH and pad_w < KW (else QG_ERR_UNSUPPORTED); M <= INT32_MAX.
 *
 * Weight-stationary form ([MNN] reorderWeight: weights reordered once at
 * load, with their per-channel sums): qconv2d_s8_pack_w packs w once into an
 * opaque buffer of qconv2d_s8_pack_w_bytes bytes (128-byte aligned), and
 * qconv2d_s8_im2col_packed runs the convolution from it in one launch, with
 * no workspace.  qconv2d_s8_im2col packs w into its workspace on every call
 * (two launches).  The gather copies 16-byte runs when Cin % 16 == 0 and x
 * is 16-byte aligned, single bytes otherwise (slower, same result).
 * ------------------------------------------------------------------------ */
size_t qconv2d_s8_pack_w_bytes(int Cout, int KH, int KW, int Cin);
int qconv2d_s8_pack_w(int Cout, int KH, int KW, int Cin, const int8_t* w,
                      void* packed_w, size_t packed_bytes, void* stream);
int qconv2d_s8_im2col_packed(int Nb, int H, int W, int Cin, int Cout, int KH, int KW,
                             int stride_h, int stride_w, int pad_h, int pad_w,
                             const int8_t* x, const void* packed_w, int8_t* y,
                             const qg_requant_t* rq, int32_t* acc_out, void* stream);
size_t qconv2d_s8_workspace_bytes(int Nb, int H, int W, int Cin, int Cout,
                                  int KH, int KW, int stride_h, int stride_w,
                                  int pad_h, int pad_w);
int qconv2d_s8_im2col(int Nb, int H, int W, int Cin, int Cout, int KH, int KW,
                      int stride_h, int stride_w, int pad_h, int pad_w,
                      const int8_t* x, const int8_t* w, int8_t* y,
                      const qg_requant_t* rq, int32_t* acc_out,
                      void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Dynamic per-row asymmetric int8 activation quantization.  [MNN]
 * BatchAsyDynamicQuant (min/max -> scale and zero-point, quantize with clamp
 * to [-128,127]); [KAI] qai8dx (int8, dynamic, per row, asymmetric); [QG]
 * section 1 (ONNX QuantizeLinear rounding: half to even).  All float32, one
 * rounding per operation:
 *   rmin = min(0, min_k x), rmax = max(0, max_k x)
 *   scale = (rmax - rmin)/255, or 1 if that is 0;  inv = 1/scale
 *   zero_point = clamp(rne(-128 - rmin*inv), -128, 127)
 *   q[k] = clamp(rne(x[k]*inv) + zero_point, -128, 127)
 *   x: f32 [M][ldx] (ldx >= K); q: int8 [M][ldq] (ldq >= K);
 *   scale: f32 [M]; zero_point: int32 [M].  Non-finite x is out of contract.
 * ------------------------------------------------------------------------ */
int quantize_rows_a8(int M, int K, const float* x, int64_t ldx,
                     int8_t* q, int64_t ldq, float* scale,
                     int32_t* zero_point, void* stream);

/* ------------------------------------------------------------------------
 * Int4 weights with one f32 scale per 32-wide K group.  [KAI] qsi4c32
 * (symmetric int4, group 32; weight zero-points absent), [MNN]
 * _computeReorderQuantInfo (int4 stored with an offset of 8).
 *
 *   w: int8 [N][ldw] (ldw >= K), values in [-8,7] (row n = output channel);
 *   group_scales: f32 [N][K/32]; K % 32 == 0.
 *   packed: opaque buffer of pack_w4_g32_bytes(N, K) bytes, 16-byte aligned:
 *     N rows of K/2 bytes, where the little-endian 32-bit word j of a row
 *     holds (w[8j+b]+8) in the low nibble and (w[8j+4+b]+8) in the high
 *     nibble of byte b (b = 0..3), followed by the f32 scales [N][K/32].
 * A weight outside [-8,7] records QG_ERR_INVALID_ARG in the device status.
 * ------------------------------------------------------------------------ */
size_t pack_w4_g32_bytes(int N, int K);
int pack_w4_g32(int N, int K, const int8_t* w, int64_t ldw,
                const float* group_scales, void* packed, size_t packed_bytes,
                void* stream);

/* ------------------------------------------------------------------------
 * A8W4 linear: y = clamp(dequant(quantize_rows_a8(x)) @ dequant(W)^T + bias).
 * [KAI] matmul_clamp_f32_qai8dxp_qsi4c32p: f32 out, clamp after bias
 * (clamp_min = -INFINITY / clamp_max = +INFINITY for none).  Per element:
 *   y[m,n] = clamp(sA[m] * sum_g sw[n,g] * I[m,n,g] + bias[n])
 *   I[m,n,g] = sum_{k in g} (qA[m,k] - zA[m]) * w[n,k]   (exact integer)
 * with the group combination in float32.
 *   x: f32 [M][ldx] (ldx >= K); packed_w from pack_w4_g32; bias f32 [N] or
 *   NULL; y: f32 [M][ldy] (ldy >= N).  K % 32 == 0 (else QG_ERR_UNSUPPORTED).
 *   q_out [M][K] int8 / scale_out [M] / zp_out [M]: optional (each may be
 *   NULL), receive the activation quantization for bit-exact checks.
 * M == 1 runs one fused kernel (quantization inside, no workspace), launched
 * so that it may start while the previous M == 1 call on the same stream is
 * still finishing: it reads packed_w (never x or bias) before that call has
 * completed.  So packed_w must not be written by the M == 1 call just before
 * it on the stream; every other ordering is kept as usual.  M > 1 with
 * K % 64 == 0 and K <= 8192 runs two kernels: the rows are quantized into
 * the workspace as bf16 tiles of qA - zA, then the tensor-core kernel forms
 * the exact per-group integer dots with bf16 MMAs, combines the groups in
 * float32 and reduces split-K partials in a fixed order.  Other M > 1 shapes
 * (K <= 25600) run a CUDA-core kernel.  q_out must then be writable as bytes
 * (any alignment).
 * ------------------------------------------------------------------------ */
size_t qgemm_a8w4_workspace_bytes(int M, int N, int K);
int qgemm_a8w4_f32(int M, int N, int K, const float* x, int64_t ldx,
                   const void* packed_w, const float* bias,
                   float clamp_min, float clamp_max,
                   float* y, int64_t ldy,
                   int8_t* q_out, float* scale_out, int32_t* zp_out,
                   void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * A8W4 with bf16 group scales.  [KAI] review of the packing call: the Kleidi
 * packing is passed a bf16 type for the group scales, kept as bf16 to save
 * space (scale bytes drop from 1/4 to 1/8 of the nibble bytes).
 *   pack_w4_g32_bf16: as pack_w4_g32, except that each f32 group scale is
 *   rounded to bf16 (round to nearest, ties to even) and stored in 2 bytes:
 *   [N][K/2] nibble bytes, then [N][K/32] bf16 scales; size from
 *   pack_w4_g32_bf16_bytes (0 when K % 32 != 0).  Same argument checks and
 *   status codes as pack_w4_g32.
 *   qgemm_a8w4_f32_bf16s: qgemm_a8w4_f32 on weights packed that way; the
 *   formula above holds with sw[n,g] the stored bf16 value (widened to f32
 *   exactly).  Arguments, workspace (qgemm_a8w4_workspace_bytes), layouts,
 *   the stream ordering note and status codes are those of qgemm_a8w4_f32.
 * ------------------------------------------------------------------------ */
size_t pack_w4_g32_bf16_bytes(int N, int K);
int pack_w4_g32_bf16(int N, int K, const int8_t* w, int64_t ldw, const float* group_scales,
                     void* packed, size_t packed_bytes, void* stream);
int qgemm_a8w4_f32_bf16s(int M, int N, int K, const float* x, int64_t ldx,
                         const void* packed_w, const float* bias,
                         float clamp_min, float clamp_max,
                         float* y, int64_t ldy,
                         int8_t* q_out, float* scale_out, int32_t* zp_out,
                         void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * A8W4 linear with the activations quantized per K block.  [MNN]
 * ConvInt8TiledExecutor, dynamic-quant option 2: the input is quantized in as
 * many K blocks as the weights have quant blocks, each block with its own
 * scale and zero-point.  Here a block is one 32-wide weight group:
 *   y[m,n] = clamp(sum_g sw[n,g] * sA[m,g] * I[m,n,g] + bias[n])
 *   I[m,n,g] = sum_{k in g} (qA[m,k] - zA[m,g]) * w[n,k]   (exact integer)
 * with sA[m,g], zA[m,g] from the per-row rule of quantize_rows_a8 applied to
 * the 32 values of block g of row m, and the group combination in float32.
 *   packed_w from pack_w4_g32 (f32 group scales).  q_out [M][K] int8,
 *   scale_out [M][K/32] f32 and zp_out [M][K/32] int32 are optional.
 *   M == 1: K % 128 == 0, K <= 8192 and x 16-byte aligned (else
 *   QG_ERR_UNSUPPORTED); no workspace; the stream note of qgemm_a8w4_f32
 *   (M == 1) applies.  M > 1: K % 64 == 0 and K <= 8192 (else
 *   QG_ERR_UNSUPPORTED), the tensor-core path of qgemm_a8w4_f32 with a
 *   workspace of qgemm_a8w4_workspace_bytes(M, N, K) bytes, 256-byte aligned.
 * ------------------------------------------------------------------------ */
int qgemm_a8w4_f32_actblock(int M, int N, int K, const float* x, int64_t ldx,
                            const void* packed_w, const float* bias,
                            float clamp_min, float clamp_max,
                            float* y, int64_t ldy,
                            int8_t* q_out, float* scale_out, int32_t* zp_out,
                            void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * A8W4 linear with asymmetric int4 weights.  [MNN] ConvInt8TiledExecutor,
 * asymmetric quant info: every (output channel, block) carries a zero and an
 * alpha, and a weight is alpha * code + zero.  Here:
 *   w_real[n,k] = sw[n,g] * w[n,k] + zw[n,g]     (w in [-8,7], g = k/32)
 *   y[m,n] = clamp(sA[m] * sum_g (sw[n,g]*I[m,n,g] + zw[n,g]*S[m,g]) + bias[n])
 *   I[m,n,g] = sum_{k in g} (qA[m,k] - zA[m]) * w[n,k],
 *   S[m,g] = sum_{k in g} (qA[m,k] - zA[m])
 * (I and S exact integers, the combination in float32).
 *   pack_w4_g32_asym: pack_w4_g32's layout followed by the f32 zeros
 *   zw[N][K/32] (row-major, contiguous), copied as given; size from
 *   pack_w4_g32_asym_bytes (0 when K % 32 != 0).  Checks as pack_w4_g32,
 *   plus group_zeros non-NULL and 4-byte aligned.
 *   qgemm_a8w4_f32_asym: arguments and outputs as qgemm_a8w4_f32.  M == 1:
 *   K % 128 == 0, K <= 8192 and x 16-byte aligned (else QG_ERR_UNSUPPORTED),
 *   no workspace, the same stream note.  M > 1: K % 64 == 0 and K <= 8192
 *   (else QG_ERR_UNSUPPORTED), a workspace of qgemm_a8w4_workspace_bytes.
 * ------------------------------------------------------------------------ */
size_t pack_w4_g32_asym_bytes(int N, int K);
int pack_w4_g32_asym(int N, int K, const int8_t* w, int64_t ldw, const float* group_scales,
                     const float* group_zeros, void* packed, size_t packed_bytes, void* stream);
int qgemm_a8w4_f32_asym(int M, int N, int K, const float* x, int64_t ldx,
                        const void* packed_w, const float* bias,
                        float clamp_min, float clamp_max,
                        float* y, int64_t ldy,
                        int8_t* q_out, float* scale_out, int32_t* zp_out,
                        void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Dynamic per-row symmetric int8 activation quantization.  [MNN]
 * ConvInt8TiledExecutor, BatchSymDynamicQuant: the absolute maximum of each
 * row gives a quantizing and a dequantizing scale, and the zero-point is 0.
 * All float32, one rounding per operation:
 *   amax = max_k |x[k]|
 *   scale = amax/127 and factor = 127/amax, both 1 if amax is 0
 *   q[k] = clamp(rne(x[k]*factor), -127, 127)
 *   x: f32 [M][ldx] (ldx >= K); q: int8 [M][ldq] (ldq >= K); scale: f32 [M].
 * Non-finite x is out of contract.
 * ------------------------------------------------------------------------ */
int quantize_rows_a8_sym(int M, int K, const float* x, int64_t ldx,
                         int8_t* q, int64_t ldq, float* scale, void* stream);

/* ------------------------------------------------------------------------
 * Convolution of a float input quantized on the fly, with int4 weights.
 * [MNN] ConvInt8TiledExecutor, low-memory path: the float input of a tile of
 * output pixels is unrolled (im2col) and every unrolled row is quantized
 * dynamically, asymmetric (BatchAsyDynamicQuant) or symmetric
 * (BatchSymDynamicQuant), before the int8 x int4 block-quantized product;
 * [QG] section 2: a tap in the padding stands for the real value 0.
 *
 *   x: f32 NHWC [Nb][H][W][Cin], 4-byte aligned
 *   packed_w: pack_w4_g32 of the int4 codes [Cout][KH][KW][Cin] read as
 *     [Cout][K], K = KH*KW*Cin in (kh, kw, ci) order, one scale per 32
 *     consecutive k of that order (K % 32 == 0, else QG_ERR_UNSUPPORTED)
 *   bias: f32 [Cout] or NULL;  y: f32 NHWC [Nb][OH][OW][Cout],
 *     OH = (H+2*pad_h-KH)/stride_h + 1 (same for W)
 * Unrolled row p = (n*OH+oh)*OW+ow holds x[n, oh*stride_h+kh-pad_h,
 * ow*stride_w+kw-pad_w, ci], 0 for a tap outside the image.  It is quantized
 * by quantize_rows_a8's rule (symmetric = 0) or quantize_rows_a8_sym's
 * (symmetric = 1, zero-point 0), and
 *   y[p, co] = clamp(sA[p] * sum_g sw[co,g] * I[p,co,g] + bias[co])
 *   I[p,co,g] = sum_{k in g} (qA[p,k] - zA[p]) * w[co,k]   (exact integer)
 * as qgemm_a8w4_f32.  q_out [P][K] int8 / scale_out [P] / zp_out [P] int32
 * (P = Nb*OH*OW): optional, receive the unrolled row quantization.
 * Workspace: qconv2d_f32_dyn_a8w4_workspace_bytes (256-byte aligned).
 * With K % 64 == 0, K <= 8192 and P >= 2 the rows are unrolled and quantized
 * straight into the tensor-core tiles of qgemm_a8w4_f32 (two kernels);
 * otherwise they are unrolled into the workspace for the CUDA-core kernel,
 * with the limits K <= 25600 and P <= 524280 (else QG_ERR_UNSUPPORTED).
 * ------------------------------------------------------------------------ */
size_t qconv2d_f32_dyn_a8w4_workspace_bytes(int Nb, int H, int W, int Cin, int Cout,
                                            int KH, int KW, int stride_h, int stride_w,
                                            int pad_h, int pad_w);
int qconv2d_f32_dyn_a8w4(int Nb, int H, int W, int Cin, int Cout, int KH, int KW,
                         int stride_h, int stride_w, int pad_h, int pad_w,
                         const float* x, const void* packed_w, const float* bias,
                         float clamp_min, float clamp_max, int symmetric, float* y,
                         int8_t* q_out, float* scale_out, int32_t* zp_out,
                         void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * qgemm_a8w4_f32 without a workspace.  The pages have no counterpart: this
 * entry point exists for callers that cannot allocate device memory for
 * scratch — a plugin inside a host framework that owns the allocator and
 * exposes none, or a serving loop that must not call cudaMalloc after
 * start-up because it can synchronise the device.
 *
 * Same arguments as qgemm_a8w4_f32 (without the optional quantization
 * outputs), and the same results within the A8W4 tolerance: M == 1 runs the
 * same fused GEMV; M > 1 always runs the CUDA-core GEMM (qgemm_a8w4_f32 may
 * take the tensor-core kernel there, which adds the same exact group dots in
 * another float order).  The scratch (per-row int8 activations, scales and
 * zero-points) lives in a fixed array in device global memory owned by the
 * library: 4 MiB + 64 KiB, held on every GPU that loads the library until
 * the process exits.  Limits when M > 1: M <= 8192 and M*K <= 4194304, else
 * QG_ERR_WORKSPACE; K <= 25600, else QG_ERR_UNSUPPORTED (8 rows of codes
 * sit in shared memory).  A rejected call launches nothing.  It never calls
 * cudaMalloc/cudaFree or any allocating routine.
 *
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  Every call on a device shares the one array
 * and each call overwrites every scratch byte it later reads, so nothing
 * needs clearing — but calls whose work overlaps on the GPU (different
 * streams, no ordering between them) race on it: order them.
 * ------------------------------------------------------------------------ */
int qgemm_a8w4_f32_noalloc(int M, int N, int K, const float* x, int64_t ldx,
                           const void* packed_w, const float* bias,
                           float clamp_min, float clamp_max,
                           float* y, int64_t ldy, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* QGEMM_H_ */
