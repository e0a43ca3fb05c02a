// A8W4 path: dynamic per-row int8 activation quantization (asymmetric, and
// symmetric or gathered from an unrolled conv input), int4 group-32 weight
// packing, and the A8W4 linear (fused M=1 GEMV; M>1 GEMM).
//
// Sources: pytorch/ao PR #997 "Kleidi 4b blockwise gemv prototype"
// (matmul_clamp_f32_qai8dxp_qsi4c32p: int8 dynamic per-row asymmetric
// activations, int4 symmetric weights with one scale per 32 K, f32 output
// clamped after the bias); MNN ConvInt8TiledExecutor.cpp
// (BatchAsyDynamicQuant min/max quantization, BatchSymDynamicQuant absolute
// maximum quantization, the low-memory float im2col path; int4 weights
// stored with an offset of 8 in _computeReorderQuantInfo).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "qg_internal.cuh"

namespace qg {


// Block-wide min/max of one row (blockDim.x threads, multiple of 32, <= 1024).
__device__ __forceinline__ void block_minmax(float& mn, float& mx, float* red /* [64] */) {
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  if (lane == 0) {
    red[warp] = mn;
    red[32 + warp] = mx;
  }
  __syncthreads();
  mn = red[0];
  mx = red[32];
  for (int i = 1; i < nw; ++i) {
    mn = fminf(mn, red[i]);
    mx = fmaxf(mx, red[32 + i]);
  }
  __syncthreads();
}

// One CTA per row.
__global__ void __launch_bounds__(256) quantize_rows_kernel(int K, const float* __restrict__ x,
                                                            int64_t ldx, int8_t* __restrict__ q,
                                                            int64_t ldq, float* __restrict__ scale,
                                                            int32_t* __restrict__ zero_point) {
  __shared__ float red[64];
  const int64_t m = blockIdx.x;
  const float* xr = x + m * ldx;
  float mn = 0.0f, mx = 0.0f;  // min(0, .) and max(0, .)
  // unrolled so that eight independent loads are in flight per thread
  int k = threadIdx.x;
  for (; k + 7 * (int)blockDim.x < K; k += 8 * blockDim.x) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = xr[k + u * blockDim.x];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      mn = fminf(mn, v[u]);
      mx = fmaxf(mx, v[u]);
    }
  }
  for (; k < K; k += blockDim.x) {
    float v = xr[k];
    mn = fminf(mn, v);
    mx = fmaxf(mx, v);
  }
  block_minmax(mn, mx, red);
  RowQuant r = row_quant_params(mn, mx);
  int8_t* qr = q + m * ldq;
  k = threadIdx.x;
  for (; k + 7 * (int)blockDim.x < K; k += 8 * blockDim.x) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = xr[k + u * blockDim.x];
#pragma unroll
    for (int u = 0; u < 8; ++u) qr[k + u * blockDim.x] = (int8_t)quant_one(v[u], r);
  }
  for (; k < K; k += blockDim.x) qr[k] = (int8_t)quant_one(xr[k], r);
  if (threadIdx.x == 0) {
    scale[m] = r.scale;
    zero_point[m] = r.zp;
  }
}

int launch_quantize_rows(int M, int K, const float* x, int64_t ldx, int8_t* q, int64_t ldq,
                         float* scale, int32_t* zp, cudaStream_t st) {
  if (M == 0) return QG_OK;
  quantize_rows_kernel<<<M, 256, 0, st>>>(K, x, ldx, q, ldq, scale, zp);
  return launch_status();
}

// ---------------------------------------------------------------------------
// Gathered rows, quantized on the fly (MNN ConvInt8TiledExecutor, low-memory
// path: the float input of a tile of output pixels is unrolled and each
// unrolled row quantized before the int8 product).  One warp per row; a row
// is `taps` runs of `run` consecutive floats.  CONV: row m is output pixel
// (n, oh, ow) of an NHWC image, run r = (kh, kw) reads pixel
// (oh*sh+kh-ph, ow*sw+kw-pw), and a run outside the image is the value 0
// ([QG] section 2), which is never read and never widens the range (0 is
// always inside it).  Otherwise row m is x + m*ldx, one run of K.
// Asymmetric rows take the per-row rule above; symmetric rows
// (BatchSymDynamicQuant) take amax = max|x|, scale = amax/127, quantizing
// factor 127/amax (both 1 when amax is 0), codes clamp(rne(x*factor), -127,
// 127) and zero-point 0.
// ---------------------------------------------------------------------------
struct GatherGeom {
  int H, W, Cin, KH, KW, sh, sw, ph, pw, OH, OW;
};

constexpr int kGatherWarps = 8;

template <bool SYM, bool CONV>
__global__ void __launch_bounds__(kGatherWarps * 32) quantize_gathered_rows_kernel(
    int M, int K, const float* __restrict__ x, int64_t ldx, GatherGeom g,
    int8_t* __restrict__ q, int64_t ldq, float* __restrict__ scale,
    int32_t* __restrict__ zero_point) {
  const int lane = threadIdx.x & 31;
  const int64_t m = (int64_t)blockIdx.x * kGatherWarps + (threadIdx.x >> 5);
  if (m >= M) return;
  const int taps = CONV ? g.KH * g.KW : 1;
  const int run = CONV ? g.Cin : K;
  int64_t n = 0;
  int oh = 0, ow = 0;
  if (CONV) {
    ow = (int)(m % g.OW);
    const int64_t t = m / g.OW;
    oh = (int)(t % g.OH);
    n = t / g.OH;
  }
  // start of run t of this row, or nullptr for a run outside the image
  auto run_ptr = [&](int t) -> const float* {
    if (!CONV) return x + m * ldx;
    const int kh = t / g.KW, kw = t - kh * g.KW;
    const int ih = oh * g.sh + kh - g.ph, iw = ow * g.sw + kw - g.pw;
    if (ih < 0 || ih >= g.H || iw < 0 || iw >= g.W) return nullptr;
    return x + ((n * g.H + ih) * g.W + iw) * (int64_t)g.Cin;
  };
  float mn = 0.0f, mx = 0.0f;
  for (int t = 0; t < taps; ++t) {
    const float* p = run_ptr(t);
    if (!p) continue;
    for (int c = lane; c < run; c += 32) {
      const float v = __ldg(p + c);
      if (SYM) {
        mx = fmaxf(mx, fabsf(v));
      } else {
        mn = fminf(mn, v);
        mx = fmaxf(mx, v);
      }
    }
  }
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  RowQuant r;
  if (SYM) {
    r.scale = mx == 0.0f ? 1.0f : __fdiv_rn(mx, 127.0f);
    r.inv = mx == 0.0f ? 1.0f : __fdiv_rn(127.0f, mx);
    r.zp = 0;
  } else {
    r = row_quant_params(mn, mx);
  }
  int8_t* qr = q + m * ldq;
  for (int t = 0; t < taps; ++t) {
    const float* p = run_ptr(t);
    int8_t* qt = qr + (int64_t)t * run;
    for (int c = lane; c < run; c += 32) {
      const float v = p ? __ldg(p + c) : 0.0f;
      int code;
      if (SYM)
        code = min(max(__float2int_rn(__fmul_rn(v, r.inv)), -127), 127);
      else
        code = quant_one(v, r);
      qt[c] = (int8_t)code;
    }
  }
  if (lane == 0) {
    scale[m] = r.scale;
    if (zero_point) zero_point[m] = r.zp;
  }
}

int launch_quantize_rows_sym(int M, int K, const float* x, int64_t ldx, int8_t* q, int64_t ldq,
                             float* scale, int32_t* zp, cudaStream_t st) {
  if (M == 0) return QG_OK;
  const GatherGeom g{};
  quantize_gathered_rows_kernel<true, false>
      <<<(unsigned)cdiv(M, kGatherWarps), kGatherWarps * 32, 0, st>>>(M, K, x, ldx, g, q, ldq,
                                                                      scale, zp);
  return launch_status();
}

// Unrolled rows of an NHWC float image: P = Nb*OH*OW rows of K = KH*KW*Cin
// codes, row-major with ld K.
int launch_im2col_quantize(int Nb, int H, int W, int Cin, int KH, int KW, int sh, int sw, int ph,
                           int pw, const float* x, bool symmetric, int8_t* q, float* scale,
                           int32_t* zp, cudaStream_t st) {
  const int OH = (H + 2 * ph - KH) / sh + 1, OW = (W + 2 * pw - KW) / sw + 1;
  const int64_t P = (int64_t)Nb * OH * OW;
  const int K = KH * KW * Cin;
  if (P == 0) return QG_OK;
  const GatherGeom g{H, W, Cin, KH, KW, sh, sw, ph, pw, OH, OW};
  const unsigned grid = (unsigned)cdiv(P, kGatherWarps);
  if (symmetric)
    quantize_gathered_rows_kernel<true, true>
        <<<grid, kGatherWarps * 32, 0, st>>>((int)P, K, x, 0, g, q, K, scale, zp);
  else
    quantize_gathered_rows_kernel<false, true>
        <<<grid, kGatherWarps * 32, 0, st>>>((int)P, K, x, 0, g, q, K, scale, zp);
  return launch_status();
}

// ---------------------------------------------------------------------------
// W4 pack: one thread per output 32-bit word (8 consecutive k of a row).
// word j of row n: byte b = (w[8j+b]+8) | (w[8j+4+b]+8) << 4.
// ---------------------------------------------------------------------------
__global__ void pack_w4_kernel(int N, int K, const int8_t* __restrict__ w, int64_t ldw,
                               const float* __restrict__ sw, uint8_t* __restrict__ packed,
                               int scale_bf16, int* status) {
  const int64_t words_per_row = K / 8;
  const int64_t total = (int64_t)N * words_per_row;
  const int G = K / 32;
  uint32_t* out = reinterpret_cast<uint32_t*>(packed);
  uint8_t* sout = packed + (size_t)N * (K / 2);  // f32 or bf16 scales [N][K/32]
  bool bad = false;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = i / words_per_row, j = i % words_per_row;
    const int8_t* src = w + n * ldw + 8 * j;
    uint32_t word = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      int lo = src[b], hi = src[4 + b];
      bad |= (lo < -8) | (lo > 7) | (hi < -8) | (hi > 7);
      word |= (uint32_t)(((lo + 8) & 0xF) | (((hi + 8) & 0xF) << 4)) << (8 * b);
    }
    out[i] = word;
  }
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < (int64_t)N * G;
       i += (int64_t)gridDim.x * blockDim.x) {
    if (scale_bf16)  // round to nearest even
      reinterpret_cast<unsigned short*>(sout)[i] = __bfloat16_as_ushort(__float2bfloat16_rn(sw[i]));
    else
      reinterpret_cast<float*>(sout)[i] = sw[i];
  }
  if (bad) record_error(status, QG_ERR_INVALID_ARG);
}

int launch_pack_w4(int N, int K, const int8_t* w, int64_t ldw, const float* sw, void* packed,
                   bool scale_bf16, cudaStream_t st) {
  const int64_t words = (int64_t)N * (K / 8);
  int blocks = (int)min64(cdiv(words, 256), (int64_t)num_sms() * 8);
  if (blocks < 1) blocks = 1;
  pack_w4_kernel<<<blocks, 256, 0, st>>>(N, K, w, ldw, sw, (uint8_t*)packed, scale_bf16 ? 1 : 0,
                                         status_word());
  return launch_status();
}

// ---------------------------------------------------------------------------
// Shared per-group arithmetic.
//
// With u = w + 8 in [0,15] stored as nibbles, for one 32-wide group g:
//   E  = sum_k qA[k] * u[k]                      (dp4a, bytes of u as s8 >= 0)
//   U  = sum_k u[k]
//   SA = sum_k qA[k]
//   I  = sum_k (qA[k] - zA) * w[k] = E - 8*SA - zA*U + 256*zA
// c = 256*zA - 8*SA depends on the activation only and seeds the dp4a chain.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int group_dot(const uint4 w, const int (&a)[8], int c, int za) {
  const uint32_t m = 0x0F0F0F0Fu;
  uint32_t l0 = w.x & m, h0 = (w.x >> 4) & m;
  uint32_t l1 = w.y & m, h1 = (w.y >> 4) & m;
  uint32_t l2 = w.z & m, h2 = (w.z >> 4) & m;
  uint32_t l3 = w.w & m, h3 = (w.w >> 4) & m;
  // two independent dp4a chains (low / high nibbles) halve the dependency depth
  int e0 = c, e1 = 0;
  e0 = __dp4a((int)l0, a[0], e0);
  e1 = __dp4a((int)h0, a[1], e1);
  e0 = __dp4a((int)l1, a[2], e0);
  e1 = __dp4a((int)h1, a[3], e1);
  e0 = __dp4a((int)l2, a[4], e0);
  e1 = __dp4a((int)h2, a[5], e1);
  e0 = __dp4a((int)l3, a[6], e0);
  e1 = __dp4a((int)h3, a[7], e1);
  // bytewise sums stay below 256 (8 nibbles of at most 15): no carries
  uint32_t t = (l0 + h0) + (l1 + h1) + (l2 + h2) + (l3 + h3);
  int U = __dp4a((int)t, 0x01010101, 0);
  return e0 + e1 - za * U;
}

__device__ __forceinline__ int act_seed(const int (&a)[8], int za) {
  int sa = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) sa = __dp4a(a[j], 0x01010101, sa);
  return 256 * za - 8 * sa;
}

__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// 16 bytes through L2 only (coherent with writes of a preceding grid).
__device__ __forceinline__ float4 ld_cg_f4(const float* p) {
  float4 v;
  asm volatile("ld.global.cg.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t ld_stream_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ float ld_stream_f32(const float* p) {
  float v;
  asm volatile("ld.global.nc.L1::no_allocate.f32 %0, [%1];" : "=f"(v) : "l"(p));
  return v;
}

// Scale of group g = lane + 32*i of row r (G groups per row) for the GEMV
// lanes.  With bf16 scales the lane reads the 32-bit word holding the scales
// of groups g and g^1; g has the lane's parity, so the half is picked with a
// byte permute whose selector `sel` the caller fixes once per lane (0x1044:
// low half, 0x3244: high half, moved to the top of an f32 pattern).
template <bool SBF>
__device__ __forceinline__ float ld_row_scale(const void* base, int64_t r, int G, int lane, int i,
                                              uint32_t sel) {
  if constexpr (SBF) {
    const uint32_t* p = reinterpret_cast<const uint32_t*>(base) + r * (G >> 1) + (lane >> 1) + 16 * i;
    uint32_t v, d;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(d) : "r"(v), "r"(sel));
    return __uint_as_float(d);
  } else {
    return ld_stream_f32(reinterpret_cast<const float*>(base) + r * G + lane + 32 * i);
  }
}

// Group scale i of a packed W4 matrix, stored as f32 or (SBF) as bf16; a bf16
// value widens to f32 exactly.  A bf16 scale is read as the aligned 32-bit
// word holding it and its neighbour (the scale array starts 16-byte aligned).
template <bool SBF>
__device__ __forceinline__ float ld_scale(const void* base, int64_t i) {
  if constexpr (SBF) {
    const uint32_t* p = reinterpret_cast<const uint32_t*>(base) + (i >> 1);
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return __uint_as_float((i & 1) ? (v & 0xFFFF0000u) : (v << 16));
  } else {
    return ld_stream_f32(reinterpret_cast<const float*>(base) + i);
  }
}

// ---------------------------------------------------------------------------
// Fused A8W4 GEMV (M = 1).
//
// Grid: a multiple of the SM count; CTA c owns the contiguous rows
// [c*N/grid, (c+1)*N/grid).  Thread 0 first asks the copy engine to stage that
// whole slice of nibbles and scales into L2 (one bulk prefetch), so HBM streams
// at full rate from the start while the CTA quantizes x into shared memory.
// Each warp then owns rows r, r+8, ...; lane l holds the activations of groups
// l, l+32, ... in registers (8 words per group) and reads the matching 16-byte
// nibble chunk and scale of each row with coalesced 128-bit loads.  Two rows
// per iteration keep eight 128-bit loads in flight per lane; their partial
// sums are reduced together with five shuffles.
// ---------------------------------------------------------------------------
template <int GPL, bool SBF>
__global__ void __launch_bounds__(256) a8w4_gemv_kernel(
    int N, int K, const float* __restrict__ x, const uint8_t* __restrict__ wq,
    const void* __restrict__ wscale, const float* __restrict__ bias, float clamp_lo,
    float clamp_hi, float* __restrict__ y, int8_t* __restrict__ q_out, float* __restrict__ scale_out,
    int32_t* __restrict__ zp_out) {
  extern __shared__ __align__(16) int8_t qa_s[];  // K bytes
  __shared__ float red[64];
  const int G = K >> 5;
  const int64_t rowbytes = K >> 1;
  const int n0 = (int)((int64_t)blockIdx.x * N / gridDim.x);
  const int n1 = (int)((int64_t)(blockIdx.x + 1) * N / gridDim.x);

  if (threadIdx.x == 0 && n1 > n0) {
    // nibbles of rows [n0, n1): contiguous, 16-byte multiple
    const uint8_t* p = wq + (int64_t)n0 * rowbytes;
    int64_t bytes = (int64_t)(n1 - n0) * rowbytes;
    while (bytes > 0) {
      uint32_t c = (uint32_t)min64(bytes, 1 << 20);
      bulk_prefetch_l2(p, c);
      p += c;
      bytes -= c;
    }
    // scales: round the start down and the end down to 16 bytes (in bounds)
    const int64_t sb = SBF ? 2 : 4;  // bytes per scale
    uintptr_t s0 = ((uintptr_t)wscale + (uintptr_t)((int64_t)n0 * G * sb)) & ~(uintptr_t)15;
    uintptr_t s1 = ((uintptr_t)wscale + (uintptr_t)((int64_t)n1 * G * sb)) & ~(uintptr_t)15;
    if (s1 > s0) bulk_prefetch_l2((const void*)s0, (uint32_t)(s1 - s0));
  }

  // ---- quantize x (row 0) into shared memory ----
  float mn = 0.0f, mx = 0.0f;
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    float v = x[k];
    mn = fminf(mn, v);
    mx = fmaxf(mx, v);
  }
  block_minmax(mn, mx, red);
  const RowQuant rq = row_quant_params(mn, mx);
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    int v = quant_one(x[k], rq);
    qa_s[k] = (int8_t)v;
    if (blockIdx.x == 0 && q_out) q_out[k] = (int8_t)v;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    if (scale_out) scale_out[0] = rq.scale;
    if (zp_out) zp_out[0] = rq.zp;
  }
  __syncthreads();

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int za = rq.zp;
  const int chunks = (G + 32 * GPL - 1) / (32 * GPL);

  int a[GPL][8];
  int cseed[GPL];
  auto load_act = [&](int chunk) {
#pragma unroll
    for (int i = 0; i < GPL; ++i) {
      const int g = chunk * 32 * GPL + lane + 32 * i;
      if (g < G) {
        const int4* src = reinterpret_cast<const int4*>(qa_s + 32 * g);
        int4 v0 = src[0], v1 = src[1];
        a[i][0] = v0.x; a[i][1] = v0.y; a[i][2] = v0.z; a[i][3] = v0.w;
        a[i][4] = v1.x; a[i][5] = v1.y; a[i][6] = v1.z; a[i][7] = v1.w;
        cseed[i] = act_seed(a[i], za);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) a[i][j] = 0;
        cseed[i] = 0;
      }
    }
  };
  if (chunks == 1) load_act(0);

  for (int r = n0 + warp; r < n1; r += 16) {
    const int rb = r + 8;
    const bool has_b = rb < n1;
    float acc0 = 0.0f, acc1 = 0.0f;
    for (int ch = 0; ch < chunks; ++ch) {
      if (chunks > 1) load_act(ch);
      uint4 w0[GPL], w1[GPL];
      float s0[GPL], s1[GPL];
#pragma unroll
      for (int i = 0; i < GPL; ++i) {
        const int g = ch * 32 * GPL + lane + 32 * i;
        if (g < G) {
          w0[i] = ld_stream_u4(wq + (int64_t)r * rowbytes + 16 * g);
          s0[i] = ld_scale<SBF>(wscale, (int64_t)r * G + g);
          if (has_b) {
            w1[i] = ld_stream_u4(wq + (int64_t)rb * rowbytes + 16 * g);
            s1[i] = ld_scale<SBF>(wscale, (int64_t)rb * G + g);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < GPL; ++i) {
        const int g = ch * 32 * GPL + lane + 32 * i;
        if (g < G) {
          acc0 = fmaf(s0[i], (float)group_dot(w0[i], a[i], cseed[i], za), acc0);
          if (has_b) acc1 = fmaf(s1[i], (float)group_dot(w1[i], a[i], cseed[i], za), acc1);
        }
      }
    }
    // lanes with bit0 = 0 finish row r, lanes with bit0 = 1 finish row rb
    const bool odd = lane & 1;
    float keep = odd ? acc1 : acc0;
    float give = odd ? acc0 : acc1;
    keep += __shfl_xor_sync(0xffffffffu, give, 1);
#pragma unroll
    for (int o = 2; o < 32; o <<= 1) keep += __shfl_xor_sync(0xffffffffu, keep, o);
    if (lane < 2) {
      const int row = lane ? rb : r;
      if (lane == 0 || has_b) {
        float v = __fmul_rn(rq.scale, keep);
        if (bias) v = __fadd_rn(v, bias[row]);
        y[row] = fminf(fmaxf(v, clamp_lo), clamp_hi);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Fused A8W4 GEMV (M = 1), register-pipelined row streaming (K % 128 == 0,
// K <= 8192).
//
// One CTA per SM owns the contiguous rows [n0, n1).  The first W * nfull
// rows (nfull = (n1 - n0) / W) go round-robin to the W warps; each of the
// L < W rows left over is split by groups across GPL warps (warp w takes
// slot w % GPL of every lane) and their partial sums meet in shared memory,
// so no warp finishes a whole extra row alone (14336 rows over 148 SMs give
// 96 or 97 rows per CTA: 6 per warp plus at most one split row).  Lane l holds the quantized activations of groups
// l, l+32, ... in registers and, for every row, loads the matching 16-byte
// nibble chunk and f32 scale of each of its groups with 128-bit / 32-bit
// non-coherent loads: each warp instruction reads 512 contiguous bytes.  Each
// warp keeps D rows of loads in flight in registers: after computing a row it
// issues the loads of its row D further on into the registers just freed.
// The weight stream therefore never passes through the copy engine (whose
// per-request cost bounds small copies) nor through shared memory.
//
// Launch overlap.  Launches use programmatic dependent launch.  Packed
// weights and scales are inputs of the call alone, so every warp issues the
// loads of its first D rows before waiting for the previous grid; x and bias
// may be outputs of that grid, so before the wait they are only prefetched
// into L2 (a prefetch cannot return stale data: L2 is where every write
// lands).  After the wait every thread loads its share of x into registers
// (through L2) and the CTA quantizes it while those weight rows are in
// flight; once x has landed the rest of the CTA's slice is prefetched into
// L2.
// ---------------------------------------------------------------------------
constexpr int kStreamSmemMax = 96 * 1024;  // qa_s + bias_s

// Warp-wide float min / max (NaN inputs ignored, as fminf / fmaxf do).
__device__ __forceinline__ float warp_min(float v) {
  float r;
  asm volatile("redux.sync.min.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}
__device__ __forceinline__ float warp_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

template <int W>
__device__ __forceinline__ void gemv_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(W * 32) : "memory");
}

// L2 prefetch of the 16-byte-aligned interior of [p, p + bytes).
__device__ __forceinline__ void prefetch_l2_interior(const void* p, int64_t bytes) {
  uintptr_t a = ((uintptr_t)p + 15) & ~(uintptr_t)15;
  const uintptr_t e = ((uintptr_t)p + (uintptr_t)bytes) & ~(uintptr_t)15;
  while (a < e) {
    const uint32_t c = (uint32_t)min64((int64_t)(e - a), 1 << 20);
    bulk_prefetch_l2((const void*)a, c);
    a += c;
  }
}

template <int GPL, int W, int D, bool SBF, bool ABLK, bool WZP, int CPS>
__global__ void __launch_bounds__(W * 32, CPS) a8w4_gemv_stream_kernel(
    int N, int K, int max_rows, const float* __restrict__ x, const uint8_t* __restrict__ wq,
    const void* __restrict__ wscale, const float* __restrict__ wzero,
    const float* __restrict__ bias, float clamp_lo,
    float clamp_hi, float* __restrict__ y, int8_t* __restrict__ q_out,
    float* __restrict__ scale_out, int32_t* __restrict__ zp_out, int* status) {
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ float red[2 * W];
  __shared__ float part_s[W * GPL];        // partial sums of the split rows
  // ABLK (activations quantized per 32-wide K block): scale and zero-point of
  // each block
  static_assert(!(ABLK && WZP), "weight zeros are taken with per-row activation scales");
  __shared__ float blk_scale_s[ABLK ? GPL * 32 : 1];
  __shared__ int blk_zp_s[ABLK ? GPL * 32 : 1];
  const int G = K >> 5;
  const int rowbytes = K >> 1;
  int8_t* qa_s = reinterpret_cast<int8_t*>(sm);      // [K] quantized x
  float* bias_s = reinterpret_cast<float*>(sm + K);  // [max_rows]

  const int n0 = (int)((int64_t)blockIdx.x * N / gridDim.x);
  const int n1 = (int)((int64_t)(blockIdx.x + 1) * N / gridDim.x);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nrows = (n1 - n0) / W;         // whole rows per warp
  const int nleft = n1 - n0 - W * nrows;   // rows split across warps
  const int slot = warp % GPL;             // this warp's slot in a split row
  static_assert(W % GPL == 0, "split rows need W to be a multiple of GPL");

  uint4 wbuf[D][GPL];
  float sbuf[SBF ? 1 : D][GPL];
  // SBF: the row's bf16 scales as 32-bit words, read whole (lane l holds
  // words l, l + 32, ...: 128 contiguous bytes per load) and handed to the
  // lanes of their groups by shuffles when the row is used
  constexpr int SW = (GPL + 1) / 2;
  uint32_t swd[SBF ? D : 1][SW];
  float zbuf[WZP ? D : 1][GPL];  // WZP: f32 weight zero of each group
  // loads of this warp's row j into buffer u (nothing past the last row)
  const uint32_t ssel = (lane & 1) ? 0x3244u : 0x1044u;  // bf16 half of the scale word
  auto load_row = [&](int u, int j) {
    if (j < nrows) {
      const int r = n0 + warp + W * j;
#pragma unroll
      for (int i = 0; i < GPL; ++i) {
        const int g = lane + 32 * i;
        if (g < G) {
          wbuf[u][i] = ld_stream_u4(wq + (int64_t)r * rowbytes + 16 * g);
          if constexpr (!SBF) sbuf[u][i] = ld_row_scale<false>(wscale, r, G, lane, i, ssel);
          if constexpr (WZP) zbuf[u][i] = ld_stream_f32(wzero + (int64_t)r * G + g);
        }
      }
      if constexpr (SBF) {
        const uint32_t* rw = reinterpret_cast<const uint32_t*>(wscale) + (int64_t)r * (G >> 1);
#pragma unroll
        for (int jj = 0; jj < SW; ++jj) {
          const int w = lane + 32 * jj;
          swd[u][jj] = w < (G >> 1) ? ld_stream_u32(rw + w) : 0u;
        }
      }
    }
  };

  if (threadIdx.x == 0) {
    prefetch_l2_interior(x, (int64_t)K * 4);
    if (bias && n1 > n0) prefetch_l2_interior(bias + n0, (int64_t)(n1 - n0) * 4);
  }
#pragma unroll
  for (int u = 0; u < D; ++u) load_row(u, u);
  // the first split row this warp takes part in
  uint4 wsplit = make_uint4(0, 0, 0, 0);
  float ssplit = 0.0f, zsplit = 0.0f;
  auto load_split = [&](int k) {
    const int r = n0 + W * nrows + k;
    const int g = lane + 32 * slot;
    if (g < G) {
      wsplit = ld_stream_u4(wq + (int64_t)r * rowbytes + 16 * g);
      ssplit = ld_row_scale<SBF>(wscale, r, G, lane, slot, ssel);
      if constexpr (WZP) zsplit = ld_stream_f32(wzero + (int64_t)r * G + g);
    }
  };
  if (warp / GPL < nleft) load_split(warp / GPL);
  __syncthreads();
  // Programmatic dependent launch: let the next grid in the stream start its
  // own prologue, then wait until the previous grid's writes are visible.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // ---------------- quantize x ----------------
  for (int i = threadIdx.x; i < n1 - n0; i += W * 32)
    bias_s[i] = bias ? bias[n0 + i] : 0.0f;
  // Each thread loads its float4 chunks of x once (through L2, coherent with
  // the previous grid's writes) and keeps them in registers for both passes
  // (K <= 1024*GPL).
  constexpr int XV = (GPL * 1024 + 4 * W * 32 - 1) / (4 * W * 32);
  float4 xv[XV];
  float mn = 0.0f, mx = 0.0f;
#pragma unroll
  for (int j = 0; j < XV; ++j) {
    const int c = threadIdx.x + j * W * 32;  // float4 chunk index
    xv[j] = 4 * c < K ? ld_cg_f4(x + 4 * c) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int j = 0; j < XV; ++j) {
    mn = fminf(mn, fminf(fminf(xv[j].x, xv[j].y), fminf(xv[j].z, xv[j].w)));
    mx = fmaxf(mx, fmaxf(fmaxf(xv[j].x, xv[j].y), fmaxf(xv[j].z, xv[j].w)));
  }
  // The rest of the slice into L2, queued only once x (on the critical path)
  // has landed: mn <= 0 always holds (the running minimum starts at 0, and
  // fminf ignores NaN), but testing it makes the prefetch wait for this
  // thread's x loads.
  if (threadIdx.x == 0 && mn <= 0.0f) {
    const int r_rest = n0 + W * min(D, nrows);  // rows beyond the ones already requested
    if (r_rest < n1) {
      prefetch_l2_interior(wq + (int64_t)r_rest * rowbytes, (int64_t)(n1 - r_rest) * rowbytes);
      constexpr int64_t sb = SBF ? 2 : 4;  // bytes per scale
      prefetch_l2_interior((const uint8_t*)wscale + (int64_t)r_rest * G * sb,
                           (int64_t)(n1 - r_rest) * G * sb);
      if (WZP) prefetch_l2_interior(wzero + (int64_t)r_rest * G, (int64_t)(n1 - r_rest) * G * 4);
    }
  }
  RowQuant rq;
  if constexpr (!ABLK) {
    mn = warp_min(mn);
    mx = warp_max(mx);
    if (lane == 0) {
      red[warp] = mn;
      red[W + warp] = mx;
    }
    gemv_bar<W>();
    // every warp combines the W per-warp results (lanes past W repeat warp 0's)
    mn = warp_min(red[lane < W ? lane : 0]);
    mx = warp_max(red[W + (lane < W ? lane : 0)]);
    rq = row_quant_params(mn, mx);
#pragma unroll
    for (int j = 0; j < XV; ++j) {
      const int c = threadIdx.x + j * W * 32;
      if (4 * c < K) {
        const uint32_t b0 = (uint32_t)quant_one(xv[j].x, rq) & 0xFFu;
        const uint32_t b1 = (uint32_t)quant_one(xv[j].y, rq) & 0xFFu;
        const uint32_t b2 = (uint32_t)quant_one(xv[j].z, rq) & 0xFFu;
        const uint32_t b3 = (uint32_t)quant_one(xv[j].w, rq) & 0xFFu;
        reinterpret_cast<uint32_t*>(qa_s)[c] = b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
        if (blockIdx.x == 0 && q_out) {
          int8_t* qo = q_out + 4 * c;
          qo[0] = (int8_t)b0; qo[1] = (int8_t)b1; qo[2] = (int8_t)b2; qo[3] = (int8_t)b3;
        }
      }
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      if (scale_out) scale_out[0] = rq.scale;
      if (zp_out) zp_out[0] = rq.zp;
    }
  } else {
    // One 32-wide block = 8 consecutive float4 chunks, held by 8 consecutive
    // lanes (K % 128 == 0: a warp's 32 chunks are all in range or all out).
    // The per-row rule applies to each block: range including 0, f32 scale.
#pragma unroll
    for (int j = 0; j < XV; ++j) {
      const int c = threadIdx.x + j * W * 32;
      float bmn = fminf(0.0f, fminf(fminf(xv[j].x, xv[j].y), fminf(xv[j].z, xv[j].w)));
      float bmx = fmaxf(0.0f, fmaxf(fmaxf(xv[j].x, xv[j].y), fmaxf(xv[j].z, xv[j].w)));
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) {
        bmn = fminf(bmn, __shfl_xor_sync(0xffffffffu, bmn, o));
        bmx = fmaxf(bmx, __shfl_xor_sync(0xffffffffu, bmx, o));
      }
      if (4 * c < K) {
        const RowQuant bq = row_quant_params(bmn, bmx);
        const uint32_t b0 = (uint32_t)quant_one(xv[j].x, bq) & 0xFFu;
        const uint32_t b1 = (uint32_t)quant_one(xv[j].y, bq) & 0xFFu;
        const uint32_t b2 = (uint32_t)quant_one(xv[j].z, bq) & 0xFFu;
        const uint32_t b3 = (uint32_t)quant_one(xv[j].w, bq) & 0xFFu;
        reinterpret_cast<uint32_t*>(qa_s)[c] = b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
        if (blockIdx.x == 0 && q_out) {
          int8_t* qo = q_out + 4 * c;
          qo[0] = (int8_t)b0; qo[1] = (int8_t)b1; qo[2] = (int8_t)b2; qo[3] = (int8_t)b3;
        }
        if ((lane & 7) == 0) {
          blk_scale_s[c >> 3] = bq.scale;
          blk_zp_s[c >> 3] = bq.zp;
          if (blockIdx.x == 0 && scale_out) scale_out[c >> 3] = bq.scale;
          if (blockIdx.x == 0 && zp_out) zp_out[c >> 3] = bq.zp;
        }
      }
    }
    rq.scale = 1.0f;  // the activation scales enter per group below
    rq.inv = 1.0f;
    rq.zp = 0;
  }
  gemv_bar<W>();

  // zero-point and scale of the activations of each of this lane's groups
  int zag[GPL];
  float sag[GPL];
#pragma unroll
  for (int i = 0; i < GPL; ++i) {
    const int g = lane + 32 * i;
    zag[i] = ABLK ? (g < G ? blk_zp_s[g] : 0) : rq.zp;
    sag[i] = ABLK ? (g < G ? blk_scale_s[g] : 0.0f) : 1.0f;
  }
  int a[GPL][8];
  int cseed[GPL];
  float asum[GPL];  // WZP: the group sums of the centred activation codes
#pragma unroll
  for (int i = 0; i < GPL; ++i) asum[i] = 0.0f;
#pragma unroll
  for (int i = 0; i < GPL; ++i) {
    const int g = lane + 32 * i;
    if (g < G) {
      const int4* src = reinterpret_cast<const int4*>(qa_s + 32 * g);
      const int4 v0 = src[0], v1 = src[1];
      a[i][0] = v0.x; a[i][1] = v0.y; a[i][2] = v0.z; a[i][3] = v0.w;
      a[i][4] = v1.x; a[i][5] = v1.y; a[i][6] = v1.z; a[i][7] = v1.w;
      cseed[i] = act_seed(a[i], zag[i]);
      if constexpr (WZP) {  // S_g = sum_k (qA[k] - zA), exact
        int sraw = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) sraw = __dp4a(a[i][j], 0x01010101, sraw);
        asum[i] = (float)(sraw - 32 * zag[i]);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) a[i][j] = 0;
      cseed[i] = 0;
    }
  }

  // ---------------- stream this warp's rows ----------------
  for (int j0 = 0; j0 < nrows; j0 += D) {
#pragma unroll
    for (int u = 0; u < D; ++u) {
      const int j = j0 + u;
      if (j < nrows) {
        float acc = 0.0f;
        float scv[GPL];
#pragma unroll
        for (int i = 0; i < GPL; ++i) {
          if constexpr (SBF) {
            // group g = lane + 32i: word g / 2 = lane / 2 + 16i of the row
            const uint32_t wv =
                __shfl_sync(0xffffffffu, swd[u][i >> 1], (lane >> 1) + 16 * (i & 1));
            uint32_t d;
            asm("prmt.b32 %0, %1, 0, %2;" : "=r"(d) : "r"(wv), "r"(ssel));
            scv[i] = __uint_as_float(d);
          } else {
            scv[i] = sbuf[u][i];
          }
        }
#pragma unroll
        for (int i = 0; i < GPL; ++i) {
          const int g = lane + 32 * i;
          if (g < G) {
            const float sc = ABLK ? __fmul_rn(scv[i], sag[i]) : scv[i];
            acc = fmaf(sc, (float)group_dot(wbuf[u][i], a[i], cseed[i], zag[i]), acc);
            if constexpr (WZP) acc = fmaf(zbuf[u][i], asum[i], acc);
          }
        }
        load_row(u, j + D);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) {
          const int r = n0 + warp + W * j;
          float v = ABLK ? acc : __fmul_rn(rq.scale, acc);
          if (bias) v = __fadd_rn(v, bias_s[r - n0]);
          y[r] = fminf(fmaxf(v, clamp_lo), clamp_hi);
        }
      }
    }
  }

  // ---------------- split rows ----------------
  if (nleft > 0) {  // uniform across the CTA
    for (int k = warp / GPL; k < nleft; k += W / GPL) {
      if (k != warp / GPL) load_split(k);
      float part = 0.0f;
      const int g = lane + 32 * slot;
#pragma unroll
      for (int i = 0; i < GPL; ++i)  // static register indexing of a[slot]
        if (i == slot && g < G)
        {
          part = __fmul_rn(ABLK ? __fmul_rn(ssplit, sag[i]) : ssplit,
                           (float)group_dot(wsplit, a[i], cseed[i], zag[i]));
          if constexpr (WZP) part = fmaf(zsplit, asum[i], part);
        }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
      if (lane == 0) part_s[k * GPL + slot] = part;
    }
    gemv_bar<W>();
    if (threadIdx.x < nleft) {
      const int k = threadIdx.x;
      float acc = part_s[k * GPL];
#pragma unroll
      for (int i = 1; i < GPL; ++i) acc += part_s[k * GPL + i];
      const int r = n0 + W * nrows + k;
      float v = ABLK ? acc : __fmul_rn(rq.scale, acc);
      if (bias) v = __fadd_rn(v, bias_s[r - n0]);
      y[r] = fminf(fmaxf(v, clamp_lo), clamp_hi);
    }
  }
}

template <int GPL, int W, int D, bool SBF, bool ABLK = false, bool WZP = false, int CPS = 1>
static int launch_stream(int N, int K, const float* x, const uint8_t* wq, const void* ws, const float* wz,
                         const float* bias, float lo, float hi, float* y, int8_t* q_out,
                         float* scale_out, int32_t* zp_out, cudaStream_t st) {
  int grid = num_sms() * CPS;  // CPS co-resident CTAs per SM
  if (grid > N) grid = N;
  const int rows_per_cta = (N + grid - 1) / grid;
  const size_t smem = (size_t)K + (size_t)rows_per_cta * 4;  // qa_s, bias_s
  if (smem > (size_t)kStreamSmemMax) return 1;  // caller uses the plain kernel
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(W * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, a8w4_gemv_stream_kernel<GPL, W, D, SBF, ABLK, WZP, CPS>, N, K, rows_per_cta,
                                     x, wq, ws, wz, bias, lo, hi, y, q_out, scale_out, zp_out,
                                     status_word());
  return e == cudaSuccess ? QG_OK : QG_ERR_CUDA;
}

template <bool SBF>
static int launch_a8w4_gemv_t(int N, int K, const float* x, const void* packed,
                              const float* bias, float lo, float hi, float* y, int8_t* q_out,
                              float* scale_out, int32_t* zp_out, cudaStream_t st) {
  const uint8_t* wq = (const uint8_t*)packed;
  const void* ws = wq + (size_t)N * (K / 2);
  const int G = K / 32;
  int grid = num_sms() * 2;
  if (grid > N) grid = N;
  if (K % 128 == 0 && K <= 8192 && ((uintptr_t)x & 15) == 0) {
    int rc;
    if (G <= 32) rc = launch_stream<1, 16, 3, SBF>(N, K, x, wq, ws, nullptr, bias, lo, hi, y, q_out, scale_out, zp_out, st);
    else if (G <= 64) rc = launch_stream<2, 16, 3, SBF>(N, K, x, wq, ws, nullptr, bias, lo, hi, y, q_out, scale_out, zp_out, st);
    // K <= 4096: two CTAs of 8 warps per SM (a CTA that finishes its slice
    // leaves the SM to the other; 1x14336x4096: 7.73 -> 7.54 us)
    else if (G <= 128) rc = launch_stream<4, 8, 2, SBF, false, false, 2>(N, K, x, wq, ws, nullptr, bias, lo, hi, y, q_out, scale_out, zp_out, st);
    else rc = launch_stream<8, 8, 3, SBF>(N, K, x, wq, ws, nullptr, bias, lo, hi, y, q_out, scale_out, zp_out, st);
    if (rc <= 0) return rc;
  }
  const size_t smem = (size_t)K;
  if (G <= 32) {
    a8w4_gemv_kernel<1, SBF><<<grid, 256, smem, st>>>(N, K, x, wq, ws, bias, lo, hi, y, q_out,
                                                      scale_out, zp_out);
  } else if (G <= 64) {
    a8w4_gemv_kernel<2, SBF><<<grid, 256, smem, st>>>(N, K, x, wq, ws, bias, lo, hi, y, q_out,
                                                      scale_out, zp_out);
  } else {
    a8w4_gemv_kernel<4, SBF><<<grid, 256, smem, st>>>(N, K, x, wq, ws, bias, lo, hi, y, q_out,
                                                      scale_out, zp_out);
  }
  return launch_status();
}

int launch_a8w4_gemv(int N, int K, const float* x, const void* packed, const float* bias,
                     float lo, float hi, float* y, int8_t* q_out, float* scale_out,
                     int32_t* zp_out, bool scale_bf16, cudaStream_t st) {
  return scale_bf16 ? launch_a8w4_gemv_t<true>(N, K, x, packed, bias, lo, hi, y, q_out,
                                               scale_out, zp_out, st)
                    : launch_a8w4_gemv_t<false>(N, K, x, packed, bias, lo, hi, y, q_out,
                                                scale_out, zp_out, st);
}

// A8W4 GEMV with the activations quantized per 32-wide K block (f32 group
// scales): the streaming kernel only (K % 128 == 0, K <= 8192, x 16-byte
// aligned), else QG_ERR_UNSUPPORTED.
int launch_a8w4_gemv_actblock(int N, int K, const float* x, const void* packed, const float* bias,
                              float lo, float hi, float* y, int8_t* q_out, float* scale_out,
                              int32_t* zp_out, cudaStream_t st) {
  if (K % 128 != 0 || K > 8192 || ((uintptr_t)x & 15) != 0) return QG_ERR_UNSUPPORTED;
  const uint8_t* wq = (const uint8_t*)packed;
  const void* ws = wq + (size_t)N * (K / 2);
  const int G = K / 32;
  int rc;
  if (G <= 32) rc = launch_stream<1, 16, 3, false, true>(N, K, x, wq, ws, nullptr, bias, lo, hi, y, q_out, scale_out, zp_out, st);
  else if (G <= 64) rc = launch_stream<2, 16, 3, false, true>(N, K, x, wq, ws, nullptr, bias, lo, hi, y, q_out, scale_out, zp_out, st);
  else if (G <= 128) rc = launch_stream<4, 16, 2, false, true>(N, K, x, wq, ws, nullptr, bias, lo, hi, y, q_out, scale_out, zp_out, st);
  else rc = launch_stream<8, 8, 3, false, true>(N, K, x, wq, ws, nullptr, bias, lo, hi, y, q_out, scale_out, zp_out, st);
  return rc > 0 ? QG_ERR_UNSUPPORTED : rc;
}

// A8W4 GEMV with asymmetric int4 weights (an f32 zero per 32-wide group
// after the f32 scales): the streaming kernel only (K % 128 == 0, K <= 8192,
// x 16-byte aligned), else QG_ERR_UNSUPPORTED.
int launch_a8w4_gemv_asym(int N, int K, const float* x, const void* packed, const float* bias,
                          float lo, float hi, float* y, int8_t* q_out, float* scale_out,
                          int32_t* zp_out, cudaStream_t st) {
  if (K % 128 != 0 || K > 8192 || ((uintptr_t)x & 15) != 0) return QG_ERR_UNSUPPORTED;
  const uint8_t* wq = (const uint8_t*)packed;
  const float* ws = (const float*)(wq + (size_t)N * (K / 2));
  const float* wz = ws + (size_t)N * (K / 32);
  const int G = K / 32;
  int rc;
  if (G <= 32) rc = launch_stream<1, 16, 3, false, false, true>(N, K, x, wq, ws, wz, bias, lo, hi, y, q_out, scale_out, zp_out, st);
  else if (G <= 64) rc = launch_stream<2, 16, 3, false, false, true>(N, K, x, wq, ws, wz, bias, lo, hi, y, q_out, scale_out, zp_out, st);
  else if (G <= 128) rc = launch_stream<4, 16, 2, false, false, true>(N, K, x, wq, ws, wz, bias, lo, hi, y, q_out, scale_out, zp_out, st);
  else rc = launch_stream<8, 8, 3, false, false, true>(N, K, x, wq, ws, wz, bias, lo, hi, y, q_out, scale_out, zp_out, st);
  return rc > 0 ? QG_ERR_UNSUPPORTED : rc;
}

template <bool SBF>
static bool setup_a8w4_gemv_t() {
  // up to 64 KiB of activations in shared memory for the plain kernel
  const void* plain[] = {(const void*)a8w4_gemv_kernel<1, SBF>, (const void*)a8w4_gemv_kernel<2, SBF>,
                         (const void*)a8w4_gemv_kernel<4, SBF>};
  const void* stream[] = {(const void*)a8w4_gemv_stream_kernel<1, 16, 3, SBF, false, false, 1>,
                          (const void*)a8w4_gemv_stream_kernel<2, 16, 3, SBF, false, false, 1>,
                          (const void*)a8w4_gemv_stream_kernel<4, 8, 2, SBF, false, false, 2>,
                          (const void*)a8w4_gemv_stream_kernel<8, 8, 3, SBF, false, false, 1>};
  bool ok = true;
  for (const void* f : plain)
    ok &= cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, 65536) == cudaSuccess;
  for (const void* f : stream)
    ok &= cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, kStreamSmemMax) ==
          cudaSuccess;
  return ok;
}

int setup_a8w4_gemv() {
  bool ok = setup_a8w4_gemv_t<false>() && setup_a8w4_gemv_t<true>();
  const void* blk[] = {(const void*)a8w4_gemv_stream_kernel<1, 16, 3, false, true, false, 1>,
                       (const void*)a8w4_gemv_stream_kernel<2, 16, 3, false, true, false, 1>,
                       (const void*)a8w4_gemv_stream_kernel<4, 16, 2, false, true, false, 1>,
                       (const void*)a8w4_gemv_stream_kernel<8, 8, 3, false, true, false, 1>};
  for (const void* f : blk)
    ok &= cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, kStreamSmemMax) ==
          cudaSuccess;
  const void* asym[] = {(const void*)a8w4_gemv_stream_kernel<1, 16, 3, false, false, true, 1>,
                        (const void*)a8w4_gemv_stream_kernel<2, 16, 3, false, false, true, 1>,
                        (const void*)a8w4_gemv_stream_kernel<4, 16, 2, false, false, true, 1>,
                        (const void*)a8w4_gemv_stream_kernel<8, 8, 3, false, false, true, 1>};
  for (const void* f : asym)
    ok &= cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, kStreamSmemMax) ==
          cudaSuccess;
  return ok ? QG_OK : QG_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// A8W4 GEMM for M > 1 on CUDA cores (dp4a): activations quantized beforehand
// (q [M][K], scale, zp in the workspace).  CTA tile: 8 rows of M staged in
// shared memory x a slice of N; each warp owns one column n at a time, lanes
// split the groups, and every weight chunk loaded into registers serves the
// 8 rows.
// ---------------------------------------------------------------------------
constexpr int kSimtRows = 8;

template <bool SBF>
__global__ void __launch_bounds__(256) a8w4_gemm_simt_kernel(
    int M, int N, int K, const int8_t* __restrict__ q, const float* __restrict__ sA,
    const int32_t* __restrict__ zA, const uint8_t* __restrict__ wq,
    const void* __restrict__ wscale, const float* __restrict__ bias, float lo, float hi,
    float* __restrict__ y, int64_t ldy) {
  extern __shared__ __align__(16) int8_t qs[];  // kSimtRows * K
  const int G = K >> 5;
  const int64_t rowbytes = K >> 1;
  const int m0 = blockIdx.y * kSimtRows;
  const int rows = min(kSimtRows, M - m0);
  for (int i = threadIdx.x; i < rows * (K / 16); i += blockDim.x) {
    const int r = i / (K / 16), c = i % (K / 16);
    reinterpret_cast<int4*>(qs + (int64_t)r * K)[c] =
        reinterpret_cast<const int4*>(q + (int64_t)(m0 + r) * K)[c];
  }
  __syncthreads();
  int za[kSimtRows];
#pragma unroll
  for (int r = 0; r < kSimtRows; ++r) za[r] = r < rows ? zA[m0 + r] : 0;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n0 = (int)((int64_t)blockIdx.x * N / gridDim.x);
  const int n1 = (int)((int64_t)(blockIdx.x + 1) * N / gridDim.x);
  for (int n = n0 + warp; n < n1; n += 8) {
    float acc[kSimtRows];
#pragma unroll
    for (int r = 0; r < kSimtRows; ++r) acc[r] = 0.0f;
    for (int g = lane; g < G; g += 32) {
      const uint4 w = ld_stream_u4(wq + (int64_t)n * rowbytes + 16 * g);
      const float s = ld_scale<SBF>(wscale, (int64_t)n * G + g);
#pragma unroll
      for (int r = 0; r < kSimtRows; ++r) {
        if (r < rows) {
          const int4* src = reinterpret_cast<const int4*>(qs + (int64_t)r * K + 32 * g);
          int4 v0 = src[0], v1 = src[1];
          int a[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
          acc[r] = fmaf(s, (float)group_dot(w, a, act_seed(a, za[r]), za[r]), acc[r]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < kSimtRows; ++r) {
      float v = acc[r];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0 && r < rows) {
        float t = __fmul_rn(sA[m0 + r], v);
        if (bias) t = __fadd_rn(t, bias[n]);
        y[(int64_t)(m0 + r) * ldy + n] = fminf(fmaxf(t, lo), hi);
      }
    }
  }
}

int launch_a8w4_gemm_simt(int M, int N, int K, const int8_t* q, const float* sA,
                          const int32_t* zA, const void* packed, const float* bias, float lo,
                          float hi, float* y, int64_t ldy, bool scale_bf16, cudaStream_t st) {
  const uint8_t* wq = (const uint8_t*)packed;
  const void* ws = wq + (size_t)N * (K / 2);
  const int mblocks = (int)cdiv(M, kSimtRows);
  int nblocks = (int)max64(1, min64(cdiv((int64_t)num_sms() * 2, mblocks), cdiv(N, 8)));
  dim3 grid(nblocks, mblocks);
  const size_t smem = (size_t)kSimtRows * K;
  if (scale_bf16)
    a8w4_gemm_simt_kernel<true><<<grid, 256, smem, st>>>(M, N, K, q, sA, zA, wq, ws, bias, lo, hi,
                                                         y, ldy);
  else
    a8w4_gemm_simt_kernel<false><<<grid, 256, smem, st>>>(M, N, K, q, sA, zA, wq, ws, bias, lo, hi,
                                                          y, ldy);
  return launch_status();
}

int setup_a8w4_gemm_simt() {
  cudaError_t e = cudaFuncSetAttribute(a8w4_gemm_simt_kernel<false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
  cudaError_t e2 = cudaFuncSetAttribute(a8w4_gemm_simt_kernel<true>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
  return (e == cudaSuccess && e2 == cudaSuccess) ? QG_OK : QG_ERR_CUDA;
}

}  // namespace qg
