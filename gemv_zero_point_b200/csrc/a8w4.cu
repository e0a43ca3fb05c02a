// A8W4 path: dynamic per-row int8 activation quantization, int4 group-32
// weight packing, and the A8W4 linear (fused M=1 GEMV; M>1 GEMM).
//
// Sources: pytorch/ao PR #997 "Kleidi 4b blockwise gemv prototype"
// (matmul_clamp_f32_qai8dxp_qsi4c32p: int8 dynamic per-row asymmetric
// activations, int4 symmetric weights with one scale per 32 K, f32 output
// clamped after the bias); MNN ConvInt8TiledExecutor.cpp
// (BatchAsyDynamicQuant min/max quantization; int4 weights stored with an
// offset of 8 in _computeReorderQuantInfo).
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "qg_internal.cuh"

namespace qg {

// ---------------------------------------------------------------------------
// Per-row quantization parameters (float32, one IEEE rounding per operation,
// no contraction): rmin = min(0, min x), rmax = max(0, max x),
// scale = (rmax-rmin)/255 (1 if 0), inv = 1/scale,
// zp = clamp(rne(-128 - rmin*inv), -128, 127).
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
// W4 pack: one thread per output 32-bit word (8 consecutive k of a row).
// word j of row n: byte b = (w[8j+b]+8) | (w[8j+4+b]+8) << 4.
// ---------------------------------------------------------------------------
__global__ void pack_w4_kernel(int N, int K, const int8_t* __restrict__ w, int64_t ldw,
                               const float* __restrict__ sw, uint8_t* __restrict__ packed,
                               int* status) {
  const int64_t words_per_row = K / 8;
  const int64_t total = (int64_t)N * words_per_row;
  const int G = K / 32;
  uint32_t* out = reinterpret_cast<uint32_t*>(packed);
  float* sout = reinterpret_cast<float*>(packed + (size_t)N * (K / 2));
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
       i += (int64_t)gridDim.x * blockDim.x)
    sout[i] = sw[i];
  if (bad) record_error(status, QG_ERR_INVALID_ARG);
}

int launch_pack_w4(int N, int K, const int8_t* w, int64_t ldw, const float* sw, void* packed,
                   cudaStream_t st) {
  const int64_t words = (int64_t)N * (K / 8);
  int blocks = (int)min64(cdiv(words, 256), (int64_t)num_sms() * 8);
  if (blocks < 1) blocks = 1;
  pack_w4_kernel<<<blocks, 256, 0, st>>>(N, K, w, ldw, sw, (uint8_t*)packed, status_word());
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

__device__ __forceinline__ float ld_stream_f32(const float* p) {
  float v;
  asm volatile("ld.global.nc.L1::no_allocate.f32 %0, [%1];" : "=f"(v) : "l"(p));
  return v;
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
template <int GPL>
__global__ void __launch_bounds__(256) a8w4_gemv_kernel(
    int N, int K, const float* __restrict__ x, const uint8_t* __restrict__ wq,
    const float* __restrict__ wscale, const float* __restrict__ bias, float clamp_lo,
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
    uintptr_t s0 = (uintptr_t)(wscale + (int64_t)n0 * G) & ~(uintptr_t)15;
    uintptr_t s1 = (uintptr_t)(wscale + (int64_t)n1 * G) & ~(uintptr_t)15;
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
          s0[i] = ld_stream_f32(wscale + (int64_t)r * G + g);
          if (has_b) {
            w1[i] = ld_stream_u4(wq + (int64_t)rb * rowbytes + 16 * g);
            s1[i] = ld_stream_f32(wscale + (int64_t)rb * G + g);
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
// Fused A8W4 GEMV (M = 1), bulk-copy ring version (K % 128 == 0, K <= 8192).
//
// One CTA per SM owns the contiguous rows [n0, n1).  Its producer warp asks
// the copy engine for whole stages of 16 rows (nibbles and scales, two bulk
// copies) into a ring of shared-memory slots, so most of the CTA's weight
// bytes are requested at kernel start and HBM streams at full rate while the
// 16 consumer warps quantize x.  Consumer warp w then takes row w of every
// stage: lane l holds the activations of groups l, l+32, ... in registers and
// reads its 16-byte nibble chunk and scale per group from shared memory.
// Slots are handed back through per-slot `empty` barriers.
// ---------------------------------------------------------------------------
constexpr int kRingWarps = 16;  // consumer warps = rows per stage
constexpr int kRingThreads = (kRingWarps + 1) * 32;
constexpr int kRingSmemMax = 220 * 1024;

__device__ __forceinline__ void consumer_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(kRingWarps * 32) : "memory");
}

template <int GPL>
__global__ void __launch_bounds__(kRingThreads, 1) a8w4_gemv_ring_kernel(
    int N, int K, int slots, int max_rows, const float* __restrict__ x,
    const uint8_t* __restrict__ wq, const float* __restrict__ wscale,
    const float* __restrict__ bias, float clamp_lo, float clamp_hi, float* __restrict__ y,
    int8_t* __restrict__ q_out, float* __restrict__ scale_out, int32_t* __restrict__ zp_out,
    int* status) {
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ float red[2 * kRingWarps];
  const int G = K >> 5;
  const int rowbytes = K >> 1;
  const int sclbytes = G * 4;
  const int stage_bytes = kRingWarps * (rowbytes + sclbytes);
  int8_t* qa_s = reinterpret_cast<int8_t*>(sm);
  float* bias_s = reinterpret_cast<float*>(sm + ((K + 127) & ~127));  // [max_rows]
  uint8_t* ring = sm + ((K + 127) & ~127) + ((max_rows * 4 + 127) & ~127);
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + (size_t)slots * stage_bytes);
  uint64_t* empty = full + slots;
  uint64_t* xfull = empty + slots;   // x has landed in x_s
  uint64_t* xfree = xfull + 1;       // every consumer warp has read x_s
  // x (4K bytes) borrows the last ring slot until the consumers hold it in
  // registers; that slot's first stage is requested afterwards.
  const int xslot = slots - 1;
  const float* x_s = reinterpret_cast<const float*>(ring + (size_t)xslot * stage_bytes);

  const int n0 = (int)((int64_t)blockIdx.x * N / gridDim.x);
  const int n1 = (int)((int64_t)(blockIdx.x + 1) * N / gridDim.x);
  const int nstages = (n1 - n0 + kRingWarps - 1) / kRingWarps;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < slots; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kRingWarps);
    }
    mbar_init(xfull, 1);
    mbar_init(xfree, kRingWarps);
    fence_mbar_init();
    // Stage this CTA's weight slice into L2 before waiting on the previous
    // grid: a prefetch cannot return stale data (L2 is where every write
    // lands), and the copies that feed the math are issued after the wait.
    if (n1 > n0) {
      const uint8_t* p = wq + (int64_t)n0 * rowbytes;
      int64_t bytes = (int64_t)(n1 - n0) * rowbytes;
      while (bytes > 0) {
        const uint32_t c = (uint32_t)min64(bytes, 1 << 20);
        bulk_prefetch_l2(p, c);
        p += c;
        bytes -= c;
      }
      bulk_prefetch_l2(wscale + (int64_t)n0 * G, (uint32_t)((n1 - n0) * sclbytes));
    }
  }
  // Programmatic dependent launch: let the next grid in the stream start its
  // own prologue, then wait until the previous grid's writes are visible.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __syncthreads();

  if (warp == kRingWarps) {
    // ---------------- producer ----------------
    if (lane == 0) {
      mbar_arrive_expect_tx(xfull, (uint32_t)(K * 4));
      bulk_g2s(const_cast<float*>(x_s), x, (uint32_t)(K * 4), xfull);
      for (int s = 0; s < nstages; ++s) {
        const int slot = s % slots;
        if (s == xslot && !mbar_wait(xfree, 0, status)) break;
        if (s >= slots && !mbar_wait(&empty[slot], ((s / slots) - 1) & 1, status)) break;
        const int r0 = n0 + kRingWarps * s;
        const int rows = min(kRingWarps, n1 - r0);
        uint8_t* dst = ring + (size_t)slot * stage_bytes;
        mbar_arrive_expect_tx(&full[slot], (uint32_t)(rows * (rowbytes + sclbytes)));
        bulk_g2s(dst, wq + (int64_t)r0 * rowbytes, (uint32_t)(rows * rowbytes), &full[slot]);
        bulk_g2s(dst + kRingWarps * rowbytes, wscale + (int64_t)r0 * G,
                 (uint32_t)(rows * sclbytes), &full[slot]);
      }
    }
    return;
  }

  // ---------------- consumers: quantize x ----------------
  for (int i = threadIdx.x; i < n1 - n0; i += kRingWarps * 32)
    bias_s[i] = bias ? bias[n0 + i] : 0.0f;
  // Each thread takes its float4 chunks of x from shared memory once and keeps
  // them in registers for both passes (K <= 1024*GPL).
  constexpr int XV = (GPL * 1024 + 4 * kRingWarps * 32 - 1) / (4 * kRingWarps * 32);
  float4 xv[XV];
  float mn = 0.0f, mx = 0.0f;
  const bool x_ok = mbar_wait(xfull, 0, status);
#pragma unroll
  for (int j = 0; j < XV; ++j) {
    const int c = threadIdx.x + j * kRingWarps * 32;  // float4 chunk index
    xv[j] = (x_ok && 4 * c < K) ? reinterpret_cast<const float4*>(x_s)[c]
                                : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(xfree);   // x_s may now be overwritten by its stage
#pragma unroll
  for (int j = 0; j < XV; ++j) {
    mn = fminf(mn, fminf(fminf(xv[j].x, xv[j].y), fminf(xv[j].z, xv[j].w)));
    mx = fmaxf(mx, fmaxf(fmaxf(xv[j].x, xv[j].y), fmaxf(xv[j].z, xv[j].w)));
  }
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (lane == 0) {
    red[warp] = mn;
    red[kRingWarps + warp] = mx;
  }
  consumer_bar();
  mn = red[0];
  mx = red[kRingWarps];
#pragma unroll
  for (int i = 1; i < kRingWarps; ++i) {
    mn = fminf(mn, red[i]);
    mx = fmaxf(mx, red[kRingWarps + i]);
  }
  const RowQuant rq = row_quant_params(mn, mx);
#pragma unroll
  for (int j = 0; j < XV; ++j) {
    const int c = threadIdx.x + j * kRingWarps * 32;
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
  consumer_bar();

  const int za = rq.zp;
  int a[GPL][8];
  int cseed[GPL];
#pragma unroll
  for (int i = 0; i < GPL; ++i) {
    const int g = lane + 32 * i;
    if (g < G) {
      const int4* src = reinterpret_cast<const int4*>(qa_s + 32 * g);
      const int4 v0 = src[0], v1 = src[1];
      a[i][0] = v0.x; a[i][1] = v0.y; a[i][2] = v0.z; a[i][3] = v0.w;
      a[i][4] = v1.x; a[i][5] = v1.y; a[i][6] = v1.z; a[i][7] = v1.w;
      cseed[i] = act_seed(a[i], za);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) a[i][j] = 0;
      cseed[i] = 0;
    }
  }

  // ---------------- consumers: stream rows ----------------
  for (int s = 0; s < nstages; ++s) {
    const int slot = s % slots;
    if (!mbar_wait(&full[slot], (s / slots) & 1, status)) break;
    const int r = n0 + kRingWarps * s + warp;
    if (r < n1) {
      const uint8_t* nib = ring + (size_t)slot * stage_bytes + warp * rowbytes;
      const float* scl = reinterpret_cast<const float*>(ring + (size_t)slot * stage_bytes +
                                                        kRingWarps * rowbytes + warp * sclbytes);
      float acc = 0.0f;
#pragma unroll
      for (int i = 0; i < GPL; ++i) {
        const int g = lane + 32 * i;
        if (g < G) {
          const uint4 wv = *reinterpret_cast<const uint4*>(nib + 16 * g);
          acc = fmaf(scl[g], (float)group_dot(wv, a[i], cseed[i], za), acc);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) {
        float v = __fmul_rn(rq.scale, acc);
        if (bias) v = __fadd_rn(v, bias_s[r - n0]);
        y[r] = fminf(fmaxf(v, clamp_lo), clamp_hi);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
  }
}

template <int GPL>
static int launch_ring(int N, int K, const float* x, const uint8_t* wq, const float* ws,
                       const float* bias, float lo, float hi, float* y, int8_t* q_out,
                       float* scale_out, int32_t* zp_out, cudaStream_t st) {
  const int G = K / 32;
  const int stage_bytes = kRingWarps * (K / 2 + G * 4);
  int grid = num_sms();
  const int max_grid = (N + kRingWarps - 1) / kRingWarps;
  if (grid > max_grid) grid = max_grid;
  const int rows_per_cta = (N + grid - 1) / grid;
  const int nstages = (rows_per_cta + kRingWarps - 1) / kRingWarps;
  const int base = ((K + 127) & ~127) + ((rows_per_cta * 4 + 127) & ~127);
  int slots = (kRingSmemMax - base - 16) / (stage_bytes + 16);
  if (slots > nstages) slots = nstages;
  if (slots < 1) return 1;  // does not fit: caller uses the register-streaming kernel
  const size_t smem = (size_t)base + (size_t)slots * (stage_bytes + 16) + 16;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kRingThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, a8w4_gemv_ring_kernel<GPL>, N, K, slots, rows_per_cta, x,
                                     wq, ws, bias, lo, hi, y, q_out, scale_out, zp_out,
                                     status_word());
  return e == cudaSuccess ? QG_OK : QG_ERR_CUDA;
}

int launch_a8w4_gemv(int N, int K, const float* x, const void* packed, const float* bias,
                     float lo, float hi, float* y, int8_t* q_out, float* scale_out,
                     int32_t* zp_out, cudaStream_t st) {
  const uint8_t* wq = (const uint8_t*)packed;
  const float* ws = (const float*)(wq + (size_t)N * (K / 2));
  const int G = K / 32;
  int grid = num_sms() * 2;
  if (grid > N) grid = N;
  if (K % 128 == 0 && K <= 8192 && ((uintptr_t)x & 15) == 0) {
    int rc;
    if (G <= 32) rc = launch_ring<1>(N, K, x, wq, ws, bias, lo, hi, y, q_out, scale_out, zp_out, st);
    else if (G <= 64) rc = launch_ring<2>(N, K, x, wq, ws, bias, lo, hi, y, q_out, scale_out, zp_out, st);
    else if (G <= 128) rc = launch_ring<4>(N, K, x, wq, ws, bias, lo, hi, y, q_out, scale_out, zp_out, st);
    else rc = launch_ring<8>(N, K, x, wq, ws, bias, lo, hi, y, q_out, scale_out, zp_out, st);
    if (rc <= 0) return rc;
  }
  const size_t smem = (size_t)K;
  if (G <= 32) {
    a8w4_gemv_kernel<1><<<grid, 256, smem, st>>>(N, K, x, wq, ws, bias, lo, hi, y, q_out,
                                                 scale_out, zp_out);
  } else if (G <= 64) {
    a8w4_gemv_kernel<2><<<grid, 256, smem, st>>>(N, K, x, wq, ws, bias, lo, hi, y, q_out,
                                                 scale_out, zp_out);
  } else {
    a8w4_gemv_kernel<4><<<grid, 256, smem, st>>>(N, K, x, wq, ws, bias, lo, hi, y, q_out,
                                                 scale_out, zp_out);
  }
  return launch_status();
}

int setup_a8w4_gemv() {
  // allow up to 64 KiB of activations in shared memory
  cudaError_t e1 = cudaFuncSetAttribute(a8w4_gemv_kernel<1>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, 65536);
  cudaError_t e2 = cudaFuncSetAttribute(a8w4_gemv_kernel<2>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, 65536);
  cudaError_t e3 = cudaFuncSetAttribute(a8w4_gemv_kernel<4>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, 65536);
  cudaError_t e4 = cudaFuncSetAttribute(a8w4_gemv_ring_kernel<1>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, kRingSmemMax);
  cudaError_t e5 = cudaFuncSetAttribute(a8w4_gemv_ring_kernel<2>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, kRingSmemMax);
  cudaError_t e6 = cudaFuncSetAttribute(a8w4_gemv_ring_kernel<4>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, kRingSmemMax);
  cudaError_t e7 = cudaFuncSetAttribute(a8w4_gemv_ring_kernel<8>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, kRingSmemMax);
  return (e1 == cudaSuccess && e2 == cudaSuccess && e3 == cudaSuccess && e4 == cudaSuccess &&
          e5 == cudaSuccess && e6 == cudaSuccess && e7 == cudaSuccess)
             ? QG_OK
             : QG_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// A8W4 GEMM for M > 1 on CUDA cores (dp4a): activations quantized beforehand
// (q [M][K], scale, zp in the workspace).  CTA tile: 8 rows of M staged in
// shared memory x a slice of N; each warp owns one column n at a time, lanes
// split the groups, and every weight chunk loaded into registers serves the
// 8 rows.
// ---------------------------------------------------------------------------
constexpr int kSimtRows = 8;

__global__ void __launch_bounds__(256) a8w4_gemm_simt_kernel(
    int M, int N, int K, const int8_t* __restrict__ q, const float* __restrict__ sA,
    const int32_t* __restrict__ zA, const uint8_t* __restrict__ wq,
    const float* __restrict__ wscale, const float* __restrict__ bias, float lo, float hi,
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
      const float s = ld_stream_f32(wscale + (int64_t)n * G + g);
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
                          float hi, float* y, int64_t ldy, cudaStream_t st) {
  const uint8_t* wq = (const uint8_t*)packed;
  const float* ws = (const float*)(wq + (size_t)N * (K / 2));
  const int mblocks = (int)cdiv(M, kSimtRows);
  int nblocks = (int)max64(1, min64(cdiv((int64_t)num_sms() * 2, mblocks), cdiv(N, 8)));
  dim3 grid(nblocks, mblocks);
  const size_t smem = (size_t)kSimtRows * K;
  a8w4_gemm_simt_kernel<<<grid, 256, smem, st>>>(M, N, K, q, sA, zA, wq, ws, bias, lo, hi, y, ldy);
  return launch_status();
}

int setup_a8w4_gemm_simt() {
  cudaError_t e = cudaFuncSetAttribute(a8w4_gemm_simt_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
  return e == cudaSuccess ? QG_OK : QG_ERR_CUDA;
}

}  // namespace qg
