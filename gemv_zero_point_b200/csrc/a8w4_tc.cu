// A8W4 linear for M > 1 on the 5th-generation tensor cores, and the same
// contraction for the unrolled rows of the float-input convolution.
//
// Sources: pytorch/ao PR #997 "Kleidi 4b blockwise gemv prototype"
// (matmul_clamp_f32_qai8dxp_qsi4c32p: int8 dynamic per-row asymmetric
// activations, int4 symmetric weights with one scale per 32-wide K group,
// f32 output clamped after the bias; m > 1 tests); MNN
// ConvInt8TiledExecutor.cpp (dynamic-quant option 2: the input quantized per
// K block; asymmetric weight quant info, w_real = alpha*code + zero; the
// low-memory float im2col path, symmetric or asymmetric rows).
//
//   y[m,n] = clamp(sA[m] * sum_g (sw[n,g]*I[m,n,g] + zw[n,g]*S[m,g]) + bias[n])
//   I[m,n,g] = sum_{k in g} (qA[m,k] - zA[m]) * w[n,k],  S[m,g] = sum_{k in g}(qA[m,k] - zA[m])
// (zw = 0 for symmetric weights; with per-block activations sA and zA are
// per (m, g) and sA moves inside the sum).
//
// Exactness: qA - zA lies in [-255,255] and w in [-8,7], both exact in
// bf16, and every partial sum of one group is an integer below 2^24, so the
// two K = 16 bf16 MMAs of a group leave the exact I[m,n,g] in an f32 TMEM
// accumulator.  Only the combination over groups is rounded (f32).
//
// Two launches per call:
//  1. a8w4_quant_tiles_kernel quantizes each activation row (per row or per
//     32-wide block, asymmetric or symmetric; plain rows or the unrolled rows
//     of an NHWC image) and writes the centred codes qA - zA as bf16 in the
//     exact byte image the tensor cores read: for every 128-row tile and
//     every 64-wide K block, 128 rows of 128 bytes with the 16-byte chunks of
//     row r permuted by r % 8 (the 128-byte swizzle).  One stage of the GEMM
//     is then one contiguous 16 KiB bulk copy.  Launched as a programmatic
//     dependent of the previous work in the stream (it waits for it on the
//     device before reading x).
//  2. a8w4_tc_kernel (programmatic dependent launch after 1) computes a tile
//     of 128 weight rows (MMA M, TMEM lanes) x 128 activation rows (MMA N,
//     TMEM columns) over a K range; the K ranges of one tile form a cluster
//     and their partial tiles are reduced through distributed shared memory
//     in a fixed order.
//
// Roles of a8w4_tc_kernel (704 threads, one CTA per SM):
//   warp 0      tensor copies of the weight scale (and zero) tables before
//               the grid dependency wait; after it the activation tables and
//               the bulk copies of the activation stages
//   warp 1      TMEM allocation; MMA issue: per 64-wide stage four K = 16
//               MMAs (two per 32-wide group) into one of 2 TMEM stage
//               buffers of 2 x 128 columns, one commit for the accumulators
//   warps 2..5  weight nibbles: a ring of 64-wide K slices of the CTA's 128
//               rows (tensor copies, issued before the grid dependency wait),
//               expanded to bf16 w = u - 8 in the swizzled stage layout
//   warps 6..21 per stage: tcgen05.ld of the exact group dots (32 columns
//               per warp), release of the buffer, acc += scale * I with
//               packed f32x2 FMAs; then the partial tile, the cluster
//               reduction and y
// One thread per warp waits on each barrier.  The waits off the critical
// path (stage slots and operands that are normally ready in time) park in
// mbarrier.try_wait with a suspend-time hint, so they take no issue slots
// from the converter and read-out warps; the two waits of the TMEM round
// trip (free accumulator buffer, accumulators ready) poll.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include "qg_internal.cuh"

namespace qg {

int make_tmap_generic(CUtensorMap* tm, CUtensorMapDataType dt, const void* base, uint64_t inner,
                      uint64_t rows, uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_rows,
                      CUtensorMapSwizzle swz);

namespace {

constexpr int TW = 128;                 // weight rows per CTA (MMA M, TMEM lanes)
constexpr int TM = 128;                 // activation rows per CTA (MMA N, TMEM columns)
constexpr int KS = 64;                  // K per stage: one 128-byte swizzle row of bf16
constexpr int STAGE_BYTES = 128 * KS * 2;  // 16 KiB, both operands
constexpr int STAGES = 4;
constexpr int NRING = 8;                // weight nibble stages in flight
constexpr int NIB_BYTES = TW * KS / 2;  // 4 KiB of nibbles per stage
constexpr int NSB = 2;                  // TMEM stage buffers: the 2 groups of a stage, 2*TM columns
constexpr int KR_MAX = 1024;            // K range per CTA
constexpr int GR_MAX = KR_MAX / 32;
constexpr int MAX_SPLITS = 8;
constexpr int THREADS = 22 * 32;
constexpr int CONV_WARP0 = 2;
constexpr int NCONV = 128;              // converter threads
constexpr int EPI_WARP0 = 6;
constexpr int NEPI = 512;               // epilogue threads: 4 lane quarters x 4 column blocks
constexpr int PST = TW + 4;             // row stride (floats) of the partial tile [m][n]

// shared-memory map (offsets from the 1024-byte aligned base)
constexpr size_t OFF_A = 0;                                        // activation stages
constexpr size_t OFF_W = OFF_A + (size_t)STAGES * STAGE_BYTES;     // weight stages
constexpr size_t OFF_N = OFF_W + (size_t)STAGES * STAGE_BYTES;     // nibble ring
constexpr size_t OFF_SCL = OFF_N + (size_t)NRING * NIB_BYTES;      // [TW][Gr] weight scales
constexpr size_t OFF_ZW = OFF_SCL + (size_t)GR_MAX * TW * 4;       // [TW][Gr] weight zeros
constexpr size_t OFF_ACT = OFF_ZW + (size_t)GR_MAX * TW * 4;       // [Gr][TM] act scales / sums
constexpr size_t OFF_BAR = OFF_ACT + (size_t)GR_MAX * TM * 4;
constexpr size_t SMEM_BYTES = 1024 + OFF_BAR + 512;
static_assert((size_t)TM * PST * 4 <= OFF_N, "partial tile reuses the stage buffers");
static_assert(OFF_SCL % 1024 == 0 && OFF_ZW % 1024 == 0 && OFF_ACT % 1024 == 0,
              "swizzled tables start on a swizzle atom");

// The per-group tables (weight scales / zeros [row][Gr], activation block
// scales / sums [row][Gr]) are kept as rows of Gr elements; when a row is
// 32, 64 or 128 bytes they arrive by one tensor copy with the matching
// swizzle (16-byte chunk c of the row at byte address a moves to
// c ^ ((a >> 7) & (span/16 - 1))), which spreads a column of the table over
// the banks; other sizes are loaded by threads into the same layout.
__device__ __forceinline__ uint32_t tbl_off(int row, int g, int esz, int rowbytes) {
  const uint32_t raw = (uint32_t)(row * rowbytes + g * esz);
  const uint32_t mask = rowbytes == 128 ? 7u : rowbytes == 64 ? 3u : rowbytes == 32 ? 1u : 0u;
  return raw ^ (((raw >> 7) & mask) << 4);
}

// kind::f16 instruction descriptor: D f32, A bf16, B bf16, both K-major,
// N = TM, M = TW.
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(TM >> 3) << 17) |
                           ((uint32_t)(TW >> 4) << 24);

__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;            // leading byte offset (unused with 128B swizzle)
  d |= (uint64_t)(1024 >> 4) << 32;  // stride byte offset between 8-row groups
  d |= (uint64_t)1 << 46;            // descriptor version
  d |= (uint64_t)2 << 61;            // SWIZZLE_128B
  return d;
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(IDESC), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
// bf16x2 (0x4300 | u) - 136 = u - 8, exact.
__device__ __forceinline__ uint32_t bf16x2_minus136(uint32_t v) {
  uint32_t d;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(v), "r"(0x43084308u));
  return d;
}
typedef unsigned long long f32x2;
__device__ __forceinline__ f32x2 pack2(float lo, float hi) {
  return ((f32x2)__float_as_uint(hi) << 32) | __float_as_uint(lo);
}
__device__ __forceinline__ f32x2 pack2u(uint32_t lo, uint32_t hi) {
  return ((f32x2)hi << 32) | lo;
}
__device__ __forceinline__ void ffma2(f32x2& acc, f32x2 a, f32x2 b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}
__device__ __forceinline__ f32x2 fmul2(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float lo_f(f32x2 v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float hi_f(f32x2 v) { return __uint_as_float((uint32_t)(v >> 32)); }

// Named barriers with an AND over a predicate, so every thread of a role
// takes the same decision after a bounded wait.
template <int ID, int N>
__device__ __forceinline__ bool bar_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(ID), "n"(N)
      : "memory");
  return r != 0;
}
template <int ID, int N>
__device__ __forceinline__ void bar_sync() {
  asm volatile("bar.sync %0, %1;" ::"n"(ID), "n"(N) : "memory");
}

// Wait for phase `parity` of `bar` with mbarrier.try_wait and a suspend-time
// hint: the hardware parks the thread until the phase completes (or the
// 20 us hint runs out, after which it asks again), so a waiting warp issues
// a few instructions per wake-up instead of a polling loop that takes issue
// slots from the converter and read-out warps on its sub-partition
// (test-and-sleep polls were about half of all instructions this kernel
// issued).  At most limit / 256 + 1 tries: about 82 ms at kSpinLimit,
// 0.3 ms at kStallSpinLimit.
__device__ __forceinline__ bool mbar_park(uint64_t* bar, uint32_t parity, int* status,
                                          uint32_t limit = kSpinLimit) {
  const uint32_t tries = (limit >> 8) + 1;
  for (uint32_t i = 0; i < tries; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
        : "memory");
    if (ok) return true;
  }
  record_error(status, QG_ERR_TIMEOUT);
  return false;
}

// Poll a barrier phase from one thread, sleeping briefly between polls;
// bounded like mbar_poll.  Kept for the two waits on the TMEM round trip
// (the MMA issuer waiting for a free accumulator buffer, an epilogue warp
// waiting for its accumulators), where the kernel measured slower with
// parked waits (mbar_park) than with these polls.
__device__ __forceinline__ bool poll_yield(uint64_t* bar, uint32_t parity, int* status,
                                           uint32_t limit) {
  for (uint32_t i = 0; i < (limit << 4); ++i) {
    if (mbar_test(bar, parity)) return true;
    __nanosleep(32);
  }
  record_error(status, QG_ERR_TIMEOUT);
  return false;
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t mapa(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// ---------------------------------------------------------------------------
// 1. Quantization of the activation rows into swizzled bf16 tiles.
// ---------------------------------------------------------------------------
enum QuantMode { kRowAsym = 0, kBlockAsym = 1, kRowSym = 2 };

struct RowSource {
  const float* x;
  int64_t ldx;  // plain rows: row m at x + m*ldx
  // unrolled NHWC rows: row m = output pixel (n, oh, ow), k = (kh*KW + kw)*Cin + ci
  int H, W, Cin, KH, KW, sh, sw, ph, pw, OH, OW;
};

struct QuantArgs {
  int M, K, Mpad;
  RowSource src;
  int vec4;             // the 8 floats of a chunk can be read as two aligned float4
  uint16_t* atile;      // [Mpad/128][K/64][128][64] bf16 (qA - zA), swizzled
  float* sA;            // per-row scale [Mpad], or per-block [K/32][Mpad] (transposed)
  float* Sg;            // per-block sums of qA - zA [K/32][Mpad] (weight zeros), or NULL
  int8_t* q_out;        // optional [M][K] codes
  int q_vec;            // q_out is 8-byte aligned
  float* scale_out;     // optional [M] (per row) or [M][K/32] (per block)
  int32_t* zp_out;      // optional, same shape as scale_out
};

constexpr int QT = 256;   // threads per quantization CTA
constexpr int QCH = 4;    // most 8-wide chunks per thread (K <= 32 * threads per row)

// Tap of each 8-wide K chunk of an unrolled row (Cin % 8 == 0: a chunk lies
// in one tap): x = input channel of its first value, y = kh << 16 | kw.  The
// same for every row, so a CTA builds it once instead of dividing per chunk.
constexpr int kMaxChunks = QCH * QT;  // K / 8 for the largest K (QCH chunks per thread)

template <bool CONV>
__device__ __forceinline__ void load_chunk(const QuantArgs& a, int64_t m, int c, int pn, int poh,
                                           int pow_, const int2* tap_tab, float (&v)[8]) {
  const RowSource& s = a.src;
  if (!CONV) {
    const float* p = s.x + m * s.ldx + 8 * c;
    if (a.vec4) {
      const float4 u0 = __ldg(reinterpret_cast<const float4*>(p));
      const float4 u1 = __ldg(reinterpret_cast<const float4*>(p) + 1);
      v[0] = u0.x; v[1] = u0.y; v[2] = u0.z; v[3] = u0.w;
      v[4] = u1.x; v[5] = u1.y; v[6] = u1.z; v[7] = u1.w;
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = __ldg(p + e);
    }
    return;
  }
  if (a.vec4) {  // Cin % 8 == 0: the chunk lies in one tap
    const int2 e = tap_tab[c];
    const int ci = e.x, kh = e.y >> 16, kw = e.y & 0xFFFF;
    const int ih = poh * s.sh + kh - s.ph, iw = pow_ * s.sw + kw - s.pw;
    if (ih < 0 || ih >= s.H || iw < 0 || iw >= s.W) {
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = 0.0f;  // a pad tap is the real value 0
      return;
    }
    const float* p = s.x + (((int64_t)pn * s.H + ih) * s.W + iw) * s.Cin + ci;
    const float4 u0 = __ldg(reinterpret_cast<const float4*>(p));
    const float4 u1 = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = u0.x; v[1] = u0.y; v[2] = u0.z; v[3] = u0.w;
    v[4] = u1.x; v[5] = u1.y; v[6] = u1.z; v[7] = u1.w;
    return;
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int k = 8 * c + e;
    const int tap = k / s.Cin, ci = k - tap * s.Cin;
    const int kh = tap / s.KW, kw = tap - kh * s.KW;
    const int ih = poh * s.sh + kh - s.ph, iw = pow_ * s.sw + kw - s.pw;
    v[e] = (ih < 0 || ih >= s.H || iw < 0 || iw >= s.W)
               ? 0.0f
               : __ldg(s.x + (((int64_t)pn * s.H + ih) * s.W + iw) * s.Cin + ci);
  }
}

// R rows per CTA, QT/R threads per row; thread t of a row owns the 8-wide K
// chunks t, t + QT/R, ... (at most QCH of them).
template <int MODE, bool CONV>
__global__ void __launch_bounds__(QT) a8w4_quant_tiles_kernel(QuantArgs a, int R) {
  // the GEMM grid may start its prologue now; it waits for this grid before
  // it reads anything written here
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ float red[2][QT / 32];
  __shared__ int2 tap_tab[CONV ? kMaxChunks : 1];
  const int T = QT / R;
  const int sub = threadIdx.x / T, t = threadIdx.x - sub * T;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t m = (int64_t)blockIdx.x * R + sub;
  const int K = a.K, G = K >> 5, nchunk = K >> 3, nkb = K >> 6;
  const bool live = m < a.M;
  int pn = 0, poh = 0, pow_ = 0;
  if (CONV && live) {  // m < Mpad <= INT32_MAX: 32-bit divisions
    const int mi = (int)m;
    const int tt = mi / a.src.OW;
    pow_ = mi - tt * a.src.OW;
    pn = tt / a.src.OH;
    poh = tt - pn * a.src.OH;
  }
  if (CONV && a.vec4) {
    for (int c = threadIdx.x; c < nchunk; c += QT) {
      const int k = 8 * c;
      const int tap = k / a.src.Cin, kh = tap / a.src.KW;
      tap_tab[c] = make_int2(k - tap * a.src.Cin, (kh << 16) | (tap - kh * a.src.KW));
    }
    __syncthreads();
  }
  // This grid is itself a programmatic dependent of the work before it in
  // the stream: x is read and the workspace written only once that is done.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  float v[QCH][8];
  float mn = 0.0f, mx = 0.0f;  // min(0, .), max(0, .); mx is max|x| when symmetric
#pragma unroll
  for (int i = 0; i < QCH; ++i) {
    const int c = t + i * T;
    if (live && c < nchunk) {
      load_chunk<CONV>(a, m, c, pn, poh, pow_, tap_tab, v[i]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) v[i][e] = 0.0f;
    }
  }
  RowQuant rowq;
  if (MODE != kBlockAsym) {
#pragma unroll
    for (int i = 0; i < QCH; ++i)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if (MODE == kRowSym) {
          mx = fmaxf(mx, fabsf(v[i][e]));
        } else {
          mn = fminf(mn, v[i][e]);
          mx = fmaxf(mx, v[i][e]);
        }
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if (T > 32) {  // combine the warps of this row
      if (lane == 0) {
        red[0][warp] = mn;
        red[1][warp] = mx;
      }
      __syncthreads();
      const int w0 = (sub * T) >> 5, nw = T >> 5;
      mn = red[0][w0];
      mx = red[1][w0];
      for (int i = 1; i < nw; ++i) {
        mn = fminf(mn, red[0][w0 + i]);
        mx = fmaxf(mx, red[1][w0 + i]);
      }
    }
    rowq = MODE == kRowSym ? row_quant_params_sym(mx) : row_quant_params(mn, mx);
  }
  const int mt = (int)(m >> 7), r = (int)(m & 127);
#pragma unroll
  for (int i = 0; i < QCH; ++i) {
    const int c = t + i * T;
    RowQuant q = rowq;
    if (MODE == kBlockAsym) {
      // the 4 chunks of a 32-wide block sit in 4 consecutive threads
      float bmn = 0.0f, bmx = 0.0f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        bmn = fminf(bmn, v[i][e]);
        bmx = fmaxf(bmx, v[i][e]);
      }
#pragma unroll
      for (int o = 1; o < 4; o <<= 1) {
        bmn = fminf(bmn, __shfl_xor_sync(0xffffffffu, bmn, o));
        bmx = fmaxf(bmx, __shfl_xor_sync(0xffffffffu, bmx, o));
      }
      q = row_quant_params(bmn, bmx);
    }
    int code[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
      code[e] = MODE == kRowSym ? quant_one_sym(v[i][e], q) : quant_one(v[i][e], q);
    // block sums of the centred codes (exact; only read with weight zeros)
    int csum = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) csum += code[e] - q.zp;
    if (a.Sg) {
#pragma unroll
      for (int o = 1; o < 4; o <<= 1) csum += __shfl_xor_sync(0xffffffffu, csum, o);
    }
    if (c >= nchunk || m >= a.Mpad) continue;
    uint32_t h[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float f0 = live ? (float)(code[2 * e] - q.zp) : 0.0f;
      const float f1 = live ? (float)(code[2 * e + 1] - q.zp) : 0.0f;
      // |code - zp| <= 255: exact in bf16
      h[e] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f0)) |
             ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f1)) << 16);
    }
    const int kb = c >> 3, j = c & 7;
    uint8_t* dst = reinterpret_cast<uint8_t*>(a.atile) +
                   (((int64_t)mt * nkb + kb) * 128 + r) * 128 + ((j ^ (r & 7)) << 4);
    *reinterpret_cast<uint4*>(dst) = make_uint4(h[0], h[1], h[2], h[3]);
    if (!live) continue;
    if (a.q_out) {
      uint32_t lo = 0, hi = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        lo |= ((uint32_t)code[e] & 0xFFu) << (8 * e);
        hi |= ((uint32_t)code[4 + e] & 0xFFu) << (8 * e);
      }
      int8_t* qo = a.q_out + m * K + 8 * c;
      if (a.q_vec) {
        *reinterpret_cast<uint2*>(qo) = make_uint2(lo, hi);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) qo[e] = (int8_t)code[e];
      }
    }
    // per-group tables for the GEMM transposed, [G][Mpad]; the caller's
    // outputs stay [M][G]
    if (MODE == kBlockAsym && (t & 3) == 0) {
      const int64_t b = m * G + (c >> 2);
      a.sA[(int64_t)(c >> 2) * a.Mpad + m] = q.scale;
      if (a.scale_out) a.scale_out[b] = q.scale;
      if (a.zp_out) a.zp_out[b] = q.zp;
    }
    if (a.Sg && (t & 3) == 0) a.Sg[(int64_t)(c >> 2) * a.Mpad + m] = (float)csum;
  }
  if (MODE != kBlockAsym && t == 0 && m < a.Mpad) {
    a.sA[m] = live ? rowq.scale : 0.0f;
    if (live && a.scale_out) a.scale_out[m] = rowq.scale;
    if (live && a.zp_out) a.zp_out[m] = rowq.zp;
  }
}

// ---------------------------------------------------------------------------
// 2. The tensor-core contraction.
// ---------------------------------------------------------------------------
struct GemmArgs {
  int M, N, K, Kr, splits, n_tiles, nkb;
  const uint16_t* atile;   // activation tiles from the quantization kernel
  const void* wscale;      // [N][K/32] f32, or bf16 when scale_bf16
  int scale_bf16;
  const float* wzero;      // [N][K/32] f32 weight zeros (WZP)
  const float* sA;         // [Mpad] or [K/32][Mpad] (ABLK)
  const float* Sg;         // [K/32][Mpad] (WZP)
  int Mpad;
  const float* bias;
  float lo, hi;
  float* y;
  int64_t ldy;
  int tma_w, tma_act;      // the weight / activation tables come by tensor copy
  int stall;               // test hook: the activation stage 1 is never issued
  uint32_t spin;           // poll limit of the pipeline waits
};

// Tensor maps of one call: nibbles, and the per-group tables when they come
// by tensor copy (otherwise unused copies of the nibble map).
struct TcMaps {
  CUtensorMap w, scl, zw, act;
};

template <bool ABLK, bool WZP>
__global__ void __launch_bounds__(THREADS, 1)
    a8w4_tc_kernel(const __grid_constant__ TcMaps tm_, GemmArgs a, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem + OFF_A;
  uint8_t* sW = smem + OFF_W;
  uint8_t* sN = smem + OFF_N;
  uint8_t* scl = smem + OFF_SCL;   // [n][Gr] weight scales (f32 or bf16), swizzled rows
  uint8_t* zws = smem + OFF_ZW;    // [n][Gr] f32 weight zeros
  // [g][m] f32 activation block scales / group sums: the 32 rows of a
  // warp's column block for one group are 128 contiguous bytes
  float* actp = reinterpret_cast<float*>(smem + OFF_ACT);
  uint64_t* a_full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* w_full = a_full + STAGES;
  uint64_t* empty = w_full + STAGES;
  uint64_t* nib_full = empty + STAGES;
  uint64_t* tfull = nib_full + NRING;
  uint64_t* tempty = tfull + NSB;
  uint64_t* prm_full = tempty + NSB;   // weight tables landed
  uint64_t* act_full = prm_full + 1;   // activation tables landed
  uint64_t* drain = act_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  float* part = reinterpret_cast<float*>(smem);  // [TM][PST], after the mainloop

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = a.splits > 1 ? (int)cluster_rank() : 0;
  const int tile = blockIdx.x / a.splits;
  const int tn = tile % a.n_tiles, tm = tile / a.n_tiles;
  const int n0 = tn * TW, m0 = tm * TM;
  const int k0 = split * a.Kr;
  const int G = a.K >> 5, g0 = k0 >> 5;
  const int Gr = a.Kr >> 5;
  const int nst = a.Kr / KS;
  const int sesz = a.scale_bf16 ? 2 : 4;  // bytes per stored weight scale
  const int srow = Gr * sesz, frow = Gr * 4;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&a_full[s], 1);
      mbar_init(&w_full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < NRING; ++s) mbar_init(&nib_full[s], 1);
    for (int b = 0; b < NSB; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], NEPI / 32);
    }
    mbar_init(prm_full, 1);
    mbar_init(act_full, 1);
    mbar_init(drain, 1);
    fence_mbar_init();
    prefetch_tmap(&tm_.w);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(NSB * 2 * TM)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------- tables and activation stages (tensor / bulk copies) -------------
    if (lane == 0) {
      uint32_t issued = 0, last_ph = 0;
      bool prm = false, act = false;
      if (a.tma_w) {  // inputs of the call: before the grid dependency wait
        mbar_arrive_expect_tx(prm_full, (uint32_t)(TW * (srow + (WZP ? frow : 0))));
        tma_load_2d(scl, &tm_.scl, g0, n0, prm_full);
        if (WZP) tma_load_2d(zws, &tm_.zw, g0, n0, prm_full);
        prm = true;
      }
      // the activation tiles and tables come from the quantization grid
      asm volatile("griddepcontrol.wait;" ::: "memory");
      if ((ABLK || WZP) && a.tma_act) {
        mbar_arrive_expect_tx(act_full, (uint32_t)(TM * frow));
        tma_load_2d(actp, &tm_.act, m0, g0, act_full);
        act = true;
      }
      const uint8_t* src = reinterpret_cast<const uint8_t*>(a.atile) +
                           ((int64_t)tm * a.nkb + (k0 / KS)) * STAGE_BYTES;
      for (int s = 0; s < nst; ++s) {
        const int slot = s % STAGES;
        if (s >= STAGES && !mbar_park(&empty[slot], ((s / STAGES) - 1) & 1, status, a.spin)) break;
        if (a.stall && s == 1) continue;
        mbar_arrive_expect_tx(&a_full[slot], STAGE_BYTES);
        bulk_g2s(sA + slot * STAGE_BYTES, src + (int64_t)s * STAGE_BYTES, STAGE_BYTES,
                 &a_full[slot]);
        issued |= 1u << slot;
        last_ph = (last_ph & ~(1u << slot)) | ((uint32_t)((s / STAGES) & 1) << slot);
      }
      // every copy issued here has landed before the CTA may exit
      for (int st = 0; st < STAGES; ++st)
        if ((issued >> st) & 1u) mbar_poll(&a_full[st], (last_ph >> st) & 1u, status);
      if (prm) mbar_poll(prm_full, 0, status);
      if (act) mbar_poll(act_full, 0, status);
    }
  } else if (warp == 1) {
    // ---------------- MMA issue ----------------
    // Per stage: both groups (two K = 16 MMAs each) into one TMEM stage
    // buffer, one commit for the accumulators and one for the stage.
    if (lane == 0) {
      bool failed = false;
      for (int s = 0; s < nst; ++s) {
        const int slot = s % STAGES, sb = s % NSB;
        const uint32_t par = (uint32_t)(s / STAGES) & 1;
        if (!mbar_park(&a_full[slot], par, status, a.spin) ||
            !mbar_park(&w_full[slot], par, status, a.spin) ||
            !poll_yield(&tempty[sb], ((uint32_t)(s / NSB) & 1) ^ 1, status, a.spin)) {
          failed = true;
          break;
        }
        tc_fence_after();
        // descriptor start addresses count 16-byte units: K = 16 more is +2
        const uint64_t dw = sdesc_sw128(smem_u32(sW + slot * STAGE_BYTES));
        const uint64_t dx = sdesc_sw128(smem_u32(sA + slot * STAGE_BYTES));
        const uint32_t d = tmem_base + (uint32_t)(sb * 2 * TM);
#pragma unroll
        for (int gi = 0; gi < 2; ++gi) {
          mma_bf16(d + gi * TM, dw + 4 * gi, dx + 4 * gi, 0);
          mma_bf16(d + gi * TM, dw + 4 * gi + 2, dx + 4 * gi + 2, 1);
        }
        mma_commit(&tfull[sb]);
        mma_commit(&empty[slot]);
      }
      if (failed) {
        // MMAs already issued finish before their operands or TMEM go away
        mma_commit(drain);
        mbar_poll(drain, 0, status);
      }
    }
  } else if (warp < EPI_WARP0) {
    // ---------------- weight nibbles -> bf16 stages ----------------
    const int ctid = threadIdx.x - CONV_WARP0 * 32;  // 0..127
    uint32_t issued = 0, last_ph = 0;                 // nibble ring (thread 0 only)
    if (ctid == 0) {
      for (int s = 0; s < nst && s < NRING; ++s) {
        mbar_arrive_expect_tx(&nib_full[s], NIB_BYTES);
        tma_load_2d(sN + s * NIB_BYTES, &tm_.w, (k0 + KS * s) / 8, n0, &nib_full[s]);
        issued |= 1u << s;
      }
    }
    bool ok = true;
    // Converter thread r owns row r of every stage: its 8 nibble words (32
    // bytes, two 128-bit loads issued before any use) become the row's 8
    // swizzled 16-byte bf16 chunks.
    const int r = ctid;
    const uint32_t nib_row = smem_u32(sN) + (uint32_t)(r * 32);
    const uint32_t dst_row = smem_u32(sW) + (uint32_t)(r * 128);
    for (int s = 0; s < nst; ++s) {
      const int slot = s % STAGES, ns = s % NRING;
      // thread 0 waits on both barriers; a hardware barrier releases the rest
      bool w = true;
      if (ctid == 0) {
        if (s >= STAGES) w = mbar_park(&empty[slot], ((s / STAGES) - 1) & 1, status, a.spin);
        w = w && mbar_park(&nib_full[ns], (s / NRING) & 1, status, a.spin);
      }
      w = bar_and<2, NCONV>(w);
      if (w) {
        uint32_t wd[8];
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(wd[0]), "=r"(wd[1]), "=r"(wd[2]), "=r"(wd[3])
                     : "r"(nib_row + (uint32_t)(ns * NIB_BYTES)));
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(wd[4]), "=r"(wd[5]), "=r"(wd[6]), "=r"(wd[7])
                     : "r"(nib_row + (uint32_t)(ns * NIB_BYTES) + 16));
        const uint32_t dst = dst_row + (uint32_t)(slot * STAGE_BYTES);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t L = wd[c] & 0x0F0F0F0Fu, H = (wd[c] >> 4) & 0x0F0F0F0Fu;
          const uint32_t o0 = bf16x2_minus136(prmt(L, 0x43434343u, 0x5140u));
          const uint32_t o1 = bf16x2_minus136(prmt(L, 0x43434343u, 0x5342u));
          const uint32_t o2 = bf16x2_minus136(prmt(H, 0x43434343u, 0x5140u));
          const uint32_t o3 = bf16x2_minus136(prmt(H, 0x43434343u, 0x5342u));
          asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(dst + ((c ^ (r & 7)) << 4)),
                       "r"(o0), "r"(o1), "r"(o2), "r"(o3)
                       : "memory");
        }
        fence_proxy_async_smem();
      }
      ok = w;
      if (!ok) break;
      bar_sync<2, NCONV>();  // every converter is done with this nibble stage
      if (ctid == 0) {
        mbar_arrive(&w_full[slot]);
        const int sn = s + NRING;
        if (sn < nst) {
          mbar_arrive_expect_tx(&nib_full[ns], NIB_BYTES);
          tma_load_2d(sN + ns * NIB_BYTES, &tm_.w, (k0 + KS * sn) / 8, n0, &nib_full[ns]);
          last_ph = (last_ph & ~(1u << ns)) | ((uint32_t)((sn / NRING) & 1) << ns);
        }
      }
    }
    if (ctid == 0) {
      for (int st = 0; st < NRING; ++st)
        if ((issued >> st) & 1u) mbar_poll(&nib_full[st], (last_ph >> st) & 1u, status);
    }
  } else {
    // ---------------- epilogue ----------------
    const int etid = threadIdx.x - EPI_WARP0 * 32;  // 0..511
    const int q = warp & 3;                         // TMEM lane quarter
    const int cb = (warp - EPI_WARP0) >> 2;         // 32-column block of a group
    const int nl = 32 * q + lane;                   // weight row within the tile
    if (!a.tma_w) {
      // tables by thread loads (row sizes the tensor copy cannot take)
      for (int i = etid; i < Gr * TW; i += NEPI) {
        const int n = i / Gr, g = i - n * Gr;
        const int64_t idx = (int64_t)(n0 + n) * G + g0 + g;
        const bool in = n0 + n < a.N;
        if (a.scale_bf16)
          *reinterpret_cast<unsigned short*>(scl + tbl_off(n, g, 2, srow)) =
              in ? __ldg(reinterpret_cast<const unsigned short*>(a.wscale) + idx) : (unsigned short)0;
        else
          *reinterpret_cast<float*>(scl + tbl_off(n, g, 4, srow)) =
              in ? __ldg(reinterpret_cast<const float*>(a.wscale) + idx) : 0.0f;
        if (WZP) *reinterpret_cast<float*>(zws + tbl_off(n, g, 4, frow)) = in ? __ldg(a.wzero + idx) : 0.0f;
      }
    }
    // activation tables come from the quantization grid
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if ((ABLK || WZP) && !a.tma_act) {
      const float* src = ABLK ? a.sA : a.Sg;  // [G][Mpad]
      for (int i = etid; i < Gr * TM; i += NEPI) {
        const int g = i / TM, mm = i - g * TM;
        actp[i] = src[(int64_t)(g0 + g) * a.Mpad + m0 + mm];
      }
    }
    bool ok = true;
    if (a.tma_w) ok = mbar_wait(prm_full, 0, status, a.spin);
    if ((ABLK || WZP) && a.tma_act) ok = mbar_wait(act_full, 0, status, a.spin) && ok;
    ok = bar_and<1, NEPI>(ok);  // also publishes the thread-loaded tables
    f32x2 acc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] = 0ull;
    for (int s = 0; s < nst && ok; ++s) {
      const int sb = s % NSB;
      // each warp waits on its own: lane 0 polls the accumulator barrier and
      // the warp takes its decision together (the TMEM loads below are
      // .sync.aligned); warps are not held in step with each other
      bool w = true;
      if (lane == 0) w = poll_yield(&tfull[sb], (uint32_t)(s / NSB) & 1, status, a.spin);
      ok = __shfl_sync(0xffffffffu, (int)w, 0) != 0;
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int gi = 0; gi < 2; ++gi) {
        const int g = 2 * s + gi;
        uint32_t p[32];
        tmem_ld32(tmem_base + ((uint32_t)(32 * q) << 16) +
                      (uint32_t)(sb * 2 * TM + gi * TM + 32 * cb), p);
        tmem_wait_ld();
        if (gi == 1) {  // both groups read: hand the stage buffer back
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[sb]);
        }
        const float sw =
            a.scale_bf16
                ? __uint_as_float((uint32_t)*reinterpret_cast<const unsigned short*>(scl + tbl_off(nl, g, 2, srow)) << 16)
                : *reinterpret_cast<const float*>(scl + tbl_off(nl, g, 4, srow));
        const f32x2 s2 = pack2(sw, sw);
        if (ABLK) {
          const float4* av = reinterpret_cast<const float4*>(actp + g * TM + 32 * cb);
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            const float4 a4 = av[j >> 1];  // same address in every lane: a broadcast
            ffma2(acc[j], pack2u(p[2 * j], p[2 * j + 1]), fmul2(s2, pack2(a4.x, a4.y)));
            ffma2(acc[j + 1], pack2u(p[2 * j + 2], p[2 * j + 3]), fmul2(s2, pack2(a4.z, a4.w)));
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) ffma2(acc[j], pack2u(p[2 * j], p[2 * j + 1]), s2);
        }
        if (WZP) {
          const float zw = *reinterpret_cast<const float*>(zws + tbl_off(nl, g, 4, frow));
          const f32x2 z2 = pack2(zw, zw);
          const float4* sv = reinterpret_cast<const float4*>(actp + g * TM + 32 * cb);
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            const float4 s4 = sv[j >> 1];
            ffma2(acc[j], pack2(s4.x, s4.y), z2);
            ffma2(acc[j + 1], pack2(s4.z, s4.w), z2);
          }
        }
      }
    }
    ok = bar_and<1, NEPI>(ok);
    // park the partial tile as [m][n]; every MMA has completed (the last
    // stage's accumulators were waited for), so the stage buffers are free
    if (ok) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        part[(32 * cb + 2 * j) * PST + nl] = lo_f(acc[j]);
        part[(32 * cb + 2 * j + 1) * PST + nl] = hi_f(acc[j]);
      }
    }
  }

  // Split-K reduction over the cluster (one CTA per K range): after the
  // first cluster barrier every partial is visible; CTA `split` sums its
  // share of the rows over all ranks in rank order (deterministic) and
  // writes y; the second barrier keeps every CTA's shared memory alive until
  // its peers have read it.  This CTA reduces rows [r0, r1) of the tile;
  // epilogue thread etid takes the 4-column chunk c = etid % 32 of rows
  // r0 + etid / 32 + 16j.  Its bias and row scales are fetched before the
  // cluster barrier, so each output waits only for the partials.
  const int rows_per = (TM + a.splits - 1) / a.splits;
  const int r0 = split * rows_per, r1 = min(TM, r0 + rows_per);
  constexpr int RSTEP = NEPI / 32;
  constexpr int RJ = TM / RSTEP;  // rows per thread at most (one split)
  float bias4[4] = {0.f, 0.f, 0.f, 0.f};
  float srow_s[RJ];
  __syncwarp();
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  if (warp >= EPI_WARP0) {
    const int etid = threadIdx.x - EPI_WARP0 * 32;
    const int c = etid & 31;
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (a.bias && n0 + 4 * c + e < a.N) bias4[e] = __ldg(a.bias + n0 + 4 * c + e);
#pragma unroll
    for (int j = 0; j < RJ; ++j) {
      const int mm = r0 + (etid >> 5) + RSTEP * j;
      srow_s[j] = (!ABLK && mm < r1 && m0 + mm < a.M) ? a.sA[m0 + mm] : 1.0f;
    }
  }
  __syncwarp();
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
  if (warp >= EPI_WARP0) {
    const int etid = threadIdx.x - EPI_WARP0 * 32;
    const uint32_t part_s = smem_u32(part);
    const bool vec = ((a.ldy & 3) == 0) && ((reinterpret_cast<uintptr_t>(a.y) & 15) == 0);
    const int c = etid & 31;
#pragma unroll
    for (int jr = 0; jr < RJ; ++jr) {
      const int mm = r0 + (etid >> 5) + RSTEP * jr;
      const int m = m0 + mm, n = n0 + 4 * c;
      if (mm >= r1 || m >= a.M || n >= a.N) continue;
      const uint32_t off = (uint32_t)((mm * PST + 4 * c) * 4);
      // every rank's partial requested before the first is added
      float4 t[MAX_SPLITS];
#pragma unroll
      for (int j = 0; j < MAX_SPLITS; ++j)
        if (j < a.splits) t[j] = ld_dsmem_f4(mapa(part_s + off, (uint32_t)j));
      const float s = srow_s[jr];
      float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int j = 0; j < MAX_SPLITS; ++j) {
        if (j < a.splits) {
          sum.x = __fadd_rn(sum.x, t[j].x);
          sum.y = __fadd_rn(sum.y, t[j].y);
          sum.z = __fadd_rn(sum.z, t[j].z);
          sum.w = __fadd_rn(sum.w, t[j].w);
        }
      }
      float t4[4] = {sum.x, sum.y, sum.z, sum.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (!ABLK) t4[e] = __fmul_rn(s, t4[e]);
        if (a.bias) t4[e] = __fadd_rn(t4[e], bias4[e]);
        t4[e] = fminf(fmaxf(t4[e], a.lo), a.hi);
      }
      float* yr = a.y + (int64_t)m * a.ldy + n;
      if (vec && n + 3 < a.N) {
        *reinterpret_cast<float4*>(yr) = make_float4(t4[0], t4[1], t4[2], t4[3]);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (n + e < a.N) yr[e] = t4[e];
      }
    }
  }
  // peers may still read this CTA's partial tile: leave only after all have
  // finished (no memory ordering is needed for that)
  __syncwarp();
  asm volatile("barrier.cluster.arrive.relaxed.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");

  // Reconverge every warp (single lanes ran the copy and MMA loops) so the
  // CTA barrier below counts complete warps, then free TMEM.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(NSB * 2 * TM)
                 : "memory");
  }
}

// Split count s (a cluster of s CTAs per output tile): K/s a multiple of 64
// and at most KR_MAX; the largest s with tiles * s within the SM count, else
// the smallest valid one; -1 if none.
int choose_splits(int64_t tiles, int K, int sms) {
  int best = -1;
  for (int s = 1; s <= MAX_SPLITS; ++s) {
    if (K % (KS * s)) continue;
    if (K / s > KR_MAX) continue;
    if (best < 0) best = s;
    if (tiles * s <= sms) best = s;
  }
  return best;
}

struct TcPlan {
  int m_tiles, n_tiles, splits, R;
  int64_t Mpad;
  size_t off_sA, off_Sg, bytes;
};

TcPlan plan_tc(int64_t M, int N, int K, int sms) {
  TcPlan p{};
  p.m_tiles = (int)cdiv(M, TM);
  p.n_tiles = (int)cdiv(N, TW);
  p.Mpad = (int64_t)p.m_tiles * TM;
  p.splits = choose_splits((int64_t)p.m_tiles * p.n_tiles, K, sms);
  int R = 1;
  while (R < 8 && (int64_t)K * 2 * R <= (int64_t)32 * QT) R *= 2;  // K <= 32 * (QT / R)
  p.R = R;
  const int G = K / 32;
  p.off_sA = (size_t)round_up(p.Mpad * K * 2, 256);
  p.off_Sg = p.off_sA + (size_t)round_up(p.Mpad * G * 4, 256);
  p.bytes = p.off_Sg + (size_t)round_up(p.Mpad * G * 4, 256);
  return p;
}

template <int MODE, bool CONV>
int launch_quant(const QuantArgs& qa, int grid, int R, cudaStream_t st) {
  // programmatic dependent launch: the CTAs are scheduled as the previous
  // kernel in the stream drains and wait for it on the device
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(QT);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, a8w4_quant_tiles_kernel<MODE, CONV>, qa, R) == cudaSuccess
             ? QG_OK
             : QG_ERR_CUDA;
}

}  // namespace

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
bool a8w4_tc_supported(int64_t M, int N, int K) {
  if (M < 2 || N < 1 || K < KS || K % KS) return false;
  if (K > QCH * 8 * QT) return false;  // one quantization CTA per row holds the row
  return choose_splits((cdiv(M, TM)) * cdiv(N, TW), K, 1 << 30) > 0;
}

size_t a8w4_tc_workspace_bytes(int64_t M, int N, int K) {
  return plan_tc(M, N, K, 1 << 30).bytes;
}

int a8w4_tc_setup() {
  const void* fns[] = {(const void*)a8w4_tc_kernel<false, false>,
                       (const void*)a8w4_tc_kernel<true, false>,
                       (const void*)a8w4_tc_kernel<false, true>};
  for (const void* f : fns)
    if (cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES) !=
        cudaSuccess)
      return QG_ERR_CUDA;
  return QG_OK;
}

int launch_a8w4_tc_call(const A8W4TcCall& c, void* ws, size_t ws_bytes, cudaStream_t st) {
  const TcPlan p = plan_tc(c.M, c.N, c.K, num_sms());
  if (p.splits <= 0) return QG_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < p.bytes) return QG_ERR_WORKSPACE;
  if ((c.mode == kBlockAsym) && c.wzero) return QG_ERR_UNSUPPORTED;
  uint8_t* w = (uint8_t*)ws;
  QuantArgs qa{};
  qa.M = (int)c.M;
  qa.K = c.K;
  qa.Mpad = (int)p.Mpad;
  qa.src.x = c.x;
  qa.src.ldx = c.ldx;
  qa.src.H = c.H; qa.src.W = c.W; qa.src.Cin = c.Cin; qa.src.KH = c.KH; qa.src.KW = c.KW;
  qa.src.sh = c.sh; qa.src.sw = c.sw; qa.src.ph = c.ph; qa.src.pw = c.pw;
  qa.src.OH = c.OH; qa.src.OW = c.OW;
  const bool x16 = ((uintptr_t)c.x & 15) == 0;
  qa.vec4 = c.conv ? (x16 && c.Cin % 8 == 0) : (x16 && c.ldx % 4 == 0);
  qa.atile = (uint16_t*)w;
  qa.sA = (float*)(w + p.off_sA);
  qa.Sg = c.wzero ? (float*)(w + p.off_Sg) : nullptr;
  qa.q_out = c.q_out;
  qa.q_vec = ((uintptr_t)c.q_out & 7) == 0;
  qa.scale_out = c.scale_out;
  qa.zp_out = c.zp_out;
  const int qgrid = (int)cdiv(p.Mpad, p.R);
  int rc;
  if (c.conv) {
    if (c.mode == kRowAsym) rc = launch_quant<kRowAsym, true>(qa, qgrid, p.R, st);
    else if (c.mode == kRowSym) rc = launch_quant<kRowSym, true>(qa, qgrid, p.R, st);
    else return QG_ERR_UNSUPPORTED;
  } else {
    if (c.mode == kRowAsym) rc = launch_quant<kRowAsym, false>(qa, qgrid, p.R, st);
    else if (c.mode == kBlockAsym) rc = launch_quant<kBlockAsym, false>(qa, qgrid, p.R, st);
    else rc = launch_quant<kRowSym, false>(qa, qgrid, p.R, st);
  }
  if (rc != QG_OK) return rc;

  const uint8_t* wq = (const uint8_t*)c.packed;
  TcMaps maps;
  rc = make_tmap_generic(&maps.w, CU_TENSOR_MAP_DATA_TYPE_UINT32, wq, (uint64_t)c.K / 8,
                         (uint64_t)c.N, (uint64_t)c.K / 2, KS / 8, TW, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (rc != QG_OK) return rc;
  maps.scl = maps.zw = maps.act = maps.w;
  GemmArgs ga{};
  ga.M = (int)c.M; ga.N = c.N; ga.K = c.K;
  ga.Kr = c.K / p.splits; ga.splits = p.splits; ga.n_tiles = p.n_tiles; ga.nkb = c.K / KS;
  ga.atile = qa.atile;
  ga.wscale = wq + (size_t)c.N * (c.K / 2);
  ga.scale_bf16 = c.scale_bf16 ? 1 : 0;
  ga.wzero = c.wzero;
  ga.sA = qa.sA;
  ga.Sg = qa.Sg;
  ga.Mpad = (int)p.Mpad;
  ga.bias = c.bias; ga.lo = c.lo; ga.hi = c.hi; ga.y = c.y; ga.ldy = c.ldy;
  // The per-group tables by tensor copy when a CTA's row of them is 32, 64
  // or 128 bytes and the global rows are 16-byte multiples (else thread loads).
  const int G = c.K / 32, Gr = ga.Kr / 32;
  auto swz_for = [](int rowbytes) {
    return rowbytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                           : rowbytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  };
  auto tma_ok = [](int rowbytes, int64_t pitch, const void* base) {
    return (rowbytes == 32 || rowbytes == 64 || rowbytes == 128) && pitch % 16 == 0 &&
           ((uintptr_t)base & 15) == 0;
  };
  const int sesz = c.scale_bf16 ? 2 : 4;
  ga.tma_w = tma_ok(Gr * sesz, (int64_t)G * sesz, ga.wscale) &&
             (!c.wzero || tma_ok(Gr * 4, (int64_t)G * 4, c.wzero));
  if (ga.tma_w) {
    rc = make_tmap_generic(&maps.scl,
                           c.scale_bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                           ga.wscale, (uint64_t)G, (uint64_t)c.N, (uint64_t)G * sesz, (uint32_t)Gr,
                           TW, swz_for(Gr * sesz));
    if (rc != QG_OK) return rc;
    if (c.wzero) {
      rc = make_tmap_generic(&maps.zw, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, c.wzero, (uint64_t)G,
                             (uint64_t)c.N, (uint64_t)G * 4, (uint32_t)Gr, TW, swz_for(Gr * 4));
      if (rc != QG_OK) return rc;
    }
  }
  // activation tables [G][Mpad] (transposed by the quantization grid): a
  // box of TM rows of Gr groups, unswizzled
  const float* act_src = c.mode == kBlockAsym ? qa.sA : qa.Sg;
  ga.tma_act = act_src && ((uintptr_t)act_src & 15) == 0 && p.Mpad % 4 == 0;
  if (ga.tma_act) {
    rc = make_tmap_generic(&maps.act, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, act_src, (uint64_t)p.Mpad,
                           (uint64_t)G, (uint64_t)p.Mpad * 4, TM, (uint32_t)Gr,
                           CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc != QG_OK) return rc;
  }
  ga.stall = take_stall(kStallA8W4TC) ? 1 : 0;
  ga.spin = ga.stall ? kStallSpinLimit : kSpinLimit;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((int64_t)p.m_tiles * p.n_tiles * p.splits));
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)p.splits;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // programmatic dependent launch: barriers, TMEM, the weight nibbles and
  // tables overlap the quantization grid
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e;
  if (c.mode == kBlockAsym)
    e = cudaLaunchKernelEx(&cfg, a8w4_tc_kernel<true, false>, maps, ga, status_word());
  else if (c.wzero)
    e = cudaLaunchKernelEx(&cfg, a8w4_tc_kernel<false, true>, maps, ga, status_word());
  else
    e = cudaLaunchKernelEx(&cfg, a8w4_tc_kernel<false, false>, maps, ga, status_word());
  return e == cudaSuccess ? QG_OK : QG_ERR_CUDA;
}

}  // namespace qg
