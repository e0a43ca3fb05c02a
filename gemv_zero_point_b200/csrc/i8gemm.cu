// Affine INT8 GEMM on the 5th-generation tensor cores (tcgen05, kind::i8)
// with the zero-point correction, bias, fixed-point requantization and clamp
// fused into the epilogue; the INT8 convolution runs through the same kernel.
//
// Sources: xidianedu "量化 GEMM：数值契约、SRAM、DMA 与结果验证" section 1
// (affine contract, int32 bias in accumulator scale, integer multiplier and
// shift), section 2 (padding stands for real zero; logical vs physical
// shape), section 4 (INT32 accumulator zeroed at the first K block, kept
// across all of K, post-processing once after the last block), section 5
// (element strides vs byte strides in copy descriptors; a double-buffer slot
// is overwritten only after its last read); MNN ConvInt8TiledExecutor.cpp
// (reorderWeight with per-column kernel sums; im2col padded with the input
// zero-point; QuanPostTreatParameters clamp bounds).
//
// Expanded form of the accumulator computed here (exact in int32 under the
// overflow bound the API enforces):
//   acc[m,n] = S[m,n] - za*colsum[n] - zb*rowsum[m] + K*za*zb + bias[n]
//   S = sum_k A[m,k]*B[k,n] (tensor cores), colsum[n] = sum_k B[k,n],
//   rowsum[m] = sum_k A[m,k].
// Padding of B beyond K is zero, so the padded K positions add nothing to S,
// colsum or rowsum whatever A holds there.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include "qg_internal.cuh"

namespace qg {

namespace {

constexpr int BM = 128;          // tile rows (TMEM lanes)
constexpr int BN = 256;          // tile columns (TMEM columns per accumulator)
constexpr int BK = 128;          // bytes of K per pipeline stage (one 128B swizzle atom)
constexpr int STAGES = 4;
constexpr int A_STAGE = BM * BK;  // 16 KiB
constexpr int B_STAGE = BN * BK;  // 32 KiB
constexpr int TMEM_COLS = 2 * BN; // double-buffered accumulator
constexpr int THREADS = 192;      // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr int CONV_PW = 4;        // implicit-im2col gather warps: one A row per thread
constexpr int THREADS_CONV = (CONV_PW + 5) * 32;  // + MMA warp + 4 epilogue warps
constexpr size_t SMEM_BYTES = 1024 /*align slack*/ + STAGES * (A_STAGE + B_STAGE) + 6144;

// Instruction descriptor for kind::i8: D s32, A s8, B s8, both K-major,
// M = BM, N = n (a multiple of 16, 16..256).
__host__ __device__ constexpr uint32_t idesc_i8(int n) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(BM >> 4) << 24);
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (sm_100 descriptor version 1).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;            // leading byte offset (unused with 128B swizzle)
  d |= (uint64_t)(1024 >> 4) << 32;  // stride byte offset between 8-row groups
  d |= (uint64_t)1 << 46;            // descriptor version
  d |= (uint64_t)2 << 61;            // SWIZZLE_128B
  return d;
}

__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void mma_i8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
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
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void epi_bar_sync() {
  asm volatile("bar.sync 1, 128;" ::: "memory");
}
// Barrier over the 128 epilogue threads that also ANDs a predicate, so every
// epilogue thread takes the same decision after a bounded wait.
__device__ __forceinline__ bool epi_bar_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

// y = clamp(zo + rne(acc*M0 / 2^(31+sh)), lo, hi).  With p = acc*M0 and
// s = 31+sh: rne(p/2^s) = (p + 2^(s-1) - 1 + ((p >> s) & 1)) >> s.
// |acc| <= 2^31 - 1 (the overflow bound) and M0 < 2^31 give |p| < 2^62, so
// the rounded quotient fits int32 and the clamp runs in 32 bits:
// clamp(q + zo, lo, hi) = clamp(q, lo - zo, hi - zo) + zo.  The epilogue
// passes s = 31 + shift and rnd = 2^(s-1) - 1 precomputed per column, and
// the clamp bounds lo - zo, hi - zo.
__device__ __forceinline__ int requant_s(int acc, int m0, int s, long long rnd, int zo, int lo_z,
                                         int hi_z) {
  const long long p = (long long)acc * (long long)m0;
  const int q = (int)((p + rnd + ((p >> s) & 1)) >> s);
  return min(max(q, lo_z), hi_z) + zo;
}

struct EpiArgs {
  int M, N, K;
  int za, zb, zo, lo, hi;
  const int32_t* colsum;   // [>= N]
  const int32_t* rowsum;   // [M] or NULL (zb == 0)
  const int32_t* bias;     // [N] or NULL
  int per_channel, m0, sh;
  const int32_t* m0v;      // [N] when per_channel
  const int32_t* shv;
  int8_t* C;
  int64_t ldc;
  int32_t* acc_out;
  int64_t ld_acc;
  int stall;        // test hook (one-CTA kernel): skip the loads of K block 1 of the first tile
  uint32_t spin;    // poll limit of the pipeline waits
  int nmma;         // one-CTA kernel: MMA N and B-tile rows (BN, or N rounded up to 16
                    // when one column tile covers N)
};

// ---------------------------------------------------------------------------
// Implicit im2col for the convolution (MNN tileSplitFunction: the unrolled
// input, with the input zero-point in padded taps; [QG] section 2).  Row m
// of the virtual A matrix is output pixel (n, oh, ow); byte k = (kh*KW +
// kw)*Cin + ci holds x[n, oh*sh+kh-ph, ow*sw+kw-pw, ci], or za outside the
// image.  The producer warp writes each stage's 128 rows x 128 bytes straight
// into the swizzled shared-memory tile: 16-byte cp.async copies when every
// 16-byte chunk of a row is one contiguous run of channels (Cin % 16 == 0,
// x 16-byte aligned), byte loads otherwise.  Bytes past K and rows past M are
// left as they are: the packed weights are zero past K, and rows past M are
// never stored.
// ---------------------------------------------------------------------------
struct ConvGather {
  const int8_t* x;
  int H, W, Cin, KH, KW, sh, sw, ph, pw, OH, OW;
  int M, K;
  int za;
  int vec16;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// The output pixel of im2col row m, decoded once per tile: its image and
// the input coordinates of tap (0, 0).
struct ConvRow {
  const int8_t* img;
  int ihb, iwb;
  bool ok;
};
__device__ __forceinline__ ConvRow conv_row(const ConvGather& g, int m) {
  ConvRow cr;
  cr.ok = m < g.M;
  const int mm = cr.ok ? m : 0;
  const int ow = mm % g.OW, t = mm / g.OW;
  const int oh = t % g.OH, n = t / g.OH;
  cr.ihb = oh * g.sh - g.ph;
  cr.iwb = ow * g.sw - g.pw;
  cr.img = g.x + (int64_t)n * g.H * g.W * g.Cin;
  return cr;
}

// Row r of K block kb into the swizzled stage (row r at byte r*128, 16-byte
// chunk c at position c ^ (r & 7)).  With Cin % 16 == 0 and a 16-byte
// aligned input, a 16-byte chunk of K lies inside one tap: lane c of the
// warp decodes chunk c of the block (tap, channel) and the warp shares it,
// then each thread copies its row's chunk with cp.async, or writes the
// input zero-point where the tap falls in the padding.  Otherwise the bytes
// are read one by one (first layers with few channels), stepping
// (kh, kw, ci) along K without divisions.  K positions at or beyond K are
// left as they are: the packed weights are zero there.
__device__ __forceinline__ void conv_gather_row(const ConvGather& g, const ConvRow& cr,
                                                uint8_t* drow, int r, int kb, int lane) {
  const uint32_t za4 = (uint32_t)(uint8_t)g.za * 0x01010101u;
  const int k0 = kb * BK;
  if (g.vec16) {
    int ckh = -1, ckw = 0, cci = 0;
    if (lane < 8) {
      const int k = k0 + 16 * lane;
      if (k < g.K) {
        const int tap = k / g.Cin;
        cci = k - tap * g.Cin;
        ckh = tap / g.KW;
        ckw = tap - ckh * g.KW;
      }
    }
    int kh[8], kw[8], ci[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      kh[c] = __shfl_sync(0xffffffffu, ckh, c);
      kw[c] = __shfl_sync(0xffffffffu, ckw, c);
      ci[c] = __shfl_sync(0xffffffffu, cci, c);
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      if (kh[c] < 0) break;
      uint8_t* d = drow + ((c ^ (r & 7)) << 4);
      const int ih = cr.ihb + kh[c], iw = cr.iwb + kw[c];
      if (cr.ok && (unsigned)ih < (unsigned)g.H && (unsigned)iw < (unsigned)g.W)
        cp_async16(smem_u32(d), cr.img + ((int64_t)ih * g.W + iw) * g.Cin + ci[c]);
      else
        *reinterpret_cast<uint4*>(d) = make_uint4(za4, za4, za4, za4);
    }
  } else {
    if (k0 >= g.K) return;
    int tap = k0 / g.Cin;
    int ci = k0 - tap * g.Cin;
    int kh = tap / g.KW;
    int kw = tap - kh * g.KW;
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      if (k0 + 16 * c >= g.K) break;
      uint32_t wv[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int b = 0; b < 16; ++b) {
        const int k = k0 + 16 * c + b;
        const int ih = cr.ihb + kh, iw = cr.iwb + kw;
        int v = g.za;
        if (k < g.K && cr.ok && (unsigned)ih < (unsigned)g.H && (unsigned)iw < (unsigned)g.W)
          v = cr.img[((int64_t)ih * g.W + iw) * g.Cin + ci];
        wv[b >> 2] |= ((uint32_t)v & 0xFFu) << (8 * (b & 3));
        if (++ci == g.Cin) {
          ci = 0;
          if (++kw == g.KW) {
            kw = 0;
            ++kh;
          }
        }
      }
      *reinterpret_cast<uint4*>(drow + ((c ^ (r & 7)) << 4)) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
    }
  }
}

// CONV = false: A is a row-major matrix read by the tensor-copy engine.
// CONV = true: A is the implicit im2col of `cg`, gathered by CONV_PW warps
// (one tile row per thread, see conv_gather_row); B still comes by tensor
// copies.  Warp roles: producers, then the MMA warp, then 4 epilogue warps.
template <bool CONV>
__global__ void __launch_bounds__(CONV ? THREADS_CONV : THREADS, 1)
    i8gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     int num_kb, int tiles_m, int tiles_n, EpiArgs ep, ConvGather cg, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_STAGE;
  uint64_t* full = (uint64_t*)(sB + STAGES * B_STAGE);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;                 // MMA completion after a failed wait
  uint32_t* tmem_slot = (uint32_t*)(drain + 1);
  // [BN] per-column constants, 16-byte aligned (read four at a time)
  int32_t* c_term = (int32_t*)(((uintptr_t)(tmem_slot + 4) + 15) & ~(uintptr_t)15);
  int32_t* c_m0 = c_term + BN;                   // [BN]
  int32_t* c_sh = c_m0 + BN;                     // [BN] 31 + shift
  long long* c_rnd = (long long*)(c_sh + BN);    // [BN] 2^(30 + shift) - 1

  constexpr int PW = CONV ? CONV_PW : 1;  // producer warps
  constexpr int MMA_WARP = PW, EPI_WARP0 = PW + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles = tiles_m * tiles_n;
  const uint32_t b_bytes = (uint32_t)ep.nmma * BK;  // B tile rows actually copied
  // Launched as a programmatic dependent: the next grid in the stream may be
  // scheduled now (on SMs this one leaves free) and set itself up; every
  // role that touches global memory waits for the previous grid first.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], CONV ? 32 * PW : 1);  // conv: every producer thread arrives
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    if (!CONV) prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == MMA_WARP) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (CONV && warp < PW) {
    // ---------------- implicit-im2col producers ----------------
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // Thread ptid gathers row ptid of every tile.  Stage s is signalled one
    // stage late: after the copies of stage s+1 are issued, each thread
    // waits for its own copies of stage s, makes them and its zero-point
    // fills visible to the tensor cores, and arrives.  Warp 0 lane 0 also
    // issues the weight tensor copies.
    const int ptid = threadIdx.x;  // 0 .. 32*PW-1
    int stage = 0, prev = -1;
    uint32_t phase = 0;
    uint32_t issued = 0, last_ph = 0;  // B tensor copies (thread 0)
    for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
      const int tm = t % tiles_m, tn = t / tiles_m;
      const ConvRow cr = conv_row(cg, tm * BM + ptid);
      for (int kb = 0; kb < num_kb; ++kb) {
        bool got = true;
        if (lane == 0) got = mbar_poll(&empty[stage], phase ^ 1, status, ep.spin);
        if (!__shfl_sync(0xffffffffu, (int)got, 0)) goto conv_done;
        if (ptid == 0) {
          mbar_expect_tx(&full[stage], b_bytes);
          tma_load_2d(sB + stage * B_STAGE, &tmB, kb * BK, tn * BN, &full[stage]);
          issued |= 1u << stage;
          last_ph = (last_ph & ~(1u << stage)) | (phase << stage);
        }
        conv_gather_row(cg, cr, sA + stage * A_STAGE + ptid * BK, ptid, kb, lane);
        cp_async_commit();
        if (prev >= 0) {
          cp_async_wait<1>();
          fence_proxy_async_smem();
          mbar_arrive(&full[prev]);
        }
        prev = stage;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
  conv_done:
    cp_async_wait<0>();
    fence_proxy_async_smem();
    if (prev >= 0) mbar_arrive(&full[prev]);
    if (ptid == 0)
      for (int st = 0; st < STAGES; ++st)
        if ((issued >> st) & 1u) mbar_poll(&full[st], (last_ph >> st) & 1u, status);
  } else if (warp == 0) {
    // ------------------------- TMA producer -------------------------
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_ph = 0;  // per slot: loads issued, parity of the last issue
      for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
        const int tm = t % tiles_m, tn = t / tiles_m;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_poll(&empty[stage], phase ^ 1, status, ep.spin)) goto producer_done;
          if (!(ep.stall && t == (int)blockIdx.x && kb == 1)) {
            mbar_arrive_expect_tx(&full[stage], A_STAGE + b_bytes);
            tma_load_2d(sA + stage * A_STAGE, &tmA, kb * BK, tm * BM, &full[stage]);
            tma_load_2d(sB + stage * B_STAGE, &tmB, kb * BK, tn * BN, &full[stage]);
            issued |= 1u << stage;
            last_ph = (last_ph & ~(1u << stage)) | (phase << stage);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    producer_done:
      // every copy this thread issued has landed before the CTA may exit
      // (after a normal run these phases completed long ago)
      for (int st = 0; st < STAGES; ++st)
        if ((issued >> st) & 1u) mbar_poll(&full[st], (last_ph >> st) & 1u, status);
    }
  } else if (warp == MMA_WARP) {
    // ------------------------- MMA issuer -------------------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool failed = false;
      for (int t = blockIdx.x; t < tiles && !failed; t += gridDim.x, ++local) {
        const int buf = local & 1;
        const uint32_t use = (uint32_t)(local >> 1);
        if (!mbar_poll(&tempty[buf], (use & 1) ^ 1, status, ep.spin)) {
          failed = true;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(buf * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_poll(&full[stage], phase, status, ep.spin)) {
            failed = true;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * A_STAGE);
          const uint32_t b0 = smem_u32(sB + stage * B_STAGE);
#pragma unroll
          for (int k = 0; k < BK / 32; ++k) {
            mma_i8(d, sdesc_sw128(a0 + 32 * k), sdesc_sw128(b0 + 32 * k), idesc_i8(ep.nmma),
                   (kb | k) != 0);
          }
          mma_commit(&empty[stage]);  // frees the stage when these MMAs finish
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!failed) mma_commit(&tfull[buf]);  // accumulator ready for the epilogue
      }
      if (failed) {
        // MMAs already issued finish before TMEM is freed
        mma_commit(drain);
        mbar_poll(drain, 0, status);
      }
    }
  } else {
    // ------------------------- epilogue -------------------------
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int etid = threadIdx.x - 32 * EPI_WARP0;  // 0..127
    const int row_in_tile = 32 * q + lane;
    const int64_t Kza_zb = (int64_t)ep.K * ep.za * ep.zb;
    const int lo_z = ep.lo - ep.zo, hi_z = ep.hi - ep.zo;
    int local = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++local) {
      const int tm = t % tiles_m, tn = t / tiles_m;
      const int buf = local & 1;
      const uint32_t use = (uint32_t)(local >> 1);
      epi_bar_sync();  // previous tile's column constants no longer read
      for (int c = etid; c < BN; c += 128) {
        const int n = tn * BN + c;
        if (n < ep.N) {
          const int64_t v = (ep.bias ? (int64_t)ep.bias[n] : 0) -
                            (int64_t)ep.za * ep.colsum[n] + Kza_zb;
          c_term[c] = (int32_t)v;  // wraps mod 2^32; the final sum is in range
          c_m0[c] = ep.per_channel ? ep.m0v[n] : ep.m0;
          const int sft = 31 + (ep.per_channel ? ep.shv[n] : ep.sh);
          c_sh[c] = sft;
          c_rnd[c] = (1LL << (sft - 1)) - 1;
        }
      }
      epi_bar_sync();
      const int m = tm * BM + row_in_tile;
      const bool row_ok = m < ep.M;
      const int32_t r_term = (ep.rowsum && row_ok) ? -ep.zb * ep.rowsum[m] : 0;
      const bool ok = epi_bar_and(mbar_wait(&tfull[buf], use & 1, status, ep.spin));
      tc_fence_after();
      if (ok) {
        for (int ch = 0; ch < BN / 32; ++ch) {
          const int nb = tn * BN + ch * 32;
          if (nb >= ep.N) break;  // warp-uniform
          uint32_t r[32];
          tmem_ld32(tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * BN + ch * 32), r);
          if (!row_ok) continue;
          const bool full_chunk = nb + 32 <= ep.N;
          int accv[32];
          uint32_t packed[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {  // four columns' constants per load
            const int4 t4 = reinterpret_cast<const int4*>(c_term + ch * 32)[jj];
            const int4 m4 = reinterpret_cast<const int4*>(c_m0 + ch * 32)[jj];
            const int4 s4 = reinterpret_cast<const int4*>(c_sh + ch * 32)[jj];
            const longlong2 r01 = reinterpret_cast<const longlong2*>(c_rnd + ch * 32)[2 * jj];
            const longlong2 r23 = reinterpret_cast<const longlong2*>(c_rnd + ch * 32)[2 * jj + 1];
            const int tt[4] = {t4.x, t4.y, t4.z, t4.w}, mv[4] = {m4.x, m4.y, m4.z, m4.w},
                      sv[4] = {s4.x, s4.y, s4.z, s4.w};
            const long long rv[4] = {r01.x, r01.y, r23.x, r23.y};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int j = 4 * jj + e;
              const int a = (int)((uint32_t)r[j] + (uint32_t)tt[e] + (uint32_t)r_term);
              accv[j] = a;
              const int yv = requant_s(a, mv[e], sv[e], rv[e], ep.zo, lo_z, hi_z);
              packed[j >> 2] |= ((uint32_t)yv & 0xFFu) << (8 * (j & 3));
            }
          }
          int8_t* cp = ep.C + (int64_t)m * ep.ldc + nb;
          if (full_chunk && (((uintptr_t)cp & 15) == 0)) {
            reinterpret_cast<uint4*>(cp)[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
            reinterpret_cast<uint4*>(cp)[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (nb + j < ep.N) cp[j] = (int8_t)((packed[j >> 2] >> (8 * (j & 3))) & 0xFF);
          }
          if (ep.acc_out) {
            int32_t* ap = ep.acc_out + (int64_t)m * ep.ld_acc + nb;
            if (full_chunk && (((uintptr_t)ap & 15) == 0)) {
#pragma unroll
              for (int j = 0; j < 32; j += 4)
                reinterpret_cast<int4*>(ap + j)[0] = make_int4(accv[j], accv[j + 1], accv[j + 2], accv[j + 3]);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (nb + j < ep.N) ap[j] = accv[j];
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
      if (!ok) break;
    }
  }

  // Reconverge every warp (lane 0 of the TMA and MMA warps ran their loops
  // alone) so the CTA barrier below counts complete warps only after all
  // of their work, in particular before TMEM is freed.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// 2-CTA version (cta_group::2).  A cluster of two CTAs on two SMs computes a
// 256 x 256 tile: CTA rank r stages rows [128r, 128r+128) of the A tile and
// columns [128r, 128r+128) of the B tile (32 KiB per stage, so 6 stages fit),
// and its TMEM receives rows [128r, 128r+128) x all 256 columns.  Rank 0 (the
// leader) issues tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 32); both
// CTAs' tensor copies complete on the leader's `full` barrier, the leader's
// commits arrive on both CTAs' `empty` / `tfull` barriers, and both epilogues
// hand the accumulator back on the leader's `tempty` barrier.  No cluster
// multicast load is used.
// ---------------------------------------------------------------------------
constexpr int P_STAGES = 6;
constexpr int P_STAGE = BM * BK;  // 16 KiB for the A half, same for the B half
constexpr size_t P_SMEM_BYTES = 1024 + (size_t)P_STAGES * 2 * P_STAGE + 6144;
constexpr int P_GROUP_M = 16;     // pair-tile rows per raster group (A slice stays in L2)
// kind::i8, D s32, A/B s8 K-major, N = 256, M = 256 (the pair)
constexpr uint32_t IDESC2 = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(256 >> 3) << 17) |
                            ((uint32_t)(256 >> 4) << 24);

__device__ __forceinline__ uint32_t cluster_rank_u32() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ uint32_t mapa_u32(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
// Tensor copy into this CTA's shared memory whose completion is counted on the
// (leader's) barrier at cluster address `bar_cluster`.
__device__ __forceinline__ void tma_load_2d_pair(void* dst_smem, const void* tmap, int32_t x,
                                                 int32_t y, uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst_smem)),
      "l"(tmap), "r"(x), "r"(y), "r"(bar_cluster)
      : "memory");
}
__device__ __forceinline__ void mma_i8_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(IDESC2), "r"(accumulate)
      : "memory");
}
// Arrive on the barrier at the same offset in both CTAs of the pair once the
// leader's prior MMAs complete.
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"((uint16_t)0x3)
      : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster)
               : "memory");
}

__device__ __forceinline__ void pair_tile_coords(int t, int tiles_m, int tiles_n, int& tm, int& tn) {
  const int per_group = P_GROUP_M * tiles_n;
  const int g = t / per_group, r = t % per_group;
  const int rows = min(P_GROUP_M, tiles_m - g * P_GROUP_M);
  tm = g * P_GROUP_M + r % rows;
  // serpentine: odd groups sweep the B panels from the last one back, so a
  // group starts on the panels the previous one read last (still in L2)
  tn = (g & 1) ? tiles_n - 1 - r / rows : r / rows;
}

__global__ void __launch_bounds__(THREADS, 1)
    i8gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      int num_kb, int tiles_m, int tiles_n, EpiArgs ep, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem;
  uint8_t* sB = smem + P_STAGES * P_STAGE;
  uint64_t* full = (uint64_t*)(sB + P_STAGES * P_STAGE);
  uint64_t* empty = full + P_STAGES;
  uint64_t* tfull = empty + P_STAGES;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = (uint32_t*)(tempty + 2);
  int32_t* c_term = (int32_t*)(((uintptr_t)(tmem_slot + 4) + 15) & ~(uintptr_t)15);
  int32_t* c_m0 = c_term + 256;
  int32_t* c_sh = c_m0 + 256;                    // 31 + shift
  long long* c_rnd = (long long*)(c_sh + 256);   // 2^(30 + shift) - 1

  // the next grid in the stream may be scheduled now (it waits for this one
  // on the device before it touches memory)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank_u32();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int tiles = tiles_m * tiles_n;

  if (threadIdx.x == 0) {
    for (int s = 0; s < P_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 8);  // 4 epilogue warps in each CTA of the pair
    }
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------- TMA producer (both CTAs) -------------------------
    if (lane == 0) {
      // B never comes from the grid this one may overlap (the A staging
      // pass, launched as its programmatic primary): the first ring's worth
      // of B tiles is requested before the grid dependency wait, A after it.
      int pre = 0;
      for (int t = pair, kb = 0; pre < P_STAGES && t < tiles; ++pre) {
        int tm, tn;
        pair_tile_coords(t, tiles_m, tiles_n, tm, tn);
        const uint32_t fb = mapa_u32(smem_u32(&full[pre]), 0);
        if (leader) mbar_arrive_expect_tx(&full[pre], 2u * 2u * P_STAGE);
        tma_load_2d_pair(sB + pre * P_STAGE, &tmB, kb * BK, tn * 256 + (int)rank * BM, fb);
        if (++kb == num_kb) {
          kb = 0;
          t += npairs;
        }
      }
      asm volatile("griddepcontrol.wait;" ::: "memory");
      int stage = 0, it = 0;
      uint32_t phase = 0;
      for (int t = pair; t < tiles; t += npairs) {
        int tm, tn;
        pair_tile_coords(t, tiles_m, tiles_n, tm, tn);
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const uint32_t fb = mapa_u32(smem_u32(&full[stage]), 0);
          if (it >= pre) {  // slots of the first ring pass were set up above
            if (!mbar_poll(&empty[stage], phase ^ 1, status)) goto producer_done;
            if (leader) mbar_arrive_expect_tx(&full[stage], 2u * 2u * P_STAGE);
            tma_load_2d_pair(sB + stage * P_STAGE, &tmB, kb * BK, tn * 256 + (int)rank * BM, fb);
          }
          tma_load_2d_pair(sA + stage * P_STAGE, &tmA, kb * BK, tm * 256 + (int)rank * BM, fb);
          if (++stage == P_STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    producer_done:;
    }
  } else if (warp == 1) {
    // ------------------------- MMA issuer (leader only) -------------------------
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      for (int t = pair; t < tiles; t += npairs, ++local) {
        const int buf = local & 1;
        const uint32_t use = (uint32_t)(local >> 1);
        if (!mbar_poll(&tempty[buf], (use & 1) ^ 1, status)) goto mma_done;
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(buf * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_poll(&full[stage], phase, status)) goto mma_done;
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * P_STAGE);
          const uint32_t b0 = smem_u32(sB + stage * P_STAGE);
#pragma unroll
          for (int k = 0; k < BK / 32; ++k)
            mma_i8_pair(d, sdesc_sw128(a0 + 32 * k), sdesc_sw128(b0 + 32 * k), (kb | k) != 0);
          mma_commit_pair(&empty[stage]);
          if (++stage == P_STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        mma_commit_pair(&tfull[buf]);
      }
    mma_done:;
    }
  } else {
    // ------------------------- epilogue (both CTAs) -------------------------
    const int q = warp & 3;
    const int etid = threadIdx.x - 64;
    const int row_in_tile = 32 * q + lane;
    const int64_t Kza_zb = (int64_t)ep.K * ep.za * ep.zb;
    const int lo_z = ep.lo - ep.zo, hi_z = ep.hi - ep.zo;
    const uint32_t tempty_leader0 = mapa_u32(smem_u32(&tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa_u32(smem_u32(&tempty[1]), 0);
    int local = 0;
    for (int t = pair; t < tiles; t += npairs, ++local) {
      int tm, tn;
      pair_tile_coords(t, tiles_m, tiles_n, tm, tn);
      const int buf = local & 1;
      const uint32_t use = (uint32_t)(local >> 1);
      epi_bar_sync();
      for (int c = etid; c < BN; c += 128) {
        const int n = tn * BN + c;
        if (n < ep.N) {
          const int64_t v = (ep.bias ? (int64_t)ep.bias[n] : 0) -
                            (int64_t)ep.za * ep.colsum[n] + Kza_zb;
          c_term[c] = (int32_t)v;
          c_m0[c] = ep.per_channel ? ep.m0v[n] : ep.m0;
          const int sft = 31 + (ep.per_channel ? ep.shv[n] : ep.sh);
          c_sh[c] = sft;
          c_rnd[c] = (1LL << (sft - 1)) - 1;
        }
      }
      epi_bar_sync();
      const int m = tm * 256 + (int)rank * BM + row_in_tile;
      const bool row_ok = m < ep.M;
      if (local == 0) asm volatile("griddepcontrol.wait;" ::: "memory");  // row sums
      const int32_t r_term = (ep.rowsum && row_ok) ? -ep.zb * ep.rowsum[m] : 0;
      const bool ok = epi_bar_and(mbar_wait(&tfull[buf], use & 1, status, ep.spin));
      tc_fence_after();
      if (ok) {
        for (int ch = 0; ch < BN / 32; ++ch) {
          const int nb = tn * BN + ch * 32;
          if (nb >= ep.N) break;  // warp-uniform
          uint32_t r[32];
          tmem_ld32(tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * BN + ch * 32), r);
          if (!row_ok) continue;
          const bool full_chunk = nb + 32 <= ep.N;
          int accv[32];
          uint32_t packed[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {  // four columns' constants per load
            const int4 t4 = reinterpret_cast<const int4*>(c_term + ch * 32)[jj];
            const int4 m4 = reinterpret_cast<const int4*>(c_m0 + ch * 32)[jj];
            const int4 s4 = reinterpret_cast<const int4*>(c_sh + ch * 32)[jj];
            const longlong2 r01 = reinterpret_cast<const longlong2*>(c_rnd + ch * 32)[2 * jj];
            const longlong2 r23 = reinterpret_cast<const longlong2*>(c_rnd + ch * 32)[2 * jj + 1];
            const int tt[4] = {t4.x, t4.y, t4.z, t4.w}, mv[4] = {m4.x, m4.y, m4.z, m4.w},
                      sv[4] = {s4.x, s4.y, s4.z, s4.w};
            const long long rv[4] = {r01.x, r01.y, r23.x, r23.y};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int j = 4 * jj + e;
              const int a = (int)((uint32_t)r[j] + (uint32_t)tt[e] + (uint32_t)r_term);
              accv[j] = a;
              const int yv = requant_s(a, mv[e], sv[e], rv[e], ep.zo, lo_z, hi_z);
              packed[j >> 2] |= ((uint32_t)yv & 0xFFu) << (8 * (j & 3));
            }
          }
          int8_t* cp = ep.C + (int64_t)m * ep.ldc + nb;
          if (full_chunk && (((uintptr_t)cp & 15) == 0)) {
            reinterpret_cast<uint4*>(cp)[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
            reinterpret_cast<uint4*>(cp)[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (nb + j < ep.N) cp[j] = (int8_t)((packed[j >> 2] >> (8 * (j & 3))) & 0xFF);
          }
          if (ep.acc_out) {
            int32_t* ap = ep.acc_out + (int64_t)m * ep.ld_acc + nb;
            if (full_chunk && (((uintptr_t)ap & 15) == 0)) {
#pragma unroll
              for (int j = 0; j < 32; j += 4)
                reinterpret_cast<int4*>(ap + j)[0] = make_int4(accv[j], accv[j + 1], accv[j + 2], accv[j + 3]);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (nb + j < ep.N) ap[j] = accv[j];
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(buf ? tempty_leader1 : tempty_leader0);
      if (!ok) break;
    }
  }

  // Reconverge every warp, then the whole pair: no CTA leaves while its peer
  // may still signal its barriers or read its shared memory; then free TMEM.
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(TMEM_COLS)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// B pack (row-major B[K][ldb] -> K-major Bp[Np][Kp], zero padded) with the
// column sums colsum[n] = sum_{k<K} B[k,n].  64x64 tiles through shared memory.
// ---------------------------------------------------------------------------
__global__ void pack_b_rowmajor_kernel(int K, int N, const int8_t* __restrict__ B, int64_t ldb,
                                       int8_t* __restrict__ Bp, int64_t Kp,
                                       int32_t* __restrict__ colsum) {
  __shared__ int8_t t[64][65];
  const int k0 = blockIdx.x * 64, n0 = blockIdx.y * 64;
  const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
  for (int r = ty; r < 64; r += 8) {
    const int k = k0 + r;
    for (int c = tx; c < 64; c += 32) {
      const int n = n0 + c;
      t[r][c] = (k < K && n < N) ? B[(int64_t)k * ldb + n] : (int8_t)0;
    }
  }
  __syncthreads();
  for (int r = ty; r < 64; r += 8) {
    const int n = n0 + r;
    for (int c = tx; c < 64; c += 32) Bp[(int64_t)n * Kp + k0 + c] = t[c][r];
  }
  if (ty == 0) {
    for (int c = tx; c < 64; c += 32) {
      int s = 0;
      for (int r = 0; r < 64; ++r) s += t[r][c];
      if (n0 + c < N && s != 0) atomicAdd(&colsum[n0 + c], s);
    }
  }
}

// K-major source (w[N][ldw], K contiguous; conv weights [Cout][KH][KW][Cin]).
__global__ void pack_b_kmajor_kernel(int K, int N, const int8_t* __restrict__ W, int64_t ldw,
                                     int8_t* __restrict__ Bp, int64_t Kp,
                                     int32_t* __restrict__ colsum) {
  __shared__ int red[8];
  const int n = blockIdx.x;
  int s = 0;
  for (int k = threadIdx.x; k < Kp; k += blockDim.x) {
    int8_t v = (n < N && k < K) ? W[(int64_t)n * ldw + k] : (int8_t)0;
    Bp[(int64_t)n * Kp + k] = v;
    s += v;
  }
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    int tot = 0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) tot += red[i];
    colsum[n] = tot;
  }
}

// ---------------------------------------------------------------------------
// A staging: copy rows into a 16-byte-aligned buffer (ld = ldw) when A's own
// rows cannot be described to the tensor-copy engine, and/or compute
// rowsum[m] = sum_k A[m,k] when zb != 0.  One CTA per row.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) stage_a_kernel(int K, const int8_t* __restrict__ A,
                                                      int64_t lda, int8_t* __restrict__ Aw,
                                                      int64_t ldw, int32_t* __restrict__ rowsum) {
  // the GEMM grid may start its prologue and its B copies now; it waits for
  // this grid before it reads the staged rows or the row sums
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // This grid is a programmatic dependent of the previous work in the
  // stream: A is read and the workspace written only once that has finished.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ int red[8];
  const int64_t m = blockIdx.x;
  const int8_t* src = A + m * lda;
  int8_t* dst = Aw ? Aw + m * ldw : nullptr;  // 16-byte aligned rows
  int s = 0;
  // Whole 16-byte chunks: output chunk j holds row bytes [16j, 16j + 16),
  // which sit at offset a = src % 16 in the aligned source chunks j and
  // j + 1.  A chunk is loaded only when it holds a byte of the row, so no
  // load leaves the pages the row lies in; bytes past K in the last chunk
  // land in the staged row's padding (never read) and are left out of the
  // sum.
  const int a = (int)((uintptr_t)src & 15);
  const uint4* s4 = reinterpret_cast<const uint4*>(src - a);
  const int nchunk = (K + 15) >> 4;
  for (int j = threadIdx.x; j < nchunk; j += blockDim.x) {
    const int end = min(16 * j + 16, K);  // row bytes [16j, end) are real
    const uint4 lo = __ldg(s4 + j);
    uint4 hi = make_uint4(0u, 0u, 0u, 0u);
    if (a != 0 && end + a > 16 * (j + 1)) hi = __ldg(s4 + j + 1);
    const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
    const int q = a >> 2, sh = 8 * (a & 3);
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      // w[k + q] and w[k + q + 1] with a uniform q in 0..3
      const uint32_t x0 = q == 0 ? w[k] : q == 1 ? w[k + 1] : q == 2 ? w[k + 2] : w[k + 3];
      const uint32_t x1 = q == 0 ? w[k + 1] : q == 1 ? w[k + 2] : q == 2 ? w[k + 3] : w[k + 4];
      o[k] = __funnelshift_r(x0, x1, sh);
    }
    if (dst) reinterpret_cast<uint4*>(dst)[j] = make_uint4(o[0], o[1], o[2], o[3]);
    if (rowsum) {
      const int nv = end - 16 * j;  // real bytes in this chunk (1..16)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int keep = min(max(nv - 4 * k, 0), 4);
        const uint32_t msk = keep == 4 ? 0xFFFFFFFFu : ((1u << (8 * keep)) - 1u);
        s = __dp4a((int)(o[k] & msk), 0x01010101, s);
      }
    }
  }
  if (rowsum) {
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
      int tot = 0;
      for (int i = 0; i < 8; ++i) tot += red[i];
      rowsum[m] = tot;
    }
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int get_encode() {
  if (g_encode) return QG_OK;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult qr;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qr) !=
          cudaSuccess ||
      qr != cudaDriverEntryPointSuccess || !fn)
    return QG_ERR_CUDA;
  g_encode = (PFN_cuTensorMapEncodeTiled_v12000)fn;
  return QG_OK;
}

// 2-D uint8 tensor [rows][cols] with row pitch `pitch` bytes, box {128, box_rows}.
int make_tmap(CUtensorMap* tm, const void* base, uint64_t cols, uint64_t rows, uint64_t pitch,
              uint32_t box_rows) {
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {pitch};
  cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? QG_OK : QG_ERR_CUDA;
}

}  // namespace

// Generic 2-D tensor map (any element type), used by the A8W4 tensor-core path.
int make_tmap_generic(CUtensorMap* tm, CUtensorMapDataType dt, const void* base, uint64_t inner,
                      uint64_t rows, uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_rows,
                      CUtensorMapSwizzle swz) {
  if (get_encode() != QG_OK) return QG_ERR_CUDA;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(tm, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? QG_OK : QG_ERR_CUDA;
}

namespace {

constexpr int kMaxDevices = 64;
int g_max_pairs[kMaxDevices];  // resident CTA pairs per device, set by i8gemm_setup

struct PackDims {
  int64_t Kp, Np;
};
PackDims pack_dims(int K, int N) { return {round_up(K, BK), round_up(N, BN)}; }

}  // namespace

size_t i8gemm_pack_b_bytes(int K, int N) {
  PackDims d = pack_dims(K, N);
  return (size_t)(d.Np * d.Kp + d.Np * 4);
}

static int pack_common(int K, int N, void* packed, cudaStream_t st, int32_t** colsum_out) {
  PackDims d = pack_dims(K, N);
  int32_t* colsum = (int32_t*)((int8_t*)packed + d.Np * d.Kp);
  if (cudaMemsetAsync(colsum, 0, (size_t)d.Np * 4, st) != cudaSuccess) return QG_ERR_CUDA;
  *colsum_out = colsum;
  return QG_OK;
}

int i8gemm_pack_b(int K, int N, const int8_t* B, int64_t ldb, void* packed, cudaStream_t st) {
  PackDims d = pack_dims(K, N);
  int32_t* colsum = nullptr;
  int rc = pack_common(K, N, packed, st, &colsum);
  if (rc != QG_OK) return rc;
  dim3 grid((unsigned)(d.Kp / 64), (unsigned)(d.Np / 64));
  pack_b_rowmajor_kernel<<<grid, dim3(32, 8), 0, st>>>(K, N, B, ldb, (int8_t*)packed, d.Kp, colsum);
  return launch_status();
}

int i8gemm_pack_b_kmajor(int K, int N, const int8_t* W, int64_t ldw, void* packed,
                         cudaStream_t st) {
  PackDims d = pack_dims(K, N);
  int32_t* colsum = nullptr;
  int rc = pack_common(K, N, packed, st, &colsum);
  if (rc != QG_OK) return rc;
  pack_b_kmajor_kernel<<<(unsigned)d.Np, 256, 0, st>>>(K, N, W, ldw, (int8_t*)packed, d.Kp, colsum);
  return launch_status();
}

static int64_t staged_lda(int K) { return round_up(K, 16); }

size_t i8gemm_packed_workspace_bytes(int M, int K) {
  return (size_t)(round_up((int64_t)M * staged_lda(K), 256) + round_up((int64_t)M * 4, 256));
}

int i8gemm_setup() {
  cudaError_t e = cudaFuncSetAttribute(i8gemm_tc_kernel<false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (e != cudaSuccess) return QG_ERR_CUDA;
  e = cudaFuncSetAttribute(i8gemm_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)SMEM_BYTES);
  if (e != cudaSuccess) return QG_ERR_CUDA;
  e = cudaFuncSetAttribute(i8gemm_tc2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)P_SMEM_BYTES);
  if (e != cudaSuccess) return QG_ERR_CUDA;
  // how many CTA pairs can be resident at once (SM pairs with a disabled
  // partner cannot host one)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QG_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = P_SMEM_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, i8gemm_tc2_kernel, &cfg) != cudaSuccess ||
      clusters < 1)
    return QG_ERR_CUDA;
  g_max_pairs[dev] = clusters;
  return get_encode();
}

static EpiArgs make_epi(int M, int N, int K, const void* packed_b, const qg_requant_t& rq,
                        const int32_t* rowsum, int8_t* C, int64_t ldc, int32_t* acc_out,
                        int64_t ld_acc) {
  const PackDims d = pack_dims(K, N);
  EpiArgs ep;
  ep.M = M; ep.N = N; ep.K = K;
  ep.za = rq.a_zero_point; ep.zb = rq.b_zero_point; ep.zo = rq.out_zero_point;
  ep.lo = rq.clamp_min; ep.hi = rq.clamp_max;
  ep.colsum = (const int32_t*)((const int8_t*)packed_b + d.Np * d.Kp);
  ep.rowsum = rowsum;
  ep.bias = rq.bias;
  ep.per_channel = rq.per_channel;
  ep.m0 = rq.multiplier0; ep.sh = rq.shift0;
  ep.m0v = rq.multiplier; ep.shv = rq.shift;
  ep.C = C; ep.ldc = ldc; ep.acc_out = acc_out; ep.ld_acc = ld_acc;
  ep.stall = 0;
  ep.spin = kSpinLimit;
  // One column tile: the MMA covers only the columns that exist, rounded up
  // to the instruction's step of 16 (the packed rows beyond N are zero).
  ep.nmma = N <= BN ? (int)round_up(N, 16) : BN;
  return ep;
}

// The one-CTA kernel as a programmatic dependent launch: its CTAs may become
// resident while the previous kernel in the stream is still running and
// wait for it on the device (griddepcontrol.wait in every role that touches
// global memory), so barrier setup, TMEM allocation and the tensor-map
// prefetch overlap the previous grid instead of following a launch gap.
template <bool CONV>
static int launch_one_cta(int grid, const CUtensorMap& tmA, const CUtensorMap& tmB, int num_kb,
                          int tiles_m, int tiles_n, const EpiArgs& ep, const ConvGather& cg,
                          cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(CONV ? THREADS_CONV : THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, i8gemm_tc_kernel<CONV>, tmA, tmB, num_kb, tiles_m,
                                           tiles_n, ep, cg, status_word());
  return e == cudaSuccess ? QG_OK : QG_ERR_CUDA;
}

int i8gemm_run_packed(int M, int N, int K, const int8_t* A, int64_t lda, const void* packed_b,
                      int8_t* C, int64_t ldc, const qg_requant_t& rq, int32_t* acc_out,
                      int64_t ld_acc, void* ws, size_t ws_bytes, cudaStream_t st) {
  const PackDims d = pack_dims(K, N);
  const bool need_copy = (((uintptr_t)A & 15) != 0) || (lda % 16) != 0;
  const bool need_rowsum = rq.b_zero_point != 0;
  const int8_t* Aeff = A;
  int64_t lda_eff = lda;
  int32_t* rowsum = nullptr;
  if (need_copy || need_rowsum) {
    if (!ws || ws_bytes < i8gemm_packed_workspace_bytes(M, K)) return QG_ERR_WORKSPACE;
    int8_t* Aw = (int8_t*)ws;
    rowsum = need_rowsum ? (int32_t*)((int8_t*)ws + round_up((int64_t)M * staged_lda(K), 256))
                         : nullptr;
    // programmatic dependent launch: scheduled while the previous kernel in
    // the stream may still run; it waits for it on the device
    cudaLaunchConfig_t scfg = {};
    scfg.gridDim = dim3((unsigned)M);
    scfg.blockDim = dim3(256);
    scfg.stream = st;
    cudaLaunchAttribute sattr[1];
    sattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    sattr[0].val.programmaticStreamSerializationAllowed = 1;
    scfg.attrs = sattr;
    scfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&scfg, stage_a_kernel, K, A, lda, need_copy ? Aw : (int8_t*)nullptr,
                           (int64_t)staged_lda(K), rowsum) != cudaSuccess)
      return QG_ERR_CUDA;
    if (need_copy) {
      Aeff = Aw;
      lda_eff = staged_lda(K);
    }
  }
  // CTA pairs (256 x 256 tiles, each CTA staging half of the B tile: box of
  // BM rows) for M > 256, or when 128 x 256 tiles of one CTA would take more
  // than one wave; otherwise the one-CTA kernel (fewer, lighter launches on a
  // small problem: 130x70x129 12.7 -> 12.0 us), which copies the ep.nmma rows
  // its MMAs read.
  const bool pair_path =
      M > BM && (M > 2 * BM || cdiv(M, BM) * cdiv(N, BN) > (int64_t)num_sms());
  EpiArgs ep = make_epi(M, N, K, packed_b, rq, rowsum, C, ldc, acc_out, ld_acc);
  CUtensorMap tmA, tmB;
  int rc = make_tmap(&tmA, Aeff, (uint64_t)K, (uint64_t)M, (uint64_t)lda_eff, BM);
  if (rc != QG_OK) return rc;
  rc = make_tmap(&tmB, packed_b, (uint64_t)d.Kp, (uint64_t)d.Np, (uint64_t)d.Kp,
                 pair_path ? BM : ep.nmma);
  if (rc != QG_OK) return rc;
  const int num_kb = (int)(d.Kp / BK);
  ep.stall = (!pair_path && num_kb > 1 && take_stall(kStallInt8Gemm)) ? 1 : 0;
  ep.spin = ep.stall ? kStallSpinLimit : kSpinLimit;
  if (pair_path) {
    // 2-CTA pairs on 256 x 256 tiles, one resident pair per SM pair
    const int tiles_m = (int)cdiv(M, 256), tiles_n = (int)cdiv(N, BN);
    const int tiles = tiles_m * tiles_n;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QG_ERR_CUDA;
    int pairs = g_max_pairs[dev] > 0 ? g_max_pairs[dev] : num_sms() / 2;
    if (pairs > tiles) pairs = tiles;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * pairs));
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = P_SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // after this call's staging pass: programmatic dependent launch.  Before
    // its grid-dependency wait the kernel reads only the packed B; the rows
    // of A, the row sums and C wait for the staging grid, which itself waits
    // for the work before it in the stream.
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = (need_copy || need_rowsum) ? 2 : 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, i8gemm_tc2_kernel, tmA, tmB, num_kb, tiles_m, tiles_n,
                                       ep, status_word());
    return e == cudaSuccess ? QG_OK : QG_ERR_CUDA;
  }
  const int tiles_m = (int)cdiv(M, BM), tiles_n = (int)cdiv(N, BN);
  const int tiles = tiles_m * tiles_n;
  const int grid = tiles < num_sms() ? tiles : num_sms();
  return launch_one_cta<false>(grid, tmA, tmB, num_kb, tiles_m, tiles_n, ep, ConvGather{}, st);
}

// ---------------------------------------------------------------------------
// INT8 convolution: the weights [Cout][KH][KW][Cin] are K-major already and
// are packed like B (padded, column sums); the one-CTA tensor-core kernel
// gathers the im2col rows itself (implicit GEMM), so a call is one launch
// with packed weights, two with raw ones (pack, then the GEMM).
// ---------------------------------------------------------------------------
static void conv_geometry(int H, int W, int KH, int KW, int sh, int sw, int ph, int pw, int* OH,
                          int* OW) {
  *OH = (H + 2 * ph - KH) / sh + 1;
  *OW = (W + 2 * pw - KW) / sw + 1;
}

size_t conv_pack_w_bytes(int Cout, int K) { return i8gemm_pack_b_bytes(K, Cout); }

int conv_pack_w(int Cout, int K, const int8_t* w, void* packed, cudaStream_t st) {
  return i8gemm_pack_b_kmajor(K, Cout, w, K, packed, st);
}

size_t conv_workspace_bytes(int Nb, int H, int W, int Cin, int Cout, int KH, int KW, int sh,
                            int sw, int ph, int pw) {
  (void)Nb; (void)H; (void)W; (void)sh; (void)sw; (void)ph; (void)pw;
  return (size_t)round_up((int64_t)i8gemm_pack_b_bytes(KH * KW * Cin, Cout), 256);
}

int conv_run_packed(int Nb, int H, int W, int Cin, int Cout, int KH, int KW, int sh, int sw,
                    int ph, int pw, const int8_t* x, const void* packed_w, int8_t* y,
                    const qg_requant_t& rq, int32_t* acc_out, cudaStream_t st) {
  int OH, OW;
  conv_geometry(H, W, KH, KW, sh, sw, ph, pw, &OH, &OW);
  const int K = KH * KW * Cin;
  const int64_t M = (int64_t)Nb * OH * OW;
  if (M > INT32_MAX) return QG_ERR_UNSUPPORTED;
  const PackDims d = pack_dims(K, Cout);
  EpiArgs ep = make_epi((int)M, Cout, K, packed_w, rq, nullptr, y, Cout, acc_out, Cout);
  CUtensorMap tmB;
  int rc = make_tmap(&tmB, packed_w, (uint64_t)d.Kp, (uint64_t)d.Np, (uint64_t)d.Kp, ep.nmma);
  if (rc != QG_OK) return rc;
  ConvGather cg;
  cg.x = x;
  cg.H = H; cg.W = W; cg.Cin = Cin; cg.KH = KH; cg.KW = KW;
  cg.sh = sh; cg.sw = sw; cg.ph = ph; cg.pw = pw; cg.OH = OH; cg.OW = OW;
  cg.M = (int)M; cg.K = K;
  cg.za = rq.a_zero_point;
  cg.vec16 = (Cin % 16 == 0) && (((uintptr_t)x & 15) == 0);
  const int num_kb = (int)(d.Kp / BK);
  const int tiles_m = (int)cdiv(M, BM), tiles_n = (int)cdiv(Cout, BN);
  const int tiles = tiles_m * tiles_n;
  const int grid = tiles < num_sms() ? tiles : num_sms();
  return launch_one_cta<true>(grid, tmB, tmB, num_kb, tiles_m, tiles_n, ep, cg, st);
}

int conv_run(int Nb, int H, int W, int Cin, int Cout, int KH, int KW, int sh, int sw, int ph,
             int pw, const int8_t* x, const int8_t* w, int8_t* y, const qg_requant_t& rq,
             int32_t* acc_out, void* ws, size_t ws_bytes, cudaStream_t st) {
  const int K = KH * KW * Cin;
  if (!ws || ws_bytes < conv_workspace_bytes(Nb, H, W, Cin, Cout, KH, KW, sh, sw, ph, pw))
    return QG_ERR_WORKSPACE;
  int rc = conv_pack_w(Cout, K, w, ws, st);
  if (rc != QG_OK) return rc;
  return conv_run_packed(Nb, H, W, Cin, Cout, KH, KW, sh, sw, ph, pw, x, ws, y, rq, acc_out, st);
}

}  // namespace qg
