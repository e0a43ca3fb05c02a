// A8W4 linear for M > 1 on the 5th-generation tensor cores.
//
// Source: pytorch/ao PR #997 "Kleidi 4b blockwise gemv prototype"
// (matmul_clamp_f32_qai8dxp_qsi4c32p: int8 dynamic per-row asymmetric
// activations, int4 symmetric weights with one f32 scale per 32-wide K group,
// f32 output clamped after the bias; m > 1 tests).
//
//   y[m,n] = clamp(sA[m] * sum_g sw[n,g] * I[m,n,g] + bias[n])
//   I[m,n,g] = sum_{k in g} (qA[m,k] - zA[m]) * w[n,k]
//
// Exactness: qA - zA lies in [-255,255] and w in [-8,7], both exact in bf16,
// and every partial sum of one group is an integer below 2^24, so one
// kind::f16 MMA pair (K = 2 x 16) per group leaves the exact I[m,n,g] in an
// f32 TMEM accumulator.  Only the combination over groups is rounded (f32).
//
// Roles (448 threads, one CTA per SM, tile 128 x 128 over a K range):
//   warp 0      TMA: the CTA's nibble slice once, then (after waiting for the
//               quantization grid) bf16 A' stages (128 rows x 64 K, 128B
//               swizzle)
//   warp 1      TMEM allocation; MMA issue, one 128-column TMEM buffer per
//               group, 4 buffers
//   warps 2..5  expand nibbles into the swizzled bf16 B' stage
//   warps 6..13 per group: tcgen05.ld the exact group dots, release the
//               buffer, acc += sw * I with packed fma.rn.f32x2; then the
//               split-K partial, and the last CTA of a tile reduces the
//               partials in split order (deterministic) and writes y.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include "qg_internal.cuh"

namespace qg {

int make_tmap_generic(CUtensorMap* tm, CUtensorMapDataType dt, const void* base, uint64_t inner,
                      uint64_t rows, uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_rows,
                      CUtensorMapSwizzle swz);

namespace {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int KS = 64;              // K (bf16 elements) per stage = one 128B swizzle row
constexpr int STAGES = 4;
constexpr int NBUF = 4;             // TMEM group buffers of BN columns
constexpr int KR_MAX = 1024;        // K range per CTA
constexpr int GR_MAX = KR_MAX / 32;
constexpr int A_STAGE = BM * KS * 2;   // 16 KiB
constexpr int B_STAGE = BN * KS * 2;   // 16 KiB
constexpr int THREADS = 22 * 32;     // TMA, MMA, 4 converter, 16 epilogue warps
constexpr int CONV_THREADS = 4 * 32;
constexpr int EPI_WARP0 = 6;
constexpr int EPI_THREADS = 16 * 32;
constexpr int PST = BN + 4;          // row stride (floats) of the split-K partial in smem
constexpr size_t SMEM_BYTES = 1024 + STAGES * (A_STAGE + B_STAGE) + (size_t)BN * KR_MAX / 2 +
                              (size_t)BN * GR_MAX * 4 + 512;

// kind::f16 instruction descriptor: D f32, A bf16, B bf16, both K-major, N = BN, M = BM.
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                           ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
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
__device__ __forceinline__ void ffma2(unsigned long long& acc, unsigned long long a,
                                      unsigned long long b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}
__device__ __forceinline__ unsigned long long pack2(uint32_t lo, uint32_t hi) {
  return ((unsigned long long)hi << 32) | lo;
}
__device__ __forceinline__ void epi_sync(int id) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "n"(EPI_THREADS) : "memory");
}
__device__ __forceinline__ bool epi_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 3, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(EPI_THREADS)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
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

struct Args {
  int M, N, K, Kr, splits, n_tiles;
  const void* wscale;   // packed group scales [N][K/32], f32 or bf16
  int scale_bf16;
  const float* sA;
  const float* bias;
  float lo, hi;
  float* y;
  int64_t ldy;
};

__global__ void __launch_bounds__(THREADS, 1)
    a8w4_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW,
                   Args a, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_STAGE;
  uint8_t* sN = sB + STAGES * B_STAGE;                         // [BN][Kr/2] nibbles of this CTA
  float* scl_t = (float*)(sN + (size_t)BN * KR_MAX / 2);      // [Gr][BN] group scales
  uint64_t* ld_full = (uint64_t*)(scl_t + BN * GR_MAX);
  uint64_t* cv_full = ld_full + STAGES;
  uint64_t* empty = cv_full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + NBUF;
  uint64_t* nib_full = tempty + NBUF;
  uint32_t* tmem_slot = (uint32_t*)(nib_full + 1);
  float* part = reinterpret_cast<float*>(smem);  // [BM][PST], reuses the A' stages after the mainloop

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = a.splits > 1 ? (int)cluster_rank() : 0;
  const int tile = blockIdx.x / a.splits;
  const int tn = tile % a.n_tiles, tm = tile / a.n_tiles;
  const int m0 = tm * BM, n0 = tn * BN;
  const int k0 = split * a.Kr;
  const int Gr = a.Kr / 32;
  const int nstages = a.Kr / KS;
  // The N tiles of one split all read the same A' K range; each tile walks its
  // stages in a rotated order so concurrent CTAs fetch different A' tiles
  // instead of hammering the same L2 lines.  Stage position s holds K block
  // kb(s) = (s + rot) % nstages (every group's dot is exact, only the f32
  // combination order depends on it, and it is fixed per tile).
  const int rot = (tn * 7) % nstages;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ld_full[s], 1);
      mbar_init(&cv_full[s], CONV_THREADS / 32);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < NBUF; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], EPI_THREADS / 32);
    }
    mbar_init(nib_full, 1);
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmW);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(NBUF * BN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------- TMA producer -------------------------
    if (lane == 0) {
      // this CTA's whole nibble slice (BN rows x Kr/2 bytes) in one box
      mbar_arrive_expect_tx(nib_full, (uint32_t)(BN * a.Kr / 2));
      tma_load_2d(sN, &tmW, k0 / 8, n0, nib_full);
      // The activation codes come from the quantization grid just before
      // this one (programmatic dependent launch): wait for it from here on.
      asm volatile("griddepcontrol.wait;" ::: "memory");
      for (int s = 0; s < nstages; ++s) {
        const int slot = s % STAGES;
        if (s >= STAGES && !mbar_poll(&empty[slot], ((s / STAGES) - 1) & 1, status)) break;
        const int kb = (s + rot) % nstages;
        mbar_arrive_expect_tx(&ld_full[slot], (uint32_t)A_STAGE);
        tma_load_2d(sA + slot * A_STAGE, &tmA, k0 + KS * kb, m0, &ld_full[slot]);
      }
    }
  } else if (warp == 1) {
    // ------------------------- MMA issuer -------------------------
    if (lane == 0) {
      bool ok = true;
      for (int s = 0; s < nstages && ok; ++s) {
        const int slot = s % STAGES;
        const uint32_t par = (uint32_t)(s / STAGES) & 1;
        if (!mbar_poll(&ld_full[slot], par, status) || !mbar_poll(&cv_full[slot], par, status)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + slot * A_STAGE);
        const uint32_t b0 = smem_u32(sB + slot * B_STAGE);
#pragma unroll
        for (int gi = 0; gi < 2; ++gi) {
          const int g = 2 * s + gi;
          const int buf = g % NBUF;
          const uint32_t use = (uint32_t)(g / NBUF);
          if (!mbar_poll(&tempty[buf], (use & 1) ^ 1, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem_base + (uint32_t)(buf * BN);
          mma_bf16(d, sdesc_sw128(a0 + 64 * gi), sdesc_sw128(b0 + 64 * gi), 0);
          mma_bf16(d, sdesc_sw128(a0 + 64 * gi + 32), sdesc_sw128(b0 + 64 * gi + 32), 1);
          mma_commit(&tfull[buf]);
        }
        mma_commit(&empty[slot]);
      }
    }
  } else if (warp < EPI_WARP0) {
    // ------------------------- nibble -> bf16 converters -------------------------
    // Stage s, row r takes nibble words 8s..8s+7 of row r's slice; word c becomes
    // the 16-byte chunk c of the row in the 128B-swizzled bf16 tile.
    const int ctid = threadIdx.x - 64;  // 0..127
    const int wpr = a.Kr / 8;           // nibble words per row
    const uint32_t* nib = (const uint32_t*)sN;
    bool ok = mbar_wait(nib_full, 0, status);
    for (int s = 0; s < nstages && ok; ++s) {
      const int slot = s % STAGES;
      if (s >= STAGES && !mbar_wait(&empty[slot], ((s / STAGES) - 1) & 1, status)) break;
      uint8_t* dst = sB + slot * B_STAGE;
      const int kb = (s + rot) % nstages;
      uint32_t w[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int idx = ctid + u * CONV_THREADS;  // 0..1023 = row * 8 + word
        w[u] = nib[(idx >> 3) * wpr + 8 * kb + (idx & 7)];
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int idx = ctid + u * CONV_THREADS;
        const int r = idx >> 3, c = idx & 7;
        const uint32_t L = w[u] & 0x0F0F0F0Fu, H = (w[u] >> 4) & 0x0F0F0F0Fu;
        uint4 o;
        o.x = bf16x2_minus136(prmt(L, 0x43434343u, 0x5140u));
        o.y = bf16x2_minus136(prmt(L, 0x43434343u, 0x5342u));
        o.z = bf16x2_minus136(prmt(H, 0x43434343u, 0x5140u));
        o.w = bf16x2_minus136(prmt(H, 0x43434343u, 0x5342u));
        *reinterpret_cast<uint4*>(dst + r * 128 + ((c ^ (r & 7)) << 4)) = o;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&cv_full[slot]);
    }
  } else {
    // ------------------------- epilogue -------------------------
    const int etid = threadIdx.x - EPI_WARP0 * 32;  // 0..511
    const int q = warp & 3;                         // TMEM lane quarter
    const int cb = (warp - EPI_WARP0) >> 2;         // 32-column block
    const int row = 32 * q + lane;
    const int m = m0 + row;
    bool ok = true;
    {
      // group scales of this tile, transposed to [g][n] (rows past N read as 0)
      const int G = a.K / 32, g0 = k0 / 32;
      for (int i = etid; i < BN * Gr; i += EPI_THREADS) {
        const int n = i / Gr, g = i - n * Gr;
        const int64_t idx = (int64_t)(n0 + n) * G + g0 + g;
        float v = 0.0f;
        if (n0 + n < a.N)  // a bf16 scale widens to f32 exactly
          v = a.scale_bf16
                  ? __uint_as_float((uint32_t)__ldg(reinterpret_cast<const unsigned short*>(a.wscale) + idx) << 16)
                  : __ldg(reinterpret_cast<const float*>(a.wscale) + idx);
        scl_t[g * BN + n] = v;
      }
    }
    epi_sync(1);
    // sA (read after the mainloop) comes from the quantization grid
    asm volatile("griddepcontrol.wait;" ::: "memory");
    unsigned long long acc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] = 0ull;
    for (int g = 0; g < Gr && ok; ++g) {
      const int buf = g % NBUF;
      const uint32_t use = (uint32_t)(g / NBUF);
      ok = mbar_wait(&tfull[buf], use & 1, status);
      tc_fence_after();
      uint32_t p[32];
      tmem_ld32(tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * BN + 32 * cb), p);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
      const int gg = 2 * (((g >> 1) + rot) % nstages) + (g & 1);  // K group held by buffer
      const float4* sc = reinterpret_cast<const float4*>(scl_t + gg * BN + 32 * cb);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 s4 = sc[j];
        ffma2(acc[2 * j], pack2(p[4 * j], p[4 * j + 1]),
              pack2(__float_as_uint(s4.x), __float_as_uint(s4.y)));
        ffma2(acc[2 * j + 1], pack2(p[4 * j + 2], p[4 * j + 3]),
              pack2(__float_as_uint(s4.z), __float_as_uint(s4.w)));
      }
    }
    ok = epi_and(ok);
    float v[32];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      v[2 * j] = __uint_as_float((uint32_t)(acc[j] & 0xFFFFFFFFull));
      v[2 * j + 1] = __uint_as_float((uint32_t)(acc[j] >> 32));
    }
    const int nb = n0 + 32 * cb;
    if (a.splits == 1) {
      // N % 4 == 0 on this path: every float4 chunk is fully in or out of range
      if (ok && m < a.M) {
        const float s = a.sA[m];
        float* yr = a.y + (int64_t)m * a.ldy;
        const bool vec = ((a.ldy & 3) == 0) && ((reinterpret_cast<uintptr_t>(a.y) & 15) == 0);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int n = nb + 4 * c;
          if (n < a.N) {
            float t[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              t[e] = __fmul_rn(s, v[4 * c + e]);
              if (a.bias) t[e] = __fadd_rn(t[e], a.bias[n + e]);
              t[e] = fminf(fmaxf(t[e], a.lo), a.hi);
            }
            if (vec) {
              *reinterpret_cast<float4*>(yr + n) = make_float4(t[0], t[1], t[2], t[3]);
            } else {
#pragma unroll
              for (int e = 0; e < 4; ++e) yr[n + e] = t[e];
            }
          }
        }
      }
    } else {
      // park this split's partial tile in shared memory for the cluster reduction
      float4* dst = reinterpret_cast<float4*>(part + row * PST + 32 * cb);
#pragma unroll
      for (int c = 0; c < 8; ++c)
        dst[c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
    }
  }

  __syncwarp();
  if (a.splits > 1) {
    // Split-K reduction over the cluster (one CTA per K range): after the
    // first cluster barrier every partial is visible; CTA `split` sums its
    // share of the rows over all ranks in rank order (deterministic) and
    // writes y; the second barrier keeps every CTA's shared memory alive
    // until its peers have read it.
    cluster_sync_all();
    if (warp >= EPI_WARP0) {
      const int etid = threadIdx.x - EPI_WARP0 * 32;
      const int rows_per = BM / a.splits;
      const uint32_t part_s = smem_u32(part);
      for (int i = etid; i < rows_per * (BN / 4); i += EPI_THREADS) {
        const int r = split * rows_per + i / (BN / 4);
        const int c = i % (BN / 4);
        const int m = m0 + r, n = n0 + 4 * c;
        const uint32_t off = (uint32_t)((r * PST + 4 * c) * 4);
        float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < a.splits; ++j) {
          const float4 t = ld_dsmem_f4(mapa(part_s + off, (uint32_t)j));
          sum.x = __fadd_rn(sum.x, t.x);
          sum.y = __fadd_rn(sum.y, t.y);
          sum.z = __fadd_rn(sum.z, t.z);
          sum.w = __fadd_rn(sum.w, t.w);
        }
        if (m < a.M && n < a.N) {
          const float s = a.sA[m];
          float t4[4] = {sum.x, sum.y, sum.z, sum.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            t4[e] = __fmul_rn(s, t4[e]);
            if (a.bias) t4[e] = __fadd_rn(t4[e], a.bias[n + e]);
            t4[e] = fminf(fmaxf(t4[e], a.lo), a.hi);
          }
          float* yr = a.y + (int64_t)m * a.ldy + n;
          if (((a.ldy & 3) == 0) && ((reinterpret_cast<uintptr_t>(a.y) & 15) == 0)) {
            *reinterpret_cast<float4*>(yr) = make_float4(t4[0], t4[1], t4[2], t4[3]);
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) yr[e] = t4[e];
          }
        }
      }
    }
    __syncwarp();
    cluster_sync_all();
  }

  // Reconverge every warp (lane 0 of the TMA and MMA warps ran their loops
  // alone) so the CTA barrier below counts complete warps only after all
  // of their work, in particular before TMEM is freed.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(NBUF * BN)
                 : "memory");
  }
}

// Per-row quantization into bf16 (q - zp) for the tensor-core operand, plus
// the scale/zero-point and (optionally) the int8 codes.
__global__ void __launch_bounds__(256) quantize_rows_centered_kernel(
    int K, const float* __restrict__ x, int64_t ldx, uint16_t* __restrict__ qc,
    int8_t* __restrict__ q_opt, float* __restrict__ scale, int32_t* __restrict__ zero_point) {
  __shared__ float red[16];
  const int64_t m = blockIdx.x;
  // let the GEMM grid start its prologue (it waits before reading our outputs)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const float* xr = x + m * ldx;
  float mn = 0.0f, mx = 0.0f;
  int k = threadIdx.x;
  for (; k + 7 * 256 < K; k += 8 * 256) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = xr[k + u * 256];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      mn = fminf(mn, v[u]);
      mx = fmaxf(mx, v[u]);
    }
  }
  for (; k < K; k += 256) {
    mn = fminf(mn, xr[k]);
    mx = fmaxf(mx, xr[k]);
  }
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if ((threadIdx.x & 31) == 0) {
    red[threadIdx.x >> 5] = mn;
    red[8 + (threadIdx.x >> 5)] = mx;
  }
  __syncthreads();
  mn = red[0];
  mx = red[8];
  for (int i = 1; i < 8; ++i) {
    mn = fminf(mn, red[i]);
    mx = fmaxf(mx, red[8 + i]);
  }
  // scale = (rmax - rmin)/255 (1 if 0), inv = 1/scale, zp = clamp(rne(-128 - rmin*inv))
  float sc = __fdiv_rn(__fsub_rn(mx, mn), 255.0f);
  if (sc == 0.0f) sc = 1.0f;
  const float inv = __fdiv_rn(1.0f, sc);
  const int zp = min(max(__float2int_rn(__fsub_rn(-128.0f, __fmul_rn(mn, inv))), -128), 127);
  uint16_t* qr = qc + m * K;
  // (v - zp) in [-255, 255] is exact in bf16: built through f32 (exact), then truncated
  k = threadIdx.x;
  for (; k + 7 * 256 < K; k += 8 * 256) {
    float xv[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) xv[u] = xr[k + u * 256];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int v = min(max(__float2int_rn(__fmul_rn(xv[u], inv)) + zp, -128), 127);
      qr[k + u * 256] = (uint16_t)(__float_as_uint((float)(v - zp)) >> 16);
      if (q_opt) q_opt[m * K + k + u * 256] = (int8_t)v;
    }
  }
  for (; k < K; k += 256) {
    const int v = min(max(__float2int_rn(__fmul_rn(xr[k], inv)) + zp, -128), 127);
    qr[k] = (uint16_t)(__float_as_uint((float)(v - zp)) >> 16);
    if (q_opt) q_opt[m * K + k] = (int8_t)v;
  }
  if (threadIdx.x == 0) {
    scale[m] = sc;
    zero_point[m] = zp;
  }
}

}  // namespace

size_t a8w4_tc_workspace_bytes(int M, int N, int K, int splits) {
  (void)N;
  (void)splits;
  return (size_t)(round_up((int64_t)M * K * 2, 256) + 2 * round_up((int64_t)M * 4, 256));
}

// Split count s in {1, 2, 4, 8} (one cluster of s CTAs per output tile, K
// range K/s a multiple of 128 and <= 1024): the largest with tiles*s no more
// than the SM count, at least the smallest valid one.
int a8w4_tc_splits(int M, int N, int K, int sms) {
  const int64_t tiles = cdiv(M, BM) * cdiv(N, BN);
  int best = -1;
  for (int s = 1; s <= 8; s *= 2) {
    if (K % s) continue;
    const int kr = K / s;
    if (kr % 128 || kr > KR_MAX) continue;  // scale tile rows must be 16-byte multiples
    if (best < 0) best = s;
    if (tiles * s <= sms) best = s;
  }
  return best;
}

bool a8w4_tc_supported(int M, int N, int K) {
  return K % 128 == 0 && N % 4 == 0 && a8w4_tc_splits(M, N, K, 1 << 30) > 0;
}

int a8w4_tc_setup() {
  cudaError_t e = cudaFuncSetAttribute(a8w4_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SMEM_BYTES);
  return e == cudaSuccess ? QG_OK : QG_ERR_CUDA;
}

int launch_a8w4_tc(int M, int N, int K, const float* x, int64_t ldx, const void* packed,
                   const float* bias, float lo, float hi, float* y, int64_t ldy, int8_t* q_out,
                   float* scale_out, int32_t* zp_out, void* ws, size_t ws_bytes, bool scale_bf16,
                   cudaStream_t st) {
  const int splits = a8w4_tc_splits(M, N, K, num_sms());
  if (splits <= 0) return QG_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < a8w4_tc_workspace_bytes(M, N, K, splits)) return QG_ERR_WORKSPACE;
  const int64_t mt = cdiv(M, BM), nt = cdiv(N, BN);
  uint8_t* w = (uint8_t*)ws;
  uint16_t* qc = (uint16_t*)w;
  w += round_up((int64_t)M * K * 2, 256);
  float* sA = (float*)w;
  w += round_up((int64_t)M * 4, 256);
  int32_t* zA = (int32_t*)w;
  quantize_rows_centered_kernel<<<M, 256, 0, st>>>(K, x, ldx, qc, q_out, sA, zA);
  int rc = launch_status();
  if (rc != QG_OK) return rc;
  if (scale_out && cudaMemcpyAsync(scale_out, sA, (size_t)M * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return QG_ERR_CUDA;
  if (zp_out && cudaMemcpyAsync(zp_out, zA, (size_t)M * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return QG_ERR_CUDA;
  const uint8_t* wq = (const uint8_t*)packed;
  const void* wsc = wq + (size_t)N * (K / 2);
  const int Kr = K / splits;
  CUtensorMap tmA, tmW;
  rc = make_tmap_generic(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, qc, (uint64_t)K, (uint64_t)M,
                         (uint64_t)K * 2, KS, BM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != QG_OK) return rc;
  rc = make_tmap_generic(&tmW, CU_TENSOR_MAP_DATA_TYPE_UINT32, wq, (uint64_t)K / 8, (uint64_t)N,
                         (uint64_t)K / 2, (uint32_t)(Kr / 8), BN, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (rc != QG_OK) return rc;
  Args a;
  a.M = M; a.N = N; a.K = K; a.Kr = Kr; a.splits = splits; a.n_tiles = (int)nt;
  a.wscale = wsc;
  a.scale_bf16 = scale_bf16 ? 1 : 0;
  a.sA = sA; a.bias = bias; a.lo = lo; a.hi = hi; a.y = y; a.ldy = ldy;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(mt * nt * splits));
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)splits;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // programmatic dependent launch: the prologue (barriers, TMEM, the weight
  // nibbles and scales) overlaps the quantization grid
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, a8w4_tc_kernel, tmA, tmW, a, status_word());
  return e == cudaSuccess ? QG_OK : QG_ERR_CUDA;
}

}  // namespace qg
