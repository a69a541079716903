// W8A16 group-wise weight-only GEMM for decode batches (M <= 64), after
// "DeepSeek-R1-0528-Qwen3-8B量化版发布" (technical details: symmetric group-wise INT8 Linear
// weights, FP16 activations), group size 128 along K:
//     y[m][n] = fp16( sum_g s[n][g] * sum_{k in g} x[m][k] * wq[n][k] ).
//
// The kernel streams the int8 weights once from HBM (the bound) and never rounds a dequantized
// weight: int8 -> f16 is exact (|q| <= 127), the tensor core forms exact f16 x f16 products with
// fp32 accumulation, and the fp16 group scale multiplies each group's fp32 partial sum.
//
// Layout: "swap-AB" - the 128 weight rows of a tile are the MMA's M dimension, the (padded) tokens
// its N dimension, so a decode batch of 1..64 tokens still fills the 128-row tensor-core tile.
//   warp 0       TMA: int8 weight slab [128 rows x 128 K] (128B swizzle) + f16 activation slab
//                [MP x 128 K] as two 64-element halves (128B swizzle), one mbarrier per stage.
//   warp 1       TMEM allocation and MMA issue: 8 x tcgen05.mma.kind::f16 (K = 16) per slab.
//   warps 4..11  converters: int8 slab -> f16 operand in shared memory (128B swizzle layout the
//                MMA descriptor expects; NA operand buffers), then fence.proxy.async and an
//                mbarrier arrival.
//   warps 12..15 epilogue: thread = weight row; per slab, sum[m] += partial[m] * s[n][g].
// Small-N MMAs have a long latency compared with their work, so consecutive MMAs never wait on
// each other: each slab's 8 k-steps alternate between NACC independent TMEM accumulators (summed
// by the epilogue), and up to NBUF slabs are in flight in a ring of TMEM accumulators.
// Split-K: the CTAs of one thread-block cluster take disjoint slab ranges of the same 128 rows;
// rank 0 adds the other ranks' fp32 partial tiles read from their shared memory (distributed
// shared memory), in rank order, and writes fp16.
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"

namespace i8q {

constexpr int W8A16_MAX_M = 64;
constexpr int W8A16_BN = 128;   // weight rows per tile (MMA M)

template <int MP>
struct W8A16Cfg {
  static constexpr int W_BYTES = W8A16_BN * 128;        // int8 slab
  static constexpr int X_HALF = MP * 128;               // one 64-element half of the f16 slab
  static constexpr int X_BYTES = 2 * X_HALF;
  static constexpr int STAGE_BYTES = W_BYTES + X_BYTES;
  static constexpr int STAGES = MP >= 32 ? 4 : 6;
  static constexpr int A_BYTES = W8A16_BN * 128 * 2;    // f16 operand of one slab: two 16 KB halves
  static constexpr int NA = 3;                          // operand buffers
  static constexpr int NACC = 2;                        // independent accumulators per slab
  static constexpr int NBUF = (512 / (NACC * MP)) < 8 ? (512 / (NACC * MP)) : 8;   // slab accumulators in TMEM
  static constexpr int TMEM_NEED = NBUF * NACC * MP;
  static constexpr int TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64 : TMEM_NEED <= 128 ? 128
                                   : TMEM_NEED <= 256 ? 256 : 512;
  static constexpr int NUM_THREADS = 512;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + NA * A_BYTES + 512 + 1024;
  static_assert(MP * W8A16_BN * 4 <= NA * A_BYTES, "reduction tile must fit in the operand buffers");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

struct W8A16Args {
  const uint16_t* s;   // [N][K/128] fp16 group scales
  int M, N, K;
  uint16_t* y;         // [M][N] fp16
};

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_dsmem_f32(uint32_t local_addr, uint32_t rank) {
  uint32_t remote;
  float v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 4 signed int8 (one 32-bit word) -> 4 exact f16 values as two half2 words.
// Byte u = q + 128 is placed in the mantissa of 1024 (f16 0x6400); subtracting 1152 = 1024 + 128
// leaves q exactly.
__device__ __forceinline__ void i8x4_to_f16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t u = w ^ 0x80808080u;
  const uint32_t a = __byte_perm(u, 0x64646464u, 0x4140);
  const uint32_t b = __byte_perm(u, 0x64646464u, 0x4342);
  const __half2 bias = __half2half2(__ushort_as_half((unsigned short)0x6480));  // 1152
  __half2 ha = __hsub2(*reinterpret_cast<const __half2*>(&a), bias);
  __half2 hb = __hsub2(*reinterpret_cast<const __half2*>(&b), bias);
  lo = *reinterpret_cast<uint32_t*>(&ha);
  hi = *reinterpret_cast<uint32_t*>(&hb);
}

template <int MP>
__global__ void __launch_bounds__(512, 1)
    k_gemm_w8a16(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                 const W8A16Args args) {
  using C = W8A16Cfg<MP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sStage = smem;                                   // STAGES x (W slab | X halves)
  uint8_t* sA = smem + C::STAGES * C::STAGE_BYTES;          // NA x f16 operand (2 x 16 KB halves each)
  uint64_t* full = reinterpret_cast<uint64_t*>(sA + C::NA * C::A_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* afull = empty + C::STAGES;
  uint64_t* aempty = afull + C::NA;
  uint64_t* tfull = aempty + C::NA;
  uint64_t* tempty = tfull + C::NBUF;
  uint64_t* done = tempty + C::NBUF;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = args.N, K = args.K;
  const int KB = K / 128;
  const uint32_t rank = cluster_ctarank(), nrank = cluster_nctarank();
  const int kb0 = (int)((int64_t)KB * rank / nrank), kb1 = (int)((int64_t)KB * (rank + 1) / nrank);
  const int nslab = kb1 - kb0;
  const int n0 = blockIdx.x * W8A16_BN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 9);   // 8 converter warps + 1 MMA commit
    }
    for (int a = 0; a < C::NA; ++a) {
      mbar_init(&afull[a], 8);
      mbar_init(&aempty[a], 1);
    }
    for (int b = 0; b < C::NBUF; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  float sum[MP];
#pragma unroll
  for (int m = 0; m < MP; ++m) sum[m] = 0.f;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t filled = 0, fill_parity = 0;
      bool ok = true;
      for (int j = 0; j < nslab; ++j) {
        const int s = j % C::STAGES;
        const uint32_t ph = (j / C::STAGES) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, SITE_EMPTY, abort_flag)) { ok = false; break; }
        uint8_t* st = sStage + s * C::STAGE_BYTES;
        mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
        const int kk = (kb0 + j) * 128;
        tma_load_2d(st, &tmW, &full[s], kk, n0);
        tma_load_2d(st + C::W_BYTES, &tmX, &full[s], kk, 0);
        tma_load_2d(st + C::W_BYTES + C::X_HALF, &tmX, &full[s], kk + 64, 0);
        filled |= 1u << s;
        fill_parity = (fill_parity & ~(1u << s)) | (ph << s);
      }
      if (!ok)
        for (int s = 0; s < C::STAGES; ++s)
          if (filled & (1u << s)) mbar_wait(&full[s], (fill_parity >> s) & 1u, SITE_DRAIN, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(W8A16_BN, MP);
      for (int j = 0; j < nslab; ++j) {
        const int s = j % C::STAGES;
        const uint32_t ph = (j / C::STAGES) & 1;
        const int a = j % C::NA;
        const uint32_t pa = (j / C::NA) & 1;
        const int b = j % C::NBUF;
        const uint32_t pb = (j / C::NBUF) & 1;
        if (!mbar_wait(&tempty[b], pb ^ 1, SITE_TMEM_EMPTY, abort_flag)) break;
        if (!mbar_wait(&afull[a], pa, SITE_CONVERT, abort_flag)) break;
        if (!mbar_wait(&full[s], ph, SITE_FULL, abort_flag)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + a * C::A_BYTES);
        const uint32_t x0 = smem_u32(sStage + s * C::STAGE_BYTES + C::W_BYTES);
        const uint32_t d0 = tmem + b * C::NACC * MP;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t h = kk >> 2, off = (kk & 3) * 32;
          mma_f16(d0 + (kk % C::NACC) * MP, sw128_kmajor_desc(a0 + h * 16384 + off),
                  sw128_kmajor_desc(x0 + h * C::X_HALF + off), idesc, kk >= C::NACC);
        }
        tc_commit(&empty[s]);
        tc_commit(&aempty[a]);
        tc_commit(&tfull[b]);
      }
      tc_commit(done);
      mbar_wait(done, 0, SITE_DRAIN, nullptr);
    }
  } else if (warp >= 4 && warp < 12) {
    // converters: warp c = warp - 4 owns weight rows 32 (c % 4) .. + 31 and K half c / 4 of the slab
    const int c = warp - 4;
    const int r = (c & 3) * 32 + lane;
    const int h = c >> 2;
    const int sw = r & 7;
    for (int j = 0; j < nslab; ++j) {
      const int s = j % C::STAGES;
      const uint32_t ph = (j / C::STAGES) & 1;
      const int a = j % C::NA;
      const uint32_t pa = (j / C::NA) & 1;
      if (!warp_wait(&full[s], ph, SITE_FULL, abort_flag)) break;
      if (!warp_wait(&aempty[a], pa ^ 1, SITE_CONVERT, abort_flag)) break;
      const uint8_t* wrow = sStage + s * C::STAGE_BYTES + r * 128;
      uint8_t* arow = sA + a * C::A_BYTES + h * 16384 + r * 128;
      uint4 v[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = *reinterpret_cast<const uint4*>(wrow + (((4 * h + i) ^ sw) << 4));
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint4 o0, o1;
        i8x4_to_f16x4(v[i].x, o0.x, o0.y);
        i8x4_to_f16x4(v[i].y, o0.z, o0.w);
        i8x4_to_f16x4(v[i].z, o1.x, o1.y);
        i8x4_to_f16x4(v[i].w, o1.z, o1.w);
        // int8 chunk 4h + i holds f16 chunks 8h + 2i, 8h + 2i + 1: chunks 2i, 2i + 1 of operand half h
        *reinterpret_cast<uint4*>(arow + (((2 * i) ^ sw) << 4)) = o0;
        *reinterpret_cast<uint4*>(arow + (((2 * i + 1) ^ sw) << 4)) = o1;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&afull[a]);
        mbar_arrive(&empty[s]);
      }
    }
  } else if (warp >= 12) {
    // epilogue: thread = weight row n0 + 32 * (warp % 4) + lane
    const int q = warp & 3;
    const int n = n0 + q * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    const int G = KB;
    float sc_next = (n < N && nslab > 0) ? __half2float(__ushort_as_half(__ldg(args.s + (int64_t)n * G + kb0))) : 0.f;
    for (int j = 0; j < nslab; ++j) {
      const int b = j % C::NBUF;
      const uint32_t pb = (j / C::NBUF) & 1;
      const float sc = sc_next;
      if (j + 1 < nslab && n < N) sc_next = __half2float(__ushort_as_half(__ldg(args.s + (int64_t)n * G + kb0 + j + 1)));
      if (!warp_wait(&tfull[b], pb, SITE_TMEM_FULL, abort_flag)) break;
      tc_fence_after();
      const uint32_t base = tmem + lane_addr + b * C::NACC * MP;
      if constexpr (MP == 16) {
        uint32_t p0[16], p1[16];
        tmem_ld16(base, p0);
        tmem_ld16(base + 16, p1);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[b]);
#pragma unroll
        for (int m = 0; m < 16; ++m) sum[m] = fmaf(__uint_as_float(p0[m]) + __uint_as_float(p1[m]), sc, sum[m]);
      } else {
#pragma unroll
        for (int c0 = 0; c0 < MP; c0 += 32) {
          uint32_t p0[32], p1[32];
          tmem_ld32(base + c0, p0);
          tmem_ld32(base + MP + c0, p1);
          tmem_ld_wait();
#pragma unroll
          for (int m = 0; m < 32; ++m) sum[c0 + m] = fmaf(__uint_as_float(p0[m]) + __uint_as_float(p1[m]), sc, sum[c0 + m]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[b]);
      }
    }
  }

  // ---- split-K reduction across the cluster through distributed shared memory
  float* red = reinterpret_cast<float*>(sA);   // [MP][128] fp32 partial tile (operand buffers are idle now)
  tc_fence_before();
  __syncthreads();
  const bool epi = warp >= 12;
  const int row = epi ? (warp & 3) * 32 + lane : 0;
  if (epi && rank != 0) {
#pragma unroll
    for (int m = 0; m < MP; ++m) red[m * W8A16_BN + row] = sum[m];
  }
  cluster_sync_all();
  if (epi && rank == 0) {
    for (uint32_t r = 1; r < nrank; ++r) {
#pragma unroll
      for (int m = 0; m < MP; ++m) sum[m] += ld_dsmem_f32(smem_u32(&red[m * W8A16_BN + row]), r);
    }
    const int n = n0 + row;
    if (n < N) {
#pragma unroll
      for (int m = 0; m < MP; ++m)
        if (m < args.M) args.y[(int64_t)m * N + n] = __half_as_ushort(__float2half_rn(sum[m]));
    }
  }
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace i8q
