// W8A8 GEMMs on the 5th-generation tensor cores (tcgen05.mma kind::i8, int32 accumulators in
// TMEM), for both schemes of "DeepSeek R1 INT8 quantization practice on SGLang", section 2.3:
//
//  * channel-wise (Fig. 3 right): the whole K reduction accumulates in TMEM; the epilogue applies
//    the per-token x per-output-channel scale once and writes bf16.
//  * block-wise (Fig. 3 left): every 128-wide K slab gets a fresh TMEM accumulator; the epilogue
//    warps read each slab's exact int32 partial sum and fold it into an fp32 running sum with the
//    slab's activation-group x weight-block scale ("several dequantizations inside the INT8
//    matmul, on the CUDA cores").  Two TMEM accumulator buffers let the tensor core run the next
//    slab while the CUDA cores dequantize the previous one.
//
// Kernel structure (persistent, one CTA per SM, 256 threads):
//   warp 0      : TMA producer - 128x128 activation tile + BNx128 weight tile per slab into a
//                 STAGES-deep ring of 128B-swizzled shared-memory buffers (mbarrier complete_tx).
//   warp 1      : TMEM allocator and MMA issuer - 4 x tcgen05.mma (K = 32 each) per slab,
//                 tcgen05.commit frees the smem stage and hands the accumulator to the epilogue.
//   warps 4..7  : epilogue - warp w reads TMEM lanes 32*(w%4).. (tile rows), one row per thread.
// Tiles are 128 tokens x BN output channels, visited in bands of 16 token-blocks so that the
// activations and weights the 148 CTAs touch at one time stay resident in L2.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace i8q {

constexpr int GEMM_BM = 128;       // tokens per tile (MMA M)
constexpr int GEMM_BK = 128;       // K per slab (bytes of int8 = one 128B swizzle row)
constexpr int GEMM_GROUP_M = 16;   // token-blocks per raster band

template <int BN>
struct W8A8Cfg {
  static constexpr int A_BYTES = GEMM_BM * GEMM_BK;
  static constexpr int B_BYTES = BN * GEMM_BK;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (BN >= 256) ? 4 : 6;
  static constexpr int TMEM_COLS = 2 * BN;               // two accumulator buffers
  static constexpr int NUM_THREADS = 256;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;  // + alignment slack
  static_assert(TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM allocation must be a power of two");
};

struct W8A8Args {
  const float* sx;      // channel: [M]; block: [KB][ld_sx]
  int64_t ld_sx;
  const float* sw;      // channel: [N]; block: [ceil(N/128)][KB]
  int M, N, K;
  void* y;              // [M][N] bf16 or fp32
  int32_t* dbg;         // channel: [M][N] accumulators; block: [M][N][KB] slab partials
};

__device__ __forceinline__ void gemm_tile_coords(int t, int Mt, int Nt, int& mb, int& nb) {
  const int band_tiles = GEMM_GROUP_M * Nt;
  const int band = t / band_tiles;
  const int first_m = band * GEMM_GROUP_M;
  const int rows = min(GEMM_GROUP_M, Mt - first_m);
  const int idx = t - band * band_tiles;
  mb = first_m + idx % rows;
  nb = idx / rows;
}

// Exact int32 -> fp32 for |p| < 2^22: place p in the mantissa of 1.5 * 2^23 and subtract.
__device__ __forceinline__ float i2f_small_exact(uint32_t p) {
  return __int_as_float(0x4B400000 + (int)p) - 12582912.0f;
}

__device__ __forceinline__ void store_row8(void* y, bool f32out, int64_t off, const float (&v)[8]) {
  if (f32out) {
    float4* p = reinterpret_cast<float4*>(reinterpret_cast<float*>(y) + off);
    p[0] = make_float4(v[0], v[1], v[2], v[3]);
    p[1] = make_float4(v[4], v[5], v[6], v[7]);
  } else {
    uint4 u;
    __nv_bfloat162 h0 = __floats2bfloat162_rn(v[0], v[1]);
    __nv_bfloat162 h1 = __floats2bfloat162_rn(v[2], v[3]);
    __nv_bfloat162 h2 = __floats2bfloat162_rn(v[4], v[5]);
    __nv_bfloat162 h3 = __floats2bfloat162_rn(v[6], v[7]);
    u.x = *reinterpret_cast<uint32_t*>(&h0);
    u.y = *reinterpret_cast<uint32_t*>(&h1);
    u.z = *reinterpret_cast<uint32_t*>(&h2);
    u.w = *reinterpret_cast<uint32_t*>(&h3);
    *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(y) + off) = u;
  }
}

template <int BN, bool BLOCKWISE, bool OUT_F32, bool DEBUG>
__global__ void __launch_bounds__(256, 1)
    k_gemm_w8a8(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const W8A8Args args) {
  using C = W8A8Cfg<BN>;
  static_assert(!BLOCKWISE || BN == 128, "block-wise tiles are one weight block wide");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int M = args.M, N = args.N, K = args.K;
  const int Mt = (M + GEMM_BM - 1) / GEMM_BM, Nt = (N + BN - 1) / BN, KB = K / GEMM_BK;
  const int num_tiles = Mt * Nt;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);   // one arrival per epilogue warp
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t filled = 0, fill_parity = 0;   // per stage: a load was issued / its phase parity
      bool ok = true;
      for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
        int mb, nb;
        gemm_tile_coords(t, Mt, Nt, mb, nb);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, SITE_EMPTY, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          tma_load_2d(sA + stage * C::A_BYTES, &tmA, &full[stage], kb * GEMM_BK, mb * GEMM_BM);
          tma_load_2d(sB + stage * C::B_BYTES, &tmB, &full[stage], kb * GEMM_BK, nb * BN);
          filled |= 1u << stage;
          fill_parity = (fill_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {  // let every copy already in flight land before the CTA can exit
        for (int s = 0; s < C::STAGES; ++s)
          if (filled & (1u << s)) mbar_wait(&full[s], (fill_parity >> s) & 1u, SITE_DRAIN, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(GEMM_BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc_iter = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
        uint32_t acc = 0;
        if (!BLOCKWISE) {
          acc = acc_iter & 1;
          if (!mbar_wait(&tempty[acc], ((acc_iter >> 1) & 1) ^ 1, SITE_TMEM_EMPTY, abort_flag)) { ok = false; break; }
          tc_fence_after();
        }
        for (int kb = 0; kb < KB; ++kb) {
          if (BLOCKWISE) {
            acc = acc_iter & 1;
            if (!mbar_wait(&tempty[acc], ((acc_iter >> 1) & 1) ^ 1, SITE_TMEM_EMPTY, abort_flag)) { ok = false; break; }
            tc_fence_after();
          }
          if (!mbar_wait(&full[stage], phase, SITE_FULL, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * C::B_BYTES);
          const uint32_t d = tmem + acc * BN;
#pragma unroll
          for (int kk = 0; kk < GEMM_BK / 32; ++kk) {
            const uint32_t accumulate = BLOCKWISE ? (kk > 0) : (kb > 0 || kk > 0);
            mma_i8(d, sw128_kmajor_desc(a0 + kk * 32), sw128_kmajor_desc(b0 + kk * 32), idesc, accumulate);
          }
          tc_commit(&empty[stage]);
          if (BLOCKWISE) {
            tc_commit(&tfull[acc]);
            ++acc_iter;
          }
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
        if (!BLOCKWISE && ok) {
          tc_commit(&tfull[acc]);
          ++acc_iter;
        }
      }
      // every MMA this thread issued has finished once `done` completes
      tc_commit(done);
      mbar_wait(done, 0, SITE_DRAIN, nullptr);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;                        // TMEM lane quarter = tile rows 32q..32q+31
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    uint32_t acc_iter = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      int mb, nb;
      gemm_tile_coords(t, Mt, Nt, mb, nb);
      const int m = mb * GEMM_BM + q * 32 + lane;
      const int n0 = nb * BN;
      const bool row_ok = m < M;
      if constexpr (!BLOCKWISE) {
        const uint32_t acc = acc_iter & 1;
        if (!warp_wait(&tfull[acc], (acc_iter >> 1) & 1, SITE_TMEM_FULL, abort_flag)) break;
        tc_fence_after();
        const float sxm = row_ok ? __ldg(args.sx + m) : 0.f;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_addr + acc * BN + c * 32, r);
          tmem_ld_wait();
          const int nc = n0 + c * 32;
          if (row_ok) {
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const int n = nc + g * 8;
              if (n < N) {
                const float4 w0 = __ldg(reinterpret_cast<const float4*>(args.sw + n));
                const float4 w1 = __ldg(reinterpret_cast<const float4*>(args.sw + n + 4));
                const float ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                float v[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) v[j] = __int2float_rn((int)r[g * 8 + j]) * (sxm * ws[j]);
                store_row8(args.y, false, (int64_t)m * N + n, v);
                if constexpr (DEBUG) {
                  int4* dp = reinterpret_cast<int4*>(args.dbg + (int64_t)m * N + n);
                  dp[0] = make_int4(r[g * 8 + 0], r[g * 8 + 1], r[g * 8 + 2], r[g * 8 + 3]);
                  dp[1] = make_int4(r[g * 8 + 4], r[g * 8 + 5], r[g * 8 + 6], r[g * 8 + 7]);
                }
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
        ++acc_iter;
      } else {
        float sum[BN];
#pragma unroll
        for (int j = 0; j < BN; ++j) sum[j] = 0.f;
        bool ok = true;
        const float* swrow = args.sw + (int64_t)nb * KB;   // BN == 128: tile n-block == weight block
        float s_next = 0.f;
        if (KB > 0 && row_ok) s_next = __ldg(args.sx + m) * __ldg(swrow);
        for (int kb = 0; kb < KB; ++kb) {
          const float s = s_next;
          if (kb + 1 < KB && row_ok)
            s_next = __ldg(args.sx + (int64_t)(kb + 1) * args.ld_sx + m) * __ldg(swrow + kb + 1);
          const uint32_t acc = acc_iter & 1;
          if (!warp_wait(&tfull[acc], (acc_iter >> 1) & 1, SITE_TMEM_FULL, abort_flag)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < BN / 32; c += 2) {
            uint32_t r0[32], r1[32];
            tmem_ld32(tmem + lane_addr + acc * BN + c * 32, r0);
            tmem_ld32(tmem + lane_addr + acc * BN + (c + 1) * 32, r1);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) sum[c * 32 + j] = fmaf(i2f_small_exact(r0[j]), s, sum[c * 32 + j]);
#pragma unroll
            for (int j = 0; j < 32; ++j) sum[(c + 1) * 32 + j] = fmaf(i2f_small_exact(r1[j]), s, sum[(c + 1) * 32 + j]);
            if constexpr (DEBUG) {
              if (row_ok) {
                for (int j = 0; j < 32; ++j) {
                  if (n0 + c * 32 + j < N) args.dbg[((int64_t)m * N + n0 + c * 32 + j) * KB + kb] = (int32_t)r0[j];
                  if (n0 + (c + 1) * 32 + j < N) args.dbg[((int64_t)m * N + n0 + (c + 1) * 32 + j) * KB + kb] = (int32_t)r1[j];
                }
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[acc]);
          ++acc_iter;
        }
        if (!ok) break;
        if (row_ok) {
#pragma unroll
          for (int g = 0; g < BN / 8; ++g) {
            const int n = n0 + g * 8;
            if (n < N) {
              float v[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) v[j] = sum[g * 8 + j];
              store_row8(args.y, OUT_F32, (int64_t)m * N + n, v);
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace i8q
