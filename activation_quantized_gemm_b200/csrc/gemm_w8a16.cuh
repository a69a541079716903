// W8A16 group-wise weight-only GEMM, after "DeepSeek-R1-0528-Qwen3-8B量化版发布" (technical
// details: symmetric group-wise INT8 Linear weights, FP16 activations), group size 128 along K:
//     y[m][n] = fp16( sum_g s[n][g] * sum_{k in g} x[m][k] * wq[n][k] ).
// BF16 = true: the same GEMM for a bf16 model (bf16 activations, group scales and output), the
// weight-only INT8 analogue of the TensorRT-LLM build in "DeepSeek-R1-Distill-Llama-8B模型量化实战"
// section 2.1.  Decode batches take one token tile of MP in {16, 32, 64} tokens (K split over a
// cluster); larger batches (prefill) run tiles of 128 tokens, the grid's z dimension.
//
// The kernel streams the int8 weights once from HBM (the bound) and never rounds a dequantized
// weight: int8 -> f16 is exact (|q| <= 127), the tensor core forms exact f16 x f16 products with
// fp32 accumulation, and the fp16 group scale multiplies each group's fp32 partial sum.
//
// Layout: "swap-AB" - the 128 weight rows of a tile are the MMA's M dimension, the (padded) tokens
// its N dimension, so a decode batch of 1..64 tokens still fills the 128-row tensor-core tile.
//   warps 0..3   epilogue: thread = weight row; per slab, sum[m] += partial[m] * s[n][g].
//   warps 4..7   converters: int8 slab (shared memory) -> exact f16 operand written straight into
//                TMEM with tcgen05.st; the MMA reads its A operand from TMEM, so shared memory only
//                carries the TMA-staged int8 weights and f16 activations.
//   warp 8       TMA: lane 0 streams the int8 weight ring ([128 rows x 128 K] slabs, 128B swizzle;
//                a stage is released as soon as the converters have read it), lane 1 the f16
//                activation ring ([MP x 128 K] as two 64-element halves, released by the MMA).
//   warp 9       TMEM allocation and MMA issue: 8 x tcgen05.mma.kind::f16 (K = 16) per slab.
// For decode batches of up to 32 tokens two CTAs share an SM (256 TMEM columns each).
// The MMA thread is the serial part of the pipeline and every mbarrier probe it makes costs about
// as much as two small MMAs, so each slab costs it one wait and two commits:
//   * TMEM holds R "slots" (an f16 operand buffer + the slab's fp32 accumulator).  ready[slot]
//     completes when the 4 converter warps have written the operand and the 4 epilogue warps have
//     read out the accumulator's previous slab (they pre-arrive once per slot at start); epilogue
//     warp 0 arrives only once the slab's activations have landed.
//   * mdone[slot] (commit) tells the epilogue the accumulator is ready and the converters that the
//     operand buffer may be overwritten; xempty (commit) releases the activation stage.
// Split-K: the CTAs of one thread-block cluster take disjoint slab ranges of the same 128 rows and
// reduce-scatter their fp32 partial tiles through distributed shared memory (each CTA sums its
// share of the rows over all ranks, in rank order, and writes fp16).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"

namespace i8q {

constexpr int W8A16_BN = 128;   // weight rows per tile (MMA M)

template <int MP>
struct W8A16Cfg {
  static_assert(MP == 16 || MP == 32 || MP == 64 || MP == 128, "token tile");
  static constexpr int W_BYTES = W8A16_BN * 128;         // int8 weight slab
  static constexpr int X_HALF = MP * 128;                // one 64-element half of the f16 slab
  static constexpr int X_BYTES = 2 * X_HALF;
  static constexpr int CTAS_PER_SM = MP <= 32 ? 2 : 1;   // two CTAs share an SM's TMEM and smem
  static constexpr int TMEM_COLS = CTAS_PER_SM == 2 ? 256 : 512;
  static constexpr int A_COLS = 64;                      // 128 K f16 values = 64 packed 32-bit columns
  static constexpr int SLOT_COLS = A_COLS + MP;          // operand buffer + accumulator
  static constexpr int R_FIT = TMEM_COLS / SLOT_COLS;
  static constexpr int R = R_FIT < 4 ? R_FIT : 4;        // TMEM slots
  static constexpr int W_STAGES = MP <= 16 ? 5 : (MP <= 32 ? 4 : (MP <= 64 ? 8 : 4));   // weight ring (freed after conversion)
  static constexpr int X_STAGES = MP <= 16 ? 6 : (MP <= 64 ? 5 : 4);   // activation ring (freed by the MMA)
  static constexpr int NUM_THREADS = 320;                // warps 0-3 epilogue, 4-7 converters, 8 TMA, 9 MMA
  static constexpr int RING_BYTES = W_STAGES * W_BYTES + X_STAGES * X_BYTES;
  static constexpr int SMEM_BYTES = RING_BYTES + 512 + 1024;
  static_assert(R >= 2 && X_STAGES > R, "pipeline depth");
  static_assert(X_BYTES % 1024 == 0, "128B-swizzled TMA boxes need 1024-byte alignment");
  static_assert(MP * W8A16_BN * 4 <= RING_BYTES, "reduction tile must fit in the ring");
  static_assert(MP % 16 == 0, "MMA N and the 16-column TMEM loads");
  static_assert(CTAS_PER_SM * (SMEM_BYTES + 1024) <= 233472, "shared memory per SM");
};

struct W8A16Args {
  const uint16_t* s;   // [N][K/128] fp16 (bf16) group scales
  int M, N, K;
  uint16_t* y;         // [M][N] fp16 (bf16)
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
// Every thread of the cluster.  The .aligned barrier needs each warp converged: callers may come
// from lane-divergent code, so the warp reconverges first.
__device__ __forceinline__ void cluster_sync_all() {
  __syncwarp();
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// 16 bytes at the same shared-memory offset in CTA `rank` of the cluster (distributed shared memory)
__device__ __forceinline__ float4 ld_dsmem_f32x4(uint32_t local_addr, uint32_t rank) {
  uint32_t remote;
  float4 v;
  asm("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(remote));
  return v;
}
// D[tmem] (+)= A[tmem] * B[smem]^T, f16 x f16 -> f32 (K = 16); A is 128 lanes x 8 packed columns.
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// 32 registers -> 32 lanes x 32 columns of TMEM (thread t writes lane base + t)
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// Instruction descriptor: kind::f16 with bf16 A and B, f32 D, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4)               // D format: f32
         | (1u << 7) | (1u << 10)  // A, B: bf16
         | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// 4 signed int8 (one 32-bit word) -> 4 exact bf16 values as two bf16x2 words.  bf16 has 8
// significant bits, so |q| <= 127 is exact, but the offset-binary trick of the f16 version below
// does not fit in its 7-bit mantissa (q + 128 spans two binades).
__device__ __forceinline__ void i8x4_to_bf16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  // a code q with sign bit s and low bits l is l - 128 s.  With 0x43 as the high byte, bf16
  // 0x43 | l is 128 + l and 0x43 | (s << 7) is 128 or 256 (all exact), so one packed subtract of
  // the two gives q exactly (+0 for q = 0).
  const uint32_t pl = __byte_perm(w, 0x43434343u, 0x4140), ph = __byte_perm(w, 0x43434343u, 0x4342);
  const uint32_t al = pl & 0xFF7FFF7Fu, sl = pl & 0xFF80FF80u, ah = ph & 0xFF7FFF7Fu, sh = ph & 0xFF80FF80u;
  __nv_bfloat162 ha = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&al), *reinterpret_cast<const __nv_bfloat162*>(&sl));
  __nv_bfloat162 hb = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&ah), *reinterpret_cast<const __nv_bfloat162*>(&sh));
  lo = *reinterpret_cast<uint32_t*>(&ha);
  hi = *reinterpret_cast<uint32_t*>(&hb);
}

// Group scale (fp16 or bf16 bits) -> fp32 (exact), and fp32 -> output bits (round to nearest even).
template <bool BF16>
__device__ __forceinline__ float half_bits_to_f32(uint16_t h) {
  if constexpr (BF16) return __uint_as_float((uint32_t)h << 16);
  else return __half2float(__ushort_as_half(h));
}
template <bool BF16>
__device__ __forceinline__ uint16_t f32_to_half_bits(float v) {
  if constexpr (BF16) return __bfloat16_as_ushort(__float2bfloat16_rn(v));
  else return __half_as_ushort(__float2half_rn(v));
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

template <int MP, bool BF16>
__global__ void __launch_bounds__(320, W8A16Cfg<MP>::CTAS_PER_SM)
    k_gemm_w8a16(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                 const W8A16Args args) {
  using C = W8A16Cfg<MP>;
  constexpr int R = C::R;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sW = smem;                                       // W_STAGES x int8 weight slab
  uint8_t* sX = smem + C::W_STAGES * C::W_BYTES;            // X_STAGES x f16 activation slab
  uint64_t* wfull = reinterpret_cast<uint64_t*>(smem + C::RING_BYTES);
  uint64_t* wempty = wfull + C::W_STAGES;
  uint64_t* xfull = wempty + C::W_STAGES;
  uint64_t* xempty = xfull + C::X_STAGES;
  uint64_t* ready = xempty + C::X_STAGES;
  uint64_t* mdone = ready + R;
  uint64_t* done = mdone + R;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = args.N, K = args.K;
  const int KB = K / 128;
  const uint32_t rank = cluster_ctarank(), nrank = cluster_nctarank();
  const int kb0 = (int)((int64_t)KB * rank / nrank), kb1 = (int)((int64_t)KB * (rank + 1) / nrank);
  const int nslab = kb1 - kb0;
  const int n0 = blockIdx.x * W8A16_BN;
  const int m0 = blockIdx.z * MP;              // first token of this CTA's token tile

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::W_STAGES; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&wempty[s], 4);   // the 4 converter warps
    }
    for (int s = 0; s < C::X_STAGES; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&xempty[s], 1);   // the MMA's commit
    }
    for (int r = 0; r < R; ++r) {
      mbar_init(&ready[r], 8);    // 4 converter warps + 4 epilogue warps
      mbar_init(&mdone[r], 1);    // the MMA's commit
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // The kernel may be launched while the preceding kernel is still running: until
  // grid_dependency_wait() it touches no global memory except L2 prefetches of its first weight
  // slabs.  It lets the next kernel launch early in turn (that kernel waits for this one the same way).
  grid_dependents_launch();
  if (warp == 8 && lane == 0)
    for (int j = 0; j < nslab && j < C::W_STAGES; ++j) tma_prefetch_l2_2d(&tmW, (kb0 + j) * 128, n0);
  if (warp == 9) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dependency_wait();

  float sum[MP];
#pragma unroll
  for (int m = 0; m < MP; ++m) sum[m] = 0.f;

  if (warp == 8) {
    if (lane < 2) {
      // lane 0 feeds the weight ring (waits only for the converters), lane 1 the activation ring
      // (waits only for the MMA); the two rings run ahead independently.
      const bool is_w = lane == 0;
      const int nst = is_w ? C::W_STAGES : C::X_STAGES;
      uint64_t* fullb = is_w ? wfull : xfull;
      uint64_t* emptyb = is_w ? wempty : xempty;
      uint32_t filled = 0, par = 0;
      bool ok = true;
      for (int j = 0; j < nslab; ++j) {
        const int st = j % nst;
        const uint32_t ph = (j / nst) & 1;
        const int kk = (kb0 + j) * 128;
        if (!mbar_wait(&emptyb[st], ph ^ 1, SITE_EMPTY, abort_flag)) { ok = false; break; }
        if (is_w) {
          mbar_arrive_expect_tx(&fullb[st], C::W_BYTES);
          tma_load_2d(sW + st * C::W_BYTES, &tmW, &fullb[st], kk, n0);
        } else {
          uint8_t* xs = sX + st * C::X_BYTES;
          mbar_arrive_expect_tx(&fullb[st], C::X_BYTES);
          tma_load_2d(xs, &tmX, &fullb[st], kk, m0);
          tma_load_2d(xs + C::X_HALF, &tmX, &fullb[st], kk + 64, m0);
        }
        filled |= 1u << st;
        par = (par & ~(1u << st)) | (ph << st);
      }
      if (!ok)   // let every copy in flight land before the CTA can exit
        for (int st = 0; st < nst; ++st)
          if (filled & (1u << st)) mbar_wait(&fullb[st], (par >> st) & 1u, SITE_DRAIN, nullptr);
    }
  } else if (warp == 9) {
    if (lane == 0) {
      constexpr uint32_t idesc = BF16 ? idesc_bf16(W8A16_BN, MP) : idesc_f16(W8A16_BN, MP);
      for (int j = 0; j < nslab; ++j) {
        const int xs = j % C::X_STAGES;
        const int r = j % R;
        if (!mbar_wait(&ready[r], (j / R) & 1, SITE_CONVERT, abort_flag)) break;
        tc_fence_after();
        const uint32_t a0 = tmem + r * C::A_COLS;                        // operand columns
        const uint32_t d0 = tmem + R * C::A_COLS + r * MP;               // accumulator columns
        const uint32_t x0 = smem_u32(sX + xs * C::X_BYTES);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t h = kk >> 2, off = (kk & 3) * 32;
          mma_f16_ts(d0, a0 + kk * 8, sw128_kmajor_desc(x0 + h * C::X_HALF + off), idesc, kk > 0 ? 1u : 0u);
        }
        tc_commit(&mdone[r]);
        tc_commit(&xempty[xs]);
      }
      tc_commit(done);
      mbar_wait(done, 0, SITE_DRAIN, nullptr);
    }
  } else if (warp >= 4 && warp < 8) {
    // converters: warp w owns weight rows 32 (w % 4) .. + 31 (its TMEM lane quarter); each thread
    // writes the exact f16 values of its row's 128 K into the slot's operand columns (two f16 per
    // 32-bit column, K order).
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int sw = row & 7;
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    for (int j = 0; j < nslab; ++j) {
      const int st = j % C::W_STAGES;
      const int r = j % R;
      if (!warp_wait(&wfull[st], (j / C::W_STAGES) & 1, SITE_FULL, abort_flag)) break;
      // the operand buffer is free once the MMAs of the slot's previous slab have completed
      if (j >= R && !warp_wait(&mdone[r], ((j / R) & 1) ^ 1, SITE_CONVERT, abort_flag)) break;
      tc_fence_after();
      const uint8_t* wrow = sW + st * C::W_BYTES + row * 128;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t o[32];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 v = *reinterpret_cast<const uint4*>(wrow + (((4 * h + i) ^ sw) << 4));
          if constexpr (BF16) {
            i8x4_to_bf16x4(v.x, o[8 * i + 0], o[8 * i + 1]);
            i8x4_to_bf16x4(v.y, o[8 * i + 2], o[8 * i + 3]);
            i8x4_to_bf16x4(v.z, o[8 * i + 4], o[8 * i + 5]);
            i8x4_to_bf16x4(v.w, o[8 * i + 6], o[8 * i + 7]);
          } else {
            i8x4_to_f16x4(v.x, o[8 * i + 0], o[8 * i + 1]);
            i8x4_to_f16x4(v.y, o[8 * i + 2], o[8 * i + 3]);
            i8x4_to_f16x4(v.z, o[8 * i + 4], o[8 * i + 5]);
            i8x4_to_f16x4(v.w, o[8 * i + 6], o[8 * i + 7]);
          }
        }
        tmem_st32(tmem + lane_addr + r * C::A_COLS + h * 32, o);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&ready[r]);
        mbar_arrive(&wempty[st]);
      }
    }
  } else if (warp < 4) {
    // epilogue: thread = weight row n0 + 32 * (warp % 4) + lane
    const int q = warp & 3;
    const int n = n0 + q * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    const int G = KB;
    // Arrival on the slot of slab t: its accumulator is free.  Epilogue warp 0 also vouches for slab
    // t's activations (it observes their TMA barrier first), so that the MMA thread needs a single
    // wait per slab.  The activation ring runs further ahead than the slots, but its stage of slab t
    // cannot be refilled before slab t's MMAs, which wait for this arrival.
    auto free_slot = [&](int t) {
      if (lane == 0) {
        bool ok = true;
        if (q == 0 && t < nslab)
          ok = mbar_wait(&xfull[t % C::X_STAGES], (t / C::X_STAGES) & 1, SITE_FULL, abort_flag);
        if (ok) mbar_arrive(&ready[t % R]);
      }
      __syncwarp();
    };
    for (int r = 0; r < R; ++r) free_slot(r);   // every accumulator starts out free
    float sc_next = (n < N && nslab > 0) ? half_bits_to_f32<BF16>(__ldg(args.s + (int64_t)n * G + kb0)) : 0.f;
    for (int j = 0; j < nslab; ++j) {
      const int r = j % R;
      const float sc = sc_next;
      if (j + 1 < nslab && n < N) sc_next = half_bits_to_f32<BF16>(__ldg(args.s + (int64_t)n * G + kb0 + j + 1));
      if (!warp_wait(&mdone[r], (j / R) & 1, SITE_TMEM_FULL, abort_flag)) break;
      tc_fence_after();
      const uint32_t base = tmem + lane_addr + R * C::A_COLS + r * MP;
#pragma unroll
      for (int c0 = 0; c0 < MP; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(base + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) sum[c0 + i] = fmaf(__uint_as_float(v[i]), sc, sum[c0 + i]);
      }
      tc_fence_before();
      __syncwarp();
      free_slot(j + R);
    }
  }

  // ---- output.  Without a split the epilogue threads write their rows directly.  With a split,
  // every CTA publishes its fp32 partial tile ([128 rows][MP] in shared memory) and CTA `rank` sums
  // its block of rows over all ranks, in rank order, 4 tokens per 16-byte load.
  tc_fence_before();
  __syncthreads();
  const int mlim = args.M - m0 < MP ? args.M - m0 : MP;   // tokens of this tile
  uint16_t* ytile = args.y + (int64_t)m0 * N;
  if (nrank == 1) {
    if (warp < 4) {
      const int n = n0 + warp * 32 + lane;
      if (n < N) {
#pragma unroll
        for (int m = 0; m < MP; ++m)
          if (m < mlim) ytile[(int64_t)m * N + n] = f32_to_half_bits<BF16>(sum[m]);
      }
    }
  } else {
    float4* red = reinterpret_cast<float4*>(smem);   // [128][MP / 4] (the rings are idle now)
    if (warp < 4) {
      const int row = warp * 32 + lane;
#pragma unroll
      for (int m4 = 0; m4 < MP / 4; ++m4)
        red[row * (MP / 4) + m4] = make_float4(sum[4 * m4], sum[4 * m4 + 1], sum[4 * m4 + 2], sum[4 * m4 + 3]);
    }
    cluster_sync_all();
    // CTA `rank` owns a contiguous block of rows; consecutive threads take consecutive rows of one
    // 4-token group, so that a warp's fp16 stores are contiguous.
    const int rb0 = W8A16_BN * (int)rank / (int)nrank, rb1 = W8A16_BN * ((int)rank + 1) / (int)nrank;
    const int owned = rb1 - rb0;
    const int items = owned * (MP / 4);
    for (int e = threadIdx.x; e < items; e += C::NUM_THREADS) {
      const int m4 = e / owned;
      const int row = rb0 + (e - m4 * owned);
      const uint32_t la = smem_u32(&red[row * (MP / 4) + m4]);
      float4 part[8];
#pragma unroll
      for (int p = 0; p < 8; ++p)
        if (p < (int)nrank) part[p] = ld_dsmem_f32x4(la, (uint32_t)p);
      float4 v = part[0];
#pragma unroll
      for (int p = 1; p < 8; ++p)
        if (p < (int)nrank) {
          v.x += part[p].x; v.y += part[p].y; v.z += part[p].z; v.w += part[p].w;
        }
      const int n = n0 + row;
      if (n < N) {
        const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (4 * m4 + k < mlim) ytile[(int64_t)(4 * m4 + k) * N + n] = f32_to_half_bits<BF16>(vv[k]);
      }
    }
  }
  cluster_sync_all();   // no CTA leaves while its shared memory may still be read
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace i8q
