// Decode-size W8A8 GEMMs (M <= 128 tokens) for both schemes of "DeepSeek R1 INT8 quantization
// practice on SGLang", section 2.3.  At these sizes the weights dominate the traffic, so the kernel
// is built to stream them once from HBM:
//
// "Swap-AB" tcgen05.mma.kind::i8 (K = 32 per instruction): the 128 weight rows of a tile are the
// MMA's M dimension, read by the tensor core straight from the TMA-staged 128B-swizzled shared
// memory, and the (padded) tokens are its N dimension, so a batch of 1..128 tokens still fills the
// 128-row tensor-core tile.  The thread-block cluster of a tile splits K; its CTAs reduce-scatter
// their partial tiles through distributed shared memory (no global scratch).
//   warps 0..3  epilogue (0..15 at 128 tokens, four token quarters per TMEM lane quarter): thread =
//               weight row (TMEM lane).  Channel-wise: the exact int32 dot
//               products are read once at the end, summed exactly over the cluster, then scaled by
//               sx[m] * sw[n].  Block-wise: each 128-K slab has its own TMEM accumulator; its int32
//               partial sums are folded into fp32 running sums with sx[m][kb] * sw[n/128][kb].
//   next warp   TMA producer: weight slab [128 rows x 128 K] + activation slab [MP x 128 K].
//   next warp   TMEM allocation and MMA issue (4 x tcgen05.mma per slab).
//   (FUSEDQ)    four quantizer warps after those.
// Two CTAs share an SM for up to 64 tokens (rings of 4..6 stages each), one CTA for 128 (TMEM and
// registers); the launch keeps all CTAs in one wave.
//
// FUSEDQ (block-wise, up to 16 tokens): the activations arrive as bf16 and are quantized inside
// the GEMM, per token and 128-wide K group, as "DeepSeek R1 INT8 quantization practice on SGLang"
// section 2.3 prescribes ("quantized online per token-group").  The TMA warp stages the bf16 slab
// [MP x 128] next to the weight slab; quantizer warps turn it into the int8 operand (128B-swizzled,
// as TMA would have written it) and the group scales, with the same device code as the stand-alone
// per-token-group quantizer, so codes and scales are bit-identical to it.  Every CTA quantizes the
// slabs of its own K range (tiles over N repeat that small amount of work instead of a separate
// launch and an HBM round trip of the int8 activations).
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"
#include "gemm_w8a16.cuh"   // cluster helpers
#include "quant.cuh"        // the quantizer (fused variant)

namespace i8q {

constexpr int W8A8_SMALL_MAX_M = 128;

// CPS CTAs share an SM; the stage ring fills the rest of its shared memory: under full streaming
// load a weight slab takes about 2 us to arrive, so an SM needs of the order of 100 KB in flight.
template <int MP, bool BLOCKWISE, int CPS, bool FUSEDQ = false>
struct W8A8SmallCfg {
  static constexpr int W_BYTES = 128 * 128;
  static constexpr int X_BYTES = MP * 128;
  static constexpr int STAGE_BYTES = W_BYTES + X_BYTES;
  // fused: the bf16 activation slab has its own ring, freed as soon as the quantizers have read it
  static constexpr int XB_HALF = MP * 128;                // one 64-column half of the bf16 slab
  static constexpr int XB_BYTES = 2 * XB_HALF;
  // bf16 ring stages: deep enough that an activation slab's L2 latency (~1 us) stays hidden
  // behind the quantization of the slabs before it (two stages left the quantizers waiting)
  // Quantizer warps.  Quantizing one slab is one long dependent chain for a warp (≈ 2000 cycles at
  // 16 tokens, measured, more than a slab's share of the weight stream), so four warps take whole
  // slabs in turn: warp q quantizes slabs j ≡ q mod 4 and owns the bf16 ring slots r ≡ q mod 4.
  // Two slots per warp keep the next slab's bf16 load (≈ 1 µs from L2 under the weight stream)
  // in flight while the warp quantizes the current one.
  static constexpr int QW = FUSEDQ ? 4 : 0;
  static constexpr int XR = FUSEDQ ? 2 * QW : 0;          // bf16 ring stages
  static constexpr int XRING_BYTES = XR * XB_BYTES;
  static constexpr bool QALT = FUSEDQ;
  static constexpr int NBUF = BLOCKWISE ? 4 : 1;          // slab accumulators in TMEM
  static constexpr int TMEM_NEED = NBUF * MP;
  static constexpr int TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64 : TMEM_NEED <= 128 ? 128 : TMEM_NEED <= 256 ? 256 : 512;
  static_assert(CPS * TMEM_COLS <= 512, "TMEM of the CTAs sharing an SM");
  // epilogue warps: 4 (one per TMEM lane quarter), or 16 at 128 tokens (four column quarters per
  // lane quarter) so that the per-slab fold of 128 columns is split over four times the threads
  // (8 warps: 41.5 µs for the DeepSeek-R1 up-projection at 128 tokens, 16: 40.3 µs)
  static constexpr int EW = MP >= 128 ? 16 : 4;
  static constexpr int MPW = MP / (EW / 4);              // token columns per epilogue thread
  static constexpr int NUM_THREADS = 32 * (EW + 2 + QW);   // + TMA warp + MMA warp (+ quantizers)
  static constexpr int BAR_BYTES = FUSEDQ ? 1024 : 512;
  static constexpr int RING_BYTES = EW * 2 * MPW * 4;    // block-wise scale-product rings, one per epilogue warp
  static constexpr int QR = 16 + NBUF;                   // fused: ring of per-token scales, >= STAGES + NBUF
  static constexpr int QSX_BYTES = FUSEDQ ? QR * MP * 4 : 0;
  static constexpr int FIXED_BYTES = XRING_BYTES + BAR_BYTES + RING_BYTES + QSX_BYTES + 1024;   // + alignment slack
  static constexpr int SM_SMEM = 233472, CTA_RESERVED = 1024, CTA_MAX = 232448;
  static constexpr int BUDGET = (SM_SMEM / CPS - CTA_RESERVED) < CTA_MAX ? (SM_SMEM / CPS - CTA_RESERVED) : CTA_MAX;
  static constexpr int STAGES_FIT = (BUDGET - FIXED_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT < 16 ? STAGES_FIT : 16;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + FIXED_BYTES;
  static_assert(MP == 16 || MP == 32 || MP == 64 || MP == 128, "MMA N");
  static_assert(CPS == 1 || CPS == 2, "CTAs per SM");
  static_assert(STAGES >= 4, "stage ring");
  static_assert(MP * 128 * 4 <= STAGES * STAGE_BYTES, "reduction tile must fit in the stage buffers");
  static_assert(CPS * (SMEM_BYTES + CTA_RESERVED) <= SM_SMEM && SMEM_BYTES <= CTA_MAX, "shared memory");
  static_assert(!FUSEDQ || (BLOCKWISE && MP == 16), "fused quantization: block-wise, up to 16 tokens");
  static_assert(STAGE_BYTES % 1024 == 0, "128B-swizzled buffers stay 1024-byte aligned");
  static_assert(QR >= STAGES + NBUF, "scale ring deeper than the lead of the quantizer over the epilogue");
  static_assert(8 * (3 * STAGES + 2 * NBUF + 1 + 2 * XR + (FUSEDQ ? QR : 0)) + 8 <= BAR_BYTES, "barrier block");
  static_assert(!QALT || (XR % (QW > 0 ? QW : 1) == 0 && QW <= STAGES), "each bf16 slot belongs to one quantizer warp");
};

// Fused quantizer: quantize the bf16 activation slab of one stage (two 128B-swizzled halves of
// [MP rows x 64 bf16]) into the int8 operand (128B-swizzled [MP rows x 128]) and the per-token
// group scales.  Warp qi handles tokens [qi * MP / QW, (qi + 1) * MP / QW); LPT lanes share a token.
template <int MP, int QW>
__device__ __forceinline__ void quantize_slab(const uint8_t* xb, uint8_t* xq, float* qs, int qi, int lane,
                                              int8_t* qx_out, float* qs_out, int M, int K, int kb,
                                              int64_t ld_qs) {
  constexpr int TPW = MP / QW;                       // tokens per quantizer warp
  constexpr int LPT = TPW >= 32 ? 1 : 32 / TPW;      // lanes per token
  constexpr int PASSES = TPW >= 32 ? TPW / 32 : 1;
  constexpr int CPL = 16 / LPT;                      // 8-value bf16 chunks per lane (of 16 per row)
#pragma unroll
  for (int ps = 0; ps < PASSES; ++ps) {
    const int m = qi * TPW + ps * 32 + lane / LPT;
    const int part = lane % LPT;
    uint4 v[CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      const int c = part * CPL + i;                  // chunk of the row: K offset 8c
      const int h = c >> 3, cc = c & 7;
      v[i] = *reinterpret_cast<const uint4*>(xb + h * (MP * 128) + m * 128 + ((cc ^ (m & 7)) << 4));
    }
    uint32_t ab = 0;
#pragma unroll
    for (int i = 0; i < CPL; ++i) ab = max_u16x2(ab, absmax_bits_x8(v[i]));
#pragma unroll
    for (int d = 1; d < LPT; d <<= 1) ab = max_u16x2(ab, __shfl_xor_sync(FULL_MASK, ab, d));
    const QScale q = make_qscale(bits_to_absmax(ab));
#pragma unroll
    for (int i = 0; i < CPL; i += 2) {
      const uint2 lo = quant_bf16x8(v[i], q, true), hi = quant_bf16x8(v[i + 1], q, true);
      const int c16 = (part * CPL + i) >> 1;         // 16-byte int8 chunk of the row
      *reinterpret_cast<uint4*>(xq + m * 128 + ((c16 ^ (m & 7)) << 4)) = make_uint4(lo.x, lo.y, hi.x, hi.y);
      if (qx_out != nullptr && m < M)
        *reinterpret_cast<uint4*>(qx_out + (int64_t)m * K + kb * 128 + c16 * 16) = make_uint4(lo.x, lo.y, hi.x, hi.y);
    }
    if (part == 0) {
      qs[m] = q.s;
      if (qs_out != nullptr && m < M) qs_out[(int64_t)kb * ld_qs + m] = q.s;
    }
  }
}

__device__ __forceinline__ int4 ld_dsmem_s32x4(uint32_t local_addr, uint32_t rank) {
  uint32_t remote;
  int4 v;
  asm("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
  asm volatile("ld.shared::cluster.v4.s32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(remote));
  return v;
}

// 32 lanes x CH columns of 32-bit TMEM (CH = 16 or 32)
template <int CH>
__device__ __forceinline__ void tmem_ld_ch(uint32_t taddr, uint32_t (&r)[CH]) {
  if constexpr (CH == 16)
    tmem_ld16(taddr, r);
  else
    tmem_ld32(taddr, r);
}

template <int MP, bool BLOCKWISE, int CPS, bool OUT_F32, bool DEBUG, bool FUSEDQ = false>
__global__ void __launch_bounds__(W8A8SmallCfg<MP, BLOCKWISE, CPS, FUSEDQ>::NUM_THREADS, CPS)
    k_gemm_w8a8_small(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                      const W8A8Args args) {
  using C = W8A8SmallCfg<MP, BLOCKWISE, CPS, FUSEDQ>;
  constexpr int EW = C::EW, MPW = C::MPW;
  constexpr int CH = MPW < 32 ? MPW : 32;   // TMEM columns per load
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xring = smem + C::STAGES * C::STAGE_BYTES;     // fused: bf16 activation slabs
  uint64_t* full = reinterpret_cast<uint64_t*>(xring + C::XRING_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + C::NBUF;
  uint64_t* done = tempty + C::NBUF;
  uint64_t* xfull = done + 1;                 // fused: bf16 activation slab landed (ring of XR)
  uint64_t* xempty = xfull + C::XR;           // fused: bf16 slab read by the quantizers
  uint64_t* qready = xempty + C::XR;          // fused: int8 operand of the stage written
  // fused: token scales of a slab written (ring of QR, the depth of the scale ring).  The epilogue
  // cannot wait on qready: the quantizers may finish slab j + STAGES before the epilogue asks for
  // slab j, and a parity wait cannot tell those two phases apart.  They cannot lap this ring (slab
  // j + QR needs the epilogue past slab j, as QR >= STAGES + NBUF).
  uint64_t* sready = qready + C::STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(FUSEDQ ? sready + C::QR : done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* qsx = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(full) + C::BAR_BYTES + C::RING_BYTES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int M = args.M, N = args.N, K = args.K;
  const int KB = K / 128;
  const uint32_t rank = cluster_ctarank(), nrank = cluster_nctarank();
  const int kb0 = (int)((int64_t)KB * rank / nrank), kb1 = (int)((int64_t)KB * (rank + 1) / nrank);
  const int nslab = kb1 - kb0;
  const int n0 = blockIdx.x * 128;

  // The kernel may be launched while the preceding kernel (typically the activation quantizer) is
  // still running: until grid_dependency_wait() it touches no global memory except L2 prefetches of
  // its first weight slabs, so that the weight stream starts as early as possible.  It lets the next
  // kernel launch early in turn (that kernel waits for this one the same way).
  grid_dependents_launch();
  if (warp == EW && lane == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < C::NBUF; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], EW);
    }
    mbar_init(done, 1);
    if constexpr (FUSEDQ) {
      for (int r = 0; r < C::XR; ++r) {
        mbar_init(&xfull[r], 1);
        mbar_init(&xempty[r], C::QALT ? 1 : C::QW);
      }
      for (int st = 0; st < C::STAGES; ++st) mbar_init(&qready[st], C::QALT ? 1 : C::QW);
      for (int q = 0; q < C::QR; ++q) mbar_init(&sready[q], C::QALT ? 1 : C::QW);
    }
    *abort_flag = 0;
    fence_mbar_init();
    for (int j = 0; j < nslab && j < C::STAGES; ++j) tma_prefetch_l2_2d(&tmW, (kb0 + j) * 128, n0);
  }
  if (warp == EW + 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dependency_wait();

  // per-thread results of the epilogue warps: channel: exact int32 dot products; block: fp32 sums
  int32_t acc[MPW];
  float sum[MPW];
#pragma unroll
  for (int m = 0; m < MPW; ++m) {
    acc[m] = 0;
    sum[m] = 0.f;
  }

  if (warp == EW) {
    if constexpr (FUSEDQ) {
     if (lane == 1) {
      // bf16 activation ring (fused): waits only for the quantizers
      uint32_t filled = 0, par = 0;
      bool ok = true;
      for (int j = 0; j < nslab; ++j) {
        const int r = j % C::XR;
        const uint32_t ph = (j / C::XR) & 1;
        if (!mbar_wait(&xempty[r], ph ^ 1, SITE_EMPTY, abort_flag)) { ok = false; break; }
        uint8_t* xb = xring + r * C::XB_BYTES;
        const int kk = (kb0 + j) * 128;
        mbar_arrive_expect_tx(&xfull[r], C::XB_BYTES);
        tma_load_2d(xb, &tmX, &xfull[r], kk, 0);
        tma_load_2d(xb + C::XB_HALF, &tmX, &xfull[r], kk + 64, 0);
        filled |= 1u << r;
        par = (par & ~(1u << r)) | (ph << r);
      }
      if (!ok)
        for (int r = 0; r < C::XR; ++r)
          if (filled & (1u << r)) mbar_wait(&xfull[r], (par >> r) & 1u, SITE_DRAIN, nullptr);
     }
    }
    if (lane == 0) {
      uint32_t filled = 0, par = 0;
      bool ok = true;
      for (int j = 0; j < nslab; ++j) {
        const int s = j % C::STAGES;
        const uint32_t ph = (j / C::STAGES) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, SITE_EMPTY, abort_flag)) { ok = false; break; }
        uint8_t* st = smem + s * C::STAGE_BYTES;
        const int kk = (kb0 + j) * 128;
        if constexpr (FUSEDQ) {          // the int8 activations are written by the quantizers
          mbar_arrive_expect_tx(&full[s], C::W_BYTES);
          tma_load_2d(st, &tmW, &full[s], kk, n0);
        } else {
          mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
          tma_load_2d(st, &tmW, &full[s], kk, n0);
          tma_load_2d(st + C::W_BYTES, &tmX, &full[s], kk, 0);
        }
        filled |= 1u << s;
        par = (par & ~(1u << s)) | (ph << s);
      }
      if (!ok)
        for (int s = 0; s < C::STAGES; ++s)
          if (filled & (1u << s)) mbar_wait(&full[s], (par >> s) & 1u, SITE_DRAIN, nullptr);
    }
  } else if (warp == EW + 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(128, MP);
      for (int j = 0; j < nslab; ++j) {
        const int s = j % C::STAGES;
        const uint32_t ph = (j / C::STAGES) & 1;
        const int b = BLOCKWISE ? j % C::NBUF : 0;
        if (BLOCKWISE) {
          if (!mbar_wait(&tempty[b], ((j / C::NBUF) & 1) ^ 1, SITE_TMEM_EMPTY, abort_flag)) break;
        }
        if (!mbar_wait(&full[s], ph, SITE_FULL, abort_flag)) break;
        if (FUSEDQ && !mbar_wait(&qready[s], ph, SITE_CONVERT, abort_flag)) break;
        tc_fence_after();
        const uint32_t w0 = smem_u32(smem + s * C::STAGE_BYTES);
        const uint32_t x0 = w0 + C::W_BYTES;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t accumulate = BLOCKWISE ? (uint32_t)(kk > 0) : (uint32_t)(j > 0 || kk > 0);
          mma_i8(tmem + b * MP, sw128_kmajor_desc(w0 + kk * 32), sw128_kmajor_desc(x0 + kk * 32), idesc, accumulate);
        }
        tc_commit(&empty[s]);
        if (BLOCKWISE) tc_commit(&tfull[b]);
      }
      if (!BLOCKWISE) {
        // test aid (see g_test_skip_acc_signal): withhold this signal once, when armed
        const bool skip = *reinterpret_cast<volatile unsigned*>(&g_test_skip_acc_signal) != 0 &&
                          atomicExch(&g_test_skip_acc_signal, 0u) != 0;
        if (!skip) tc_commit(&tfull[0]);
      }
      tc_commit(done);
      mbar_wait(done, 0, SITE_DRAIN, nullptr);
    }
  } else if (FUSEDQ && warp >= EW + 2) {
    // quantizers: bf16 activation slab -> int8 operand + per-token group scales (see quantize_slab)
    if constexpr (FUSEDQ) {
      const int qi = warp - (EW + 2);
      // ALT: this warp's slabs are qi, qi + QW, ... (whole slabs); otherwise every slab, its tokens
      for (int j = C::QALT ? qi : 0; j < nslab; j += C::QALT ? C::QW : 1) {
        const int s = j % C::STAGES, r = j % C::XR;
        if (!warp_wait(&xfull[r], (j / C::XR) & 1, SITE_FULL, abort_flag)) break;
        // the int8 operand buffer of stage s is free once the MMAs of slab j - STAGES are done
        if (!warp_wait(&empty[s], ((j / C::STAGES) & 1) ^ 1, SITE_EMPTY, abort_flag)) break;
        quantize_slab<MP, C::QALT ? 1 : C::QW>(xring + r * C::XB_BYTES, smem + s * C::STAGE_BYTES + C::W_BYTES,
                                               qsx + (j % C::QR) * MP, C::QALT ? 0 : qi, lane,
                                               blockIdx.x == 0 ? args.qx_out : nullptr,
                                               blockIdx.x == 0 ? args.qs_out : nullptr, M, K, kb0 + j, args.ld_sx);
        // generic-proxy reads and writes of shared memory before the tensor core and TMA touch it
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&xempty[r]);
          mbar_arrive(&qready[s]);
          mbar_arrive(&sready[j % C::QR]);
        }
      }
    }
  } else {
    // epilogue: thread = weight row n0 + 32 * (warp % 4) + lane (TMEM lane quarter = warp % 4),
    // token columns cb .. cb + MPW - 1
    const int row = (warp & 3) * 32 + lane;
    const int n = n0 + row;
    const int cb = (warp >> 2) * MPW;
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
    if constexpr (!BLOCKWISE) {
      if (nslab > 0 && warp_wait(&tfull[0], 0, SITE_TMEM_FULL, abort_flag)) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < MPW / CH; ++c) {
          uint32_t r[CH];
          tmem_ld_ch<CH>(tmem + lane_addr + cb + c * CH, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < CH; ++i) acc[c * CH + i] = (int32_t)r[i];
        }
      }
    } else {
      // Scale products sx[kb][m] * sw[tile][kb] of a slab go through a per-warp two-slot ring in
      // shared memory: lane l loads token l (and l + 32) of slab j + 1 while slab j is folded, so
      // the global-load latency is hidden behind one slab of streaming.
      const float* swrow = args.sw + (int64_t)(n0 / 128) * KB;
      float* ring = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(full) + C::BAR_BYTES) + warp * 2 * MPW;
      constexpr int PER_LANE = (MPW + 31) / 32;
      float nsx[PER_LANE], nsw = 0.f;
      auto load_scales = [&](int kb) {
        nsw = __ldg(swrow + kb);
        if constexpr (!FUSEDQ) {
#pragma unroll
          for (int i = 0; i < PER_LANE; ++i) {
            const int m = cb + lane + 32 * i;
            nsx[i] = (lane + 32 * i < MPW && m < M) ? __ldg(args.sx + (int64_t)kb * args.ld_sx + m) : 0.f;
          }
        }
      };
      if (nslab > 0) load_scales(kb0);
      for (int j = 0; j < nslab; ++j) {
        const int b = j % C::NBUF;
        const int kb = kb0 + j;
        float* slot = ring + (j & 1) * MPW;
        if constexpr (FUSEDQ) {
          // token scales of slab j come from the quantizer warps through shared memory
          if (!warp_wait(&sready[j % C::QR], (j / C::QR) & 1, SITE_CONVERT, abort_flag)) break;
#pragma unroll
          for (int i = 0; i < PER_LANE; ++i) {
            const int m = cb + lane + 32 * i;
            nsx[i] = (lane + 32 * i < MPW && m < M) ? qsx[(j % C::QR) * MP + m] : 0.f;
          }
        }
#pragma unroll
        for (int i = 0; i < PER_LANE; ++i)
          if (lane + 32 * i < MPW) slot[lane + 32 * i] = nsx[i] * nsw;
        __syncwarp();
        if (j + 1 < nslab) load_scales(kb + 1);
        if (!warp_wait(&tfull[b], (j / C::NBUF) & 1, SITE_TMEM_FULL, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < MPW / CH; ++c) {
          uint32_t r[CH];
          tmem_ld_ch<CH>(tmem + lane_addr + b * MP + cb + c * CH, r);
          tmem_ld_wait();
          if (c == MPW / CH - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[b]);
          }
          // int32 partial P (|P| <= 127^2 * 128 < 2^22) -> exact float.  Up to 64 tokens: the integer
          // add puts P into the mantissa of 1.5 * 2^23 (the bit pattern of 12582912 + P) and a packed
          // subtract removes the offset (full-rate ALU and FMA pipes rather than the conversion
          // unit); at 128 tokens the register budget favours the plain conversion (measured).
#pragma unroll
          for (int i = 0; i < CH; i += 4) {
            const float4 q = *reinterpret_cast<const float4*>(slot + c * CH + i);
            float p[4];
            if constexpr (MPW <= 64) {
              const float2 nb = make_float2(-12582912.0f, -12582912.0f);
              const float2 p01 = __fadd2_rn(make_float2(__uint_as_float(r[i + 0] + 0x4B400000u),
                                                        __uint_as_float(r[i + 1] + 0x4B400000u)), nb);
              const float2 p23 = __fadd2_rn(make_float2(__uint_as_float(r[i + 2] + 0x4B400000u),
                                                        __uint_as_float(r[i + 3] + 0x4B400000u)), nb);
              p[0] = p01.x; p[1] = p01.y; p[2] = p23.x; p[3] = p23.y;
            } else {
#pragma unroll
              for (int t = 0; t < 4; ++t) p[t] = __int2float_rn((int)r[i + t]);
            }
            sum[c * CH + i + 0] = fmaf(p[0], q.x, sum[c * CH + i + 0]);
            sum[c * CH + i + 1] = fmaf(p[1], q.y, sum[c * CH + i + 1]);
            sum[c * CH + i + 2] = fmaf(p[2], q.z, sum[c * CH + i + 2]);
            sum[c * CH + i + 3] = fmaf(p[3], q.w, sum[c * CH + i + 3]);
          }
          if constexpr (DEBUG) {
            if (n < N) {
#pragma unroll
              for (int i = 0; i < CH; ++i)
                if (cb + c * CH + i < M) args.dbg[((int64_t)(cb + c * CH + i) * N + n) * KB + kb] = (int32_t)r[i];
            }
          }
        }
      }
    }
  }

  // ---- output: reduce-scatter over the cluster (every CTA sums rows r % nrank == rank over all
  // ranks, in rank order); without a split the epilogue threads write their rows directly.
  tc_fence_before();
  __syncthreads();
  const int mlim = M < MP ? M : MP;
  auto write_out = [&](int n, int m, float v) {
    if (OUT_F32)
      reinterpret_cast<float*>(args.y)[(int64_t)m * N + n] = v;
    else
      reinterpret_cast<uint16_t*>(args.y)[(int64_t)m * N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
  };
  if (nrank == 1) {
    if (warp < EW) {
      const int n = n0 + (warp & 3) * 32 + lane;
      const int cb = (warp >> 2) * MPW;
      if (n < N) {
        const float swn = BLOCKWISE ? 0.f : __ldg(args.sw + n);
#pragma unroll
        for (int i = 0; i < MPW; ++i) {
          const int m = cb + i;
          if (m < mlim) {
            if constexpr (BLOCKWISE) {
              write_out(n, m, sum[i]);
            } else {
              write_out(n, m, __int2float_rn(acc[i]) * (__ldg(args.sx + m) * swn));
              if constexpr (DEBUG) args.dbg[(int64_t)m * N + n] = acc[i];
            }
          }
        }
      }
    }
  } else {
    // partial tiles in [MP / 4][128 rows] of 4 x 32-bit (the stage buffers are idle now); CTA `rank`
    // owns rows [128 * rank / nrank, 128 * (rank + 1) / nrank) and sums them over all ranks in rank order
    uint4* red = reinterpret_cast<uint4*>(smem);
    if (warp < EW) {
      const int row = (warp & 3) * 32 + lane;
      const int c4 = (warp >> 2) * (MPW / 4);
#pragma unroll
      for (int m4 = 0; m4 < MPW / 4; ++m4) {
        if constexpr (BLOCKWISE)
          red[(c4 + m4) * 128 + row] = make_uint4(__float_as_uint(sum[4 * m4]), __float_as_uint(sum[4 * m4 + 1]),
                                                  __float_as_uint(sum[4 * m4 + 2]), __float_as_uint(sum[4 * m4 + 3]));
        else
          red[(c4 + m4) * 128 + row] = make_uint4(acc[4 * m4], acc[4 * m4 + 1], acc[4 * m4 + 2], acc[4 * m4 + 3]);
      }
    }
    cluster_sync_all();
    const int r0 = (int)(128 * rank / nrank), r1 = (int)(128 * (rank + 1) / nrank);
    const int owned = r1 - r0;
    const int items = owned * ((mlim + 3) >> 2);
    for (int e = threadIdx.x; e < items; e += C::NUM_THREADS) {
      const int m4 = e / owned, row = r0 + (e - m4 * owned);
      const int n = n0 + row;
      const uint32_t la = smem_u32(&red[m4 * 128 + row]);
      if constexpr (BLOCKWISE) {
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
        if (n < N) {
          const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int k = 0; k < 4; ++k)
            if (4 * m4 + k < mlim) write_out(n, 4 * m4 + k, vv[k]);
        }
      } else {
        int4 part[8];
#pragma unroll
        for (int p = 0; p < 8; ++p)
          if (p < (int)nrank) part[p] = ld_dsmem_s32x4(la, (uint32_t)p);
        int4 v = part[0];
#pragma unroll
        for (int p = 1; p < 8; ++p)
          if (p < (int)nrank) {
            v.x += part[p].x; v.y += part[p].y; v.z += part[p].z; v.w += part[p].w;
          }
        if (n < N) {
          const int32_t vv[4] = {v.x, v.y, v.z, v.w};
          const float swn = __ldg(args.sw + n);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int m = 4 * m4 + k;
            if (m < mlim) {
              write_out(n, m, __int2float_rn(vv[k]) * (__ldg(args.sx + m) * swn));
              if constexpr (DEBUG) args.dbg[(int64_t)m * N + n] = vv[k];
            }
          }
        }
      }
    }
    cluster_sync_all();   // no CTA leaves while its shared memory may still be read
  }
  tc_fence_after();
  if (warp == EW + 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace i8q
