// Bandwidth kernels of the quantization steps: per-token-group and per-token activation
// quantization, 128x128 block weight quantization (bf16 input, or FP8-E4M3 input dequantized to
// bf16 first) and per-channel requantization of FP8 weights.
//
// Quantizer ("FP8与INT8量化对决：DeepSeek模型存储优化的企业实战指南", section 3.2.1, applied per group
// as "DeepSeek R1 INT8 quantization practice on SGLang" section 2.3 prescribes):
//   s = max|v| / 127 (IEEE fp32 divide), q = clamp(rint_half_even(v / s), -127, 127) where v / s
//   is the correctly rounded fp32 quotient; s == 0 gives q == 0.
//
// How the quotient is formed.  y0 = RN(v * r) with r the hardware reciprocal of s (rcp.approx,
// within 1 ulp), then one FMA correction: e = RN(v - y0 * s) (a single fma), y1 = RN(y0 + e * r)
// (a single fma) - the division scheme of P. Markstein ("Computation of elementary functions on
// the IBM RISC System/6000 processor", 1990).  The quantizer only ever divides a bf16 value v by
// s = RN(a / 127) with a (the absmax) bf16 as well, so the whole input domain is finite up to
// power-of-two scaling: 128 mantissas of a times every bf16 v with |v| <= a.  Over that complete
// domain (both signs, v down to 2^-11 a, below which every code is 0) rint(y1) equals the code of
// the IEEE quotient v / s exactly; the GPU parity tests re-check the domain through the library's
// own entry points.  Groups whose 1/s is not a normal float (|s| < 2^-125 or > 2^125, outside the
// scaling argument) use the IEEE division.  Rounding to nearest even uses z = y1 + 1.5 * 2^23
// (exact for |y1| < 2^22): the fp32 addition rounds y1 to an integer, and the low byte of z's bit
// pattern is that integer's two's-complement int8 code.
//
// Memory side: 16-byte vector loads, several in flight per thread (the next row / block is
// loaded while the current one is quantized), codes written as 8- or 16-byte vectors.  The FP8
// block requantization instead streams whole 128x128 blocks into shared memory with TMA and turns
// each block into a code table (k_requant_fp8_block below).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"

namespace i8q {

constexpr unsigned FULL_MASK = 0xFFFFFFFFu;
constexpr float kRoundMagic = 12582912.0f;          // 1.5 * 2^23

struct QScale {
  float s, r;
  bool r_ok;
};
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ QScale make_qscale(float absmax) {
  QScale q;
  q.s = absmax / 127.0f;                 // IEEE division: the stored scale is exact
  q.r = rcp_approx(q.s);                 // within 1 ulp of 1 / s
  q.r_ok = q.s >= 0x1p-125f && q.s <= 0x1p125f;
  return q;
}

// Reference-exact slow path for one value: IEEE quotient, round half to even, clamp.
__device__ __forceinline__ uint32_t quant_div(float v, float s) {
  const int q = __float2int_rn(__fdiv_rn(v, s));
  return (uint32_t)(max(-127, min(127, q)) & 0xFF);
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// per-halfword unsigned maximum
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
// magnitudes (bf16 bit patterns without sign) of a 16-byte vector, folded to one u16x2 word
__device__ __forceinline__ uint32_t absmax_bits_x8(const uint4& v) {
  const uint32_t m = 0x7FFF7FFFu;
  return max_u16x2(max_u16x2(v.x & m, v.y & m), max_u16x2(v.z & m, v.w & m));
}
__device__ __forceinline__ float bits_to_absmax(uint32_t a) { return __uint_as_float(max(a & 0xFFFFu, a >> 16) << 16); }
// max |x| over the 8 bf16 values of a 16-byte vector (exact; returned as fp32)
__device__ __forceinline__ float absmax_bf16x8(const uint4& v) { return bits_to_absmax(absmax_bits_x8(v)); }

// Codes of two values v: quotient v / s by the corrected reciprocal product, rounded to an integer
// with the magic constant; the low byte of each returned word is the int8 code.
__device__ __forceinline__ float2 code2(float2 v, float2 r2, float2 ns2) {
  const float2 y0 = __fmul2_rn(v, r2);
  const float2 e = __ffma2_rn(y0, ns2, v);
  const float2 y1 = __ffma2_rn(e, r2, y0);
  return __fadd2_rn(y1, make_float2(kRoundMagic, kRoundMagic));
}
__device__ __forceinline__ uint32_t pack4(float2 a, float2 b) {
  const uint32_t t = __byte_perm(__float_as_uint(a.x), __float_as_uint(a.y), 0x0040);
  const uint32_t u = __byte_perm(__float_as_uint(b.x), __float_as_uint(b.y), 0x0040);
  return __byte_perm(t, u, 0x5410);
}

// IEEE-division codes of 8 values, for groups whose 1/s is not a normal float.  Kept out of line
// so that the compiler cannot fold it into the common path as predicated code.
__device__ __noinline__ uint2 quant_bf16x8_div(uint4 v, float s) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t c[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    c[2 * i] = quant_div(bf16lo(w[i]), s);
    c[2 * i + 1] = quant_div(bf16hi(w[i]), s);
  }
  return make_uint2(c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24), c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24));
}

// 8 bf16 values (one 16-byte vector) -> 8 int8 codes.  Warp-collective (a warp vote decides the
// rare extreme-scale path); lanes with `active` false still take part in the vote.
__device__ __forceinline__ uint2 quant_bf16x8(const uint4& v, const QScale& q, bool active) {
  const float2 r2 = make_float2(q.r, q.r);
  const float2 ns2 = make_float2(-q.s, -q.s);
  const float2 z0 = code2(make_float2(bf16lo(v.x), bf16hi(v.x)), r2, ns2);
  const float2 z1 = code2(make_float2(bf16lo(v.y), bf16hi(v.y)), r2, ns2);
  const float2 z2 = code2(make_float2(bf16lo(v.z), bf16hi(v.z)), r2, ns2);
  const float2 z3 = code2(make_float2(bf16lo(v.w), bf16hi(v.w)), r2, ns2);
  uint2 out = make_uint2(pack4(z0, z1), pack4(z2, z3));
  const bool slow = active && q.s > 0.f && !q.r_ok;
  if (__builtin_expect(__any_sync(FULL_MASK, slow), 0)) {
    if (slow) out = quant_bf16x8_div(v, q.s);
  }
  if (!(q.s > 0.f)) out = make_uint2(0, 0);
  return out;
}

// ----------------------------------------------------------------------------------------------
// a1: per-token-group (128) activation quantization.
// Four lanes share a group (each holds 32 of its values as 4 vectors, interleaved so that the four
// lanes read 64 contiguous bytes per load), so a warp step covers 8 groups = 1024 values and the
// per-group scale computation is paid once per 1024 values.  A work item is U consecutive warp
// steps of one row; warps walk the items grid-stride and keep the loads of their next item in
// flight while they quantize the current one.  Scales are token-contiguous: sx[kb * ld_sx + m].
// ----------------------------------------------------------------------------------------------
template <int U>
__global__ void __launch_bounds__(256) k_quant_act_token_group(const uint16_t* __restrict__ x, int M, int KB,
                                                               int64_t ldx, int8_t* __restrict__ xq,
                                                               float* __restrict__ sx, int64_t ld_sx) {
  // Launched with programmatic stream serialization: the launch may overlap the end of the kernel
  // before it (often the GEMM that produced x, or one that still reads the xq / sx being
  // overwritten), so no global memory is touched before that kernel has completed.  A GEMM
  // launched behind this kernel may start its prologue at once.
  grid_dependents_launch();
  grid_dependency_wait();
  const int lane = threadIdx.x & 31;
  const int gl = lane >> 2;                        // group within the warp step (0..7)
  const int sub = lane & 3;                        // lane within the group
  const int warp = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int nwarps = (int)((gridDim.x * blockDim.x) >> 5);
  const int K = KB * 128;
  const int steps = (KB + 7) >> 3;                 // warp steps per row (8 groups each)
  const int nchunks = (steps + U - 1) / U;
  const int items = M * nchunks;
  // vector i of a lane: group elements 8 * (sub + 4 i) .. + 8
  auto load_item = [&](int item, uint4 (&v)[U][4]) {
    const int m = item / nchunks;
    const int st0 = (item - m * nchunks) * U;
    const uint16_t* xr = x + (int64_t)m * ldx + gl * 128 + sub * 8;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int kb = 8 * (st0 + u) + gl;
      const bool ok = item < items && st0 + u < steps && kb < KB;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[u][i] = make_uint4(0, 0, 0, 0);
        if (ok) v[u][i] = __ldg(reinterpret_cast<const uint4*>(xr + (st0 + u) * 1024 + i * 32));
      }
    }
  };
  uint4 cur[U][4], nxt[U][4];
  int item = warp;
  if (item < items) load_item(item, cur);
  for (; item < items; item += nwarps) {
    load_item(item + nwarps, nxt);
    const int m = item / nchunks;
    const int st0 = (item - m * nchunks) * U;
    int8_t* qr = xq + (int64_t)m * K + gl * 128 + sub * 8;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (st0 + u >= steps) break;                     // warp-uniform
      const int kb = 8 * (st0 + u) + gl;
      const bool ok = kb < KB;
      uint32_t ab = max_u16x2(max_u16x2(absmax_bits_x8(cur[u][0]), absmax_bits_x8(cur[u][1])),
                              max_u16x2(absmax_bits_x8(cur[u][2]), absmax_bits_x8(cur[u][3])));
      ab = max_u16x2(ab, __shfl_xor_sync(FULL_MASK, ab, 1));
      ab = max_u16x2(ab, __shfl_xor_sync(FULL_MASK, ab, 2));
      const QScale qs = make_qscale(bits_to_absmax(ab));
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint2 c = quant_bf16x8(cur[u][i], qs, ok);
        if (ok) *reinterpret_cast<uint2*>(qr + (st0 + u) * 1024 + i * 32) = c;
      }
      if (ok && sub == 0) sx[(int64_t)kb * ld_sx + m] = qs.s;
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int i = 0; i < 4; ++i) cur[u][i] = nxt[u][i];
  }
}

// ----------------------------------------------------------------------------------------------
// a2: per-token (per-row) quantization.
// Rows of at most 256 * CH elements: warp per row, the row in registers, shuffle reduction; each
// warp walks rows m, m + nwarps, ...  PREFETCH: the next row is loaded while the current one is
// quantized (used when warps own several rows); otherwise fewer registers give more resident
// warps, so that one launch has every row in flight at once.
// ----------------------------------------------------------------------------------------------
template <int CH, bool PREFETCH>
__global__ void __launch_bounds__(256) k_quant_act_token_warp(const uint16_t* __restrict__ x, int M, int K,
                                                              int64_t ldx, int8_t* __restrict__ xq,
                                                              float* __restrict__ sx) {
  // Launched with programmatic stream serialization: the launch may overlap the end of the kernel
  // before it (often the GEMM that produced x, or one that still reads the xq / sx being
  // overwritten), so no global memory is touched before that kernel has completed.  A GEMM
  // launched behind this kernel may start its prologue at once.
  grid_dependents_launch();
  grid_dependency_wait();
  const int lane = threadIdx.x & 31;
  const int warp = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int nwarps = (int)((gridDim.x * blockDim.x) >> 5);
  const int nv = K / 8;
  uint4 cur[CH], nxt[PREFETCH ? CH : 1];
  auto load_row = [&](int m, uint4 (&v)[CH]) {
    const uint16_t* xr = x + (int64_t)m * ldx;
#pragma unroll
    for (int j = 0; j < CH; ++j) {
      const int c = lane + j * 32;
      v[j] = make_uint4(0, 0, 0, 0);
      if (m < M && c < nv) v[j] = __ldg(reinterpret_cast<const uint4*>(xr + c * 8));
    }
  };
  int m = warp;
  if (m < M) load_row(m, cur);
  for (; m < M; m += nwarps) {
    if constexpr (PREFETCH) load_row(m + nwarps, nxt);
    float a = 0.f;
#pragma unroll
    for (int j = 0; j < CH; ++j) a = fmaxf(a, absmax_bf16x8(cur[j]));
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(FULL_MASK, a, off));
    const QScale qs = make_qscale(a);
    int8_t* qr = xq + (int64_t)m * K;
#pragma unroll
    for (int j = 0; j < CH; ++j) {
      const int c = lane + j * 32;
      const bool ok = c < nv;
      const uint2 code = quant_bf16x8(cur[j], qs, ok);
      if (ok) *reinterpret_cast<uint2*>(qr + c * 8) = code;
    }
    if (lane == 0) sx[m] = qs.s;
    if constexpr (PREFETCH) {
#pragma unroll
      for (int j = 0; j < CH; ++j) cur[j] = nxt[j];
    } else {
      if (m + nwarps < M) load_row(m + nwarps, cur);
    }
  }
}

// Longer rows: CTA of 256 threads per row, two passes (the second re-reads the row from L2).
__device__ __forceinline__ float block_absmax(float a, float* red, int nwarps) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(FULL_MASK, a, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
  __syncthreads();
  a = red[0];
  for (int i = 1; i < nwarps; ++i) a = fmaxf(a, red[i]);
  return a;
}

__global__ void __launch_bounds__(256) k_quant_act_token_cta(const uint16_t* __restrict__ x, int K, int64_t ldx,
                                                             int8_t* __restrict__ xq, float* __restrict__ sx) {
  // Launched with programmatic stream serialization: the launch may overlap the end of the kernel
  // before it (often the GEMM that produced x, or one that still reads the xq / sx being
  // overwritten), so no global memory is touched before that kernel has completed.  A GEMM
  // launched behind this kernel may start its prologue at once.
  grid_dependents_launch();
  grid_dependency_wait();
  __shared__ float red[8];
  const int64_t m = blockIdx.x;
  const int nv = K / 8;
  const uint16_t* xr = x + m * ldx;
  int8_t* qr = xq + m * K;
  float a = 0.f;
  for (int c = threadIdx.x; c < nv; c += 256) a = fmaxf(a, absmax_bf16x8(__ldg(reinterpret_cast<const uint4*>(xr + c * 8))));
  a = block_absmax(a, red, 8);
  const QScale qs = make_qscale(a);
  const int iters = (nv + 255) / 256;                    // block-uniform trip count
  for (int it = 0; it < iters; ++it) {
    const int c = threadIdx.x + it * 256;
    const bool ok = c < nv;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (ok) v = __ldg(reinterpret_cast<const uint4*>(xr + c * 8));
    const uint2 code = quant_bf16x8(v, qs, ok);
    if (ok) *reinterpret_cast<uint2*>(qr + c * 8) = code;
  }
  if (threadIdx.x == 0) sx[m] = qs.s;
}

// ----------------------------------------------------------------------------------------------
// FP8-E4M3 -> BF16 of 16 bytes: e4m3 -> f16 (exact, hardware convert) -> fp32 (exact), times the
// fp32 block scale (one rounding), rounded to nearest even into bf16.  Output: 8 words, each two
// bf16 values (element order preserved).
// ----------------------------------------------------------------------------------------------
__device__ __forceinline__ void e4m3x16_to_bf16x16(const uint4& v, float scale, uint32_t (&o)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  const float2 s2 = make_float2(scale, scale);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const __nv_fp8x2_storage_t pair = (__nv_fp8x2_storage_t)((w[i] >> (16 * h)) & 0xFFFFu);
      const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
      const float2 f = __fmul2_rn(__half22float2(*reinterpret_cast<const __half2*>(&hr)), s2);
      const __nv_bfloat162 b = __float22bfloat162_rn(f);
      o[2 * i + h] = *reinterpret_cast<const uint32_t*>(&b);
    }
  }
}

// ----------------------------------------------------------------------------------------------
// a3': 128x128 block quantization of a bf16 weight, one CTA of 256 threads per block, persistent
// over blocks (the next block's input is loaded while the current one is quantized).  Thread t
// owns 64 values of the block as 8 bf16x8 vectors (vector j: row (t + 256 j) / 16, elements
// (t % 16) * 8 .. +8); rows past N (partial last block) are neither read nor written.
// ----------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_quant_weight_block(const uint16_t* __restrict__ w, int N, int K,
                                                            int8_t* __restrict__ wq, float* __restrict__ sw) {
  __shared__ float red[8];
  const int KB = K / 128;
  const int nblocks = ((N + 127) / 128) * KB;
  auto row_of = [&](int j) { return (int)((threadIdx.x + 256 * j) >> 4); };
  const int col = (int)((threadIdx.x & 15) * 8);
  auto load = [&](int b, uint4 (&raw)[8]) {
    const int nb = b / KB, kb = b - (b / KB) * KB;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int row = nb * 128 + row_of(j);
      raw[j] = make_uint4(0, 0, 0, 0);
      if (b < nblocks && row < N) raw[j] = __ldg(reinterpret_cast<const uint4*>(w + (int64_t)row * K + kb * 128 + col));
    }
  };
  uint4 cur[8], nxt[8];
  int b = blockIdx.x;
  load(b, cur);
  for (; b < nblocks; b += gridDim.x) {
    load(b + gridDim.x, nxt);
    const int nb = b / KB, kb = b - (b / KB) * KB;
    float a = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) a = fmaxf(a, absmax_bf16x8(cur[j]));
    a = block_absmax(a, red, 8);
    const QScale qs = make_qscale(a);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int row = nb * 128 + row_of(j);
      const bool ok = row < N;
      const uint2 c = quant_bf16x8(cur[j], qs, ok);
      if (ok) *reinterpret_cast<uint2*>(wq + (int64_t)row * K + kb * 128 + col) = c;
    }
    if (threadIdx.x == 0) sw[b] = qs.s;
    __syncthreads();                            // red[] is reused by the next block
#pragma unroll
    for (int j = 0; j < 8; ++j) cur[j] = nxt[j];
  }
}

// ----------------------------------------------------------------------------------------------
// a3, TMA-fed: FP8-E4M3 -> BF16 -> INT8 128x128 block requantization, two warps per block.
//
// A CTA holds NP shared-memory stages of one 16 KB FP8 block each; a pair of warps owns a stage
// and streams its blocks (gp, gp + TP, ... for global pair gp of TP) through it with TMA, warp h
// of the pair taking rows 64 h .. 64 h + 63.  The two warps exchange their halves' code maxima
// and, once both have finished with the block, the stage is refilled - two named barriers of 64
// threads per block, no CTA-wide barrier.  Two warps per block keep the time a stage is occupied
// by its quantization short, so that most of the NP stages of an SM are loading at any time.
//
// Block absmax from the codes: E4M3 -> f16 -> fp32 is exact and increasing in the code's magnitude
// bits, and the fp32 product with |sf| and the bf16 rounding are monotone and odd, so the block's
// max |bf16 value| is the dequantization of its largest code magnitude (NaN codes, 0x7F / 0xFF, are
// outside the contract).  Pass 1 only takes byte maxima over the raw block.
//
// Codes by table: inside a block the INT8 code of an element is a function of its FP8 byte alone,
// and odd in it (dequantization and quantization are both odd).  So each warp quantizes the 128
// magnitudes once per block - with the same device arithmetic as the element-wise kernels, so the
// table is bit-identical to what they compute per element - into a 128-byte table (one 32-bit
// word per shared-memory bank: any lookup pattern is conflict-free).  Pass 2 then costs per
// element one byte load from the table plus a few integer operations, instead of the
// dequantization and the corrected quotient; the signs are applied to four packed codes at once.
// A negative sf flips every sign: the table is built with |sf| and the sign bits are XORed.
// Rows past N of the last block row arrive as zeros (TMA bounds fill) and are not written.
// ----------------------------------------------------------------------------------------------
template <int NP>
struct RequantCfg {
  static constexpr int BLOCK_BYTES = 128 * 128;
  static constexpr int NUM_THREADS = 64 * NP;
  static constexpr int TABLE_BYTES = 256;                  // per warp (128 used, 256-byte aligned)
  static constexpr int XCH_BYTES = 8 * NP;                 // per pair: both warps' code maxima
  static constexpr int BAR_BYTES = 8 * NP + 16;
  static constexpr int SMEM_BYTES = NP * BLOCK_BYTES + 2 * NP * TABLE_BYTES + XCH_BYTES + BAR_BYTES + 1024;
  static_assert(NP >= 1 && NP <= 15, "one named barrier per pair (ids 1 .. NP)");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// largest E4M3 magnitude code (0..0x7E) among the 16 bytes of v, folded into two u16x2 maxima
__device__ __forceinline__ void code_absmax16(const uint4& v, uint32_t& hi, uint32_t& lo) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t m = w[i] & 0x7F7F7F7Fu;
    hi = max_u16x2(hi, m);                          // bytes 1 and 3 exact (bytes 0, 2 only break ties)
    lo = max_u16x2(lo, __byte_perm(m, 0u, 0x2404)); // bytes 0 and 2 moved up, zeros below
  }
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
__device__ __forceinline__ uint32_t lds_u8(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// Four codes of the FP8 word w from the magnitude table at shared address tbl (256-byte aligned):
// table codes P (bytes 0..127), then negation of the bytes whose sign (w's, XOR sfm) is set and
// whose code is not 0: -q = (q ^ 0xFF) + 1, carry-free for q >= 1.
__device__ __forceinline__ uint32_t table_codes4(uint32_t w, uint32_t tbl, uint32_t sfm) {
  const uint32_t wm = w & 0x7F7F7F7Fu;
  const uint32_t c0 = lds_u8(prmt(wm, tbl, 0x7650u)), c1 = lds_u8(prmt(wm, tbl, 0x7651u));
  const uint32_t c2 = lds_u8(prmt(wm, tbl, 0x7652u)), c3 = lds_u8(prmt(wm, tbl, 0x7653u));
  const uint32_t P = prmt(prmt(c0, c1, 0x0040u), prmt(c2, c3, 0x0040u), 0x5410u);
  const uint32_t nn = (P + 0x7F7F7F7Fu) & (w ^ sfm) & 0x80808080u;   // negative, non-zero code
  const uint32_t mf = prmt(nn, 0u, 0xBA98u);                         // 0xFF in those bytes
  return (P ^ mf) + (nn >> 7);
}

__device__ __forceinline__ void pair_sync(int id) { asm volatile("bar.sync %0, 64;" ::"r"(id) : "memory"); }

template <int NP>
__global__ void __launch_bounds__(RequantCfg<NP>::NUM_THREADS, 1)
    k_requant_fp8_block(const __grid_constant__ CUtensorMap tmW, const float* __restrict__ sf, int N, int K,
                        int8_t* __restrict__ wq, float* __restrict__ sw) {
  using C = RequantCfg<NP>;
  constexpr uint32_t kFailed = 0xFFFFFFFFu;                // exchange word of a warp whose wait expired
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tables = smem + NP * C::BLOCK_BYTES;
  volatile uint32_t* xch = reinterpret_cast<volatile uint32_t*>(tables + 2 * NP * C::TABLE_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(tables + 2 * NP * C::TABLE_BYTES + C::XCH_BYTES);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(full + NP);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p = warp >> 1, h = warp & 1;
  const int KB = K / 128;
  const int nblocks = ((N + 127) / 128) * KB;
  const int TP = gridDim.x * NP;
  const int gp = blockIdx.x * NP + p;
  // Launched with programmatic stream serialization: the set-up below overlaps the end of the
  // kernel before it, and no global memory is touched before that kernel has completed.
  grid_dependents_launch();
  if (threadIdx.x == 0) {
    for (int q = 0; q < NP; ++q) mbar_init(&full[q], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  grid_dependency_wait();
  uint64_t* bar = &full[p];
  uint8_t* stage = smem + p * C::BLOCK_BYTES;
  const uint8_t* half = stage + h * (C::BLOCK_BYTES / 2);
  uint32_t* table = reinterpret_cast<uint32_t*>(tables + warp * C::TABLE_BYTES);
  const uint32_t tbl = smem_u32(table);
  volatile uint32_t* xs = xch + 2 * p;
  const bool issuer = h == 0 && lane == 0;
  const int nmine = gp < nblocks ? (nblocks - 1 - gp) / TP + 1 : 0;
  auto issue = [&](int i) {                       // this pair's i-th block into its stage
    const int b = gp + i * TP;
    const int nb = b / KB, kb = b - nb * KB;
    mbar_arrive_expect_tx(bar, C::BLOCK_BYTES);
    tma_load_2d(stage, &tmW, bar, kb * 128, nb * 128);
  };
  if (issuer && nmine > 0) issue(0);
  int i = 0;
  for (; i < nmine; ++i) {
    const int b = gp + i * TP;
    const int nb = b / KB, kb = b - nb * KB;
    const float scale = __ldg(sf + b);
    const bool ok = warp_wait(bar, i & 1, SITE_FULL, abort_flag);
    // pass 1: largest code magnitude of this warp's half
    uint32_t m = 0;
    if (ok) {
      uint32_t hi = 0, lo = 0;
#pragma unroll 8
      for (int t = 0; t < 16; ++t) code_absmax16(*reinterpret_cast<const uint4*>(half + (t * 32 + lane) * 16), hi, lo);
      m = max_u16x2(hi, lo);
      m = max(m >> 24, (m >> 8) & 0xFFu);
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) m = max(m, __shfl_xor_sync(FULL_MASK, m, off));
    }
    if (lane == 0) xs[h] = ok ? m : kFailed;
    pair_sync(1 + p);
    const uint32_t m0 = xs[0], m1 = xs[1];
    if (m0 == kFailed || m1 == kFailed) break;    // both warps leave together
    m = max(m0, m1);
    const float asf = fabsf(scale);
    const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)m, __NV_E4M3);
    const float cmax = __half2float(__low2half(*reinterpret_cast<const __half2*>(&hr)));
    const QScale qs = make_qscale(__bfloat162float(__float2bfloat16_rn(__fmul_rn(cmax, asf))));
    // the codes of magnitudes 4 lane .. 4 lane + 3 (element-wise arithmetic, |sf|)
    {
      uint32_t o[8];
      e4m3x16_to_bf16x16(make_uint4(0x03020100u + 0x04040404u * (uint32_t)lane, 0u, 0u, 0u), asf, o);
      table[lane] = quant_bf16x8(make_uint4(o[0], o[1], 0u, 0u), qs, true).x;
    }
    __syncwarp();
    const uint32_t sfm = __float_as_uint(scale) >> 31 ? 0x80808080u : 0u;
    // pass 2: 16 codes per lane per step; a warp step covers 4 rows of 128 bytes
    const int row0 = nb * 128 + h * 64;
    int8_t* dst0 = wq + (int64_t)row0 * K + kb * 128 + (lane & 7) * 16;
#pragma unroll 4
    for (int t = 0; t < 16; ++t) {
      const int row = t * 4 + (lane >> 3);
      const uint4 v = *reinterpret_cast<const uint4*>(half + (t * 32 + lane) * 16);
      const uint4 c = make_uint4(table_codes4(v.x, tbl, sfm), table_codes4(v.y, tbl, sfm),
                                 table_codes4(v.z, tbl, sfm), table_codes4(v.w, tbl, sfm));
      if (row0 + row < N) *reinterpret_cast<uint4*>(dst0 + (int64_t)row * K) = c;
    }
    if (issuer) sw[b] = qs.s;
    // both halves read (generic proxy) before TMA writes the stage again
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    pair_sync(1 + p);
    if (issuer && i + 1 < nmine) issue(i + 1);
  }
  // a wait expired: the block in flight lands before the CTA exits
  if (i < nmine && issuer) mbar_wait(bar, i & 1, SITE_DRAIN, nullptr);
}

// ----------------------------------------------------------------------------------------------
// FP8 -> BF16 -> INT8 per-output-channel requantization: one CTA of 256 threads per weight row;
// the second pass rebuilds the bf16 values from the FP8 bytes (re-read from L2).
// ----------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_requant_fp8_channel(const uint8_t* __restrict__ w, const float* __restrict__ sf,
                                                             int K, int8_t* __restrict__ wq, float* __restrict__ sw) {
  __shared__ float red[8];
  const int64_t n = blockIdx.x;
  const int KB = K / 128;
  const uint8_t* wr = w + n * K;
  const float* sfr = sf + (n / 128) * KB;
  const int nv = K / 16;
  float a = 0.f;
  for (int c = threadIdx.x; c < nv; c += 256) {
    uint32_t o[8];
    e4m3x16_to_bf16x16(__ldg(reinterpret_cast<const uint4*>(wr + c * 16)), __ldg(sfr + (c * 16) / 128), o);
    a = fmaxf(a, absmax_bf16x8(make_uint4(o[0], o[1], o[2], o[3])));
    a = fmaxf(a, absmax_bf16x8(make_uint4(o[4], o[5], o[6], o[7])));
  }
  a = block_absmax(a, red, 8);
  const QScale qs = make_qscale(a);
  const int iters = (nv + 255) / 256;
  for (int it = 0; it < iters; ++it) {
    const int c = threadIdx.x + it * 256;
    const bool ok = c < nv;
    uint32_t o[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (ok) e4m3x16_to_bf16x16(__ldg(reinterpret_cast<const uint4*>(wr + c * 16)), __ldg(sfr + (c * 16) / 128), o);
    const uint2 lo = quant_bf16x8(make_uint4(o[0], o[1], o[2], o[3]), qs, ok);
    const uint2 hi = quant_bf16x8(make_uint4(o[4], o[5], o[6], o[7]), qs, ok);
    if (ok) *reinterpret_cast<uint4*>(wq + n * K + c * 16) = make_uint4(lo.x, lo.y, hi.x, hi.y);
  }
  if (threadIdx.x == 0) sw[n] = qs.s;
}

}  // namespace i8q
