// Bandwidth kernels of the quantization steps: per-token-group and per-token activation
// quantization, 128x128 block weight quantization (bf16 input, or FP8-E4M3 input dequantized to
// bf16 first) and per-channel requantization of FP8 weights.
//
// Quantizer ("FP8与INT8量化对决：DeepSeek模型存储优化的企业实战指南", section 3.2.1, applied per group
// as "DeepSeek R1 INT8 quantization practice on SGLang" section 2.3 prescribes):
//   s = max|v| / 127 (IEEE fp32 divide), q = clamp(rint_half_even(v / s), -127, 127) with an
//   IEEE fp32 divide per element; s == 0 gives q == 0.
// All loads are 16-byte vectors; codes are written as packed 8- or 16-byte vectors.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"

namespace i8q {

constexpr unsigned FULL_MASK = 0xFFFFFFFFu;

__device__ __forceinline__ int quant_one(float v, float s) {
  int q = __float2int_rn(__fdiv_rn(v, s));  // IEEE divide, then round half to even
  return max(-127, min(127, q));
}

// 8 bf16 (one 16-byte vector) -> 8 floats
__device__ __forceinline__ void unpack_bf16x8(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ float absmax8(const float (&f)[8]) {
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(f[i]));
  return a;
}

// quantize 8 floats with scale s (s == 0 -> zeros), pack into 8 bytes
__device__ __forceinline__ uint2 quant_pack8(const float (&f)[8], float s) {
  uint32_t lo = 0, hi = 0;
  if (s > 0.f) {
#pragma unroll
    for (int i = 0; i < 4; ++i) lo |= (uint32_t)(quant_one(f[i], s) & 0xFF) << (8 * i);
#pragma unroll
    for (int i = 0; i < 4; ++i) hi |= (uint32_t)(quant_one(f[4 + i], s) & 0xFF) << (8 * i);
  }
  return make_uint2(lo, hi);
}

// ----------------------------------------------------------------------------------------------
// a1: per-token-group (128) activation quantization.
// A half-warp owns one group (16 lanes x 8 bf16); a warp owns two adjacent groups per step and
// keeps two steps in flight.  Scales are written token-contiguous: sx[kb * ld_sx + m].
// ----------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_quant_act_token_group(const uint16_t* __restrict__ x, int64_t M,
                                                               int64_t KB, int64_t ldx,
                                                               int8_t* __restrict__ xq,
                                                               float* __restrict__ sx, int64_t ld_sx) {
  const int lane = threadIdx.x & 31;
  const int half = lane >> 4;
  const int l16 = lane & 15;
  const int64_t G = M * KB;                 // groups
  const int64_t npairs = (G + 1) >> 1;      // warp work items (2 groups each)
  const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (gridDim.x * (int64_t)blockDim.x) >> 5;
  const int64_t K = KB * 128;

  for (int64_t p0 = warp; p0 < npairs; p0 += 2 * nwarps) {
    uint4 v[2];
    int64_t g[2];
    bool ok[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int64_t p = p0 + u * nwarps;
      g[u] = 2 * p + half;
      ok[u] = (p < npairs) && (g[u] < G);
      v[u] = make_uint4(0, 0, 0, 0);
      if (ok[u]) {
        const int64_t m = g[u] / KB, kb = g[u] - (g[u] / KB) * KB;
        v[u] = __ldg(reinterpret_cast<const uint4*>(x + m * ldx + kb * 128 + l16 * 8));
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      float f[8];
      unpack_bf16x8(v[u], f);
      float a = absmax8(f);
#pragma unroll
      for (int off = 8; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(FULL_MASK, a, off));
      const float s = a / 127.0f;
      if (ok[u]) {
        const int64_t m = g[u] / KB, kb = g[u] - (g[u] / KB) * KB;
        *reinterpret_cast<uint2*>(xq + m * K + kb * 128 + l16 * 8) = quant_pack8(f, s);
        if (l16 == 0) sx[kb * ld_sx + m] = s;
      }
    }
  }
}

// ----------------------------------------------------------------------------------------------
// a2: per-token (per-row) quantization, one CTA of 128 threads per row.  The row stays in
// registers between the absmax and the quantize pass when it has at most 128 * CH vectors;
// CH == 0 selects the two-pass variant (second pass re-reads the row, from L2).
// ----------------------------------------------------------------------------------------------
__device__ __forceinline__ float block_absmax_128(float a, float* red /* smem[4] */) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(FULL_MASK, a, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
  __syncthreads();
  a = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  return a;
}

template <int CH>
__global__ void __launch_bounds__(128) k_quant_act_token(const uint16_t* __restrict__ x, int64_t K, int64_t ldx,
                                                         int8_t* __restrict__ xq, float* __restrict__ sx) {
  __shared__ float red[4];
  const int64_t m = blockIdx.x;
  const int64_t nv = K / 8;  // 16-byte vectors in the row
  const uint16_t* xr = x + m * ldx;
  int8_t* qr = xq + m * K;
  float a = 0.f;
  if constexpr (CH > 0) {
    uint4 v[CH];
#pragma unroll
    for (int j = 0; j < CH; ++j) {
      const int64_t c = threadIdx.x + j * 128;
      v[j] = make_uint4(0, 0, 0, 0);
      if (c < nv) v[j] = __ldg(reinterpret_cast<const uint4*>(xr + c * 8));
    }
#pragma unroll
    for (int j = 0; j < CH; ++j) {
      float f[8];
      unpack_bf16x8(v[j], f);
      a = fmaxf(a, absmax8(f));
    }
    a = block_absmax_128(a, red);
    const float s = a / 127.0f;
#pragma unroll
    for (int j = 0; j < CH; ++j) {
      const int64_t c = threadIdx.x + j * 128;
      if (c < nv) {
        float f[8];
        unpack_bf16x8(v[j], f);
        *reinterpret_cast<uint2*>(qr + c * 8) = quant_pack8(f, s);
      }
    }
    if (threadIdx.x == 0) sx[m] = s;
  } else {
    for (int64_t c = threadIdx.x; c < nv; c += 128) {
      float f[8];
      unpack_bf16x8(__ldg(reinterpret_cast<const uint4*>(xr + c * 8)), f);
      a = fmaxf(a, absmax8(f));
    }
    a = block_absmax_128(a, red);
    const float s = a / 127.0f;
    for (int64_t c = threadIdx.x; c < nv; c += 128) {
      float f[8];
      unpack_bf16x8(__ldg(reinterpret_cast<const uint4*>(xr + c * 8)), f);
      *reinterpret_cast<uint2*>(qr + c * 8) = quant_pack8(f, s);
    }
    if (threadIdx.x == 0) sx[m] = s;
  }
}

// ----------------------------------------------------------------------------------------------
// FP8-E4M3 -> bf16 dequantization of 16 bytes: e4m3 -> f16 (exact, hardware convert) -> fp32
// (exact), times the fp32 block scale (one rounding), then rounded to nearest even into bf16
// and widened back to fp32.  Returns the 16 bf16-valued floats.
// ----------------------------------------------------------------------------------------------
__device__ __forceinline__ void dequant_e4m3x16_to_bf16(const uint4& v, float scale, float (&f)[16]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const __nv_fp8x2_storage_t pair = (__nv_fp8x2_storage_t)((w[i] >> (16 * h)) & 0xFFFFu);
      const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
      const float2 ff = __half22float2(*reinterpret_cast<const __half2*>(&hr));
      f[4 * i + 2 * h] = __bfloat162float(__float2bfloat16_rn(ff.x * scale));
      f[4 * i + 2 * h + 1] = __bfloat162float(__float2bfloat16_rn(ff.y * scale));
    }
  }
}

// ----------------------------------------------------------------------------------------------
// a3 / a3': 128x128 block quantization, one CTA of 256 threads per block.
// FP8 == true : input is E4M3 bytes with fp32 block scales sf (dequantized to bf16 first).
// FP8 == false: input is bf16.
// Rows past N (partial last block) are neither read nor written.
// ----------------------------------------------------------------------------------------------
template <bool FP8>
__global__ void __launch_bounds__(256) k_quant_weight_block(const void* __restrict__ w, const float* __restrict__ sf,
                                                            int64_t N, int64_t K, int8_t* __restrict__ wq,
                                                            float* __restrict__ sw) {
  constexpr int EPV = FP8 ? 16 : 8;          // elements per 16-byte vector
  constexpr int VPR = 128 / EPV;             // vectors per block row
  constexpr int VPT = 128 * VPR / 256;       // vectors per thread
  __shared__ float red[8];
  const int64_t KB = K / 128;
  const int64_t nb = blockIdx.x / KB, kb = blockIdx.x - (blockIdx.x / KB) * KB;
  const int64_t r0 = nb * 128;
  const float scale = FP8 ? __ldg(sf + nb * KB + kb) : 1.0f;

  float f[VPT][EPV];
  float a = 0.f;
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int c = threadIdx.x + j * 256;
    const int r = c / VPR, cv = c % VPR;
    const int64_t row = r0 + r;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (row < N) {
      if constexpr (FP8)
        v = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(w) + row * K + kb * 128 + cv * 16));
      else
        v = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(w) + row * K + kb * 128 + cv * 8));
    }
    if constexpr (FP8) {
      dequant_e4m3x16_to_bf16(v, scale, f[j]);
    } else {
      float t[8];
      unpack_bf16x8(v, t);
#pragma unroll
      for (int e = 0; e < 8; ++e) f[j][e] = t[e];
    }
#pragma unroll
    for (int e = 0; e < EPV; ++e) a = fmaxf(a, fabsf(f[j][e]));
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(FULL_MASK, a, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
  __syncthreads();
  a = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) a = fmaxf(a, red[i]);
  const float s = a / 127.0f;

#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int c = threadIdx.x + j * 256;
    const int r = c / VPR, cv = c % VPR;
    const int64_t row = r0 + r;
    if (row >= N) continue;
    int8_t* dst = wq + row * K + kb * 128 + cv * EPV;
    if constexpr (FP8) {
      float lo[8], hi[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) { lo[e] = f[j][e]; hi[e] = f[j][8 + e]; }
      const uint2 a2 = quant_pack8(lo, s), b2 = quant_pack8(hi, s);
      *reinterpret_cast<uint4*>(dst) = make_uint4(a2.x, a2.y, b2.x, b2.y);
    } else {
      float t[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) t[e] = f[j][e];
      *reinterpret_cast<uint2*>(dst) = quant_pack8(t, s);
    }
  }
  if (threadIdx.x == 0) sw[nb * KB + kb] = s;
}

// ----------------------------------------------------------------------------------------------
// FP8 -> BF16 -> INT8 per-output-channel requantization: one CTA of 128 threads per weight row;
// the row's bf16 values are rebuilt in both passes (the second pass re-reads the FP8 bytes).
// ----------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(128) k_requant_fp8_channel(const uint8_t* __restrict__ w, const float* __restrict__ sf,
                                                             int64_t K, int8_t* __restrict__ wq,
                                                             float* __restrict__ sw) {
  __shared__ float red[4];
  const int64_t n = blockIdx.x;
  const int64_t KB = K / 128;
  const uint8_t* wr = w + n * K;
  const float* sfr = sf + (n / 128) * KB;
  const int64_t nv = K / 16;
  float a = 0.f;
  for (int64_t c = threadIdx.x; c < nv; c += 128) {
    float f[16];
    dequant_e4m3x16_to_bf16(__ldg(reinterpret_cast<const uint4*>(wr + c * 16)), __ldg(sfr + (c * 16) / 128), f);
#pragma unroll
    for (int e = 0; e < 16; ++e) a = fmaxf(a, fabsf(f[e]));
  }
  a = block_absmax_128(a, red);
  const float s = a / 127.0f;
  for (int64_t c = threadIdx.x; c < nv; c += 128) {
    float f[16];
    dequant_e4m3x16_to_bf16(__ldg(reinterpret_cast<const uint4*>(wr + c * 16)), __ldg(sfr + (c * 16) / 128), f);
    float lo[8], hi[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) { lo[e] = f[e]; hi[e] = f[8 + e]; }
    const uint2 a2 = quant_pack8(lo, s), b2 = quant_pack8(hi, s);
    *reinterpret_cast<uint4*>(wq + n * K + c * 16) = make_uint4(a2.x, a2.y, b2.x, b2.y);
  }
  if (threadIdx.x == 0) sw[n] = s;
}

}  // namespace i8q
