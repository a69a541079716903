// CPU oracle, plain C++ version (test infrastructure only).
//
// TEST INFRASTRUCTURE ONLY.  Only tests/ load this library; the product path (the CUDA library and
// its Python binding) never calls it and it includes nothing of the product path.  It restates,
// in plain sequential loops, the same definitions as the numpy oracle (oracle/i8q_oracle.py), which
// the tests pin against golden values, brute force and invariants; the tests then check this
// version against that one element by element.
//
// Sources (cited by page title and section):
//   [R1-INT8]  "DeepSeek R1 INT8 quantization practice on SGLang" (Meituan), section 2.1 (symmetric
//              INT8: compute the scale, quantize, dequantize) and section 2.3 (block-wise: 128x128
//              weight blocks, FP8 -> BF16 -> INT8, per-token-group activations, dequantization per
//              128-wide K slab; channel-wise: per-output-channel and per-token scales, one
//              dequantization after the INT8 GEMM).
//   [FP8-vs-INT8] "FP8与INT8量化对决：DeepSeek模型存储优化的企业实战指南", section 3.2.1
//              (scale = max|x| / 127, q = round(x / scale) clamped to [-127, 127]).
//   [Qwen3-8B-W8A16] "DeepSeek-R1-0528-Qwen3-8B量化版发布", technical details (symmetric
//              group-wise INT8 weights, FP16 activations).
// Readings where the sources are silent: round half to even; a true fp32 division; a zero group
// gets scale 0; E4M3 is the OCP "E4M3FN" encoding; FP8 -> BF16 is one fp32 multiply by the block
// scale, then round to nearest even into bf16; W8A16 group size 128 with exact products.
//
// Build: g++ -O2 -std=c++17 -ffp-contract=off -shared -fPIC (no fast-math: every fp32 operation
// is a single IEEE operation, as the definitions state).
#include <cmath>
#include <cstdint>
#include <cstring>

namespace {

constexpr int kGroup = 128;
constexpr int kQmax = 127;

float bits_to_f32(uint32_t u) {
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}
uint32_t f32_to_bits(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return u;
}

// bf16 bits are the top half of an fp32
float bf16_to_f32(uint16_t b) { return bits_to_f32((uint32_t)b << 16); }

// fp32 -> bf16, round to nearest, ties to even (finite inputs)
uint16_t f32_to_bf16_rne(float x) {
  const uint32_t u = f32_to_bits(x);
  const uint32_t hi = u >> 16, lo = u & 0xFFFFu;
  const bool up = lo > 0x8000u || (lo == 0x8000u && (hi & 1u));
  return (uint16_t)(hi + (up ? 1u : 0u));
}

// IEEE binary16 -> fp32 (exact, subnormals included)
float f16_to_f32(uint16_t h) {
  const int sign = (h >> 15) & 1, e = (h >> 10) & 0x1F, m = h & 0x3FF;
  double v;
  if (e == 0)
    v = std::ldexp((double)m, -24);                       // subnormal: m * 2^-24
  else if (e == 31)
    v = m ? NAN : INFINITY;
  else
    v = std::ldexp(1.0 + m / 1024.0, e - 15);
  return (float)(sign ? -v : v);
}

// FP8 E4M3 ("FN"): bias 7, subnormal m * 2^-9, S.1111.111 is NaN, no infinities
float e4m3_to_f32(uint8_t c) {
  const int sign = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
  double v;
  if (e == 15 && m == 7)
    v = NAN;
  else if (e == 0)
    v = m * std::ldexp(1.0, -9);
  else
    v = (1.0 + m / 8.0) * std::ldexp(1.0, e - 7);
  return (float)(sign ? -v : v);
}

// The quantizer over one group of n fp32 values ([FP8-vs-INT8] section 3.2.1; [R1-INT8] 2.1).
void quantize_group(const float* v, int64_t n, int64_t stride, int8_t* q, int64_t qstride, float* s_out) {
  float a = 0.f;
  for (int64_t i = 0; i < n; ++i) a = std::fmax(a, std::fabs(v[i * stride]));   // exact
  const float s = a / (float)kQmax;                                             // IEEE fp32 divide
  for (int64_t i = 0; i < n; ++i) {
    int code = 0;
    if (s > 0.f) {
      const float r = v[i * stride] / s;                                        // IEEE fp32 divide
      float t = std::nearbyint(r);                                               // half to even
      if (t > kQmax) t = kQmax;
      if (t < -kQmax) t = -kQmax;
      code = (int)t;
    }
    q[i * qstride] = (int8_t)code;
  }
  *s_out = s;
}

}  // namespace

extern "C" {

void ior_bf16_to_f32(const uint16_t* in, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = bf16_to_f32(in[i]);
}
void ior_f32_to_bf16_rne(const float* in, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16_rne(in[i]);
}
void ior_f16_to_f32(const uint16_t* in, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = f16_to_f32(in[i]);
}
void ior_e4m3_to_f32(const uint8_t* in, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_to_f32(in[i]);
}

// G groups of n consecutive fp32 values -> codes [G][n], scales [G]
void ior_quantize_groups(const float* v, int64_t G, int64_t n, int8_t* q, float* s) {
  for (int64_t g = 0; g < G; ++g) quantize_group(v + g * n, n, 1, q + g * n, 1, s + g);
}

// a1: per-token-group (128) quantization of bf16 X [M][K]; sx [M][K/128]  ([R1-INT8] 2.3 block-wise)
void ior_quant_act_token_group(const uint16_t* x, int64_t M, int64_t K, int8_t* xq, float* sx) {
  const int64_t KB = K / kGroup;
  float v[kGroup];
  for (int64_t m = 0; m < M; ++m)
    for (int64_t kb = 0; kb < KB; ++kb) {
      for (int i = 0; i < kGroup; ++i) v[i] = bf16_to_f32(x[m * K + kb * kGroup + i]);
      quantize_group(v, kGroup, 1, xq + m * K + kb * kGroup, 1, sx + m * KB + kb);
    }
}

// a2 (and channel-wise weights): one group per row of a bf16 [R][K]; s [R]  ([R1-INT8] 2.3 channel-wise)
void ior_quant_act_token(const uint16_t* x, int64_t R, int64_t K, int8_t* q, float* s) {
  float* v = new float[K > 0 ? K : 1];
  for (int64_t r = 0; r < R; ++r) {
    for (int64_t k = 0; k < K; ++k) v[k] = bf16_to_f32(x[r * K + k]);
    quantize_group(v, K, 1, q + r * K, 1, s + r);
  }
  delete[] v;
}

// 128x128 block quantization of fp32 W [N][K] (rows of a partial last block: those present);
// sw [ceil(N/128)][K/128]  ([R1-INT8] 2.3 block-wise)
static void quant_weight_block_f32(const float* w, int64_t N, int64_t K, int8_t* wq, float* sw) {
  const int64_t NB = (N + kGroup - 1) / kGroup, KB = K / kGroup;
  float* blk = new float[kGroup * kGroup];
  int8_t* q = new int8_t[kGroup * kGroup];
  for (int64_t i = 0; i < NB; ++i) {
    const int64_t r0 = i * kGroup, r1 = (i + 1) * kGroup < N ? (i + 1) * kGroup : N;
    for (int64_t j = 0; j < KB; ++j) {
      int64_t n = 0;
      for (int64_t r = r0; r < r1; ++r)
        for (int c = 0; c < kGroup; ++c) blk[n++] = w[r * K + j * kGroup + c];
      quantize_group(blk, n, 1, q, 1, sw + i * KB + j);
      n = 0;
      for (int64_t r = r0; r < r1; ++r)
        for (int c = 0; c < kGroup; ++c) wq[r * K + j * kGroup + c] = q[n++];
    }
  }
  delete[] blk;
  delete[] q;
}

void ior_quant_weight_block(const uint16_t* w, int64_t N, int64_t K, int8_t* wq, float* sw) {
  float* f = new float[N * K > 0 ? N * K : 1];
  for (int64_t i = 0; i < N * K; ++i) f[i] = bf16_to_f32(w[i]);
  quant_weight_block_f32(f, N, K, wq, sw);
  delete[] f;
}

// FP8 -> BF16: one fp32 multiply by the block scale, then RNE into bf16  ([R1-INT8] 2.3)
void ior_dequant_fp8_block_to_bf16(const uint8_t* w, const float* sf, int64_t N, int64_t K, uint16_t* out) {
  const int64_t KB = (K + kGroup - 1) / kGroup;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      const float v = e4m3_to_f32(w[n * K + k]) * sf[(n / kGroup) * KB + k / kGroup];
      out[n * K + k] = f32_to_bf16_rne(v);
    }
}

// Block-wise W8A8 GEMM ([R1-INT8] 2.3 block-wise, Fig. 3 left):
//   P[m][n][kb] = sum over the slab (int64, exact);
//   Y[m][n] = sum_kb P * (double)(float)(sx[m][kb] * sw[n/128][kb]), kb ascending, in fp64;
//   T[m][n] = sum_kb |that term|.  P may be null.
void ior_gemm_w8a8_block(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw, int64_t M,
                         int64_t N, int64_t K, double* Y, double* T, int64_t* P) {
  const int64_t KB = K / kGroup;
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      double y = 0.0, t = 0.0;
      for (int64_t kb = 0; kb < KB; ++kb) {
        int64_t p = 0;
        for (int i = 0; i < kGroup; ++i)
          p += (int64_t)xq[m * K + kb * kGroup + i] * (int64_t)wq[n * K + kb * kGroup + i];
        if (P) P[(m * N + n) * KB + kb] = p;
        const float s = sx[m * KB + kb] * sw[(n / kGroup) * KB + kb];        // fp32 product
        const double term = (double)p * (double)s;
        y += term;
        t += std::fabs(term);
      }
      Y[m * N + n] = y;
      T[m * N + n] = t;
    }
}

// Channel-wise W8A8 GEMM ([R1-INT8] 2.3 channel-wise, Fig. 3 right):
//   A = xq wq^T exact in int64; Y = A * sx[m] * sw[n] in fp64 (left to right).
void ior_gemm_w8a8_channel(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw, int64_t M,
                           int64_t N, int64_t K, double* Y, int64_t* A) {
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      int64_t a = 0;
      for (int64_t k = 0; k < K; ++k) a += (int64_t)xq[m * K + k] * (int64_t)wq[n * K + k];
      A[m * N + n] = a;
      Y[m * N + n] = (double)a * (double)sx[m] * (double)sw[n];
    }
}

// W8A16 group-wise GEMM ([Qwen3-8B-W8A16]): Y[m][n] = sum_g s[n][g] * sum_{k in g} x[m][k] * wq[n][k]
// in fp64 (exact products); T = sum_g |s * partial_g|.
void ior_gemm_w8a16_group(const uint16_t* x, const int8_t* wq, const uint16_t* s, int64_t M, int64_t N,
                          int64_t K, double* Y, double* T) {
  const int64_t G = K / kGroup;
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      double y = 0.0, t = 0.0;
      for (int64_t g = 0; g < G; ++g) {
        double part = 0.0;
        for (int i = 0; i < kGroup; ++i)
          part += (double)f16_to_f32(x[m * K + g * kGroup + i]) * (double)wq[n * K + g * kGroup + i];
        const double term = part * (double)f16_to_f32(s[n * G + g]);
        y += term;
        t += std::fabs(term);
      }
      Y[m * N + n] = y;
      T[m * N + n] = t;
    }
}

}  // extern "C"
