// CPU oracle, plain C++ version (test infrastructure only).
//
// TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check and the benchmark's CPU-baseline leg load
// this library (through oracle/ref_cpp.py); the product path (the CUDA library and its Python
// binding) never calls it and it includes nothing of the product path.  It is the oracle the GPU
// parity tests compare with.  It restates, in plain loops, the same definitions as the numpy oracle
// (oracle/i8q_oracle.py); the CPU tests pin both against golden values, brute force, library
// routines and invariants, and check the two against each other element by element.
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
// Build: g++ -O2 -std=c++17 -ffp-contract=off -fopenmp -shared -fPIC (no fast-math: every fp32
// operation is a single IEEE operation, as the definitions state).  OpenMP only distributes
// independent outputs (rows, blocks, sampled positions) over the host cores: every output is
// computed by one thread in the order written here, so results do not depend on the thread count.
#include <omp.h>

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


// Row m of a grouped (MoE) problem belongs to the expert e with off[e] <= m < off[e + 1].
int64_t expert_of_row(const int64_t* off, int64_t E, int64_t m) {
  int64_t e = 0;
  while (e + 1 < E && off[e + 1] <= m) ++e;
  return e;
}

// Exact int64 dot product of two int8 rows of length n.
int64_t dot_i8(const int8_t* a, const int8_t* b, int64_t n) {
  int64_t s = 0;
  for (int64_t i = 0; i < n; ++i) s += (int64_t)a[i] * (int64_t)b[i];
  return s;
}

// Block-wise output (m, n) ([R1-INT8] 2.3 block-wise, Fig. 3 left):
//   P[kb] = exact slab sum; Y = sum_kb P * (double)(float)(sx[m][kb] * sw[n/128][kb]) in fp64,
//   kb ascending; T = sum_kb |term|.  sx_row = sx + m * KB, sw_row = sw + (n / 128) * KB.
void block_output(const int8_t* xrow, const float* sx_row, const int8_t* wrow, const float* sw_row, int64_t K,
                  double* Y, double* T, int64_t* P) {
  const int64_t KB = K / kGroup;
  double y = 0.0, t = 0.0;
  for (int64_t kb = 0; kb < KB; ++kb) {
    const int64_t p = dot_i8(xrow + kb * kGroup, wrow + kb * kGroup, kGroup);
    if (P) P[kb] = p;
    const float s = sx_row[kb] * sw_row[kb];                             // fp32 product
    const double term = (double)p * (double)s;
    y += term;
    t += std::fabs(term);
  }
  *Y = y;
  *T = t;
}

// Channel-wise output (m, n) ([R1-INT8] 2.3 channel-wise, Fig. 3 right): A exact, Y = A * sx * sw in fp64.
void channel_output(const int8_t* xrow, float sxm, const int8_t* wrow, float swn, int64_t K, double* Y, int64_t* A) {
  const int64_t a = dot_i8(xrow, wrow, K);
  *A = a;
  *Y = (double)a * (double)sxm * (double)swn;
}

// Activation / scale formats of the W8A16 GEMM: 0 = fp16, 1 = bf16.
float half_to_f32(uint16_t h, int fmt) { return fmt == 1 ? bf16_to_f32(h) : f16_to_f32(h); }

// W8A16 output (m, n) ([Qwen3-8B-W8A16]): Y = sum_g s[n][g] * sum_{k in g} x[m][k] * wq[n][k] in fp64
// (exact products); T = sum_g |s * partial_g|.
void w8a16_output(const uint16_t* xrow, const int8_t* wrow, const uint16_t* srow, int64_t K, int fmt, double* Y,
                  double* T) {
  const int64_t G = K / kGroup;
  double y = 0.0, t = 0.0;
  for (int64_t g = 0; g < G; ++g) {
    double part = 0.0;
    for (int i = 0; i < kGroup; ++i)
      part += (double)half_to_f32(xrow[g * kGroup + i], fmt) * (double)wrow[g * kGroup + i];
    const double term = part * (double)half_to_f32(srow[g], fmt);
    y += term;
    t += std::fabs(term);
  }
  *Y = y;
  *T = t;
}

}  // namespace

extern "C" {

// Host threads OpenMP will use for the parallel loops below.
int ior_num_threads(void) { return omp_get_max_threads(); }

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
#pragma omp parallel for schedule(static)
  for (int64_t g = 0; g < G; ++g) quantize_group(v + g * n, n, 1, q + g * n, 1, s + g);
}

// a1: per-token-group (128) quantization of bf16 X [M][K]; sx [M][K/128]  ([R1-INT8] 2.3 block-wise)
void ior_quant_act_token_group(const uint16_t* x, int64_t M, int64_t K, int8_t* xq, float* sx) {
  const int64_t KB = K / kGroup;
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    float v[kGroup];
    for (int64_t kb = 0; kb < KB; ++kb) {
      for (int i = 0; i < kGroup; ++i) v[i] = bf16_to_f32(x[m * K + kb * kGroup + i]);
      quantize_group(v, kGroup, 1, xq + m * K + kb * kGroup, 1, sx + m * KB + kb);
    }
  }
}

// a2 (and channel-wise weights): one group per row of a bf16 [R][K]; s [R]  ([R1-INT8] 2.3 channel-wise)
void ior_quant_act_token(const uint16_t* x, int64_t R, int64_t K, int8_t* q, float* s) {
#pragma omp parallel
  {
    float* v = new float[K > 0 ? K : 1];
#pragma omp for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
      for (int64_t k = 0; k < K; ++k) v[k] = bf16_to_f32(x[r * K + k]);
      quantize_group(v, K, 1, q + r * K, 1, s + r);
    }
    delete[] v;
  }
}

// 128x128 block quantization of fp32 W [N][K] (rows of a partial last block: those present);
// sw [ceil(N/128)][K/128]  ([R1-INT8] 2.3 block-wise)
static void quant_weight_block_f32(const float* w, int64_t N, int64_t K, int8_t* wq, float* sw) {
  const int64_t NB = (N + kGroup - 1) / kGroup, KB = K / kGroup;
#pragma omp parallel
  {
    float* blk = new float[kGroup * kGroup];
    int8_t* q = new int8_t[kGroup * kGroup];
#pragma omp for schedule(static) collapse(2)
    for (int64_t i = 0; i < NB; ++i)
      for (int64_t j = 0; j < KB; ++j) {
        const int64_t r0 = i * kGroup, r1 = (i + 1) * kGroup < N ? (i + 1) * kGroup : N;
        int64_t n = 0;
        for (int64_t r = r0; r < r1; ++r)
          for (int c = 0; c < kGroup; ++c) blk[n++] = w[r * K + j * kGroup + c];
        quantize_group(blk, n, 1, q, 1, sw + i * KB + j);
        n = 0;
        for (int64_t r = r0; r < r1; ++r)
          for (int c = 0; c < kGroup; ++c) wq[r * K + j * kGroup + c] = q[n++];
      }
    delete[] blk;
    delete[] q;
  }
}

void ior_quant_weight_block(const uint16_t* w, int64_t N, int64_t K, int8_t* wq, float* sw) {
  float* f = new float[N * K > 0 ? N * K : 1];
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < N * K; ++i) f[i] = bf16_to_f32(w[i]);
  quant_weight_block_f32(f, N, K, wq, sw);
  delete[] f;
}

// FP8 -> BF16: one fp32 multiply by the block scale, then RNE into bf16  ([R1-INT8] 2.3)
void ior_dequant_fp8_block_to_bf16(const uint8_t* w, const float* sf, int64_t N, int64_t K, uint16_t* out) {
  const int64_t KB = (K + kGroup - 1) / kGroup;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      const float v = e4m3_to_f32(w[n * K + k]) * sf[(n / kGroup) * KB + k / kGroup];
      out[n * K + k] = f32_to_bf16_rne(v);
    }
}

// Block-wise W8A8 GEMM ([R1-INT8] 2.3 block-wise, Fig. 3 left): every output by block_output.
// xq [M][K], sx [M][K/128], wq [N][K], sw [ceil(N/128)][K/128]; Y, T [M][N]; P [M][N][K/128] or null.
void ior_gemm_w8a8_block(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw, int64_t M,
                         int64_t N, int64_t K, double* Y, double* T, int64_t* P) {
  const int64_t KB = K / kGroup;
#pragma omp parallel for schedule(static) collapse(2)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n)
      block_output(xq + m * K, sx + m * KB, wq + n * K, sw + (n / kGroup) * KB, K, Y + m * N + n, T + m * N + n,
                   P ? P + (m * N + n) * KB : nullptr);
}

// The same outputs at S sampled positions (ms[i], ns[i]); P [S][K/128] or null.
void ior_gemm_w8a8_block_at(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw, int64_t M,
                            int64_t N, int64_t K, const int64_t* ms, const int64_t* ns, int64_t S, double* Y,
                            double* T, int64_t* P) {
  const int64_t KB = K / kGroup;
  (void)M;
  (void)N;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < S; ++i)
    block_output(xq + ms[i] * K, sx + ms[i] * KB, wq + ns[i] * K, sw + (ns[i] / kGroup) * KB, K, Y + i, T + i,
                 P ? P + i * KB : nullptr);
}

// Channel-wise W8A8 GEMM ([R1-INT8] 2.3 channel-wise, Fig. 3 right): every output by channel_output.
void ior_gemm_w8a8_channel(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw, int64_t M,
                           int64_t N, int64_t K, double* Y, int64_t* A) {
#pragma omp parallel for schedule(static) collapse(2)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n)
      channel_output(xq + m * K, sx[m], wq + n * K, sw[n], K, Y + m * N + n, A + m * N + n);
}

void ior_gemm_w8a8_channel_at(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw, int64_t M,
                              int64_t N, int64_t K, const int64_t* ms, const int64_t* ns, int64_t S, double* Y,
                              int64_t* A) {
  (void)M;
  (void)N;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < S; ++i) channel_output(xq + ms[i] * K, sx[ms[i]], wq + ns[i] * K, sw[ns[i]], K, Y + i, A + i);
}

// Grouped (MoE) W8A8 GEMMs: expert e owns the token rows off[e] .. off[e + 1] - 1 of xq [M][K]
// (off[0] = 0, off[E] = M) and its own weight wq[e] [N][K] with its own scales; every row is the
// dense definition above with its expert's weight.  Channel: sw [E][N].  Block: sw [E][ceil(N/128)][K/128].
void ior_gemm_w8a8_channel_grouped_at(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw,
                                      const int64_t* off, int64_t E, int64_t M, int64_t N, int64_t K,
                                      const int64_t* ms, const int64_t* ns, int64_t S, double* Y, int64_t* A) {
  (void)M;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < S; ++i) {
    const int64_t e = expert_of_row(off, E, ms[i]);
    channel_output(xq + ms[i] * K, sx[ms[i]], wq + (e * N + ns[i]) * K, sw[e * N + ns[i]], K, Y + i, A + i);
  }
}

void ior_gemm_w8a8_block_grouped_at(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw,
                                    const int64_t* off, int64_t E, int64_t M, int64_t N, int64_t K,
                                    const int64_t* ms, const int64_t* ns, int64_t S, double* Y, double* T,
                                    int64_t* P) {
  const int64_t KB = K / kGroup, NB = (N + kGroup - 1) / kGroup;
  (void)M;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < S; ++i) {
    const int64_t e = expert_of_row(off, E, ms[i]);
    block_output(xq + ms[i] * K, sx + ms[i] * KB, wq + (e * N + ns[i]) * K, sw + (e * NB + ns[i] / kGroup) * KB, K,
                 Y + i, T + i, P ? P + i * KB : nullptr);
  }
}

// W8A16 group-wise GEMM ([Qwen3-8B-W8A16]): x [M][K] and s [N][K/128] in format fmt (0 fp16, 1 bf16).
void ior_gemm_w8a16_group_fmt(const uint16_t* x, const int8_t* wq, const uint16_t* s, int64_t M, int64_t N,
                              int64_t K, int64_t fmt, double* Y, double* T) {
  const int64_t G = K / kGroup;
#pragma omp parallel for schedule(static) collapse(2)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n)
      w8a16_output(x + m * K, wq + n * K, s + n * G, K, (int)fmt, Y + m * N + n, T + m * N + n);
}

void ior_gemm_w8a16_group(const uint16_t* x, const int8_t* wq, const uint16_t* s, int64_t M, int64_t N, int64_t K,
                          double* Y, double* T) {
  ior_gemm_w8a16_group_fmt(x, wq, s, M, N, K, 0, Y, T);
}

void ior_gemm_w8a16_group_at(const uint16_t* x, const int8_t* wq, const uint16_t* s, int64_t M, int64_t N, int64_t K,
                             int64_t fmt, const int64_t* ms, const int64_t* ns, int64_t S, double* Y, double* T) {
  const int64_t G = K / kGroup;
  (void)M;
  (void)N;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < S; ++i) w8a16_output(x + ms[i] * K, wq + ns[i] * K, s + ns[i] * G, K, (int)fmt, Y + i, T + i);
}

}  // extern "C"
