/*
 * i8q.h — C ABI of libi8q.so: symmetric INT8 activation-quantized GEMM on B200 (sm_100a).
 *
 * Method (cited by page title and section):
 *   [R1-INT8]  "DeepSeek R1 INT8 quantization practice on SGLang" (Meituan), section 2.1
 *              (symmetric INT8: compute the scale, quantize, dequantize) and section 2.3
 *              (block-wise: 128x128 weight blocks, FP8 -> BF16 -> INT8, activations quantized
 *              online per token-group, dequantization inside the INT8 matmul for every K block;
 *              channel-wise: one scale per output channel, per-token activation scales, one
 *              dequantization after the INT8 GEMM; Fig. 3).
 *   [FP8-vs-INT8] "FP8与INT8量化对决：DeepSeek模型存储优化的企业实战指南", section 3.2.1
 *              (scale = max|x| / 127, q = round(x / scale) clamped to [-127, 127]).
 *   [Qwen3-8B-W8A16] "DeepSeek-R1-0528-Qwen3-8B量化版发布", technical details section
 *              (symmetric group-wise INT8 weights, FP16 activations).
 *
 * Quantizer used by every quantizing entry point: for a group v, a = max|v| (fp32),
 * s = a / 127 (IEEE fp32 division), q = clamp(round_half_even(v / s), -127, 127) with a true
 * IEEE fp32 division; a group with a = 0 gets s = 0 and q = 0.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The library never
 *     allocates, frees or retains user memory and keeps no pointer after the call returns.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  Nothing synchronizes except i8q_status_check.
 *   - Row-major layouts; "[A][B]" means B is the contiguous index.
 *   - Every pointer must be 16-byte aligned (I8Q_ERR_ALIGN otherwise).
 *   - K must be a multiple of 128 where stated (I8Q_ERR_SHAPE otherwise); negative sizes give
 *     I8Q_ERR_SHAPE; a zero M, N or K is a valid empty problem (see each call).
 *   - The first call on a device checks that it is compute capability 10.0 (B200);
 *     other devices give I8Q_ERR_UNSUPPORTED.
 *   - Errors never cross the ABI as exceptions; a failed launch gives I8Q_ERR_CUDA
 *     (i8q_last_error_string() then describes it).
 *   - Device-side waits are bounded: a wait that expires sets a device error word and the
 *     kernel returns early; i8q_status_check() reports it as I8Q_ERR_TIMEOUT.
 */
#ifndef I8Q_H
#define I8Q_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  I8Q_OK = 0,
  I8Q_ERR_NULL = 1,         /* a required pointer is NULL */
  I8Q_ERR_SHAPE = 2,        /* a size or leading dimension is invalid */
  I8Q_ERR_ALIGN = 3,        /* a pointer is not 16-byte aligned */
  I8Q_ERR_DTYPE = 4,        /* an enum argument is out of range */
  I8Q_ERR_CUDA = 5,         /* a CUDA runtime / driver call failed */
  I8Q_ERR_TIMEOUT = 6,      /* a bounded device wait expired (reported by i8q_status_check) */
  I8Q_ERR_UNSUPPORTED = 7   /* the current device is not sm_100 */
} i8q_status;

typedef enum { I8Q_OUT_BF16 = 0, I8Q_OUT_FP32 = 1 } i8q_out_dtype;

/*
 * Online per-token-group activation quantization (block-wise scheme).
 * [R1-INT8] section 2.3, block-wise paragraph: every token's vector is split into groups of
 * 128 consecutive K and each group is quantized with its own scale.
 *   x_bf16 : [M][ldx] bf16 bit patterns, K valid columns; ldx >= K, ldx % 8 == 0.
 *   M, K   : M >= 0; K >= 0, K % 128 == 0.
 *   xq     : [M][K] int8 output.
 *   sx     : [K/128][ld_sx] fp32 output; sx[kb * ld_sx + m] is the scale of token m, group kb
 *            (token-contiguous, the layout i8q_gemm_w8a8_block reads); ld_sx >= M, ld_sx % 4 == 0.
 * M == 0 or K == 0 is a no-op.
 */
i8q_status i8q_quant_act_token_group(const uint16_t* x_bf16, int64_t M, int64_t K, int64_t ldx,
                                     int8_t* xq, float* sx, int64_t ld_sx, void* stream);

/*
 * Online per-token activation quantization (channel-wise scheme); also the channel-wise weight
 * quantizer (one scale per output channel = per row of W [N][K]).
 * [R1-INT8] section 2.3, channel-wise paragraph.
 *   x_bf16 : [M][ldx] bf16, K valid columns; ldx >= K, ldx % 8 == 0.
 *   M, K   : M >= 0; K >= 0, K % 8 == 0 (rows move as 16-byte vectors of 8 values; every K of
 *            the pages' layers is a multiple of 128).
 *   xq     : [M][K] int8 output.   sx : [M] fp32 output (one scale per row).
 * M == 0 is a no-op; K == 0 writes sx = 0.
 */
i8q_status i8q_quant_act_token(const uint16_t* x_bf16, int64_t M, int64_t K, int64_t ldx,
                               int8_t* xq, float* sx, void* stream);

/*
 * Block-wise 128x128 weight quantization of a BF16 weight.
 * [R1-INT8] section 2.3, block-wise paragraph (quantization within 128x128 blocks).
 *   w_bf16 : [N][K] bf16;  N >= 0;  K >= 0, K % 128 == 0;  ceil(N/128) * K/128 < 2^30 blocks.
 *   wq     : [N][K] int8 output.
 *   sw     : [ceil(N/128)][K/128] fp32 output; a partial last row-block takes the absmax over
 *            the rows present.
 */
i8q_status i8q_quant_weight_block(const uint16_t* w_bf16, int64_t N, int64_t K,
                                  int8_t* wq, float* sw, void* stream);

/*
 * Offline FP8-E4M3 -> BF16 -> INT8 128x128 block requantization.
 * [R1-INT8] section 2.3, block-wise paragraph: DeepSeek ships FP8 weights with one fp32 scale
 * per 128x128 block and no BF16 weights, so the weights are dequantized to BF16 first
 * (bf16 = round_to_nearest_even(fp32(e4m3) * sf), one fp32 multiply) and then block-quantized.
 * E4M3 is the OCP "E4M3FN" encoding (no infinities; NaN codes are outside the contract).
 *   w_e4m3 : [N][K] bytes;   sf : [ceil(N/128)][K/128] finite fp32 block scales of the FP8 tensor.
 *   N >= 0;  K >= 0, K % 128 == 0;  ceil(N/128) * K/128 < 2^30 blocks (I8Q_ERR_SHAPE otherwise).
 *   wq     : [N][K] int8 output;   sw : [ceil(N/128)][K/128] fp32 output.
 */
i8q_status i8q_requant_fp8_to_int8_block(const uint8_t* w_e4m3, const float* sf, int64_t N, int64_t K,
                                         int8_t* wq, float* sw, void* stream);

/*
 * Offline FP8-E4M3 -> BF16 -> INT8 per-output-channel requantization.
 * [R1-INT8] section 2.3, channel-wise paragraph (FP8 weights dequantized to BF16, then
 * quantized to INT8 channel by channel).
 *   w_e4m3 : [N][K] bytes;   sf : [ceil(N/128)][K/128] fp32;  N >= 0;  K >= 0, K % 128 == 0.
 *   wq     : [N][K] int8 output;   sw : [N] fp32 output (one scale per output channel).
 */
i8q_status i8q_requant_fp8_to_int8_channel(const uint8_t* w_e4m3, const float* sf, int64_t N, int64_t K,
                                           int8_t* wq, float* sw, void* stream);

/*
 * Block-wise W8A8 GEMM: y = x w^T with a dequantization per 128-wide K slab.
 * [R1-INT8] section 2.3, block-wise paragraph and Fig. 3 (left): because activation groups and
 * weight blocks carry different scales, every slab's exact int32 partial sum
 * P[m][n][kb] = sum_{k in slab kb} xq[m][k] * wq[n][k] is scaled by sx[m][kb] * sw[n/128][kb]
 * (fp32 product) and accumulated in fp32; the result is cast once at the end.
 *   xq  : [M][K] int8;   sx : [K/128][ld_sx] fp32 (token-contiguous, as written by
 *         i8q_quant_act_token_group); ld_sx >= M, ld_sx % 4 == 0.
 *   wq  : [N][K] int8;   sw : [ceil(N/128)][K/128] fp32.
 *   M >= 0; N >= 0 (any N: a partial last weight block shares that block's scale and the
 *   output columns past N are never written); K >= 0, K % 128 == 0.
 *   y   : [M][N], bf16 (out == I8Q_OUT_BF16, round to nearest even) or fp32 (I8Q_OUT_FP32).
 *   debug_partials : NULL, or [M][N][K/128] int32 receiving every P (checking aid; slower).
 * M == 0 or N == 0 is a no-op; K == 0 writes y = 0.
 */
i8q_status i8q_gemm_w8a8_block(const int8_t* xq, const float* sx, int64_t ld_sx,
                               const int8_t* wq, const float* sw,
                               int64_t M, int64_t N, int64_t K,
                               void* y, i8q_out_dtype out, int32_t* debug_partials, void* stream);

/*
 * Block-wise W8A8 GEMM with the online per-token-group activation quantization fused in
 * (decode batches).  [R1-INT8] section 2.3, block-wise paragraph: the activations are quantized
 * online per token-group of 128 and consumed by the INT8 matmul with a dequantization per K slab.
 * The result is the composition i8q_quant_act_token_group followed by i8q_gemm_w8a8_block, and is
 * bit-identical to it (the same quantizer code runs inside the GEMM, on the activation slab each
 * CTA stages next to its weight slab), without the separate launch and the HBM round trip of the
 * int8 activations.
 *   x_bf16 : [M][ldx] bf16, K valid columns; ldx >= K, ldx % 8 == 0.
 *   wq, sw : as i8q_gemm_w8a8_block ([N][K] int8, [ceil(N/128)][K/128] fp32).
 *   1 <= M <= 16: decode batches only (I8Q_ERR_SHAPE above).  Every N tile quantizes the
 *   activation slabs it reads, so the in-GEMM work grows with M: up to 16 tokens it is hidden
 *   behind the weight stream (measured, DeepSeek-R1 up-projection), beyond that the separate
 *   quantizer is cheaper; use i8q_quant_act_token_group + i8q_gemm_w8a8_block there.
 *   N >= 0 (any N); K >= 0, K % 128 == 0.
 *   y : [M][N] bf16 or fp32 (out).
 *   xq_out, sx_out : NULL, or receive the quantized activations exactly as
 *            i8q_quant_act_token_group writes them ([M][K] int8; [K/128][ld_sx] fp32,
 *            ld_sx >= M, ld_sx % 4 == 0); ld_sx is ignored when sx_out is NULL.
 * M == 0 or N == 0 is a no-op; K == 0 writes y = 0.
 */
i8q_status i8q_gemm_w8a8_block_fused_quant(const uint16_t* x_bf16, int64_t ldx, const int8_t* wq,
                                           const float* sw, int64_t M, int64_t N, int64_t K, void* y,
                                           i8q_out_dtype out, int8_t* xq_out, float* sx_out, int64_t ld_sx,
                                           void* stream);

/*
 * Channel-wise W8A8 GEMM: y[m][n] = bf16( float(A[m][n]) * (sx[m] * sw[n]) ),
 * A = xq wq^T accumulated exactly in int32.
 * [R1-INT8] section 2.3, channel-wise paragraph and Fig. 3 (right): a single dequantization
 * after the INT8 GEMM with the per-token and per-output-channel scales.
 *   xq : [M][K] int8;  sx : [M] fp32;  wq : [N][K] int8;  sw : [N] fp32.
 *   M >= 0; N >= 0 (any N); K >= 0, K % 128 == 0 (127^2 * K < 2^31 keeps int32 exact).
 *   y_bf16 : [M][N] bf16 output (round to nearest even).
 *   debug_acc : NULL, or [M][N] int32 receiving A (checking aid).
 * M == 0 or N == 0 is a no-op; K == 0 writes y = 0.
 */
i8q_status i8q_gemm_w8a8_channel(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw,
                                 int64_t M, int64_t N, int64_t K,
                                 uint16_t* y_bf16, int32_t* debug_acc, void* stream);

/*
 * Grouped (MoE) W8A8 GEMMs: many experts, each with its own quantized weight and scales, over
 * one batch of token rows sorted by expert.
 * [R1-INT8] section 2.3 (the block-wise and channel-wise schemes above, applied per expert);
 * [FP8-vs-INT8] section 3.1.2 (the MoE expert weights of DeepSeek models are quantized like the
 * dense ones).  Row m of xq belongs to the expert e with off[e] <= m < off[e + 1]; its output row
 * is the dense GEMM of that row with expert e's weight:
 *   channel: y[m][n] = bf16( float(A) * (sx[m] * sw[e][n]) ),  A = sum_k xq[m][k] * wq[e][n][k];
 *   block:   y[m][n] = sum_kb P * (sx[m][kb] * sw[e][n/128][kb]) in fp32, as i8q_gemm_w8a8_block.
 *   xq  : [M][K] int8, rows sorted by expert.
 *   sx  : channel [M] fp32; block [K/128][ld_sx] fp32 (token-contiguous, ld_sx >= M, % 4 == 0).
 *   wq  : [E][N][K] int8 (the experts' weights stacked);  sw : channel [E][N]; block
 *         [E][ceil(N/128)][K/128] fp32.
 *   expert_offsets : DEVICE array of E + 1 int32, non-decreasing, off[0] = 0, off[E] = M (routing
 *         is device data: the host need not know the per-expert counts; an expert may have none).
 *         The kernel clamps the offsets to be non-decreasing within [0, M], so rows outside
 *         [off[0], off[E]) are never written and no row outside [0, M) is ever touched.
 *   1 <= E <= 1024; E * N < 2^31; N >= 0 (any N); K >= 0, K % 128 == 0; M >= 0.
 *   y : [M][N] bf16 (channel) or bf16 / fp32 by `out` (block).
 *   debug_acc / debug_partials : NULL or as in the dense calls ([M][N], [M][N][K/128]).
 * M == 0 or N == 0 is a no-op; K == 0 writes y = 0.
 */
i8q_status i8q_gemm_w8a8_channel_grouped(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw,
                                         const int32_t* expert_offsets, int64_t E, int64_t M, int64_t N,
                                         int64_t K, uint16_t* y_bf16, int32_t* debug_acc, void* stream);
i8q_status i8q_gemm_w8a8_block_grouped(const int8_t* xq, const float* sx, int64_t ld_sx, const int8_t* wq,
                                       const float* sw, const int32_t* expert_offsets, int64_t E, int64_t M,
                                       int64_t N, int64_t K, void* y, i8q_out_dtype out,
                                       int32_t* debug_partials, void* stream);

/*
 * W8A16 group-wise weight-only GEMM.
 * [Qwen3-8B-W8A16], technical details: Linear weights are symmetric group-wise INT8, the
 * activations stay FP16.  Group size 128 along K:
 *   y[m][n] = fp16( sum_g s[n][g] * sum_{k in g} x[m][k] * wq[n][k] )
 * with the products exact in fp32 and fp32 accumulation (the dequantized weight is never rounded).
 *   x_f16 : [M][K] fp16;  wq : [N][K] int8;  s_f16 : [N][K/128] fp16 group scales.
 *   M >= 0 (decode batches of up to 64 tokens run one token tile with K split over a cluster;
 *   larger batches run 128-token tiles, ceil(M / 128) < 65536); N >= 0 (any N);
 *   K >= 0, K % 128 == 0.
 *   y_f16 : [M][N] fp16 output (round to nearest even).
 * M == 0 or N == 0 is a no-op; K == 0 writes y = 0.
 */
i8q_status i8q_gemm_w8a16_group(const uint16_t* x_f16, const int8_t* wq, const uint16_t* s_f16,
                                int64_t M, int64_t N, int64_t K, uint16_t* y_f16, void* stream);

/*
 * The same W8A16 group-wise GEMM for a BF16 model: bf16 activations, bf16 group scales, bf16
 * output (round to nearest even).  The weight-only INT8 path of "DeepSeek-R1-Distill-Llama-8B
 * 模型量化实战" section 2.1 (TensorRT-LLM, weights INT8, activations kept in 16-bit) with the group
 * scales of [Qwen3-8B-W8A16].  int8 -> bf16 is exact (|q| <= 127 needs 7 bits); products are
 * exact in fp32.  Arguments, layouts and limits as i8q_gemm_w8a16_group.
 */
i8q_status i8q_gemm_w8a16_group_bf16(const uint16_t* x_bf16, const int8_t* wq, const uint16_t* s_bf16,
                                     int64_t M, int64_t N, int64_t K, uint16_t* y_bf16, void* stream);

/* Human-readable name of a status code (static storage). */
const char* i8q_status_string(i8q_status status);

/* Text of the last CUDA error seen by this thread inside the library ("" if none). */
const char* i8q_last_error_string(void);

/*
 * Synchronizes `stream`, then reads and clears the current device's error word.
 * Returns I8Q_ERR_TIMEOUT if a bounded device wait expired since the last check,
 * I8Q_ERR_CUDA if the stream reported an error, I8Q_OK otherwise.
 */
i8q_status i8q_status_check(void* stream);

/*
 * Test aids for the bounded device waits (no counterpart in the pages; used by the test suite).
 * i8q_test_set_wait_limit_ns: limit of every pipeline wait on the current device, in ns
 *   (0 restores the default of 2 s).  Waits that drain copies already in flight keep 2 s.
 * i8q_test_skip_accumulator_signal: armed != 0 makes the next decode-size (M <= 128) channel-wise
 *   W8A8 GEMM launch withhold one accumulator-ready signal in one CTA, so that its epilogue's wait
 *   expires (after the limit above), the kernel returns early, and i8q_status_check() reports
 *   I8Q_ERR_TIMEOUT; the output of that launch is undefined.  armed == 0 disarms it.
 * Both write a device variable synchronously (cudaMemcpyToSymbol); do not call them while
 * kernels of this library are running.
 */
i8q_status i8q_test_set_wait_limit_ns(uint64_t ns);
i8q_status i8q_test_skip_accumulator_signal(int armed);

/* Library version, as major * 10000 + minor * 100 + patch. */
int i8q_version(void);

#ifdef __cplusplus
}
#endif

#endif /* I8Q_H */
