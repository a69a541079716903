"""CPU oracle for symmetric INT8 activation-quantized GEMM (test infrastructure).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The product path
(the CUDA library and its Python binding) never calls it, and this module
never calls the product path: the two share no code.

Everything here is the plain definition of what the method computes, written
out with numpy in the order the sources state it.  Library primitives used as
single steps: numpy fp32 division and multiplication (IEEE round-to-nearest),
``numpy.rint`` (round half to even), numpy int64 matmul, the numpy float16
cast (IEEE round-to-nearest-even).

Sources (cited by page title and section):

* [R1-INT8] "DeepSeek R1 INT8 quantization practice on SGLang" (Meituan
  search & recommendation team), section 2.1 "quantization basics"
  (symmetric INT8, Fig. 1: compute the scale, then quant/dequant) and
  section 2.3 "quantization method design": block-wise paragraph (128x128
  weight blocks, FP8 -> BF16 -> INT8, activations quantized online per
  token-group, several dequantizations inside the INT8 matmul) and
  channel-wise paragraph (one scale per weight column = output channel,
  per-token activation scales, a single dequantization after the INT8 GEMM).
* [FP8-vs-INT8] "FP8与INT8量化对决：DeepSeek模型存储优化的企业实战指南",
  section 3.2.1 (the quantizer formula: scale = max|w| / 127,
  q = round(w / scale).clamp(-127, 127)) and section 2.1 table
  (FP8 E4M3 = 4 exponent bits + 3 mantissa bits).
* [Qwen3-8B-W8A16] "DeepSeek-R1-0528-Qwen3-8B量化版发布", sections
  "模型简介与核心特性" and "技术实现与优化细节" (symmetric group-wise
  INT8 weights, FP16 activations, W8A16).

Readings taken where the sources are silent or garbled (each one is listed
with its justification in the design notes):

1. Rounding is half-to-even (torch ``round`` in the [FP8-vs-INT8] formula).
2. ``x / scale`` is a true fp32 division, not a multiply by a reciprocal.
3. A group whose absmax is 0 gets scale 0 and all-zero codes.
4. "Each column of the weight" in the channel-wise scheme is one output
   channel, i.e. one row of W stored [N, K].
5. E4M3 follows the OCP FP8 "E4M3FN" definition (bias 7, no infinities,
   0x7F/0xFF NaN, max 448); the [FP8-vs-INT8] range table is garbled.
6. FP8 -> BF16 is one fp32 multiply by the block scale, rounded to nearest
   even, then rounded to nearest even into bf16.
7. Partial weight blocks (N not a multiple of 128) take the absmax over the
   rows present; K must be a multiple of 128.
8. W8A16: group size 128 along K; the int8 x fp16 products are exact in fp32
   and the group scale multiplies the group's partial sum, without rounding
   the dequantized weight to fp16 first.

Every function is pinned by tests (``tests/test_oracle_*.py``) against brute
force, library routines, closed forms and invariants; none is "parity
unpinned".
"""
from __future__ import annotations

import numpy as np

GROUP = 128          # activation token-group size and weight block edge
QMAX = 127           # symmetric int8 range [-127, 127]


# ----------------------------------------------------------------------------
# number formats
# ----------------------------------------------------------------------------

def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> fp32: the bf16 bits are the top half of an fp32."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


def f32_to_bf16_rne(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bits, round to nearest, ties to even (finite inputs).

    Keep the top 16 bits of the fp32 pattern; round up when the dropped low
    16 bits exceed half, or equal half with an odd kept part.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    hi = u >> np.uint64(16)
    lo = u & np.uint64(0xFFFF)
    up = (lo > 0x8000) | ((lo == 0x8000) & ((hi & np.uint64(1)) == 1))
    return (hi + up.astype(np.uint64)).astype(np.uint16)


def f16_to_f32(bits: np.ndarray) -> np.ndarray:
    """fp16 bit patterns (uint16) -> fp32 (exact widening, subnormals included)."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float32)


def f32_to_f16_rne(x) -> np.ndarray:
    """fp32/fp64 -> fp16 bits, IEEE round to nearest even."""
    return np.asarray(x).astype(np.float16).view(np.uint16)


def e4m3_to_f32(codes: np.ndarray) -> np.ndarray:
    """FP8 E4M3 (OCP "FN" variant) byte -> fp32.

    sign = bit 7, exponent = bits 6..3 (bias 7), mantissa = bits 2..0.
    exponent 0: subnormal, value = mantissa * 2^-9.
    exponent 15 with mantissa 7: NaN (the format has no infinities).
    otherwise: value = (1 + mantissa / 8) * 2^(exponent - 7).
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = (1.0 + m / 8.0) * np.exp2(e - 7.0)
    sub = m * 2.0 ** -9
    v = sign * np.where(e == 0, sub, normal)
    v = np.where((e == 15) & (m == 7), np.nan, v)
    return v.astype(np.float32)


# ----------------------------------------------------------------------------
# the symmetric quantizer
# ----------------------------------------------------------------------------

def quantize_groups(v: np.ndarray):
    """Symmetric INT8 quantization of each row of ``v`` (fp32, shape [G, n]) as one group.

    [FP8-vs-INT8] section 3.2.1: scale = max|v| / 127 (fp32), then
    q = round(v / scale) clamped to [-127, 127].  [R1-INT8] section 2.1: the
    scale is computed first, then the values are quantized with it.
    Returns (q int8 [G, n], scale fp32 [G]).
    """
    v = np.asarray(v, dtype=np.float32)
    a = np.max(np.abs(v), axis=1)                       # exact: max does not round
    s = (a / np.float32(QMAX)).astype(np.float32)       # fp32 IEEE divide
    q = np.zeros(v.shape, dtype=np.int8)
    nz = s > 0
    if np.any(nz):
        r = v[nz] / s[nz, None]                         # fp32 IEEE divide, element-wise
        q[nz] = np.clip(np.rint(r), -QMAX, QMAX).astype(np.int8)   # rint: half to even
    return q, s


def quant_act_token_group(x_bf16: np.ndarray):
    """Online per-token-group activation quantization (block-wise scheme).

    [R1-INT8] section 2.3, block-wise paragraph: each token's vector is split
    into groups (of 128, matching the 128-wide weight blocks) and each group
    is quantized on its own.  x_bf16: bf16 bits [M, K], K % 128 == 0.
    Returns (xq int8 [M, K], sx fp32 [M, K/128]) with sx indexed (m, kb).
    """
    M, K = x_bf16.shape
    assert K % GROUP == 0
    kb = K // GROUP
    q, s = quantize_groups(bf16_to_f32(x_bf16).reshape(M * kb, GROUP))
    return q.reshape(M, K), s.reshape(M, kb)


def quant_act_token(x_bf16: np.ndarray):
    """Online per-token activation quantization (channel-wise scheme).

    [R1-INT8] section 2.3, channel-wise paragraph: activations are quantized
    online per token, i.e. one scale per row of X.  Also used for the
    channel-wise weight scales: one scale per output channel = per row of W
    [N, K].  Returns (q int8 [R, K], s fp32 [R]).
    """
    return quantize_groups(bf16_to_f32(x_bf16))


def quant_weight_block_f32(w: np.ndarray):
    """Block-wise weight quantization with one scale per 128x128 block.

    [R1-INT8] section 2.3, block-wise paragraph: quantization acts within
    128x128 blocks of the weight matrix.  w: fp32 values [N, K], K % 128 == 0;
    a partial last row-block uses the rows present.
    Returns (wq int8 [N, K], sw fp32 [ceil(N/128), K/128]).
    """
    N, K = w.shape
    assert K % GROUP == 0
    nb, kb = -(-N // GROUP), K // GROUP
    wq = np.zeros((N, K), dtype=np.int8)
    sw = np.zeros((nb, kb), dtype=np.float32)
    for i in range(nb):
        r0, r1 = i * GROUP, min(N, (i + 1) * GROUP)
        for j in range(kb):
            blk = w[r0:r1, j * GROUP:(j + 1) * GROUP]
            q, s = quantize_groups(blk.reshape(1, -1))
            wq[r0:r1, j * GROUP:(j + 1) * GROUP] = q.reshape(blk.shape)
            sw[i, j] = s[0]
    return wq, sw


def quant_weight_block(w_bf16: np.ndarray):
    """Block-wise 128x128 quantization of a bf16 weight (bf16 bits [N, K])."""
    return quant_weight_block_f32(bf16_to_f32(w_bf16))


def dequant_fp8_block_to_bf16(w_e4m3: np.ndarray, sf: np.ndarray) -> np.ndarray:
    """FP8-E4M3 checkpoint -> BF16 (the first half of the offline conversion).

    [R1-INT8] section 2.3: DeepSeek publishes no BF16 weights, so the native
    FP8 weights are first dequantized to BF16.  The FP8 tensor carries one
    fp32 scale per 128x128 block: value = e4m3 * sf[n/128, k/128], one fp32
    multiply, then rounded to bf16 (reading 6).  Returns bf16 bits [N, K].
    """
    N, K = w_e4m3.shape
    v = e4m3_to_f32(w_e4m3)
    sfe = np.repeat(np.repeat(np.asarray(sf, np.float32), GROUP, axis=0), GROUP, axis=1)[:N, :K]
    return f32_to_bf16_rne((v * sfe).astype(np.float32))


def requant_fp8_to_int8_block(w_e4m3: np.ndarray, sf: np.ndarray):
    """Offline FP8 -> BF16 -> INT8 128x128 block requantization ([R1-INT8] section 2.3)."""
    return quant_weight_block(dequant_fp8_block_to_bf16(w_e4m3, sf))


def requant_fp8_to_int8_channel(w_e4m3: np.ndarray, sf: np.ndarray):
    """Offline FP8 -> BF16 -> INT8 per-output-channel requantization.

    [R1-INT8] section 2.3, channel-wise paragraph: the native FP8 weights are
    dequantized to BF16, then quantized to INT8 channel by channel.
    Returns (wq int8 [N, K], sw fp32 [N]).
    """
    return quant_act_token(dequant_fp8_block_to_bf16(w_e4m3, sf))


# ----------------------------------------------------------------------------
# GEMMs
# ----------------------------------------------------------------------------

def _assert_int32_safe(K: int):
    # |sum of K products of two int8 in [-127, 127]| <= 127^2 * K must fit int32
    assert QMAX * QMAX * K < 2 ** 31, K


def gemm_w8a8_block_partials(xq: np.ndarray, wq: np.ndarray) -> np.ndarray:
    """Per-slab integer partial sums P[m, n, kb] = sum_{k in slab kb} xq[m,k] * wq[n,k] (int64, exact)."""
    M, K = xq.shape
    N = wq.shape[0]
    assert wq.shape[1] == K and K % GROUP == 0
    _assert_int32_safe(K)
    kb = K // GROUP
    P = np.empty((M, N, kb), dtype=np.int64)
    x64 = xq.astype(np.int64)
    w64 = wq.astype(np.int64)
    for j in range(kb):
        sl = slice(j * GROUP, (j + 1) * GROUP)
        P[:, :, j] = x64[:, sl] @ w64[:, sl].T
    return P


def gemm_w8a8_block(xq, sx, wq, sw):
    """Block-wise W8A8 GEMM ([R1-INT8] section 2.3 block-wise paragraph, Fig. 3 left).

    Because activation groups and weight blocks carry different scales, the
    INT8 matmul is dequantized once per 128-wide K slab:
        Y[m, n] = sum_kb P[m, n, kb] * (sx[m, kb] * sw[n // 128, kb])
    with the scale product taken in fp32 and everything else exact in fp64.
    Returns (Y fp64 [M, N], T fp64 [M, N], P int64 [M, N, KB]) where
    T = sum_kb |P * s| is the magnitude scale used by the error criteria.
    """
    P = gemm_w8a8_block_partials(xq, wq)
    M, N, kb = P.shape
    sxs = np.asarray(sx, np.float32)
    sws = np.asarray(sw, np.float32)[np.arange(N) // GROUP]          # [N, KB]
    s = (sxs[:, None, :] * sws[None, :, :]).astype(np.float32)     # fp32 product [M, N, KB]
    terms = P.astype(np.float64) * s.astype(np.float64)
    return terms.sum(axis=2), np.abs(terms).sum(axis=2), P


def gemm_w8a8_channel(xq, sx, wq, sw):
    """Channel-wise W8A8 GEMM ([R1-INT8] section 2.3 channel-wise paragraph, Fig. 3 right).

    One INT8 GEMM, then a single dequantization with the per-token and
    per-output-channel scales: Y[m, n] = A[m, n] * sx[m] * sw[n],
    A = xq @ wq^T exact in int64, the scaling in fp64.
    Returns (Y fp64 [M, N], A int64 [M, N]).
    """
    M, K = xq.shape
    assert wq.shape[1] == K
    _assert_int32_safe(K)
    A = xq.astype(np.int64) @ wq.astype(np.int64).T
    Y = A.astype(np.float64) * np.asarray(sx, np.float64)[:, None] * np.asarray(sw, np.float64)[None, :]
    return Y, A


def gemm_w8a16_group(x_f16, wq, s_f16, group: int = GROUP):
    """W8A16 group-wise weight-only GEMM ([Qwen3-8B-W8A16], technical details).

    Weights are symmetric INT8 with one fp16 scale per group of ``group``
    consecutive K of each output channel; activations stay fp16:
        Y[m, n] = sum_g s[n, g] * sum_{k in g} x[m, k] * wq[n, k]
    evaluated in fp64 (exact products; reading 8).
    Returns (Y fp64 [M, N], T fp64 [M, N]) with T = sum_g |s * partial_g|.
    """
    x = f16_to_f32(x_f16).astype(np.float64)
    M, K = x.shape
    N = wq.shape[0]
    assert wq.shape[1] == K and K % group == 0
    g = K // group
    s = f16_to_f32(s_f16).astype(np.float64).reshape(N, g)
    w = wq.astype(np.float64)
    Y = np.zeros((M, N))
    T = np.zeros((M, N))
    for j in range(g):
        sl = slice(j * group, (j + 1) * group)
        part = (x[:, sl] @ w[:, sl].T) * s[None, :, j]
        Y += part
        T += np.abs(part)
    return Y, T


# ----------------------------------------------------------------------------
# sampled evaluation (large shapes: the oracle computes chosen outputs one by one)
# ----------------------------------------------------------------------------

def gemm_w8a8_block_at(xq, sx, wq, sw, ms, ns):
    """Block-wise GEMM at the sampled output positions (ms[i], ns[i]); same definition as gemm_w8a8_block."""
    ms = np.asarray(ms)
    ns = np.asarray(ns)
    K = xq.shape[1]
    _assert_int32_safe(K)
    kb = K // GROUP
    xr = xq[ms].astype(np.int64).reshape(len(ms), kb, GROUP)
    wr = wq[ns].astype(np.int64).reshape(len(ns), kb, GROUP)
    P = np.einsum('ijk,ijk->ij', xr, wr)                          # [S, KB]
    s = (np.asarray(sx, np.float32)[ms] * np.asarray(sw, np.float32)[ns // GROUP]).astype(np.float32)
    terms = P.astype(np.float64) * s.astype(np.float64)
    return terms.sum(axis=1), np.abs(terms).sum(axis=1), P


def gemm_w8a8_channel_at(xq, sx, wq, sw, ms, ns):
    """Channel-wise GEMM at sampled positions; same definition as gemm_w8a8_channel."""
    ms = np.asarray(ms)
    ns = np.asarray(ns)
    _assert_int32_safe(xq.shape[1])
    A = np.einsum('ik,ik->i', xq[ms].astype(np.int64), wq[ns].astype(np.int64))
    Y = A.astype(np.float64) * np.asarray(sx, np.float64)[ms] * np.asarray(sw, np.float64)[ns]
    return Y, A


def gemm_w8a16_group_at(x_f16, wq, s_f16, ms, ns, group: int = GROUP):
    """W8A16 GEMM at sampled positions; same definition as gemm_w8a16_group."""
    ms = np.asarray(ms)
    ns = np.asarray(ns)
    K = wq.shape[1]
    g = K // group
    x = f16_to_f32(x_f16[ms]).astype(np.float64).reshape(len(ms), g, group)
    w = wq[ns].astype(np.float64).reshape(len(ns), g, group)
    s = f16_to_f32(s_f16[ns]).astype(np.float64).reshape(len(ns), g)
    parts = np.einsum('ijk,ijk->ij', x, w) * s
    return parts.sum(axis=1), np.abs(parts).sum(axis=1)
