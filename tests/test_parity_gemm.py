"""CUDA W8A8 GEMMs (tcgen05 kind::i8) against the oracle.

Integer partial sums are compared bit-exactly through the debug outputs; the fp32 / bf16 outputs
within the criteria of tests/criteria.py.  Inputs are quantized by the oracle, so the GEMM is
checked on its own."""
import numpy as np
import pytest
import torch

from oracle import ref_cpp as O
from activation_quantized_gemm_b200 import synth
from criteria import check_fp32, check_half
from gpu_util import dev, empty, host, setup_library

pytestmark = pytest.mark.gpu

SHAPES = [(1, 8, 128), (16, 256, 512), (7, 200, 384), (130, 264, 1024), (300, 520, 2048),
          (129, 1032, 768), (260, 136, 128),
          # decode-size batches (M <= 64): token padding to 16 / 32 / 64, K split over clusters of
          # 1..8 CTAs with slab counts that do not divide evenly, ragged last weight tile
          (17, 136, 896), (33, 520, 1152), (64, 1032, 4096), (48, 8, 256), (2, 2056, 1920),
          (65, 264, 1024),
          # decode kernel with 128-token padding (65..128 tokens, one CTA per SM)
          (100, 1032, 1536), (128, 264, 4096),
          # channel-wise pair-tile widths 224 and 256 (chosen by wave fill; smaller shapes take 192)
          (200, 16384, 256), (130, 18944, 256),
          # any N: masked tails (unaligned output rows, a partial last weight block), decode and
          # prefill kernels
          (1, 1, 128), (16, 7, 256), (40, 129, 512), (300, 7, 384), (257, 129, 256), (33, 7170, 512),
          (260, 7170, 256),
          # M >= 512: several pair-tile rows, ragged last tile
          (512, 1032, 1024), (600, 520, 768), (777, 7170, 512), (1024, 136, 2048)]


@pytest.fixture(scope="module")
def q():
    return setup_library()


def _inputs(M, N, K, seed, kind="synthetic"):
    if kind == "synthetic":
        x = synth.activation_bf16(M, K, seed=seed, outlier_p=0.005, outlier_mult=20.0)
        w = synth.weight_bf16(N, K, seed=seed)
        return x, w
    rng = np.random.default_rng(seed)
    if kind == "uniform":
        x = O.f32_to_bf16_rne(rng.uniform(-1, 1, (M, K)).astype(np.float32))
        w = O.f32_to_bf16_rne(rng.uniform(-1, 1, (N, K)).astype(np.float32))
        return x, w
    if kind == "extreme":   # every code +-127 with one sign: int32 accumulators at their maximum
        x = np.full((M, K), 0x3F80, np.uint16)                  # 1.0
        w = np.full((N, K), 0xBF80, np.uint16)                  # -1.0
        return x, w
    raise ValueError(kind)


def _block_operands(x, w):
    xq, sx = O.quant_act_token_group(x)
    wq, sw = O.quant_weight_block(w)
    return xq, sx, wq, sw


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("kind", ["synthetic", "uniform"])
def test_channel(q, M, N, K, kind):
    x, w = _inputs(M, N, K, seed=M * 31 + N + K, kind=kind)
    xq, sx = O.quant_act_token(x)
    wq, sw = O.quant_act_token(w)          # per-output-channel weight scales
    Y, A = O.gemm_w8a8_channel(xq, sx, wq, sw)
    y = empty((M, N), torch.int16, 0x7FC0)
    acc = empty((M, N), torch.int32, 0x7FFFFFFF)
    q.i8q_gemm_w8a8_channel(dev(xq), dev(sx), dev(wq), dev(sw), y, debug_acc=acc)
    torch.cuda.synchronize()
    assert np.array_equal(host(acc), A.astype(np.int32))
    T = np.abs(Y)
    check_half(host(y, np.uint16), Y, T, "bf16", f"channel {M}x{N}x{K}", strict=True)
    # the production variant (no debug output) writes the same bits
    y2 = empty((M, N), torch.int16, 0x7FC0)
    q.i8q_gemm_w8a8_channel(dev(xq), dev(sx), dev(wq), dev(sw), y2)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("kind", ["synthetic", "uniform"])
def test_block(q, M, N, K, kind):
    x, w = _inputs(M, N, K, seed=M * 17 + N + 3 * K, kind=kind)
    xq, sx, wq, sw = _block_operands(x, w)
    Y, T, P = O.gemm_w8a8_block(xq, sx, wq, sw)
    ld = (M + 3) // 4 * 4
    sxd = torch.zeros((K // 128, ld), dtype=torch.float32, device="cuda")
    sxd[:, :M] = dev(np.ascontiguousarray(sx.T))
    dbg = empty((M, N, K // 128), torch.int32, 0x7FFFFFFF)
    y32 = empty((M, N), torch.float32, float("nan"))
    q.i8q_gemm_w8a8_block(dev(xq), sxd, dev(wq), dev(sw), y32, out=q.I8Q_OUT_FP32, debug_partials=dbg)
    torch.cuda.synchronize()
    assert np.array_equal(host(dbg), P.astype(np.int32))
    check_fp32(host(y32), Y, T, f"block fp32 {M}x{N}x{K}")
    yb = empty((M, N), torch.int16, 0x7FC0)
    q.i8q_gemm_w8a8_block(dev(xq), sxd, dev(wq), dev(sw), yb)
    torch.cuda.synchronize()
    check_half(host(yb, np.uint16), Y, T, "bf16", f"block bf16 {M}x{N}x{K}")
    # production fp32 variant equals the debug variant bit for bit
    y32b = empty((M, N), torch.float32)
    q.i8q_gemm_w8a8_block(dev(xq), sxd, dev(wq), dev(sw), y32b, out=q.I8Q_OUT_FP32)
    torch.cuda.synchronize()
    assert torch.equal(y32, y32b)


def test_tiny_blockwise_config(q):
    """Tiny block-wise W8A8: X [16, 512] ~N(0,1) with 0.5% x20 outliers, W [256, 512] ~N(0,0.02), seed 0,
    per-token-group activation quantization on the GPU, 128x128 weight blocks, fp32 out."""
    x = synth.activation_bf16(16, 512, seed=0, outlier_p=0.005, outlier_mult=20.0)
    w = synth.weight_bf16(256, 512, seed=0)
    xq_ref, sx_ref, wq_ref, sw_ref = _block_operands(x, w)
    Y, T, P = O.gemm_w8a8_block(xq_ref, sx_ref, wq_ref, sw_ref)
    xq = empty((16, 512), torch.int8)
    sx = empty((4, 16), torch.float32)
    wq = empty((256, 512), torch.int8)
    sw = empty((2, 4), torch.float32)
    q.i8q_quant_act_token_group(dev(x), xq, sx)
    q.i8q_quant_weight_block(dev(w), wq, sw)
    dbg = empty((16, 256, 4), torch.int32)
    y = empty((16, 256), torch.float32)
    q.i8q_gemm_w8a8_block(xq, sx, wq, sw, y, out=q.I8Q_OUT_FP32, debug_partials=dbg)
    torch.cuda.synchronize()
    assert np.array_equal(host(xq), xq_ref) and np.array_equal(host(sx).T, sx_ref)
    assert np.array_equal(host(wq), wq_ref) and np.array_equal(host(sw), sw_ref)
    assert np.array_equal(host(dbg), P.astype(np.int32))
    check_fp32(host(y), Y, T, "tiny block-wise")


@pytest.mark.parametrize("M,N,K", [(130, 264, 18432), (5, 16, 18432)])
def test_extreme_accumulators(q, M, N, K):
    """All codes +-127: int32 partials reach 127^2 * 128 per slab and 127^2 * K in total."""
    x, w = _inputs(M, N, K, seed=1, kind="extreme")
    xq, sx = O.quant_act_token(x)
    wq, sw = O.quant_act_token(w)
    Y, A = O.gemm_w8a8_channel(xq, sx, wq, sw)
    assert A.min() == -127 * 127 * K
    y = empty((M, N), torch.int16)
    acc = empty((M, N), torch.int32)
    q.i8q_gemm_w8a8_channel(dev(xq), dev(sx), dev(wq), dev(sw), y, debug_acc=acc)
    xqb, sxb, wqb, swb = _block_operands(x, w)
    Yb, Tb, Pb = O.gemm_w8a8_block(xqb, sxb, wqb, swb)
    sxd = dev(np.ascontiguousarray(np.pad(sxb.T, ((0, 0), (0, (-M) % 4)))))
    dbg = empty((M, N, K // 128), torch.int32)
    y32 = empty((M, N), torch.float32)
    q.i8q_gemm_w8a8_block(dev(xqb), sxd, dev(wqb), dev(swb), y32, out=q.I8Q_OUT_FP32, debug_partials=dbg)
    torch.cuda.synchronize()
    assert np.array_equal(host(acc), A.astype(np.int32))
    check_half(host(y, np.uint16), Y, np.abs(Y), "bf16", "extreme channel", strict=True)
    assert np.array_equal(host(dbg), Pb.astype(np.int32))
    check_fp32(host(y32), Yb, Tb, "extreme block")


@pytest.mark.parametrize("M,N", [(16, 7), (70, 129), (300, 7), (260, 7170)])
def test_ragged_n_stays_in_bounds(q, M, N):
    """N not a multiple of 8: every output element is written exactly where it belongs and nothing
    past the packed [M, N] output (all four kernels: decode / pair tiles, channel / block, bf16 and fp32)."""
    K = 256
    x, w = _inputs(M, N, K, seed=M + N)
    xq, sx = O.quant_act_token(x)
    wq, sw = O.quant_act_token(w)
    Y, A = O.gemm_w8a8_channel(xq, sx, wq, sw)
    big = empty((M * N + 96,), torch.int16, 0x1234)
    q.i8q_gemm_w8a8_channel(dev(xq), dev(sx), dev(wq), dev(sw), big[: M * N].view(M, N))
    xqb, sxb, wqb, swb = _block_operands(x, w)
    Yb, Tb, Pb = O.gemm_w8a8_block(xqb, sxb, wqb, swb)
    sxd = dev(np.ascontiguousarray(np.pad(sxb.T, ((0, 0), (0, (-M) % 4)))))
    big16 = empty((M * N + 96,), torch.int16, 0x1234)
    q.i8q_gemm_w8a8_block(dev(xqb), sxd, dev(wqb), dev(swb), big16[: M * N].view(M, N))
    big32 = empty((M * N + 96,), torch.float32, 1234.5)
    q.i8q_gemm_w8a8_block(dev(xqb), sxd, dev(wqb), dev(swb), big32[: M * N].view(M, N), out=q.I8Q_OUT_FP32)
    torch.cuda.synchronize()
    h, h16, h32 = host(big).view(np.uint16), host(big16).view(np.uint16), host(big32)
    assert np.all(h[M * N:] == 0x1234) and np.all(h16[M * N:] == 0x1234) and np.all(h32[M * N:] == 1234.5)
    check_half(h[: M * N].reshape(M, N), Y, np.abs(Y), "bf16", f"channel ragged {M}x{N}", strict=True)
    check_half(h16[: M * N].reshape(M, N), Yb, Tb, "bf16", f"block ragged {M}x{N}")
    check_fp32(h32[: M * N].reshape(M, N), Yb, Tb, f"block fp32 ragged {M}x{N}")


def test_outputs_stay_in_bounds(q):
    """Rows past M and columns past N of a padded output buffer are never written."""
    M, N, K = 70, 136, 256
    x, w = _inputs(M, N, K, seed=9)
    xq, sx = O.quant_act_token(x)
    wq, sw = O.quant_act_token(w)
    big = empty((M + 3, N + 64), torch.int16, 0x1234)
    view = big.view(-1)[: M * N].view(M, N)          # the GEMM writes a packed [M, N] prefix
    q.i8q_gemm_w8a8_channel(dev(xq), dev(sx), dev(wq), dev(sw), view)
    torch.cuda.synchronize()
    rest = host(big).reshape(-1)[M * N:]
    assert np.all(rest == 0x1234)


def test_k_zero_writes_zeros(q):
    y = empty((4, 16), torch.int16, 0x1234)
    z8 = empty((4, 16), torch.int8)
    f = empty((16,), torch.float32)
    q.load().i8q_gemm_w8a8_channel(z8.data_ptr(), f.data_ptr(), z8.data_ptr(), f.data_ptr(), 4, 16, 0,
                                   y.data_ptr(), None, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert torch.all(y == 0)
