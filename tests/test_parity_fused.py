"""Block-wise W8A8 GEMM with the per-token-group activation quantization fused in (decode batches)
against the C++ oracle's a1 -> a4 chain: the quantized activations the kernel produced internally
(codes and group scales) bit-exact, outputs within the criteria of tests/criteria.py; plus the
same layer through the unfused entry points."""
import numpy as np
import pytest
import torch

from oracle import ref_cpp as O
from activation_quantized_gemm_b200 import synth
from criteria import check_fp32, check_half
from gpu_util import dev, empty, host, setup_library

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    return setup_library()


def _acts(M, K, seed):
    x = synth.activation_bf16(M, K, seed=seed, outlier_p=0.005, outlier_mult=50.0)
    rng = np.random.default_rng(seed)
    if M >= 4:
        x[0, 128:256] = 0                                            # an all-zero group
        e = int(rng.integers(-8, 8))
        t = (rng.integers(-126, 126, K) + 0.5) * 2.0 ** e              # exact ties
        t[::128] = 127 * 2.0 ** e
        x[1] = O.f32_to_bf16_rne(t.astype(np.float32))
        x[2] = O.f32_to_bf16_rne((rng.standard_normal(K) * 1e-38).astype(np.float32))   # subnormal range
        x[3, :] = 0x8000                                             # negative zeros
    return x


def _run(q, M, N, K, seed, sampled=False):
    x = _acts(M, K, seed)
    w = synth.weight_bf16(N, K, seed=seed + 1)
    wq, sw = O.quant_weight_block(w)
    xq_ref, sx_ref = O.quant_act_token_group(x)
    ld = (M + 3) // 4 * 4 + 4
    xq = empty((M, K), torch.int8, 99)
    sx = empty((K // 128, ld), torch.float32, -1.0)
    y32 = empty((M, N), torch.float32, float("nan"))
    yb = empty((M, N), torch.int16, 0x7FC0)
    xd, wqd, swd = dev(x), dev(wq), dev(sw)
    q.i8q_gemm_w8a8_block_fused_quant(xd, wqd, swd, y32, out=q.I8Q_OUT_FP32, xq_out=xq, sx_out=sx)
    q.i8q_gemm_w8a8_block_fused_quant(xd, wqd, swd, yb)
    torch.cuda.synchronize()
    assert np.array_equal(host(xq), xq_ref), "fused codes"
    sxh = host(sx)
    assert np.array_equal(sxh[:, :M].T.view(np.uint32), sx_ref.view(np.uint32)), "fused scales"
    assert np.all(sxh[:, M:] == -1.0)
    if sampled:
        rng = np.random.default_rng(seed)
        mm, nn = np.meshgrid(np.arange(M), np.unique(np.concatenate([[0, N - 1], rng.integers(0, N, 300)])),
                             indexing="ij")
        ms, ns = mm.ravel(), nn.ravel()
        Y, T, P = O.gemm_w8a8_block_at(xq_ref, sx_ref, wq, sw, ms, ns)
        check_fp32(host(y32)[ms, ns], Y, T, f"fused fp32 {M}x{N}x{K}")
        check_half(host(yb, np.uint16)[ms, ns], Y, T, "bf16", f"fused bf16 {M}x{N}x{K}")
    else:
        Y, T, P = O.gemm_w8a8_block(xq_ref, sx_ref, wq, sw)
        check_fp32(host(y32), Y, T, f"fused fp32 {M}x{N}x{K}")
        check_half(host(yb, np.uint16), Y, T, "bf16", f"fused bf16 {M}x{N}x{K}")
    return xd, wqd, swd, y32, yb


@pytest.mark.parametrize("M,N,K", [(1, 256, 512), (4, 136, 384), (16, 256, 512), (5, 1032, 1024),
                                   (13, 264, 896), (16, 520, 1152), (7, 7, 256), (16, 1032, 2048),
                                   (9, 129, 128), (16, 4104, 4096), (2, 1032, 18432)])
def test_fused_quant_block(q, M, N, K):
    _run(q, M, N, K, seed=M * 7 + N + K)


@pytest.mark.parametrize("M", [1, 11, 16])
def test_fused_matches_unfused_path(q, M):
    """The fused call and the two-call path (a1 kernel, then the block GEMM) agree: codes and scales
    bit for bit, outputs within the criteria (the K split of the two launches may differ)."""
    N, K = 1032, 2048
    xd, wqd, swd, y32, yb = _run(q, M, N, K, seed=900 + M)
    ld = (M + 3) // 4 * 4
    xq = empty((M, K), torch.int8)
    sx = empty((K // 128, ld), torch.float32, 0.0)
    q.i8q_quant_act_token_group(xd, xq, sx, ld_sx=ld)
    y2 = empty((M, N), torch.float32)
    q.i8q_gemm_w8a8_block(xq, sx, wqd, swd, y2, out=q.I8Q_OUT_FP32)
    torch.cuda.synchronize()
    Y = host(y2).astype(np.float64)
    T = np.abs(Y) + 1e-30
    check_fp32(host(y32), Y, np.maximum(T, np.abs(host(y32))) * 2, f"fused vs unfused M={M}")


@pytest.mark.parametrize("proj,N,K", [("up", 18432, 7168), ("down", 7168, 18432)])
def test_fused_dense_mlp_decode(q, proj, N, K):
    """DeepSeek-R1 dense-MLP shapes at decode batch 16 (the launch bench.py times)."""
    _run(q, 16, N, K, seed=77 if proj == "up" else 78, sampled=True)


def test_fused_rejects_larger_batch(q):
    x = empty((17, 128), torch.int16)
    wq = empty((128, 128), torch.int8)
    sw = empty((1, 1), torch.float32)
    y = empty((17, 128), torch.int16)
    with pytest.raises(q.I8QError):
        q.i8q_gemm_w8a8_block_fused_quant(x, wq, sw, y)


@pytest.mark.parametrize("M,proj,N,K", [(16, "up", 18432, 7168), (16, "down", 7168, 18432), (1, "up", 18432, 7168),
                                        (8, "up", 18432, 7168)])
def test_fused_back_to_back_launches(q, M, proj, N, K):
    """Many launches queued back to back at the timed decode shapes, each result equal to the
    first one bit for bit.  The quantizer warps then run a whole stage ring ahead of the epilogue,
    which a barrier protocol that cannot tell those phases apart turns into an expired wait."""
    x = _acts(M, K, seed=300 + M)
    w = synth.weight_bf16(N, K, seed=301)
    wq, sw = O.quant_weight_block(w)
    xd, wqd, swd = dev(x), dev(wq), dev(sw)
    y0 = empty((M, N), torch.float32)
    q.i8q_gemm_w8a8_block_fused_quant(xd, wqd, swd, y0, out=q.I8Q_OUT_FP32)
    ys = [empty((M, N), torch.float32, float("nan")) for _ in range(4)]
    for i in range(40):
        q.i8q_gemm_w8a8_block_fused_quant(xd, wqd, swd, ys[i % 4], out=q.I8Q_OUT_FP32)
    torch.cuda.synchronize()
    q.i8q_status_check()
    ref = host(y0).view(np.uint32)
    for y in ys:
        assert np.array_equal(host(y).view(np.uint32), ref), f"fused {proj} M={M}: repeated launch differs"
