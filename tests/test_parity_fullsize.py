"""Full-size parity: the DeepSeek-R1 / Qwen3-8B layer shapes, through the same entry points and
therefore the same launch configurations that bench.py times.

Quantized tensors and scales (activation quantizers, weight quantizers, the whole FP8 requant of
the [18432, 7168] layer) are compared bit-exactly in full; GEMM outputs and their int32 partial
sums on sampled rows and columns that the C++ oracle computes one by one (first/last rows and
columns, tile edges, random)."""
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


def _samples(n, count, seed):
    """Sorted unique indices in [0, n): both ends, both sides of every 128 boundary near the
    start, and random ones."""
    rng = np.random.default_rng(seed)
    base = [0, 1, n - 1, n - 2] + [b + d for b in (127, 255) for d in (0, 1)]
    idx = np.concatenate([np.array([i for i in base if 0 <= i < n], np.int64),
                          rng.integers(0, n, size=count)])
    return np.unique(idx)


def _grid(M, N, count_m, count_n, seed):
    """Flattened (row, column) pairs of the product of sampled rows and sampled columns."""
    mm, nn = np.meshgrid(_samples(M, count_m, seed), _samples(N, count_n, seed + 1), indexing="ij")
    return mm.ravel(), nn.ravel()


# ------------------------------------------------------------------ channel-wise, MoE down-proj
@pytest.fixture(scope="module")
def channel_layer(q):
    N, K, Mmax = 7168, 2048, 4096
    x = synth.activation_bf16(Mmax, K, seed=1, outlier_p=0.001, outlier_mult=50.0)
    w = synth.weight_bf16(N, K, seed=1)
    xq_ref, sx_ref = O.quant_act_token(x)
    wq_ref, sw_ref = O.quant_act_token(w)
    xd, wd = dev(x), dev(w)
    wq, sw = empty((N, K), torch.int8), empty((N,), torch.float32)
    q.i8q_quant_act_token(wd, wq, sw)
    torch.cuda.synchronize()
    assert np.array_equal(host(wq), wq_ref) and np.array_equal(host(sw), sw_ref)
    return dict(N=N, K=K, xd=xd, xq_ref=xq_ref, sx_ref=sx_ref, wq=wq, sw=sw, wq_ref=wq_ref, sw_ref=sw_ref)


@pytest.mark.parametrize("M", [1, 16, 128, 1024, 4096])
def test_channel_moe_down_proj(q, channel_layer, M):
    L = channel_layer
    N, K = L["N"], L["K"]
    xq, sx = empty((M, K), torch.int8), empty((M,), torch.float32)
    q.i8q_quant_act_token(L["xd"][:M], xq, sx)
    y = empty((M, N), torch.int16, 0x7FC0)
    acc = empty((M, N), torch.int32, 0x7FFFFFFF)
    q.i8q_gemm_w8a8_channel(xq, sx, L["wq"], L["sw"], y, debug_acc=acc)
    torch.cuda.synchronize()
    assert np.array_equal(host(xq), L["xq_ref"][:M]) and np.array_equal(host(sx), L["sx_ref"][:M])
    ms, ns = _grid(M, N, 48, 96, seed=M)
    Y, A = O.gemm_w8a8_channel_at(L["xq_ref"][:M], L["sx_ref"][:M], L["wq_ref"], L["sw_ref"], ms, ns)
    assert np.array_equal(host(acc)[ms, ns], A.astype(np.int32))
    check_half(host(y, np.uint16)[ms, ns], Y, np.abs(Y), "bf16", f"channel {M}x{N}x{K}", strict=True)


# ------------------------------------------------------------------ block-wise, dense MLP
@pytest.fixture(scope="module")
def block_x():
    """Prefill activation of the up projection [16384, 7168] and its oracle quantization."""
    x = synth.activation_bf16(16384, 7168, seed=2, outlier_p=0.001, outlier_mult=50.0)
    xq, sx = O.quant_act_token_group(x)
    return x, xq, sx


def _block_weights(q, N, K, seed):
    w = synth.weight_bf16(N, K, seed=seed)
    wq_ref, sw_ref = O.quant_weight_block(w)
    wq, sw = empty((N, K), torch.int8), empty(((N + 127) // 128, K // 128), torch.float32)
    q.i8q_quant_weight_block(dev(w), wq, sw)
    torch.cuda.synchronize()
    assert np.array_equal(host(wq), wq_ref) and np.array_equal(host(sw), sw_ref)
    return wq, sw, wq_ref, sw_ref


@pytest.mark.parametrize("proj,N,K", [("up", 18432, 7168), ("down", 7168, 18432)])
def test_block_dense_mlp(q, block_x, proj, N, K):
    wq, sw, wq_ref, sw_ref = _block_weights(q, N, K, seed=2)
    if K == block_x[0].shape[1]:
        x_all, xq_all, sx_all = block_x
    else:   # the down projection consumes an activation of the MLP's inner width
        x_all = synth.activation_bf16(16384, K, seed=5, outlier_p=0.001, outlier_mult=50.0)
        xq_all, sx_all = O.quant_act_token_group(x_all)
    xd_all = dev(x_all)
    for M in [1, 16, 128, 1024, 4096, 16384]:
        if M > x_all.shape[0]:
            continue
        ld = (M + 3) // 4 * 4
        xq = empty((M, K), torch.int8)
        sxd = empty((K // 128, ld), torch.float32, 0.0)
        q.i8q_quant_act_token_group(xd_all[:M], xq, sxd, ld_sx=ld)
        y = empty((M, N), torch.int16, 0x7FC0)
        q.i8q_gemm_w8a8_block(xq, sxd, wq, sw, y)
        y32 = empty((M, N), torch.float32, float("nan"))
        q.i8q_gemm_w8a8_block(xq, sxd, wq, sw, y32, out=q.I8Q_OUT_FP32)
        torch.cuda.synchronize()
        assert np.array_equal(host(xq), xq_all[:M]), f"{proj} M={M} codes"
        assert np.array_equal(host(sxd)[:, :M].T, sx_all[:M]), f"{proj} M={M} scales"
        ms, ns = _grid(M, N, 24, 64, seed=M + N)
        Y, T, P = O.gemm_w8a8_block_at(xq_all[:M], sx_all[:M], wq_ref, sw_ref, ms, ns)
        check_fp32(host(y32)[ms, ns], Y, T, f"block fp32 {proj} {M}x{N}x{K}")
        check_half(host(y, np.uint16)[ms, ns], Y, T, "bf16", f"block bf16 {proj} {M}x{N}x{K}")


@pytest.mark.parametrize("M", [1, 16, 64])
def test_block_decode_partials(q, M):
    """Decode batches on the up projection: every sampled int32 slab partial bit-exact."""
    N, K = 18432, 7168
    x = synth.activation_bf16(M, K, seed=11, outlier_p=0.001, outlier_mult=50.0)
    w = synth.weight_bf16(N, K, seed=11)
    xq_ref, sx_ref = O.quant_act_token_group(x)
    wq_ref, sw_ref = O.quant_weight_block(w)
    ld = (M + 3) // 4 * 4
    sxd = np.zeros((K // 128, ld), np.float32)
    sxd[:, :M] = sx_ref.T
    dbg = empty((M, N, K // 128), torch.int32, 0x7FFFFFFF)
    y32 = empty((M, N), torch.float32, float("nan"))
    q.i8q_gemm_w8a8_block(dev(xq_ref), dev(sxd), dev(wq_ref), dev(sw_ref), y32, out=q.I8Q_OUT_FP32,
                          debug_partials=dbg)
    torch.cuda.synchronize()
    ms, ns = _grid(M, N, 8, 256, seed=3 * M)
    Y, T, P = O.gemm_w8a8_block_at(xq_ref, sx_ref, wq_ref, sw_ref, ms, ns)
    assert np.array_equal(host(dbg)[ms, ns], P.astype(np.int32))
    check_fp32(host(y32)[ms, ns], Y, T, f"block decode {M}x{N}x{K}")


# ------------------------------------------------------------------ offline requant + act quant
def test_requant_fp8_full_layer(q):
    N, K = 18432, 7168
    w8, sf = synth.fp8_checkpoint(N, K, seed=3)
    wq, sw = empty((N, K), torch.int8), empty((N // 128, K // 128), torch.float32)
    q.i8q_requant_fp8_to_int8_block(dev(w8), dev(sf), wq, sw)
    torch.cuda.synchronize()
    wq_ref, sw_ref = O.requant_fp8_to_int8_block(w8, sf)       # the whole layer
    assert np.array_equal(host(sw).view(np.uint32), sw_ref.view(np.uint32))
    bad = np.argwhere(host(wq) != wq_ref)
    assert bad.size == 0, f"{len(bad)} codes differ, first at {bad[:4].tolist()}"


def test_act_quant_full_prefill(q, block_x):
    x, xq_ref, sx_ref = block_x
    M, K = x.shape
    xq, sx = empty((M, K), torch.int8), empty((K // 128, M), torch.float32)
    q.i8q_quant_act_token_group(dev(x), xq, sx)
    torch.cuda.synchronize()
    assert np.array_equal(host(xq), xq_ref)
    assert np.array_equal(host(sx).T, sx_ref)


# ------------------------------------------------------------------ W8A16 decode, Qwen3-8B
@pytest.mark.parametrize("N,K", [(12288, 4096), (4096, 12288)])
def test_w8a16_qwen3_8b(q, N, K):
    wq, s = synth.int8_weight_groups(N, K, seed=4)
    wqd, sd = dev(wq), dev(s)
    x_all = synth.activation_f16(64, K, seed=4)
    for M in [1, 4, 16, 64]:
        x = x_all[:M]
        y = empty((M, N), torch.int16, 0x7E00)
        q.i8q_gemm_w8a16_group(dev(x), wqd, sd, y)
        torch.cuda.synchronize()
        ms, ns = _grid(M, N, 8, 256, seed=N + M)
        Y, T = O.gemm_w8a16_group_at(x, wq, s, ms, ns)
        check_half(host(y, np.uint16)[ms, ns], Y, T, "fp16", f"w8a16 {M}x{N}x{K}")


@pytest.mark.parametrize("N,K", [(12288, 4096), (4096, 12288)])
def test_w8a16_qwen3_8b_prefill_and_bf16(q, N, K):
    """Qwen3-8B shapes at prefill batches (fp16) and with bf16 activations (decode and prefill)."""
    wq, s = synth.int8_weight_groups(N, K, seed=4)
    wqd, sd = dev(wq), dev(s)
    x_all = synth.activation_f16(2048, K, seed=4)
    for M in [512, 2048]:
        x = x_all[:M]
        y = empty((M, N), torch.int16, 0x7E00)
        q.i8q_gemm_w8a16_group(dev(x), wqd, sd, y)
        torch.cuda.synchronize()
        ms, ns = _grid(M, N, 16, 128, seed=N + M)
        Y, T = O.gemm_w8a16_group_at(x, wq, s, ms, ns)
        check_half(host(y, np.uint16)[ms, ns], Y, T, "fp16", f"w8a16 prefill {M}x{N}x{K}")
    wqb, sb = synth.int8_weight_groups(N, K, seed=5, scale_fmt="bf16")
    wqbd, sbd = dev(wqb), dev(sb)
    xb_all = synth.activation_bf16_plain(2048, K, seed=5)
    for M in [1, 16, 64, 2048]:
        x = xb_all[:M]
        y = empty((M, N), torch.int16, 0x7FC0)
        q.i8q_gemm_w8a16_group_bf16(dev(x), wqbd, sbd, y)
        torch.cuda.synchronize()
        ms, ns = _grid(M, N, 16, 128, seed=N + M + 1)
        Y, T = O.gemm_w8a16_group_at(x, wqb, sb, ms, ns, fmt="bf16")
        check_half(host(y, np.uint16)[ms, ns], Y, T, "bf16", f"w8a16 bf16 {M}x{N}x{K}")
