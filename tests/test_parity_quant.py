"""CUDA quantization kernels against the oracle: codes and scales bit-exact."""
import numpy as np
import pytest
import torch

import oracle as O
from activation_quantized_gemm_b200 import synth
from gpu_util import dev, empty, host, setup_library

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    return setup_library()


def _edge_activations(M, K, seed):
    """Synthetic activations plus rows that exercise the quantizer's edge cases."""
    x = synth.activation_bf16(M, K, seed=seed, outlier_p=0.01, outlier_mult=50.0)
    rng = np.random.default_rng(seed)
    if M >= 6:
        x[0, :] = 0                                              # all-zero token
        e = int(rng.integers(-8, 8))                             # exact ties under a power-of-two scale
        t = (rng.integers(-126, 126, K) + 0.5) * 2.0 ** e
        t[::128] = 127 * 2.0 ** e
        x[1] = O.f32_to_bf16_rne(t.astype(np.float32))
        x[2] = O.f32_to_bf16_rne((rng.standard_normal(K) * 1e-38).astype(np.float32))   # subnormal range
        x[3] = O.f32_to_bf16_rne((rng.standard_normal(K) * 1e37).astype(np.float32))    # near the top
        x[4, :] = 0x8000                                         # negative zeros
        x[5] = O.f32_to_bf16_rne(np.where(rng.random(K) < 0.5, -1.0, 1.0).astype(np.float32))
    return x


@pytest.mark.parametrize("M,K", [(16, 512), (1, 128), (300, 1024), (37, 7168), (6, 18432)])
def test_act_token_group(q, M, K):
    x = _edge_activations(M, K, seed=M + K)
    xq_ref, sx_ref = O.quant_act_token_group(x)
    ld_sx = (M + 3) // 4 * 4 + 4
    xd = dev(x)
    xq = empty((M, K), torch.int8, 99)
    sx = empty((K // 128, ld_sx), torch.float32, -1.0)
    q.i8q_quant_act_token_group(xd, xq, sx)
    torch.cuda.synchronize()
    assert np.array_equal(host(xq), xq_ref)
    sxh = host(sx)
    assert np.array_equal(sxh[:, :M].T.view(np.uint32), sx_ref.view(np.uint32))
    assert np.all(sxh[:, M:] == -1.0)              # padding of the scale rows untouched


def test_act_token_group_strided_input(q):
    M, K, ldx = 33, 384, 512
    full = synth.activation_bf16(M, ldx, seed=3)
    xq_ref, sx_ref = O.quant_act_token_group(np.ascontiguousarray(full[:, :K]))
    xd = dev(full)
    xq = empty((M, K), torch.int8)
    sx = empty((K // 128, 36), torch.float32)
    q.i8q_quant_act_token_group(xd[:, :K], xq, sx)
    torch.cuda.synchronize()
    assert np.array_equal(host(xq), xq_ref)
    assert np.array_equal(host(sx)[:, :M].T, sx_ref)


@pytest.mark.parametrize("M,K", [(16, 2048), (1, 16), (300, 2048), (6, 7168), (7, 18432), (130, 4096)])
def test_act_token(q, M, K):
    x = _edge_activations(M, K, seed=2 * M + K)
    xq_ref, sx_ref = O.quant_act_token(x)
    xq = empty((M, K), torch.int8, 99)
    sx = empty((M,), torch.float32)
    q.i8q_quant_act_token(dev(x), xq, sx)
    torch.cuda.synchronize()
    assert np.array_equal(host(xq), xq_ref)
    assert np.array_equal(host(sx).view(np.uint32), sx_ref.view(np.uint32))


@pytest.mark.parametrize("N,K", [(130, 256), (256, 7168), (1000, 384), (1, 128)])
def test_weight_block(q, N, K):
    w = synth.weight_bf16(N, K, seed=N + K)
    if N >= 200:
        w[128:256, 128:256] = 0                      # an all-zero block
    wq_ref, sw_ref = O.quant_weight_block(w)
    wq = empty((N, K), torch.int8, 99)
    sw = empty(sw_ref.shape, torch.float32)
    q.i8q_quant_weight_block(dev(w), wq, sw)
    torch.cuda.synchronize()
    assert np.array_equal(host(wq), wq_ref)
    assert np.array_equal(host(sw), sw_ref)


@pytest.mark.parametrize("N,K", [(260, 384), (129, 128), (384, 2048)])
def test_requant_fp8_block(q, N, K):
    w8, sf = synth.fp8_checkpoint(N, K, seed=N * 7 + K)
    wq_ref, sw_ref = O.requant_fp8_to_int8_block(w8, sf)
    wq = empty((N, K), torch.int8, 99)
    sw = empty(sw_ref.shape, torch.float32)
    q.i8q_requant_fp8_to_int8_block(dev(w8), dev(sf), wq, sw)
    torch.cuda.synchronize()
    assert np.array_equal(host(wq), wq_ref)
    assert np.array_equal(host(sw), sw_ref)


def test_requant_fp8_all_codes(q):
    """Every finite E4M3 code appears, including subnormals and +-448."""
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    w8 = np.resize(codes, (128, 256)).astype(np.uint8)
    sf = np.array([[0.5, 3.0e-3]], np.float32)
    wq_ref, sw_ref = O.requant_fp8_to_int8_block(w8, sf)
    wq = empty((128, 256), torch.int8)
    sw = empty((1, 2), torch.float32)
    q.i8q_requant_fp8_to_int8_block(dev(w8), dev(sf), wq, sw)
    torch.cuda.synchronize()
    assert np.array_equal(host(wq), wq_ref) and np.array_equal(host(sw), sw_ref)


@pytest.mark.parametrize("N,K", [(260, 384), (3, 2048)])
def test_requant_fp8_channel(q, N, K):
    w8, sf = synth.fp8_checkpoint(N, K, seed=N + 5 * K)
    wq_ref, sw_ref = O.requant_fp8_to_int8_channel(w8, sf)
    wq = empty((N, K), torch.int8, 99)
    sw = empty((N,), torch.float32)
    q.i8q_requant_fp8_to_int8_channel(dev(w8), dev(sf), wq, sw)
    torch.cuda.synchronize()
    assert np.array_equal(host(wq), wq_ref)
    assert np.array_equal(host(sw), sw_ref)


def test_status_check_clean(q):
    q.i8q_status_check()
