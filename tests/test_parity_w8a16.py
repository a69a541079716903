"""CUDA W8A16 group-wise decode GEMM (tcgen05 kind::f16, cluster split-K) against the oracle."""
import numpy as np
import pytest
import torch

from oracle import ref_cpp as O
from activation_quantized_gemm_b200 import synth
from criteria import check_half
from gpu_util import dev, empty, host, setup_library

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    return setup_library()


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 16, 17, 33, 64])
@pytest.mark.parametrize("N,K", [(128, 128), (264, 512), (1024, 4096), (136, 3072)])
def test_w8a16(q, M, N, K):
    x = synth.activation_f16(M, K, seed=M + N)
    wq, s = synth.int8_weight_groups(N, K, seed=N + K)
    Y, T = O.gemm_w8a16_group(x, wq, s)
    y = empty((M, N), torch.int16, 0x7E00)
    q.i8q_gemm_w8a16_group(dev(x), dev(wq), dev(s), y)
    torch.cuda.synchronize()
    check_half(host(y, np.uint16), Y, T, "fp16", f"w8a16 {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(1, 264, 16384), (3, 136, 18432), (4, 8, 256), (2, 4104, 1024),
                                   (1, 1, 128), (5, 7, 256), (16, 129, 512), (64, 4097, 1024)])
def test_w8a16_small_batches_long_rows(q, M, N, K):
    """Small decode batches with long rows (K up to 18432: 144 groups split over clusters of up to
    8 CTAs), a single ragged tile and many tiles."""
    x = synth.activation_f16(M, K, seed=M + K)
    wq, s = synth.int8_weight_groups(N, K, seed=N)
    Y, T = O.gemm_w8a16_group(x, wq, s)
    y = empty((M, N), torch.int16, 0x7E00)
    q.i8q_gemm_w8a16_group(dev(x), dev(wq), dev(s), y)
    torch.cuda.synchronize()
    check_half(host(y, np.uint16), Y, T, "fp16", f"w8a16 {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(65, 264, 512), (128, 136, 1024), (200, 1032, 2048), (1000, 520, 384),
                                   (129, 7, 256)])
def test_w8a16_prefill(q, M, N, K):
    """Batches above 64 tokens: 128-token tiles over the grid's z dimension, ragged last tile."""
    x = synth.activation_f16(M, K, seed=M + 3 * N)
    wq, s = synth.int8_weight_groups(N, K, seed=N + 5)
    Y, T = O.gemm_w8a16_group(x, wq, s)
    y = empty((M + 1, N), torch.int16, 0x7E00)                 # one row past the output
    q.i8q_gemm_w8a16_group(dev(x), dev(wq), dev(s), y[:M])
    torch.cuda.synchronize()
    check_half(host(y[:M], np.uint16), Y, T, "fp16", f"w8a16 prefill {M}x{N}x{K}")
    assert np.all(host(y[M:], np.uint16) == 0x7E00)


@pytest.mark.parametrize("M,N,K", [(1, 256, 512), (4, 136, 1024), (16, 1032, 4096), (33, 264, 3072), (64, 7, 256),
                                   (100, 520, 1024), (300, 264, 2048)])
def test_w8a16_bf16(q, M, N, K):
    """bf16 activations, bf16 group scales, bf16 output; exact int8 -> bf16 conversion."""
    x = synth.activation_bf16_plain(M, K, seed=7 * M + N)
    wq, s = synth.int8_weight_groups(N, K, seed=N + K, scale_fmt="bf16")
    Y, T = O.gemm_w8a16_group_fmt(x, wq, s, "bf16")
    y = empty((M, N), torch.int16, 0x7FC0)
    q.i8q_gemm_w8a16_group_bf16(dev(x), dev(wq), dev(s), y)
    torch.cuda.synchronize()
    check_half(host(y, np.uint16), Y, T, "bf16", f"w8a16 bf16 {M}x{N}x{K}")


def test_w8a16_bf16_all_codes(q):
    """Every int8 code -127..127 through the bf16 converter: x = one-hot, scale 1, so the output
    is the code itself (exact in bf16)."""
    N, K = 256, 256
    wq = np.zeros((N, K), np.int8)
    codes = np.arange(-127, 128, dtype=np.int64)
    wq[: codes.size, 5] = codes.astype(np.int8)
    wq[: codes.size, 130] = (-codes).astype(np.int8)
    x = np.zeros((2, K), np.uint16)
    x[0, 5] = 0x3F80                                           # bf16 1.0
    x[1, 130] = 0x3F80
    s = np.full((N, K // 128), 0x3F80, np.uint16)
    y = empty((2, N), torch.int16)
    q.i8q_gemm_w8a16_group_bf16(dev(x), dev(wq), dev(s), y)
    torch.cuda.synchronize()
    got = host(y, np.uint16)
    vals = (got.astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(vals[0, : codes.size], codes.astype(np.float32))
    assert np.array_equal(vals[1, : codes.size], -codes.astype(np.float32))
