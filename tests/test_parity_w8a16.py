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


def test_w8a16_rejects_prefill_batch(q):
    x = empty((65, 128), torch.float16)
    with pytest.raises(q.I8QError):
        q.i8q_gemm_w8a16_group(x, empty((8, 128), torch.int8), empty((8, 1), torch.float16), empty((65, 8), torch.float16))
