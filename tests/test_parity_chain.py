"""Layer chains without host synchronisation: each layer's output is the next layer's input and
every layer reuses the same quantized-activation and scale buffers, so the kernels' dependent
launches (a GEMM or quantizer may start while the kernel before it still runs) are exercised
against both hazards they must respect: reading an input the previous kernel is still writing, and
overwriting a buffer the previous kernel is still reading.  Each layer is checked against the
oracle applied to the GPU's own input of that layer."""
import numpy as np
import pytest
import torch

from oracle import ref_cpp as O
from activation_quantized_gemm_b200 import synth
from criteria import check_fp32, check_half
from gpu_util import dev, empty, host, setup_library

pytestmark = pytest.mark.gpu
LAYERS = 6


@pytest.fixture(scope="module")
def q():
    return setup_library()


@pytest.mark.parametrize("M,D", [(16, 1024), (300, 768)])
def test_block_chain(q, M, D):
    ws = [synth.weight_bf16(D, D, seed=40 + i, sigma=0.05) for i in range(LAYERS)]
    wqs, sws = [], []
    for w in ws:
        wq, sw = empty((D, D), torch.int8), empty((D // 128, D // 128), torch.float32)
        q.i8q_quant_weight_block(dev(w), wq, sw)
        wqs.append(wq)
        sws.append(sw)
    ld = (M + 3) // 4 * 4
    xq, sx = empty((M, D), torch.int8), empty((D // 128, ld), torch.float32, 0.0)   # shared by every layer
    x0 = synth.activation_bf16(M, D, seed=3)
    acts = [dev(x0)] + [empty((M, D), torch.int16) for _ in range(LAYERS)]
    torch.cuda.synchronize()
    for i in range(LAYERS):
        q.i8q_quant_act_token_group(acts[i], xq, sx, ld_sx=ld)
        q.i8q_gemm_w8a8_block(xq, sx, wqs[i], sws[i], acts[i + 1])
    torch.cuda.synchronize()
    for i in range(LAYERS):
        xi = host(acts[i], np.uint16)
        xq_r, sx_r = O.quant_act_token_group(xi)
        wq_r, sw_r = O.quant_weight_block(ws[i])
        Y, T, _ = O.gemm_w8a8_block(xq_r, sx_r, wq_r, sw_r)
        check_half(host(acts[i + 1], np.uint16), Y, T, "bf16", f"block chain layer {i} M={M}")


@pytest.mark.parametrize("M,D", [(16, 1024), (300, 768)])
def test_channel_chain(q, M, D):
    ws = [synth.weight_bf16(D, D, seed=50 + i, sigma=0.05) for i in range(LAYERS)]
    wqs, sws = [], []
    for w in ws:
        wq, sw = empty((D, D), torch.int8), empty((D,), torch.float32)
        q.i8q_quant_act_token(dev(w), wq, sw)
        wqs.append(wq)
        sws.append(sw)
    xq, sx = empty((M, D), torch.int8), empty((M,), torch.float32)
    acts = [dev(synth.activation_bf16(M, D, seed=4))] + [empty((M, D), torch.int16) for _ in range(LAYERS)]
    torch.cuda.synchronize()
    for i in range(LAYERS):
        q.i8q_quant_act_token(acts[i], xq, sx)
        q.i8q_gemm_w8a8_channel(xq, sx, wqs[i], sws[i], acts[i + 1])
    torch.cuda.synchronize()
    for i in range(LAYERS):
        xq_r, sx_r = O.quant_act_token(host(acts[i], np.uint16))
        wq_r, sw_r = O.quant_act_token(ws[i])
        Y, _ = O.gemm_w8a8_channel(xq_r, sx_r, wq_r, sw_r)
        check_half(host(acts[i + 1], np.uint16), Y, np.abs(Y), "bf16", f"channel chain layer {i} M={M}", strict=True)


@pytest.mark.parametrize("M", [1, 16])
def test_w8a16_chain(q, M):
    D = 2048
    layers = [synth.int8_weight_groups(D, D, seed=60 + i) for i in range(LAYERS)]
    dl = [(dev(wq), dev(s)) for wq, s in layers]
    acts = [dev(synth.activation_f16(M, D, seed=5))] + [empty((M, D), torch.int16) for _ in range(LAYERS)]
    torch.cuda.synchronize()
    for i in range(LAYERS):
        q.i8q_gemm_w8a16_group(acts[i], dl[i][0], dl[i][1], acts[i + 1])
    torch.cuda.synchronize()
    for i in range(LAYERS):
        Y, T = O.gemm_w8a16_group(host(acts[i], np.uint16), *layers[i])
        check_half(host(acts[i + 1], np.uint16), Y, T, "fp16", f"w8a16 chain layer {i} M={M}")
