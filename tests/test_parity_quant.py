"""CUDA quantization kernels against the oracle: codes and scales bit-exact."""
import numpy as np
import pytest
import torch

from oracle import ref_cpp as O
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


@pytest.mark.parametrize("M,K", [(16, 512), (1, 128), (300, 1024), (37, 7168), (6, 18432), (9, 24576), (1000, 256)])
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


@pytest.mark.parametrize("M,K", [(16, 2048), (1, 16), (300, 2048), (6, 7168), (7, 18432), (130, 4096), (5, 24576), (1001, 384),
                                 (1, 8), (9, 24), (33, 40), (6, 1000)])
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


def test_requant_fp8_block_streams(q):
    """More blocks than the kernel has warps (each warp streams several blocks through its stage),
    a ragged last row-block, negative and zero block scales, an all-zero block and a block whose
    largest magnitude is a subnormal code."""
    N, K = 4100, 7168
    w8, sf = synth.fp8_checkpoint(N, K, seed=41)
    sf[1, 2] = -sf[1, 2]
    sf[5, :] = -sf[5, :]
    sf[3, 3] = 0.0
    w8[256:384, 512:640] = 0
    w8[0:128, 0:128] &= 0x87                      # E4M3 subnormals (exponent field 0) only
    wq_ref, sw_ref = O.requant_fp8_to_int8_block(w8, sf)
    wq = empty((N, K), torch.int8, 99)
    sw = empty(sw_ref.shape, torch.float32)
    q.i8q_requant_fp8_to_int8_block(dev(w8), dev(sf), wq, sw)
    torch.cuda.synchronize()
    assert np.array_equal(host(sw).view(np.uint32), sw_ref.view(np.uint32))
    bad = np.argwhere(host(wq) != wq_ref)
    assert bad.size == 0, f"{len(bad)} codes differ, first at {bad[:4].tolist()}"


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


def _reciprocal_traps(n_scales=400, seed=21):
    """bf16 groups in which x * fp32(1/s) and the true quotient x / s round to different codes.

    For random bf16 absmax values a, every positive bf16 x <= a is tried; the ones where the
    reciprocal product lands on the other side of a half-integer (or on a tie the quotient does
    not reach) are collected, and each group is [a, traps..., random fill <= a], with random signs.
    """
    rng = np.random.default_rng(seed)
    all_pos = (np.arange(1, 0x7F80, dtype=np.uint32) << 16).view(np.float32)     # positive finite bf16
    rows = []
    for _ in range(n_scales):
        a = np.float32(all_pos[rng.integers(0x3000, 0x5000)])                       # ~1e-5 .. 1e10
        s = np.float32(a / np.float32(127))
        xs = all_pos[all_pos <= a]
        q_div = np.rint(xs / s)
        q_rec = np.rint(xs * (np.float32(1) / s))
        traps = xs[q_div != q_rec]
        if traps.size == 0:
            continue
        row = np.empty(128, np.float32)
        row[0] = a
        k = min(traps.size, 100)
        row[1:1 + k] = rng.choice(traps, k, replace=False)
        row[1 + k:] = rng.choice(xs, 127 - k)
        row[1:] *= np.where(rng.random(127) < 0.5, -1, 1).astype(np.float32)
        rows.append(row)
    assert len(rows) >= 50, len(rows)
    return O.f32_to_bf16_rne(np.stack(rows))


def test_quantizer_reciprocal_traps(q):
    x = _reciprocal_traps()
    M = x.shape[0]
    xq_ref, sx_ref = O.quant_act_token_group(x)
    xq = empty((M, 128), torch.int8)
    sx = empty((1, (M + 3) // 4 * 4), torch.float32)
    q.i8q_quant_act_token_group(dev(x), xq, sx)
    xq2 = empty((M, 128), torch.int8)
    sx2 = empty((M,), torch.float32)
    q.i8q_quant_act_token(dev(x), xq2, sx2)
    torch.cuda.synchronize()
    assert np.array_equal(host(xq), xq_ref) and np.array_equal(host(sx)[0, :M], sx_ref[:, 0])
    assert np.array_equal(host(xq2), xq_ref) and np.array_equal(host(sx2), sx_ref[:, 0])


def test_quantizer_random_magnitudes(q):
    """4M elements: each 128-group has a random bf16 absmax (1e-30 .. 1e30) and uniform codes below it."""
    rng = np.random.default_rng(22)
    G = 32768
    e = rng.uniform(-100, 100, G)
    a = (2.0 ** e).astype(np.float32)
    v = (rng.uniform(-1, 1, (G, 128)) * a[:, None]).astype(np.float32)
    v[np.arange(G), rng.integers(0, 128, G)] = a * np.where(rng.random(G) < 0.5, -1, 1)
    x = O.f32_to_bf16_rne(v).reshape(1024, 32 * 128)
    xq_ref, sx_ref = O.quant_act_token_group(x)
    xq = empty(x.shape, torch.int8)
    sx = empty((32, 1024), torch.float32)
    q.i8q_quant_act_token_group(dev(x), xq, sx)
    torch.cuda.synchronize()
    assert np.array_equal(host(xq), xq_ref)
    assert np.array_equal(host(sx).T, sx_ref)


def _exhaustive_groups(exponents=(127, 100, 160)):
    """Every absmax mantissa x every bf16 value below it (12 binades, both signs), as 128-groups.

    The quantizer divides bf16 values v by s = RN(a / 127) with a bf16, so up to power-of-two
    scaling this is its complete input domain (below 2^-11 a every code is 0)."""
    rows = []
    for ea in exponents:
        for ma in range(128):
            a_bits = (ea << 7) | ma
            a = np.array([a_bits << 16], np.uint32).view(np.float32)[0]
            ex = np.arange(ea - 11, ea + 1)
            mant = np.arange(128)
            bits = ((ex[:, None] << 7) | mant[None, :]).ravel().astype(np.uint32)
            vals = (bits << 16).view(np.float32)
            vals = vals[vals <= a]
            vals = np.concatenate([vals, -vals])
            for i in range(0, vals.size, 127):
                row = np.zeros(128, np.float32)
                row[0] = a
                chunk = vals[i:i + 127]
                row[1:1 + chunk.size] = chunk
                rows.append(row)
    return O.f32_to_bf16_rne(np.stack(rows))


def test_quantizer_exhaustive_bf16_domain(q):
    x = _exhaustive_groups()
    M = x.shape[0]
    xq_ref, sx_ref = O.quant_act_token_group(x)
    xd = dev(x)
    xq = empty((M, 128), torch.int8)
    sx = empty((1, (M + 3) // 4 * 4), torch.float32)
    q.i8q_quant_act_token_group(xd, xq, sx)
    xq2 = empty((M, 128), torch.int8)
    sx2 = empty((M,), torch.float32)
    q.i8q_quant_act_token(xd, xq2, sx2)
    # the same values as 128x128 weight blocks (rows padded to a multiple of 128)
    Mp = (M + 127) // 128 * 128
    xpad = np.zeros((Mp, 128), np.uint16)
    xpad[:M] = x
    wq = empty((Mp, 128), torch.int8)
    sw = empty((Mp // 128, 1), torch.float32)
    q.i8q_quant_weight_block(dev(xpad), wq, sw)
    torch.cuda.synchronize()
    assert np.array_equal(host(xq), xq_ref) and np.array_equal(host(sx)[0, :M], sx_ref[:, 0])
    assert np.array_equal(host(xq2), xq_ref) and np.array_equal(host(sx2), sx_ref[:, 0])
    wq_ref, sw_ref = O.quant_weight_block(xpad)
    assert np.array_equal(host(wq), wq_ref) and np.array_equal(host(sw), sw_ref)
