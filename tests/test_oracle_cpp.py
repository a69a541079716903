"""The plain C++ oracle (oracle/i8q_oracle_ref.cpp): pinned by the same checks as the numpy oracle
(golden fixtures, brute force, library routines, invariants) and equal to it element by element on
seeded inputs of every kind (bit-exact for codes, scales, formats and integer partial sums)."""
import numpy as np
import pytest

import oracle as O
import oracle_pins as pins
from activation_quantized_gemm_b200 import synth
from oracle import ref_cpp as R


@pytest.fixture(scope="module", autouse=True)
def _built():
    R.build()
    R.load()


def test_pins_quantizer():
    pins.check_quantizer_golden(R.quantize_groups)
    pins.check_quantizer_brute(R.quantize_groups)
    pins.check_quantizer_invariants(R.quantize_groups)


def test_pins_formats():
    pins.check_bf16_rne(R.f32_to_bf16_rne)
    pins.check_bf16_widen(R.bf16_to_f32)
    pins.check_e4m3(R.e4m3_to_f32)


def test_pins_gemms():
    pins.check_block_gemm_golden(R.gemm_w8a8_block)
    pins.check_channel_gemm_golden(R.gemm_w8a8_channel)
    pins.check_block_gemm_brute(R.gemm_w8a8_block)
    pins.check_block_vs_integer_matmul(R.gemm_w8a8_block)
    pins.check_channel_vs_library(R.gemm_w8a8_channel)
    pins.check_w8a16(R.gemm_w8a16_group)


def test_formats_exhaustive_agree():
    every16 = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    assert np.array_equal(R.bf16_to_f32(every16).view(np.uint32), O.bf16_to_f32(every16).view(np.uint32))
    a, b = R.f16_to_f32(every16), O.f16_to_f32(every16)
    assert np.array_equal(a, b, equal_nan=True)
    codes = np.arange(256, dtype=np.uint32).astype(np.uint8)
    assert np.array_equal(R.e4m3_to_f32(codes), O.e4m3_to_f32(codes), equal_nan=True)
    rng = np.random.default_rng(11)
    u = rng.integers(0, 0x7F800000, 200_000, dtype=np.uint32)
    u[:4096] = (u[:4096] & 0xFFFF0000) | 0x8000          # exact ties, both parities
    x = u.view(np.float32) * np.where(rng.random(u.size) < 0.5, -1, 1).astype(np.float32)
    assert np.array_equal(R.f32_to_bf16_rne(x), O.f32_to_bf16_rne(x))


def test_quantizers_agree():
    x = synth.activation_bf16(37, 1024, seed=21, outlier_p=0.001, outlier_mult=50.0)
    x[3, 128:256] = 0                                       # an all-zero group
    for got, ref in ((R.quant_act_token_group(x), O.quant_act_token_group(x)),
                     (R.quant_act_token(x), O.quant_act_token(x))):
        assert np.array_equal(got[0], ref[0]) and np.array_equal(got[1], ref[1])
    w = synth.weight_bf16(300, 384, seed=22)               # partial last row block
    got, ref = R.quant_weight_block(w), O.quant_weight_block(w)
    assert np.array_equal(got[0], ref[0]) and np.array_equal(got[1], ref[1])
    w8, sf = synth.fp8_checkpoint(260, 512, seed=23)
    assert np.array_equal(R.dequant_fp8_block_to_bf16(w8, sf), O.dequant_fp8_block_to_bf16(w8, sf))
    for fr, fo in ((R.requant_fp8_to_int8_block, O.requant_fp8_to_int8_block),
                   (R.requant_fp8_to_int8_channel, O.requant_fp8_to_int8_channel)):
        got, ref = fr(w8, sf), fo(w8, sf)
        assert np.array_equal(got[0], ref[0]) and np.array_equal(got[1], ref[1])


def test_gemms_agree():
    x = synth.activation_bf16(9, 768, seed=24, outlier_p=0.001, outlier_mult=50.0)
    w = synth.weight_bf16(260, 768, seed=25)
    xq, sx = O.quant_act_token_group(x)
    wq, sw = O.quant_weight_block(w)
    Y, T, P = R.gemm_w8a8_block(xq, sx, wq, sw)
    Yr, Tr, Pr = O.gemm_w8a8_block(xq, sx, wq, sw)
    assert np.array_equal(P, Pr)
    assert np.all(np.abs(Y - Yr) <= 1e-12 * Tr) and np.allclose(T, Tr, rtol=1e-12, atol=0)
    xq, sx = O.quant_act_token(x)
    wq, sw = O.quant_act_token(w)
    Y, A = R.gemm_w8a8_channel(xq, sx, wq, sw)
    Yr, Ar = O.gemm_w8a8_channel(xq, sx, wq, sw)
    assert np.array_equal(A, Ar) and np.array_equal(Y, Yr)
    xf = synth.activation_f16(5, 1024, seed=26)
    wq, s = synth.int8_weight_groups(130, 1024, seed=27)
    Y, T = R.gemm_w8a16_group(xf, wq, s)
    Yr, Tr = O.gemm_w8a16_group(xf, wq, s)
    assert np.all(np.abs(Y - Yr) <= 1e-12 * Tr) and np.allclose(T, Tr, rtol=1e-12, atol=0)


def test_threads_reported():
    assert R.num_threads() >= 1


def test_sampled_equals_full():
    """The sampled (one output at a time) functions give exactly the full functions' outputs."""
    rng = np.random.default_rng(31)
    x = synth.activation_bf16(11, 640, seed=31)
    w = synth.weight_bf16(300, 640, seed=32)
    ms, ns = rng.integers(0, 11, 200), rng.integers(0, 300, 200)
    xq, sx = R.quant_act_token_group(x)
    wq, sw = R.quant_weight_block(w)
    Y, T, P = R.gemm_w8a8_block(xq, sx, wq, sw)
    Ys, Ts, Ps = R.gemm_w8a8_block_at(xq, sx, wq, sw, ms, ns)
    assert np.array_equal(Ys, Y[ms, ns]) and np.array_equal(Ts, T[ms, ns]) and np.array_equal(Ps, P[ms, ns])
    xq, sx = R.quant_act_token(x)
    wq, sw = R.quant_act_token(w)
    Y, A = R.gemm_w8a8_channel(xq, sx, wq, sw)
    Ys, As = R.gemm_w8a8_channel_at(xq, sx, wq, sw, ms, ns)
    assert np.array_equal(Ys, Y[ms, ns]) and np.array_equal(As, A[ms, ns])
    xf = synth.activation_f16(11, 640, seed=33)
    wq, s = synth.int8_weight_groups(300, 640, seed=34)
    Y, T = R.gemm_w8a16_group(xf, wq, s)
    Ys, Ts = R.gemm_w8a16_group_at(xf, wq, s, ms, ns)
    assert np.array_equal(Ys, Y[ms, ns]) and np.array_equal(Ts, T[ms, ns])
    # and they agree with the numpy oracle's sampled functions
    Yn, Tn = O.gemm_w8a16_group_at(xf, wq, s, ms, ns)
    assert np.all(np.abs(Ys - Yn) <= 1e-12 * Tn)


def _grouped_problem(E, N, K, counts, seed):
    x = synth.activation_bf16(int(sum(counts)), K, seed=seed, outlier_p=0.001, outlier_mult=50.0)
    w = np.stack([synth.weight_bf16(N, K, seed=seed + 1 + e) for e in range(E)])
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    return x, w, off


def test_grouped_channel_is_per_expert_dense():
    """Grouped channel-wise GEMM = a loop over experts of the numpy oracle's dense definition,
    including experts without tokens."""
    E, N, K = 6, 136, 384
    counts = [3, 0, 17, 1, 0, 9]
    x, w, off = _grouped_problem(E, N, K, counts, seed=40)
    xq, sx = O.quant_act_token(x)
    wq = np.empty((E, N, K), np.int8)
    sw = np.empty((E, N), np.float32)
    for e in range(E):
        wq[e], sw[e] = O.quant_act_token(w[e])
    Y, A = R.gemm_w8a8_channel_grouped(xq, sx, wq, sw, off)
    for e in range(E):
        r = slice(off[e], off[e + 1])
        Ye, Ae = O.gemm_w8a8_channel(xq[r], sx[r], wq[e], sw[e])
        assert np.array_equal(A[r], Ae) and np.array_equal(Y[r], Ye)
    # one expert is the dense GEMM
    Y1, A1 = R.gemm_w8a8_channel_grouped(xq, sx, wq[:1], sw[:1], np.array([0, xq.shape[0]]))
    Yd, Ad = O.gemm_w8a8_channel(xq, sx, wq[0], sw[0])
    assert np.array_equal(A1, Ad) and np.array_equal(Y1, Yd)


def test_grouped_block_is_per_expert_dense():
    E, N, K = 5, 200, 512
    counts = [0, 4, 11, 0, 2]
    x, w, off = _grouped_problem(E, N, K, counts, seed=50)
    xq, sx = O.quant_act_token_group(x)
    wq = np.empty((E, N, K), np.int8)
    sw = np.empty((E, (N + 127) // 128, K // 128), np.float32)
    for e in range(E):
        wq[e], sw[e] = O.quant_weight_block(w[e])
    Y, T, P = R.gemm_w8a8_block_grouped(xq, sx, wq, sw, off)
    for e in range(E):
        r = slice(off[e], off[e + 1])
        Ye, Te, Pe = O.gemm_w8a8_block(xq[r], sx[r], wq[e], sw[e])
        assert np.array_equal(P[r], Pe)
        assert np.all(np.abs(Y[r] - Ye) <= 1e-12 * Te)


def test_w8a16_bf16_pins():
    pins.check_w8a16_bf16(lambda x, w, s: R.gemm_w8a16_group_fmt(x, w, s, "bf16"))
    # the fp16 format of the same entry is the pinned fp16 definition
    pins.check_w8a16(lambda x, w, s: R.gemm_w8a16_group_fmt(x, w, s, "fp16"))
