"""The CPU oracle against what the sources and the mathematics fix (no GPU needed)."""
import numpy as np
import pytest

import oracle as O
import oracle_pins as pins
from activation_quantized_gemm_b200 import synth


def test_quantizer_golden():
    pins.check_quantizer_golden(O.quantize_groups)


def test_quantizer_brute_force():
    pins.check_quantizer_brute(O.quantize_groups)


def test_quantizer_invariants():
    pins.check_quantizer_invariants(O.quantize_groups)


def test_bf16_rne_vs_torch():
    pins.check_bf16_rne(O.f32_to_bf16_rne)


def test_bf16_widen_vs_torch():
    pins.check_bf16_widen(O.bf16_to_f32)


def test_e4m3_exhaustive():
    pins.check_e4m3(O.e4m3_to_f32)


def test_f16_roundtrip():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(4096).astype(np.float32)
    b = O.f32_to_f16_rne(x)
    assert np.array_equal(b, x.astype(np.float16).view(np.uint16))
    assert np.array_equal(O.f16_to_f32(b), x.astype(np.float16).astype(np.float32))
    sub = np.array([1, 2, 0x3FF, 0x8001], np.uint16)   # subnormals widen exactly
    assert np.array_equal(O.f16_to_f32(sub), np.array([2.0 ** -24, 2.0 ** -23, 1023 * 2.0 ** -24, -(2.0 ** -24)], np.float32))


def test_act_token_group_brute():
    x = synth.activation_bf16(5, 384, seed=11, outlier_p=0.02, outlier_mult=20.0)
    x[3, 128:256] = 0          # a zero group
    xq, sx = O.quant_act_token_group(x)
    xf = O.bf16_to_f32(x)
    assert sx.shape == (5, 3)
    for m in range(5):
        for g in range(3):
            bq, bs = pins.brute_quantize([float(v) for v in xf[m, g * 128:(g + 1) * 128]])
            assert float(sx[m, g]) == bs
            assert list(map(int, xq[m, g * 128:(g + 1) * 128])) == bq


def test_act_token_brute():
    x = synth.activation_bf16(4, 256, seed=12, outlier_p=0.01)
    xq, sx = O.quant_act_token(x)
    xf = O.bf16_to_f32(x)
    for m in range(4):
        bq, bs = pins.brute_quantize([float(v) for v in xf[m]])
        assert float(sx[m]) == bs and list(map(int, xq[m])) == bq


def test_weight_block_brute_with_partial_block():
    w = synth.weight_bf16(130, 256, seed=13)
    wq, sw = O.quant_weight_block(w)
    wf = O.bf16_to_f32(w)
    assert sw.shape == (2, 2)
    for i in range(2):
        for j in range(2):
            blk = wf[i * 128:min(130, (i + 1) * 128), j * 128:(j + 1) * 128]
            bq, bs = pins.brute_quantize([float(v) for v in blk.ravel()])
            assert float(sw[i, j]) == bs
            assert list(map(int, wq[i * 128:min(130, (i + 1) * 128), j * 128:(j + 1) * 128].ravel())) == bq


def test_fp8_dequant_vs_torch_route():
    """E4M3 -> fp32 (torch decode) x block scale (fp32 multiply) -> bf16 (torch cast) gives the same bits."""
    import torch
    w8, sf = synth.fp8_checkpoint(260, 384, seed=14)
    got = O.dequant_fp8_block_to_bf16(w8, sf)
    v = torch.from_numpy(w8.copy()).view(torch.float8_e4m3fn).float()
    sfe = torch.from_numpy(sf).repeat_interleave(128, 0).repeat_interleave(128, 1)[:260, :384]
    ref = (v * sfe).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


def test_fp8_block_absmax_is_the_largest_code_dequantized():
    """bf16(fp32(e) * sf) is monotone in |e| for sf > 0, and |e| is monotone in the code's low 7 bits,
    so a block's BF16 absmax is the dequantization of its largest code: checked on every block of a
    checkpoint, including all-zero and single-code blocks."""
    w8, sf = synth.fp8_checkpoint(384, 512, seed=16)
    w8 = w8.copy()
    w8[:128, :128] = 0                      # all-zero block
    w8[128:256, 128:256] = 0x80 | 0x35      # one negative code everywhere
    bf = O.dequant_fp8_block_to_bf16(w8, sf)
    mag = np.abs(O.bf16_to_f32(bf))
    for i in range(3):
        for j in range(4):
            blk = (slice(i * 128, (i + 1) * 128), slice(j * 128, (j + 1) * 128))
            code = int((w8[blk] & 0x7F).max())
            one = np.array([[code]], dtype=np.uint8)
            expect = float(np.abs(O.bf16_to_f32(O.dequant_fp8_block_to_bf16(one, sf[i:i + 1, j:j + 1])))[0, 0])
            assert float(mag[blk].max()) == expect


def test_requant_codes_are_an_odd_function_of_the_byte():
    """Within a 128x128 block the requantized code of an element depends on its E4M3 byte alone and
    is odd in it: q(b | 0x80) = -q(b & 0x7F).  Dequantization (an fp32 product and a bf16 rounding)
    and quantization (an IEEE quotient, half-to-even, clamp) are both odd, and the block scale is
    shared, so a per-block table of 128 magnitude codes reproduces every element.  Checked on
    blocks with positive, negative and zero scales, every finite code in each block, and on the
    block absmax taken from the largest code magnitude with |sf|."""
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    w8 = np.resize(codes, (256, 512)).astype(np.uint8)
    rng = np.random.default_rng(23)
    rng.shuffle(w8.reshape(-1))
    sf = np.array([[0.5, -3.0e-3, 0.0, -7.5], [2.0 ** -20, -0.25, 1.0e-2, 3.0]], np.float32)
    wq, sw = O.requant_fp8_to_int8_block(w8, sf)
    for i in range(2):
        for j in range(4):
            blk = (slice(i * 128, (i + 1) * 128), slice(j * 128, (j + 1) * 128))
            b, q = w8[blk].ravel(), wq[blk].ravel().astype(int)
            table = {}
            for bb, qq in zip(b.tolist(), q.tolist()):
                assert table.setdefault(bb, qq) == qq, (i, j, bb)
            for bb, qq in table.items():
                if bb & 0x80 and (bb & 0x7F) in table:
                    assert qq == -table[bb & 0x7F], (i, j, bb)
            # the block scale from the largest magnitude code and |sf|
            top = np.array([[int((b & 0x7F).max())]], np.uint8)
            a = float(O.bf16_to_f32(O.dequant_fp8_block_to_bf16(top, np.abs(sf[i:i + 1, j:j + 1])))[0, 0])
            assert sw[i, j] == np.float32(a) / np.float32(127.0), (i, j)


def test_requant_is_dequant_then_block_quant():
    w8, sf = synth.fp8_checkpoint(256, 256, seed=15)
    wq, sw = O.requant_fp8_to_int8_block(w8, sf)
    wq2, sw2 = O.quant_weight_block(O.dequant_fp8_block_to_bf16(w8, sf))
    assert np.array_equal(wq, wq2) and np.array_equal(sw, sw2)
    # every non-zero block reaches |q| = 127
    for i in range(2):
        for j in range(2):
            assert np.abs(wq[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128].astype(int)).max() == 127
    wqc, swc = O.requant_fp8_to_int8_channel(w8, sf)
    assert swc.shape == (256,) and np.all(np.abs(wqc.astype(int)).max(axis=1) == 127)


def test_block_gemm_golden():
    pins.check_block_gemm_golden(O.gemm_w8a8_block)


def test_channel_gemm_golden():
    pins.check_channel_gemm_golden(O.gemm_w8a8_channel)


def test_block_gemm_brute():
    pins.check_block_gemm_brute(O.gemm_w8a8_block)


def test_block_gemm_integer_matmul():
    pins.check_block_vs_integer_matmul(O.gemm_w8a8_block)


def test_channel_gemm_library():
    pins.check_channel_vs_library(O.gemm_w8a8_channel)


def test_block_equals_channel_single_slab():
    """K = 128, N <= 128: one activation group per token and one weight block, so the two schemes coincide."""
    x = synth.activation_bf16(6, 128, seed=16)
    w = synth.weight_bf16(100, 128, seed=16)
    xq_g, sx_g = O.quant_act_token_group(x)
    xq_t, sx_t = O.quant_act_token(x)
    assert np.array_equal(xq_g, xq_t) and np.array_equal(sx_g[:, 0], sx_t)
    wq, sw = O.quant_weight_block(w)
    Yb, Tb, Pb = O.gemm_w8a8_block(xq_g, sx_g, wq, sw)
    Yc, Ac = O.gemm_w8a8_channel(xq_t, sx_t, wq, np.full(100, sw[0, 0], np.float32))
    assert np.array_equal(Pb[:, :, 0], Ac)
    assert np.allclose(Yb, Yc, rtol=1e-7, atol=0)


def test_w8a16():
    pins.check_w8a16(O.gemm_w8a16_group)


def test_sampled_equals_full():
    rng = np.random.default_rng(17)
    M, N, K = 7, 260, 512
    xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    wq = rng.integers(-127, 128, (N, K)).astype(np.int8)
    sx = rng.uniform(1e-3, 1e-1, (M, K // 128)).astype(np.float32)
    sw = rng.uniform(1e-4, 1e-2, (3, K // 128)).astype(np.float32)
    Y, T, P = O.gemm_w8a8_block(xq, sx, wq, sw)
    ms, ns = rng.integers(0, M, 50), rng.integers(0, N, 50)
    Ys, Ts, Ps = O.gemm_w8a8_block_at(xq, sx, wq, sw, ms, ns)
    assert np.array_equal(Ps, P[ms, ns]) and np.allclose(Ys, Y[ms, ns], rtol=1e-15, atol=0)
    sxc, swc = sx[:, 0].copy(), rng.uniform(1e-4, 1e-2, N).astype(np.float32)
    Yc, A = O.gemm_w8a8_channel(xq, sxc, wq, swc)
    Ycs, As = O.gemm_w8a8_channel_at(xq, sxc, wq, swc, ms, ns)
    assert np.array_equal(As, A[ms, ns]) and np.array_equal(Ycs, Yc[ms, ns])
    x16 = synth.activation_f16(M, K, seed=17)
    w8, s16 = synth.int8_weight_groups(N, K, seed=17)
    Yw, Tw = O.gemm_w8a16_group(x16, w8, s16)
    Yws, Tws = O.gemm_w8a16_group_at(x16, w8, s16, ms, ns)
    assert np.allclose(Yws, Yw[ms, ns], rtol=1e-13, atol=1e-13)


def test_int32_accumulation_is_exact_for_all_configured_K():
    for K in (512, 2048, 4096, 7168, 12288, 18432):
        assert 127 * 127 * K < 2 ** 31
    with pytest.raises(AssertionError):
        O.gemm_w8a8_channel(np.zeros((1, 133248), np.int8), np.ones(1, np.float32),
                            np.zeros((1, 133248), np.int8), np.ones(1, np.float32))
