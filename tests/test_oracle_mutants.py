"""Planted mistakes in copies of the oracle must fail the pins (the pins are not vacuous).

Each mutant is a small edit of an oracle function (done here, on the CPU, never
in the oracle itself): a wrong rounding mode, a reciprocal multiply instead of
a divide, -128 allowed, the wrong divisor, a dropped term, a transposed scale
index.  Every mutant must fail at least one pin check.
"""
import numpy as np
import pytest

import oracle as O
import oracle_pins as pins


def _quant_with(round_fn=np.rint, lo=-127, div=127.0, recip=False, eps=0.0):
    def quantize_groups(v):
        v = np.asarray(v, dtype=np.float32)
        a = np.max(np.abs(v), axis=1)
        s = np.maximum((a / np.float32(div)).astype(np.float32), np.float32(eps))
        q = np.zeros(v.shape, dtype=np.int8)
        nz = s > 0
        if np.any(nz):
            if recip:
                r = v[nz] * (np.float32(1.0) / s[nz, None])
            else:
                r = v[nz] / s[nz, None]
            q[nz] = np.clip(round_fn(r), lo, 127).astype(np.int8)
        return q, s
    return quantize_groups


QUANT_MUTANTS = {
    "round_half_away": _quant_with(round_fn=lambda r: np.sign(r) * np.floor(np.abs(r) + 0.5)),
    "round_half_up": _quant_with(round_fn=lambda r: np.floor(r + 0.5)),
    "truncate": _quant_with(round_fn=np.trunc),
    "reciprocal_multiply": _quant_with(recip=True),
    "divide_by_128": _quant_with(div=128.0),
    "eps_floor_on_scale": _quant_with(eps=1e-8),
}


def _fails(check, fn):
    try:
        check(fn)
    except AssertionError:
        return True
    return False


@pytest.mark.parametrize("name", sorted(QUANT_MUTANTS))
def test_quantizer_mutant_is_caught(name):
    m = QUANT_MUTANTS[name]
    assert any(_fails(c, m) for c in (pins.check_quantizer_golden, pins.check_quantizer_brute,
                                       pins.check_quantizer_invariants)), name


def test_real_quantizer_passes_all():
    for c in (pins.check_quantizer_golden, pins.check_quantizer_brute, pins.check_quantizer_invariants):
        c(O.quantize_groups)


def test_bf16_truncation_is_caught():
    def trunc(x):
        return (np.ascontiguousarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)

    def half_up(x):
        u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
        return ((u + 0x8000) >> 16).astype(np.uint16)
    assert _fails(pins.check_bf16_rne, trunc)
    assert _fails(pins.check_bf16_rne, half_up)


def test_e4m3_mutants_are_caught():
    def bias8(codes):
        c = np.asarray(codes, np.uint8).astype(np.int64)
        sign = np.where((c >> 7) & 1, -1.0, 1.0)
        e, m = (c >> 3) & 0xF, c & 7
        v = sign * np.where(e == 0, m * 2.0 ** -10, (1 + m / 8) * np.exp2(e - 8.0))
        return np.where((e == 15) & (m == 7), np.nan, v).astype(np.float32)

    def no_subnormal(codes):
        c = np.asarray(codes, np.uint8).astype(np.int64)
        sign = np.where((c >> 7) & 1, -1.0, 1.0)
        e, m = (c >> 3) & 0xF, c & 7
        v = sign * (1 + m / 8) * np.exp2(e - 7.0)
        return np.where((e == 15) & (m == 7), np.nan, v).astype(np.float32)

    def ieee_like_inf(codes):
        v = O.e4m3_to_f32(codes).copy()
        c = np.asarray(codes, np.uint8)
        v[(c & 0x78) == 0x78] = np.inf
        return v
    for f in (bias8, no_subnormal, ieee_like_inf):
        assert _fails(pins.check_e4m3, f), f.__name__


def test_block_gemm_mutants_are_caught():
    def wrong_block_index(xq, sx, wq, sw):
        P = O.gemm_w8a8_block_partials(xq, wq)
        N = wq.shape[0]
        sws = np.asarray(sw, np.float32)[np.minimum(np.arange(N) // 64, sw.shape[0] - 1)]
        s = (np.asarray(sx, np.float32)[:, None, :] * sws[None]).astype(np.float32)
        t = P * s.astype(np.float64)
        return t.sum(2), np.abs(t).sum(2), P

    def dropped_last_slab(xq, sx, wq, sw):
        Y, T, P = O.gemm_w8a8_block(xq, sx, wq, sw)
        s = (np.asarray(sx, np.float32)[:, None, -1] * np.asarray(sw, np.float32)[np.arange(wq.shape[0]) // 128][None, :, -1])
        return Y - P[:, :, -1] * s.astype(np.float32).astype(np.float64), T, P

    def single_scale(xq, sx, wq, sw):   # channel-style dequant with the first slab's scales only
        P = O.gemm_w8a8_block_partials(xq, wq)
        s = (np.asarray(sx, np.float32)[:, None, 0] * np.asarray(sw, np.float32)[np.arange(wq.shape[0]) // 128][None, :, 0])
        return P.sum(2) * s.astype(np.float64), np.abs(P.sum(2) * s.astype(np.float64)), P

    for f in (wrong_block_index, dropped_last_slab, single_scale):
        assert _fails(pins.check_block_gemm_brute, f) or _fails(pins.check_block_gemm_golden, f), f.__name__


def test_channel_gemm_mutants_are_caught():
    def transposed_scales(xq, sx, wq, sw):
        Y, A = O.gemm_w8a8_channel(xq, sx, wq, sw)
        return A * np.resize(np.asarray(sw, np.float64), sx.shape)[:, None] * np.resize(np.asarray(sx, np.float64), sw.shape)[None, :], A

    def int8_wrap(xq, sx, wq, sw):
        A = (xq.astype(np.int32) @ wq.astype(np.int32).T).astype(np.int16).astype(np.int64)
        return A * np.asarray(sx, np.float64)[:, None] * np.asarray(sw, np.float64)[None, :], A
    for f in (transposed_scales, int8_wrap):
        assert _fails(pins.check_channel_vs_library, f) or _fails(pins.check_channel_gemm_golden, f), f.__name__


def test_w8a16_mutants_are_caught():
    def fp16_dequant(x_f16, wq, s_f16):   # rounds s*q to fp16 before the dot product
        s = O.f16_to_f32(s_f16)
        N, K = wq.shape
        w = (wq.astype(np.float32).reshape(N, -1, 128) * s[:, :, None]).astype(np.float16).astype(np.float64).reshape(N, K)
        x = O.f16_to_f32(x_f16).astype(np.float64)
        Y = x @ w.T
        return Y, np.abs(x) @ np.abs(w).T * 0 + 1e-30

    def wrong_group(x_f16, wq, s_f16):
        s = O.f16_to_f32(s_f16).astype(np.float64)
        return O.gemm_w8a16_group(x_f16, wq, O.f32_to_f16_rne(np.roll(s, 1, axis=1)))
    for f in (fp16_dequant, wrong_group):
        assert _fails(pins.check_w8a16, f), f.__name__
