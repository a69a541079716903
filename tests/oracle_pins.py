"""Pin checks for the CPU oracle, written as functions so that a planted mistake can be shown to fail them.

Each ``check_*`` takes the oracle function under test (or a deliberately broken
copy of it) and raises AssertionError when it disagrees with something fixed
independently of the oracle: a hand-worked golden fixture, a brute-force
evaluation in plain Python integers / fractions, a library routine, or an
invariant of the mathematics.
"""
from __future__ import annotations

import os
import struct
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ---------------------------------------------------------------- helpers ---

def f32(x: float) -> float:
    """Round a Python float (fp64) to the nearest fp32 value, ties to even."""
    return struct.unpack("<f", struct.pack("<f", x))[0]


def bf16_bits_exact(values) -> np.ndarray:
    """bf16 bit patterns of values that bf16 represents exactly (asserts exactness)."""
    a = np.asarray(values, dtype=np.float32)
    u = a.view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "value not exactly representable in bf16"
    return (u >> 16).astype(np.uint16)


def brute_quantize(vals):
    """Symmetric INT8 quantization of one group in plain Python.

    scale = fp32(absmax / 127); r = fp32(v / scale); q = the integer in
    [-127, 127] nearest to r, ties to the even one, found by search.  Python
    divides in fp64; rounding that quotient to fp32 gives the correctly
    rounded fp32 quotient because 53 >= 2 * 24 + 2 (double rounding is
    innocuous for division at that precision gap).
    """
    a = max(abs(v) for v in vals)
    s = f32(a / 127.0)
    if s == 0.0:
        return [0] * len(vals), 0.0
    out = []
    for v in vals:
        r = f32(v / s)
        best, bd = None, None
        for q in range(-127, 128):
            d = abs(r - q)
            if best is None or d < bd or (d == bd and q % 2 == 0):
                best, bd = q, d
        out.append(best)
    return out, s


def load_quantizer_examples():
    cases = []
    with open(os.path.join(GOLDEN, "quantizer_examples.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, vals, scale, codes = [p.strip() for p in line.split("|")]
            v = [float(t) for t in vals.split()]
            c = [int(t) for t in codes.split()]
            cases.append((name, v, float(scale), c))
    return cases


def load_e4m3_codes():
    out = []
    with open(os.path.join(GOLDEN, "e4m3_codes.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            code, val = line.split()
            out.append((int(code, 16), float(val)))
    return out


def load_gemm_examples():
    block, channel = [], []
    with open(os.path.join(GOLDEN, "gemm_examples.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = [p.strip() for p in line.split("|")]
            nums = [[float(t) for t in p.split()] for p in parts[1:]]
            (block if parts[0] == "block" else channel).append(nums)
    return block, channel


# ------------------------------------------------------------- quantizer ---

def check_quantizer_golden(quantize_groups):
    """Hand-worked cases from the quantizer formula (tests/golden/quantizer_examples.txt)."""
    for name, vals, scale, codes in load_quantizer_examples():
        g = np.zeros((1, 128), np.float32)
        g[0, :len(vals)] = vals
        q, s = quantize_groups(g)
        assert float(s[0]) == scale, (name, float(s[0]), scale)
        assert list(q[0, :len(codes)]) == codes, (name, list(q[0, :len(codes)]), codes)
        assert np.all(q[0, len(codes):] == 0), name


def check_quantizer_brute(quantize_groups, seed=0, groups=28, n=128):
    """Against brute_quantize on random groups (normal, outliers, ties, tiny and huge magnitudes)."""
    rng = np.random.default_rng(seed)
    rows = []
    for i in range(groups):
        kind = i % 7
        if kind == 0:
            v = rng.standard_normal(n)
        elif kind == 1:
            v = rng.standard_normal(n)
            v[rng.integers(0, n)] *= 50.0
        elif kind == 2:  # exact ties: absmax 127 * 2^e, entries (k + 1/2) * 2^e
            e = int(rng.integers(-6, 6))
            v = (rng.integers(-126, 126, n) + 0.5) * 2.0 ** e
            v[0] = 127 * 2.0 ** e
        elif kind == 3:
            v = rng.standard_normal(n) * 1e-30
        elif kind == 4:
            v = rng.standard_normal(n) * 1e30
        elif kind == 5:  # few distinct values, many repeats
            v = rng.integers(-3, 4, n).astype(np.float64) * 0.37
        else:  # exact ties under a scale that is not a power of two: s = 7 * 2^e
            e = int(rng.integers(-6, 6))
            v = (rng.integers(-126, 126, n) + 0.5) * 7.0 * 2.0 ** e
            v[0] = 889 * 2.0 ** e
        rows.append(np.asarray(v, np.float32))
    V = np.stack(rows)
    q, s = quantize_groups(V)
    for i in range(groups):
        bq, bs = brute_quantize([float(t) for t in V[i]])
        assert float(s[i]) == bs, (i, float(s[i]), bs)
        assert list(map(int, q[i])) == bq, (i, [(j, int(q[i, j]), bq[j]) for j in range(n) if q[i, j] != bq[j]][:5])


def check_quantizer_invariants(quantize_groups, seed=1):
    """Invariants fixed by the mathematics of the symmetric absmax quantizer."""
    rng = np.random.default_rng(seed)
    V = rng.standard_normal((64, 128)).astype(np.float32)
    V[5, 7] *= 50.0
    V[9] = 0.0
    q, s = quantize_groups(V)
    nz = np.any(V != 0, axis=1)
    # every non-zero group reaches |q| = 127 (at its absmax entry)
    assert np.all(np.max(np.abs(q[nz].astype(np.int32)), axis=1) == 127)
    # zero group -> scale 0, codes 0
    assert s[9] == 0 and np.all(q[9] == 0)
    # reconstruction error at most half a step (plus the fp32 rounding of x / s)
    err = np.abs(V[nz].astype(np.float64) - q[nz].astype(np.float64) * s[nz, None].astype(np.float64))
    assert np.all(err <= s[nz, None].astype(np.float64) * (0.5 + 2.0 ** -16))
    # sign symmetry: quant(-x) = (-q, s)
    q2, s2 = quantize_groups(-V)
    assert np.array_equal(s2, s) and np.array_equal(q2, -q)
    # power-of-two equivariance: quant(2^e x) = (q, 2^e s)
    for e in (-3, 5):
        q3, s3 = quantize_groups((V * np.float32(2.0 ** e)).astype(np.float32))
        assert np.array_equal(q3, q) and np.array_equal(s3, (s * np.float32(2.0 ** e)).astype(np.float32))
    # permutation equivariance within a group
    perm = rng.permutation(128)
    q4, s4 = quantize_groups(V[:, perm])
    assert np.array_equal(s4, s) and np.array_equal(q4, q[:, perm])
    # codes are always in the symmetric range (never -128)
    assert q.min() >= -127 and q.max() <= 127


# --------------------------------------------------------------- formats ---

def check_bf16_rne(f32_to_bf16_rne, seed=2):
    """fp32 -> bf16 against torch's CPU cast (round to nearest even) on random and halfway patterns."""
    import torch
    rng = np.random.default_rng(seed)
    u = rng.integers(0, 2 ** 32, 1 << 20, dtype=np.uint64).astype(np.uint32)
    ties = (rng.integers(0, 2 ** 16, 1 << 14, dtype=np.uint64).astype(np.uint32) << 16) | 0x8000
    u = np.concatenate([u, ties, ties + 1, ties - 1])
    x = u.view(np.float32)
    x = x[np.isfinite(x) & (np.abs(x) < 3.3e38)]
    ref = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = f32_to_bf16_rne(x)
    assert np.array_equal(got, ref), int(np.sum(got != ref))


def check_bf16_widen(bf16_to_f32, seed=3):
    import torch
    rng = np.random.default_rng(seed)
    b = rng.integers(0, 2 ** 16, 1 << 16, dtype=np.uint64).astype(np.uint16)
    ref = torch.from_numpy(b.view(np.int16).copy()).view(torch.bfloat16).float().numpy()
    got = bf16_to_f32(b)
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin].view(np.uint32), ref[fin].view(np.uint32))


def check_e4m3(e4m3_to_f32):
    """All 256 codes against torch's float8_e4m3fn decode, plus the hand-worked spot values."""
    import torch
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).float().numpy()
    got = e4m3_to_f32(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(got[fin].view(np.uint32), ref[fin].view(np.uint32))
    for code, val in load_e4m3_codes():
        g = float(e4m3_to_f32(np.array([code], np.uint8))[0])
        if np.isnan(val):
            assert np.isnan(g), hex(code)
        else:
            assert g == val and np.signbit(g) == np.signbit(val), (hex(code), g, val)


# ----------------------------------------------------------------- GEMMs ---

def _frac(x) -> Fraction:
    return Fraction(float(x))


def check_block_gemm_golden(gemm_w8a8_block):
    block, _ = load_gemm_examples()
    for xs, ws, sxs, sws, ps, (y,) in block:
        xq = np.concatenate([np.full(128, xs[0]), np.full(128, xs[1])]).astype(np.int8)[None, :]
        wq = np.concatenate([np.full(128, ws[0]), np.full(128, ws[1])]).astype(np.int8)[None, :]
        sx = np.array([sxs], np.float32)
        sw = np.array([sws], np.float32)
        Y, T, P = gemm_w8a8_block(xq, sx, wq, sw)
        assert list(P[0, 0]) == [int(p) for p in ps]
        assert Y[0, 0] == y, (Y[0, 0], y)


def check_channel_gemm_golden(gemm_w8a8_channel):
    _, channel = load_gemm_examples()
    for (xv,), (wv,), (sx,), (sw,), (a,), (y,) in channel:
        xq = np.full((1, 256), xv, np.int8)
        wq = np.full((1, 256), wv, np.int8)
        Y, A = gemm_w8a8_channel(xq, np.array([sx], np.float32), wq, np.array([sw], np.float32))
        assert A[0, 0] == a and Y[0, 0] == y, (A[0, 0], a, Y[0, 0], y)


def check_block_gemm_brute(gemm_w8a8_block, seed=4, M=3, N=130, K=256):
    """P by a pure-Python triple loop; Y as an exact rational, compared within 1e-15 of T."""
    rng = np.random.default_rng(seed)
    xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    wq = rng.integers(-127, 128, (N, K)).astype(np.int8)
    sx = rng.uniform(1e-3, 1e-1, (M, K // 128)).astype(np.float32)
    sw = rng.uniform(1e-4, 1e-2, ((N + 127) // 128, K // 128)).astype(np.float32)
    Y, T, P = gemm_w8a8_block(xq, sx, wq, sw)
    for m in range(M):
        for n in range(0, N, 7):
            y = Fraction(0)
            for kb in range(K // 128):
                p = 0
                for k in range(kb * 128, kb * 128 + 128):
                    p += int(xq[m, k]) * int(wq[n, k])
                assert P[m, n, kb] == p
                s = f32(float(sx[m, kb]) * float(sw[n // 128, kb]))  # product of two fp32 is exact in fp64
                y += p * _frac(s)
            assert abs(_frac(Y[m, n]) - y) <= Fraction(1, 10 ** 15) * _frac(T[m, n]) + Fraction(1, 10 ** 300)


def check_block_vs_integer_matmul(gemm_w8a8_block, seed=5, M=17, N=300, K=640):
    """With every scale equal to 1 the block GEMM is the integer matmul (torch int64 as the library routine)."""
    import torch
    rng = np.random.default_rng(seed)
    xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    wq = rng.integers(-127, 128, (N, K)).astype(np.int8)
    Y, T, P = gemm_w8a8_block(xq, np.ones((M, K // 128), np.float32), wq, np.ones(((N + 127) // 128, K // 128), np.float32))
    ref = (torch.from_numpy(xq).long() @ torch.from_numpy(wq).long().T).numpy()
    assert np.array_equal(Y, ref.astype(np.float64))
    assert np.array_equal(P.sum(axis=2), ref)
    # all-127 inputs: each slab's partial is 127^2 * 128
    Y1, T1, P1 = gemm_w8a8_block(np.full((2, K), 127, np.int8), np.ones((2, K // 128), np.float32),
                                 np.full((3, K), 127, np.int8), np.ones((1, K // 128), np.float32))
    assert np.all(P1 == 127 * 127 * 128)


def check_channel_vs_library(gemm_w8a8_channel, seed=6, M=9, N=200, K=384):
    import torch
    rng = np.random.default_rng(seed)
    xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    wq = rng.integers(-127, 128, (N, K)).astype(np.int8)
    sx = rng.uniform(1e-3, 1e-1, M).astype(np.float32)
    sw = rng.uniform(1e-4, 1e-2, N).astype(np.float32)
    Y, A = gemm_w8a8_channel(xq, sx, wq, sw)
    ref = torch.from_numpy(xq).long() @ torch.from_numpy(wq).long().T
    assert np.array_equal(A, ref.numpy())
    refY = ref.double() * torch.from_numpy(sx).double()[:, None] * torch.from_numpy(sw).double()[None, :]
    assert np.allclose(Y, refY.numpy(), rtol=1e-15, atol=0)


def check_w8a16(gemm_w8a16_group, seed=7, M=4, N=33, K=384):
    """Scale 1 reduces to a plain fp64 matmul (torch); random scales against exact fractions."""
    import torch
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)).astype(np.float16)
    xb = x.view(np.uint16)
    wq = rng.integers(-127, 128, (N, K)).astype(np.int8)
    one = np.full((N, K // 128), 1.0, np.float16).view(np.uint16)
    Y, T = gemm_w8a16_group(xb, wq, one)
    ref = torch.from_numpy(x.astype(np.float64)) @ torch.from_numpy(wq.astype(np.float64)).T
    assert np.allclose(Y, ref.numpy(), rtol=1e-13, atol=1e-12)
    s = rng.uniform(1e-4, 1e-3, (N, K // 128)).astype(np.float16)
    Y, T = gemm_w8a16_group(xb, wq, s.view(np.uint16))
    for m in range(M):
        for n in range(0, N, 5):
            y = Fraction(0)
            for g in range(K // 128):
                part = Fraction(0)
                for k in range(g * 128, g * 128 + 128):
                    part += _frac(x[m, k]) * int(wq[n, k])
                y += part * _frac(s[n, g])
            assert abs(_frac(Y[m, n]) - y) <= Fraction(1, 10 ** 14) * _frac(T[m, n]) + Fraction(1, 10 ** 300)


def check_w8a16_bf16(gemm_w8a16_group_bf16, seed=8, M=3, N=21, K=384):
    """bf16 activations and group scales: scale 1 reduces to a plain fp64 matmul of the bf16 values
    (torch's bf16 decode as the library routine); random scales against exact fractions."""
    import torch
    rng = np.random.default_rng(seed)
    xt = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)).to(torch.bfloat16)
    xb = xt.view(torch.int16).numpy().view(np.uint16)
    xv = xt.double().numpy()
    wq = rng.integers(-127, 128, (N, K)).astype(np.int8)
    one = np.full((N, K // 128), 0x3F80, np.uint16)                         # bf16 1.0
    Y, T = gemm_w8a16_group_bf16(xb, wq, one)
    ref = torch.from_numpy(xv) @ torch.from_numpy(wq.astype(np.float64)).T
    assert np.allclose(Y, ref.numpy(), rtol=1e-13, atol=1e-12)
    st = torch.from_numpy(rng.uniform(1e-4, 1e-3, (N, K // 128)).astype(np.float32)).to(torch.bfloat16)
    sb = st.view(torch.int16).numpy().view(np.uint16)
    sv = st.double().numpy()
    Y, T = gemm_w8a16_group_bf16(xb, wq, sb)
    for m in range(M):
        for n in range(0, N, 4):
            y = Fraction(0)
            for g in range(K // 128):
                part = Fraction(0)
                for k in range(g * 128, g * 128 + 128):
                    part += _frac(xv[m, k]) * int(wq[n, k])
                y += part * _frac(sv[n, g])
            assert abs(_frac(Y[m, n]) - y) <= Fraction(1, 10 ** 14) * _frac(T[m, n]) + Fraction(1, 10 ** 300)
