"""Agreement criteria between the CUDA path and the oracle.

* int8 codes, fp32 scales, int32 partial sums: bit-exact.
* fp32 outputs: |y - Y| <= 1e-5 * T, with T the sum of the magnitudes of the terms the oracle adds
  (T >= |Y|, so this is a relative error wherever no cancellation occurs).
* bf16 / fp16 outputs of an fp32 accumulation chain (block-wise W8A8, W8A16): y is within 1 ulp
  of round_to_nearest_even(Y) in the output format, or |y - Y| <= 1e-5 * T + ulp(Y) / 2.  The
  second form is needed there: the slab sums are added in fp32, so where they cancel the fp32
  result can sit several output ulps from Y although its error is within 1e-5 * T.
  1e-5 covers that chain: the longest here is K = 18432 (144 slabs), whose worst-case fp32 FMA
  chain error is about 145 * 2^-24 * T = 8.6e-6 * T.
* bf16 outputs of the channel-wise GEMM (``strict=True``): y within 1 ulp of
  round_to_nearest_even(Y), with no escape.  The int32 accumulator is exact and the epilogue is
  three fp32 roundings (int -> float, the scale product, the final product), at most
  3 * 2^-24 relative, far below half a bf16 ulp.
"""
import numpy as np

REL = 1e-5


def _ordered(bits: np.ndarray, sign_bit: int) -> np.ndarray:
    b = bits.astype(np.int64)
    mag = b & (sign_bit - 1)
    return np.where(b & sign_bit, -mag, mag)


def bf16_bits_to_f64(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f16_bits_to_f64(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def f64_to_bf16_bits(Y):
    """round to nearest even directly from fp64 (via exact integer arithmetic on the fp64 bits)."""
    y = np.asarray(Y, np.float64)
    f = y.astype(np.float32)                      # may round; repair double rounding below
    u = f.view(np.uint32).astype(np.int64)
    cand = [(u >> 16) & 0xFFFF, ((u >> 16) + 1) & 0xFFFF, ((u >> 16) - 1) & 0xFFFF]
    best = cand[0].copy()
    bestd = np.abs(bf16_bits_to_f64(cand[0].astype(np.uint16)) - y)
    for c in cand[1:]:
        d = np.abs(bf16_bits_to_f64(c.astype(np.uint16)) - y)
        better = (d < bestd) | ((d == bestd) & ((c & 1) == 0) & ((best & 1) == 1))
        best = np.where(better, c, best)
        bestd = np.where(better, d, bestd)
    return best.astype(np.uint16)


def check_fp32(y, Y, T, what=""):
    y = np.asarray(y, np.float64)
    err = np.abs(y - Y)
    bad = err > REL * T
    assert not bad.any(), f"{what}: {int(bad.sum())} fp32 outputs off; worst rel {float(np.max(err / np.maximum(T, 1e-300))):.3g}"


def f64_to_f16_bits(Y):
    """round to nearest even directly from fp64 (numpy's double -> half conversion rounds once)."""
    return np.asarray(Y, np.float64).astype(np.float16).view(np.uint16)


def check_half(bits, Y, T, fmt: str, what="", strict: bool = False):
    """bits: uint16 output of the CUDA path; fmt 'bf16' or 'fp16'.  strict: <= 1 ulp, no T escape."""
    bits = np.asarray(bits, np.uint16)
    if fmt == "bf16":
        ref = f64_to_bf16_bits(Y)
        dec = bf16_bits_to_f64(bits)
        ulp = np.abs(bf16_bits_to_f64(ref ^ 1) - bf16_bits_to_f64(ref))
    else:
        ref = f64_to_f16_bits(Y)
        dec = f16_bits_to_f64(bits)
        ulp = np.abs(f16_bits_to_f64(ref ^ 1) - f16_bits_to_f64(ref))
    sb = 0x8000
    ulps = np.abs(_ordered(bits, sb) - _ordered(ref, sb))
    if strict:
        bad = ulps > 1
    else:
        close = np.abs(dec - Y) <= REL * T + ulp / 2
        bad = (ulps > 1) & ~close
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bits.size} {fmt} outputs off by >1 ulp; "
                           f"max ulps {int(ulps.max())}")
    return int((ulps > 0).sum())
