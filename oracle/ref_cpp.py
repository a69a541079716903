"""ctypes front end of the plain C++ oracle (oracle/i8q_oracle_ref.cpp); test infrastructure only.

The same functions, names and return conventions as the numpy oracle.  ``build()`` compiles the
library in-tree with g++ (no GPU, no CUDA); ``load()`` fails loudly if it has not been built.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "i8q_oracle_ref.cpp")
LIB = os.path.join(HERE, "libi8q_oracle_ref.so")
GROUP = 128
_lib = None


def build() -> str:
    """Compile the oracle library if it is missing or older than its source."""
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        subprocess.run(["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-shared", "-fPIC", "-o", LIB, SRC],
                       check=True)
    return LIB


def load() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise RuntimeError(f"C++ oracle not built: call oracle.ref_cpp.build() ({LIB})")
        _lib = ctypes.CDLL(LIB)
    return _lib


def _p(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _call(name, *args):
    getattr(load(), name)(*[a if isinstance(a, ctypes.c_void_p) else ctypes.c_int64(int(a)) for a in args])


def bf16_to_f32(bits):
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(b.shape, np.float32)
    _call("ior_bf16_to_f32", _p(b), b.size, _p(out))
    return out


def f32_to_bf16_rne(x):
    f = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(f.shape, np.uint16)
    _call("ior_f32_to_bf16_rne", _p(f), f.size, _p(out))
    return out


def f16_to_f32(bits):
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(b.shape, np.float32)
    _call("ior_f16_to_f32", _p(b), b.size, _p(out))
    return out


def e4m3_to_f32(codes):
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, np.float32)
    _call("ior_e4m3_to_f32", _p(c), c.size, _p(out))
    return out


def quantize_groups(v):
    f = np.ascontiguousarray(v, dtype=np.float32)
    G, n = f.shape
    q = np.empty((G, n), np.int8)
    s = np.empty(G, np.float32)
    _call("ior_quantize_groups", _p(f), G, n, _p(q), _p(s))
    return q, s


def quant_act_token_group(x_bf16):
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    M, K = x.shape
    assert K % GROUP == 0
    xq = np.empty((M, K), np.int8)
    sx = np.empty((M, K // GROUP), np.float32)
    _call("ior_quant_act_token_group", _p(x), M, K, _p(xq), _p(sx))
    return xq, sx


def quant_act_token(x_bf16):
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    R, K = x.shape
    q = np.empty((R, K), np.int8)
    s = np.empty(R, np.float32)
    _call("ior_quant_act_token", _p(x), R, K, _p(q), _p(s))
    return q, s


def quant_weight_block(w_bf16):
    w = np.ascontiguousarray(w_bf16, dtype=np.uint16)
    N, K = w.shape
    assert K % GROUP == 0
    wq = np.empty((N, K), np.int8)
    sw = np.empty((-(-N // GROUP), K // GROUP), np.float32)
    _call("ior_quant_weight_block", _p(w), N, K, _p(wq), _p(sw))
    return wq, sw


def dequant_fp8_block_to_bf16(w_e4m3, sf):
    w = np.ascontiguousarray(w_e4m3, dtype=np.uint8)
    f = np.ascontiguousarray(sf, dtype=np.float32)
    N, K = w.shape
    assert f.shape == (-(-N // GROUP), -(-K // GROUP))
    out = np.empty((N, K), np.uint16)
    _call("ior_dequant_fp8_block_to_bf16", _p(w), _p(f), N, K, _p(out))
    return out


def requant_fp8_to_int8_block(w_e4m3, sf):
    return quant_weight_block(dequant_fp8_block_to_bf16(w_e4m3, sf))


def requant_fp8_to_int8_channel(w_e4m3, sf):
    return quant_act_token(dequant_fp8_block_to_bf16(w_e4m3, sf))


def gemm_w8a8_block(xq, sx, wq, sw):
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    wq = np.ascontiguousarray(wq, dtype=np.int8)
    sx = np.ascontiguousarray(sx, dtype=np.float32)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    M, K = xq.shape
    N = wq.shape[0]
    KB = K // GROUP
    assert sx.shape == (M, KB) and sw.shape == (-(-N // GROUP), KB)
    Y = np.empty((M, N), np.float64)
    T = np.empty((M, N), np.float64)
    P = np.empty((M, N, KB), np.int64)
    _call("ior_gemm_w8a8_block", _p(xq), _p(sx), _p(wq), _p(sw), M, N, K, _p(Y), _p(T), _p(P))
    return Y, T, P


def gemm_w8a8_channel(xq, sx, wq, sw):
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    wq = np.ascontiguousarray(wq, dtype=np.int8)
    sx = np.ascontiguousarray(sx, dtype=np.float32)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    M, K = xq.shape
    N = wq.shape[0]
    Y = np.empty((M, N), np.float64)
    A = np.empty((M, N), np.int64)
    _call("ior_gemm_w8a8_channel", _p(xq), _p(sx), _p(wq), _p(sw), M, N, K, _p(Y), _p(A))
    return Y, A


def gemm_w8a16_group(x_f16, wq, s_f16):
    x = np.ascontiguousarray(x_f16, dtype=np.uint16)
    wq = np.ascontiguousarray(wq, dtype=np.int8)
    s = np.ascontiguousarray(s_f16, dtype=np.uint16)
    M, K = x.shape
    N = wq.shape[0]
    assert K % GROUP == 0 and s.size == N * (K // GROUP)
    Y = np.empty((M, N), np.float64)
    T = np.empty((M, N), np.float64)
    _call("ior_gemm_w8a16_group", _p(x), _p(wq), _p(s), M, N, K, _p(Y), _p(T))
    return Y, T
