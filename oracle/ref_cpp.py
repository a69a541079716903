"""ctypes front end of the plain C++ oracle (oracle/i8q_oracle_ref.cpp); test infrastructure only.

This is the oracle the GPU parity tests, ``__graft_entry__.smoke()`` and bench.py's CPU baseline
compare with and time.  Only ``tests/``, ``__graft_entry__.smoke()`` and bench.py's CPU-baseline
leg may import it.  The same functions, names and return conventions as the numpy oracle
(oracle/i8q_oracle.py), which stays as the cross-check the CPU tests run it against, plus the
grouped (MoE) and bf16 W8A16 definitions.  ``build()`` compiles the library in-tree with g++ and
OpenMP (no GPU, no CUDA); ``load()`` builds it when missing and fails loudly if g++ does.  OpenMP spreads
independent outputs over the host cores (``OMP_NUM_THREADS`` caps them); each output is computed
by one thread in a fixed order, so results do not depend on the thread count.
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
        subprocess.run(["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fopenmp", "-shared", "-fPIC",
                        "-o", LIB + ".tmp", SRC], check=True)
        os.replace(LIB + ".tmp", LIB)
    return LIB


def load() -> ctypes.CDLL:
    """Load the oracle library, compiling it first if it is missing or stale (g++ only)."""
    global _lib
    if _lib is None:
        build()
        _lib = ctypes.CDLL(LIB)
    return _lib


def num_threads() -> int:
    """Host threads the oracle's parallel loops use."""
    f = load().ior_num_threads
    f.restype = ctypes.c_int
    return int(f())


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


# ------------------------------------------------------------------ sampled evaluation
# Large shapes: the oracle computes chosen outputs (ms[i], ns[i]) one by one, by the same
# per-output definition as the full functions above.

def _idx(ms, ns):
    ms = np.ascontiguousarray(ms, dtype=np.int64).ravel()
    ns = np.ascontiguousarray(ns, dtype=np.int64).ravel()
    assert ms.shape == ns.shape
    return ms, ns


def gemm_w8a8_block_at(xq, sx, wq, sw, ms, ns):
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    wq = np.ascontiguousarray(wq, dtype=np.int8)
    sx = np.ascontiguousarray(sx, dtype=np.float32)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    M, K = xq.shape
    N = wq.shape[0]
    KB = K // GROUP
    assert sx.shape == (M, KB) and sw.shape == (-(-N // GROUP), KB)
    ms, ns = _idx(ms, ns)
    S = ms.size
    Y, T, P = np.empty(S), np.empty(S), np.empty((S, KB), np.int64)
    _call("ior_gemm_w8a8_block_at", _p(xq), _p(sx), _p(wq), _p(sw), M, N, K, _p(ms), _p(ns), S, _p(Y), _p(T), _p(P))
    return Y, T, P


def gemm_w8a8_channel_at(xq, sx, wq, sw, ms, ns):
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    wq = np.ascontiguousarray(wq, dtype=np.int8)
    sx = np.ascontiguousarray(sx, dtype=np.float32)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    M, K = xq.shape
    N = wq.shape[0]
    ms, ns = _idx(ms, ns)
    S = ms.size
    Y, A = np.empty(S), np.empty(S, np.int64)
    _call("ior_gemm_w8a8_channel_at", _p(xq), _p(sx), _p(wq), _p(sw), M, N, K, _p(ms), _p(ns), S, _p(Y), _p(A))
    return Y, A


def gemm_w8a16_group_fmt(x, wq, s, fmt: str = "fp16"):
    """W8A16 GEMM with activations and group scales in ``fmt`` ('fp16' or 'bf16')."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    wq = np.ascontiguousarray(wq, dtype=np.int8)
    s = np.ascontiguousarray(s, dtype=np.uint16)
    M, K = x.shape
    N = wq.shape[0]
    assert K % GROUP == 0 and s.size == N * (K // GROUP)
    Y, T = np.empty((M, N)), np.empty((M, N))
    _call("ior_gemm_w8a16_group_fmt", _p(x), _p(wq), _p(s), M, N, K, {"fp16": 0, "bf16": 1}[fmt], _p(Y), _p(T))
    return Y, T


def gemm_w8a16_group_at(x, wq, s, ms, ns, fmt: str = "fp16"):
    x = np.ascontiguousarray(x, dtype=np.uint16)
    wq = np.ascontiguousarray(wq, dtype=np.int8)
    s = np.ascontiguousarray(s, dtype=np.uint16)
    M, K = x.shape
    N = wq.shape[0]
    assert K % GROUP == 0 and s.size == N * (K // GROUP)
    ms, ns = _idx(ms, ns)
    S = ms.size
    Y, T = np.empty(S), np.empty(S)
    _call("ior_gemm_w8a16_group_at", _p(x), _p(wq), _p(s), M, N, K, {"fp16": 0, "bf16": 1}[fmt], _p(ms), _p(ns), S,
          _p(Y), _p(T))
    return Y, T


# ------------------------------------------------------------------ grouped (MoE) GEMMs
# Expert e owns token rows off[e] .. off[e+1]-1 of xq [M, K] and its own weight wq[e] [N, K].

def _offsets(off, M):
    off = np.ascontiguousarray(off, dtype=np.int64)
    assert off[0] == 0 and off[-1] == M and np.all(np.diff(off) >= 0)
    return off


def gemm_w8a8_channel_grouped_at(xq, sx, wq, sw, off, ms, ns):
    """xq [M, K], sx [M], wq [E, N, K], sw [E, N], off [E + 1]."""
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    wq = np.ascontiguousarray(wq, dtype=np.int8)
    sx = np.ascontiguousarray(sx, dtype=np.float32)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    M, K = xq.shape
    E, N, _ = wq.shape
    assert sw.shape == (E, N)
    off = _offsets(off, M)
    ms, ns = _idx(ms, ns)
    S = ms.size
    Y, A = np.empty(S), np.empty(S, np.int64)
    _call("ior_gemm_w8a8_channel_grouped_at", _p(xq), _p(sx), _p(wq), _p(sw), _p(off), E, M, N, K, _p(ms), _p(ns), S,
          _p(Y), _p(A))
    return Y, A


def gemm_w8a8_channel_grouped(xq, sx, wq, sw, off):
    M, N = xq.shape[0], wq.shape[1]
    ms, ns = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
    Y, A = gemm_w8a8_channel_grouped_at(xq, sx, wq, sw, off, ms, ns)
    return Y.reshape(M, N), A.reshape(M, N)


def gemm_w8a8_block_grouped_at(xq, sx, wq, sw, off, ms, ns):
    """xq [M, K], sx [M, K/128], wq [E, N, K], sw [E, ceil(N/128), K/128], off [E + 1]."""
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    wq = np.ascontiguousarray(wq, dtype=np.int8)
    sx = np.ascontiguousarray(sx, dtype=np.float32)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    M, K = xq.shape
    E, N, _ = wq.shape
    KB = K // GROUP
    assert sx.shape == (M, KB) and sw.shape == (E, -(-N // GROUP), KB)
    off = _offsets(off, M)
    ms, ns = _idx(ms, ns)
    S = ms.size
    Y, T, P = np.empty(S), np.empty(S), np.empty((S, KB), np.int64)
    _call("ior_gemm_w8a8_block_grouped_at", _p(xq), _p(sx), _p(wq), _p(sw), _p(off), E, M, N, K, _p(ms), _p(ns), S,
          _p(Y), _p(T), _p(P))
    return Y, T, P


def gemm_w8a8_block_grouped(xq, sx, wq, sw, off):
    M, N = xq.shape[0], wq.shape[1]
    ms, ns = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
    Y, T, P = gemm_w8a8_block_grouped_at(xq, sx, wq, sw, off, ms, ns)
    return Y.reshape(M, N), T.reshape(M, N), P.reshape(M, N, -1)
