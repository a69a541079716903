"""Thin Python binding of libi8q.so (ctypes).  Same names as the C ABI in include/i8q.h.

Each function takes torch tensors that live on the current CUDA device, passes
their data pointers, sizes and leading dimensions to the C entry point of the
same name, and raises ``I8QError`` on a non-OK status.  No arithmetic of the
method happens here: every step runs in the CUDA kernels of libi8q.so.  There
is no fallback: a missing library or a device the library does not support is
an error.

Tensor conventions (torch dtypes used to carry the bits):
  bf16 / fp16 tensors may be torch.bfloat16 / torch.float16 or int16 views of
  the same bits; int8 tensors are torch.int8; FP8-E4M3 bytes are torch.uint8
  (or torch.float8_e4m3fn); scales are torch.float32.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libi8q.so")
HEADER_PATH = os.path.join(os.path.dirname(PKG), "include", "i8q.h")

I8Q_OK = 0
I8Q_OUT_BF16 = 0
I8Q_OUT_FP32 = 1
STATUS_NAMES = {0: "I8Q_OK", 1: "I8Q_ERR_NULL", 2: "I8Q_ERR_SHAPE", 3: "I8Q_ERR_ALIGN", 4: "I8Q_ERR_DTYPE",
                5: "I8Q_ERR_CUDA", 6: "I8Q_ERR_TIMEOUT", 7: "I8Q_ERR_UNSUPPORTED"}


class I8QError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str):
        super().__init__(f"{fn}: {STATUS_NAMES.get(status, status)}" + (f" ({detail})" if detail else ""))
        self.status = status


_P = ctypes.c_void_p
_I = ctypes.c_int64
_SIGS = {
    "i8q_quant_act_token_group": [_P, _I, _I, _I, _P, _P, _I, _P],
    "i8q_quant_act_token": [_P, _I, _I, _I, _P, _P, _P],
    "i8q_quant_weight_block": [_P, _I, _I, _P, _P, _P],
    "i8q_requant_fp8_to_int8_block": [_P, _P, _I, _I, _P, _P, _P],
    "i8q_requant_fp8_to_int8_channel": [_P, _P, _I, _I, _P, _P, _P],
    "i8q_gemm_w8a8_block": [_P, _P, _I, _P, _P, _I, _I, _I, _P, ctypes.c_int, _P, _P],
    "i8q_gemm_w8a8_channel": [_P, _P, _P, _P, _I, _I, _I, _P, _P, _P],
    "i8q_gemm_w8a16_group": [_P, _P, _P, _I, _I, _I, _P, _P],
    "i8q_gemm_w8a16_group_bf16": [_P, _P, _P, _I, _I, _I, _P, _P],
    "i8q_gemm_w8a8_channel_grouped": [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P],
    "i8q_gemm_w8a8_block_fused_quant": [_P, _I, _P, _P, _I, _I, _I, _P, ctypes.c_int, _P, _P, _I, _P],
    "i8q_gemm_w8a8_block_grouped": [_P, _P, _I, _P, _P, _P, _I, _I, _I, _I, _P, ctypes.c_int, _P, _P],
    "i8q_status_check": [_P],
    "i8q_test_set_wait_limit_ns": [ctypes.c_uint64],
    "i8q_test_skip_accumulator_signal": [ctypes.c_int],
    "i8q_status_string": [ctypes.c_int],
    "i8q_last_error_string": [],
    "i8q_version": [],
}

_lib: Optional[ctypes.CDLL] = None


def load() -> ctypes.CDLL:
    """Load libi8q.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libi8q.so not built: run `python -m activation_quantized_gemm_b200.build` ({LIB_PATH})")
        lib = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGS.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        lib.i8q_status_string.restype = ctypes.c_char_p
        lib.i8q_last_error_string.restype = ctypes.c_char_p
        _lib = lib
    return _lib


def declared_symbols() -> list:
    """Function names declared in include/i8q.h."""
    with open(HEADER_PATH) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(i8q_[a-z0-9_]+)\s*\(", text)))


def _call(name: str, *args) -> None:
    lib = load()
    st = getattr(lib, name)(*args)
    if st != I8Q_OK:
        raise I8QError(name, st, lib.i8q_last_error_string().decode())


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ld(t) -> int:
    return t.stride(0) if t.dim() == 2 else t.shape[-1]


# ------------------------------------------------------------------------------- entry points

def i8q_quant_act_token_group(x, xq, sx, ld_sx: Optional[int] = None, stream=None) -> None:
    """x [M, K] bf16 -> xq [M, K] int8, sx [K/128, ld_sx] fp32 (token-contiguous)."""
    M, K = x.shape
    _call("i8q_quant_act_token_group", _ptr(x), M, K, _ld(x), _ptr(xq), _ptr(sx),
          sx.shape[1] if ld_sx is None else ld_sx, _stream(stream))


def i8q_quant_act_token(x, xq, sx, stream=None) -> None:
    """x [M, K] bf16 -> xq [M, K] int8, sx [M] fp32."""
    M, K = x.shape
    _call("i8q_quant_act_token", _ptr(x), M, K, _ld(x), _ptr(xq), _ptr(sx), _stream(stream))


def i8q_quant_weight_block(w, wq, sw, stream=None) -> None:
    """w [N, K] bf16 -> wq [N, K] int8, sw [ceil(N/128), K/128] fp32."""
    N, K = w.shape
    _call("i8q_quant_weight_block", _ptr(w), N, K, _ptr(wq), _ptr(sw), _stream(stream))


def i8q_requant_fp8_to_int8_block(w_e4m3, sf, wq, sw, stream=None) -> None:
    """w_e4m3 [N, K] bytes + sf [ceil(N/128), K/128] -> wq [N, K] int8, sw like sf."""
    N, K = w_e4m3.shape
    _call("i8q_requant_fp8_to_int8_block", _ptr(w_e4m3), _ptr(sf), N, K, _ptr(wq), _ptr(sw), _stream(stream))


def i8q_requant_fp8_to_int8_channel(w_e4m3, sf, wq, sw, stream=None) -> None:
    """w_e4m3 [N, K] bytes + sf [ceil(N/128), K/128] -> wq [N, K] int8, sw [N] fp32."""
    N, K = w_e4m3.shape
    _call("i8q_requant_fp8_to_int8_channel", _ptr(w_e4m3), _ptr(sf), N, K, _ptr(wq), _ptr(sw), _stream(stream))


def i8q_gemm_w8a8_block(xq, sx, wq, sw, y, out: int = I8Q_OUT_BF16, debug_partials=None,
                        ld_sx: Optional[int] = None, stream=None) -> None:
    """y [M, N] = block-wise W8A8 GEMM; sx is [K/128, ld_sx] as written by i8q_quant_act_token_group."""
    M, K = xq.shape
    N = wq.shape[0]
    _call("i8q_gemm_w8a8_block", _ptr(xq), _ptr(sx), sx.shape[1] if ld_sx is None else ld_sx, _ptr(wq), _ptr(sw),
          M, N, K, _ptr(y), int(out), _ptr(debug_partials), _stream(stream))


def i8q_gemm_w8a8_block_fused_quant(x, wq, sw, y, out: int = I8Q_OUT_BF16, xq_out=None, sx_out=None,
                                    ld_sx: Optional[int] = None, stream=None) -> None:
    """y [M, N] = block-wise W8A8 GEMM of bf16 x [M, K] (1 <= M <= 16) with the per-token-group
    quantization done inside the GEMM; xq_out [M, K] / sx_out [K/128, ld_sx] optionally receive the
    quantized activations."""
    M, K = x.shape
    N = wq.shape[0]
    if ld_sx is None:
        ld_sx = sx_out.shape[1] if sx_out is not None else 0
    _call("i8q_gemm_w8a8_block_fused_quant", _ptr(x), _ld(x), _ptr(wq), _ptr(sw), M, N, K, _ptr(y), int(out),
          _ptr(xq_out), _ptr(sx_out), ld_sx, _stream(stream))


def i8q_gemm_w8a8_channel(xq, sx, wq, sw, y, debug_acc=None, stream=None) -> None:
    """y [M, N] bf16 = channel-wise W8A8 GEMM with sx [M], sw [N]."""
    M, K = xq.shape
    N = wq.shape[0]
    _call("i8q_gemm_w8a8_channel", _ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), M, N, K, _ptr(y), _ptr(debug_acc),
          _stream(stream))


def i8q_gemm_w8a8_channel_grouped(xq, sx, wq, sw, expert_offsets, y, debug_acc=None, stream=None) -> None:
    """Grouped (MoE) channel-wise GEMM: xq [M, K] sorted by expert, wq [E, N, K], sw [E, N],
    expert_offsets int32 [E + 1] on the device, y [M, N] bf16."""
    M, K = xq.shape
    E, N = wq.shape[0], wq.shape[1]
    _call("i8q_gemm_w8a8_channel_grouped", _ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), _ptr(expert_offsets), E, M, N,
          K, _ptr(y), _ptr(debug_acc), _stream(stream))


def i8q_gemm_w8a8_block_grouped(xq, sx, wq, sw, expert_offsets, y, out: int = I8Q_OUT_BF16, debug_partials=None,
                                ld_sx: Optional[int] = None, stream=None) -> None:
    """Grouped (MoE) block-wise GEMM: xq [M, K] sorted by expert, sx [K/128, ld_sx], wq [E, N, K],
    sw [E, ceil(N/128), K/128], expert_offsets int32 [E + 1] on the device, y [M, N]."""
    M, K = xq.shape
    E, N = wq.shape[0], wq.shape[1]
    _call("i8q_gemm_w8a8_block_grouped", _ptr(xq), _ptr(sx), sx.shape[1] if ld_sx is None else ld_sx, _ptr(wq),
          _ptr(sw), _ptr(expert_offsets), E, M, N, K, _ptr(y), int(out), _ptr(debug_partials), _stream(stream))


def i8q_gemm_w8a16_group(x, wq, s, y, stream=None) -> None:
    """y [M, N] fp16 = W8A16 group-wise GEMM; x [M, K] fp16, wq [N, K] int8, s [N, K/128] fp16."""
    M, K = x.shape
    N = wq.shape[0]
    _call("i8q_gemm_w8a16_group", _ptr(x), _ptr(wq), _ptr(s), M, N, K, _ptr(y), _stream(stream))


def i8q_gemm_w8a16_group_bf16(x, wq, s, y, stream=None) -> None:
    """y [M, N] bf16 = W8A16 group-wise GEMM; x [M, K] bf16, wq [N, K] int8, s [N, K/128] bf16."""
    M, K = x.shape
    N = wq.shape[0]
    _call("i8q_gemm_w8a16_group_bf16", _ptr(x), _ptr(wq), _ptr(s), M, N, K, _ptr(y), _stream(stream))


def i8q_status_check(stream=None) -> None:
    """Synchronize the stream; raise I8QError(I8Q_ERR_TIMEOUT) if a bounded device wait expired."""
    _call("i8q_status_check", _stream(stream))


def i8q_test_set_wait_limit_ns(ns: int) -> None:
    """Test aid: limit of the pipeline waits on the current device in ns (0 = the 2 s default)."""
    _call("i8q_test_set_wait_limit_ns", int(ns))


def i8q_test_skip_accumulator_signal(armed: bool = True) -> None:
    """Test aid: the next decode-size channel-wise W8A8 GEMM withholds one accumulator signal."""
    _call("i8q_test_skip_accumulator_signal", 1 if armed else 0)


def i8q_status_string(status: int) -> str:
    return load().i8q_status_string(int(status)).decode()


def i8q_version() -> int:
    return load().i8q_version()
