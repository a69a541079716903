"""The C ABI on the host: the library loads, exports every declared symbol, and rejects bad
arguments with the documented status before touching a device (no GPU needed)."""
import ctypes

import numpy as np
import pytest

from activation_quantized_gemm_b200 import build, i8q


@pytest.fixture(scope="module")
def lib():
    build.build()
    return i8q.load()


def test_every_declared_symbol_is_exported(lib):
    names = i8q.declared_symbols()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    # the binding wraps every compute entry point under the same name
    for n in names:
        if n not in ("i8q_last_error_string",):
            assert hasattr(i8q, n), n


def test_status_strings(lib):
    for code, name in i8q.STATUS_NAMES.items():
        assert i8q.i8q_status_string(code) == name
    assert i8q.i8q_version() == 100


P = 0x10000   # an aligned fake device address; never dereferenced by the host checks
U = 0x10008   # 8-byte aligned only


def _st(lib, name, *args):
    return getattr(lib, name)(*args)


def test_shape_checks(lib):
    # K not a multiple of 128
    assert _st(lib, "i8q_quant_act_token_group", P, 4, 100, 100, P, P, 4, None) == 2
    assert _st(lib, "i8q_gemm_w8a8_channel", P, P, P, P, 4, 8, 200, P, None, None) == 2
    # a2: K not a multiple of 8 (its rows move as 8-value vectors)
    assert _st(lib, "i8q_quant_act_token", P, 4, 12, 16, P, P, None) == 2
    # negative sizes
    assert _st(lib, "i8q_quant_act_token", P, -1, 128, 128, P, P, None) == 2
    # ldx < K, ld_sx < M, ld_sx not a multiple of 4
    assert _st(lib, "i8q_quant_act_token_group", P, 4, 256, 128, P, P, 4, None) == 2
    assert _st(lib, "i8q_quant_act_token_group", P, 8, 256, 256, P, P, 4, None) == 2
    assert _st(lib, "i8q_quant_act_token_group", P, 3, 256, 256, P, P, 3, None) == 2
    # K so large that int32 accumulation could overflow
    assert _st(lib, "i8q_gemm_w8a8_channel", P, P, P, P, 4, 8, 133248, P, None, None) == 2
    # W8A16: K not a multiple of 128
    assert _st(lib, "i8q_gemm_w8a16_group_bf16", P, P, P, 65, 128, 100, P, None) == 2


def test_new_entry_point_checks(lib):
    # grouped: E out of range, offsets missing or misaligned
    assert _st(lib, "i8q_gemm_w8a8_channel_grouped", P, P, P, P, P, 0, 4, 8, 128, P, None, None) == 2
    assert _st(lib, "i8q_gemm_w8a8_channel_grouped", P, P, P, P, P, 1025, 4, 8, 128, P, None, None) == 2
    assert _st(lib, "i8q_gemm_w8a8_channel_grouped", P, P, P, P, None, 4, 4, 8, 128, P, None, None) == 1
    assert _st(lib, "i8q_gemm_w8a8_block_grouped", P, P, 4, P, P, U, 4, 4, 8, 128, P, 0, None, None) == 3
    assert _st(lib, "i8q_gemm_w8a8_block_grouped", P, P, 4, P, P, P, 4, 4, 8, 128, P, 9, None, None) == 4
    # fused quantization: decode batches only, K % 128, ldx >= K
    assert _st(lib, "i8q_gemm_w8a8_block_fused_quant", P, 128, P, P, 17, 8, 128, P, 0, None, None, 0, None) == 2
    assert _st(lib, "i8q_gemm_w8a8_block_fused_quant", P, 200, P, P, 4, 8, 200, P, 0, None, None, 0, None) == 2
    assert _st(lib, "i8q_gemm_w8a8_block_fused_quant", P, 64, P, P, 4, 8, 128, P, 0, None, None, 0, None) == 2
    assert _st(lib, "i8q_gemm_w8a8_block_fused_quant", P, 128, P, P, 4, 8, 128, P, 0, None, P, 2, None) == 2
    # empty problems need no pointers
    assert _st(lib, "i8q_gemm_w8a8_channel_grouped", None, None, None, None, None, 4, 0, 8, 128, None, None, None) == 0
    assert _st(lib, "i8q_gemm_w8a8_block_fused_quant", None, 0, None, None, 0, 8, 128, None, 0, None, None, 0, None) == 0
    assert _st(lib, "i8q_gemm_w8a16_group_bf16", None, None, None, 0, 8, 128, None, None) == 0


def test_null_align_dtype_checks(lib):
    assert _st(lib, "i8q_quant_act_token_group", None, 4, 128, 128, P, P, 4, None) == 1
    assert _st(lib, "i8q_gemm_w8a8_channel", P, None, P, P, 4, 8, 128, P, None, None) == 1
    assert _st(lib, "i8q_quant_act_token", U, 4, 128, 128, P, P, None) == 3
    assert _st(lib, "i8q_requant_fp8_to_int8_block", P, U, 128, 128, P, P, None) == 3
    assert _st(lib, "i8q_gemm_w8a8_block", P, P, 4, P, P, 4, 8, 128, P, 7, None, None) == 4


def test_empty_problems_are_noops(lib):
    # M == 0 / N == 0 return OK without any CUDA call (null pointers allowed)
    assert _st(lib, "i8q_quant_act_token_group", None, 0, 128, 128, None, None, 0, None) == 0
    assert _st(lib, "i8q_gemm_w8a8_channel", None, None, None, None, 0, 8, 128, None, None, None) == 0
    assert _st(lib, "i8q_gemm_w8a8_block", None, None, 0, None, None, 4, 0, 128, None, 0, None, None) == 0
    assert _st(lib, "i8q_gemm_w8a16_group", None, None, None, 0, 8, 128, None, None) == 0


def test_any_n_passes_the_shape_checks(lib):
    """N need not be a multiple of 8 (masked tails): with no GPU such a call gets past every
    argument check and fails only at the device (I8Q_ERR_CUDA), never with I8Q_ERR_SHAPE."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    for n in (1, 7, 129, 7170):
        assert _st(lib, "i8q_gemm_w8a8_block", P, P, 4, P, P, 4, n, 128, P, 0, None, None) == 5
        assert _st(lib, "i8q_gemm_w8a8_channel", P, P, P, P, 4, n, 128, P, None, None) == 5
        assert _st(lib, "i8q_gemm_w8a16_group", P, P, P, 4, n, 128, P, None) == 5
    assert _st(lib, "i8q_quant_act_token", P, 4, 24, 24, P, P, None) == 5


def test_valid_call_without_device_fails_loudly(lib):
    """With no usable GPU a well-formed call reports I8Q_ERR_CUDA; there is no CPU fallback."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    st = _st(lib, "i8q_quant_act_token", P, 4, 128, 128, P, P, None)
    assert st == 5
    assert lib.i8q_last_error_string().decode() != ""
    with pytest.raises(i8q.I8QError):
        i8q._call("i8q_quant_act_token", P, 4, 128, 128, P, P, None)
