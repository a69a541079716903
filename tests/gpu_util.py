"""Host<->device helpers for the GPU parity tests (torch is only the memory carrier)."""
import numpy as np
import torch

from activation_quantized_gemm_b200 import build


def setup_library():
    from oracle import ref_cpp
    ref_cpp.load()                 # the C++ oracle every GPU parity test compares with
    build.build()
    from activation_quantized_gemm_b200 import i8q
    i8q.load()
    return i8q


def dev(a: np.ndarray) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).cuda()


def host(t: torch.Tensor, dtype=None) -> np.ndarray:
    a = t.cpu().numpy()
    return a.view(dtype) if dtype is not None else a


def empty(shape, dtype, fill=None) -> torch.Tensor:
    t = torch.empty(shape, dtype=dtype, device="cuda")
    if fill is not None:
        t.fill_(fill)
    return t
