"""Device-side twin of the synthetic value generator (``synth/fill.cu``).

Fills torch CUDA tensors in place with the values that
``synth.counter_values`` gives on the host for flat indices 0..numel-1.
Input generation only: nothing of the lookup's arithmetic lives here.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

from . import DTYPE_BF16, DTYPE_E4M3, DTYPE_F32, value_scale

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsynth_fill.so")
_lib = None


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "fill.cu")
    if not force and os.path.exists(LIB_PATH) and os.path.getmtime(LIB_PATH) >= os.path.getmtime(src):
        return LIB_PATH
    cmd = ["nvcc", "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
           "-shared", "-Xcompiler", "-fPIC", "-o", LIB_PATH, src]
    subprocess.run(cmd, check=True)
    return LIB_PATH


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run synth.gpu.build()")
        lib = ctypes.CDLL(LIB_PATH)
        lib.synth_fill.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_float, ctypes.c_int,
                                   ctypes.c_void_p, ctypes.c_void_p]
        lib.synth_fill.restype = ctypes.c_int
        _lib = lib
    return _lib


def fill_(tensor, seed: int, sigma: float) -> None:
    """Fill a contiguous fp32, bf16 or fp8 e4m3 CUDA tensor with generator values."""
    import torch

    if not tensor.is_cuda or not tensor.is_contiguous():
        raise ValueError("fill_ wants a contiguous CUDA tensor")
    if tensor.dtype == torch.float32:
        code = DTYPE_F32
    elif tensor.dtype == torch.bfloat16:
        code = DTYPE_BF16
    elif tensor.dtype == torch.float8_e4m3fn:
        code = DTYPE_E4M3
    else:
        raise ValueError(f"unsupported dtype {tensor.dtype}")
    stream = torch.cuda.current_stream(tensor.device).cuda_stream
    with torch.cuda.device(tensor.device):
        rc = _load().synth_fill(seed, tensor.numel(), float(value_scale(sigma)), code,
                                tensor.data_ptr(), stream)
    if rc != 0:
        raise RuntimeError(f"synth_fill failed with code {rc}")
