"""Device-side draws with the generator of ``gen.py`` (identical bits).

Builds ``libseeded_gen.so`` next to this file (nvcc, sm_100a) and fills torch
CUDA tensors in place. Used only to create large synthetic inputs quickly.
"""
from __future__ import annotations

import ctypes
import os
import shutil
import subprocess

from .gen import normal_scale, stream_key

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "libseeded_gen.so")
SRC = os.path.join(HERE, "gen_kernels.cu")
_lib = None


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-shared", "-Xcompiler", "-fPIC",
                    "-Xcompiler", "-fvisibility=hidden", "-o", LIB + ".tmp", SRC], check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            build()
        _lib = ctypes.CDLL(LIB)
        for fn in (_lib.sg_normal_bf16, _lib.sg_normal_f32):
            fn.restype = ctypes.c_int
            fn.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_double,
                           ctypes.c_void_p]
    return _lib


def fill_normal(t, seed: int, stream, sigma: float, start: int = 0):
    """Fill a contiguous CUDA tensor (bfloat16 or float32) with the draws of
    (seed, stream) at flat indices start .. start + numel - 1."""
    import torch
    assert t.is_cuda and t.is_contiguous()
    lib = _load()
    key = stream_key(seed, stream)
    s = torch.cuda.current_stream(t.device).cuda_stream
    if t.dtype == torch.bfloat16:
        rc = lib.sg_normal_bf16(t.data_ptr(), t.numel(), key, start, normal_scale(sigma), s)
    elif t.dtype == torch.float32:
        rc = lib.sg_normal_f32(t.data_ptr(), t.numel(), key, start, normal_scale(sigma), s)
    else:
        raise TypeError("fill_normal: bfloat16 or float32 only")
    if rc != 0:
        raise RuntimeError(f"seeded generator launch failed ({rc})")
    return t
