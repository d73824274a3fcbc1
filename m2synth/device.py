"""Device fills with the seeded generator (twin of the host generator).

Builds ``libm2synth.so`` from ``fill.cu`` with nvcc (sm_100a) and fills torch
CUDA tensors in place. Bit-identical to ``m2synth.normal_storage`` for the same
key and element range; ``tests/test_synth_device.py`` checks that on a GPU.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fill.cu")
LIB_PATH = os.path.join(_HERE, "libm2synth.so")
_lib = None


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB_PATH) and os.path.getmtime(LIB_PATH) >= os.path.getmtime(_SRC):
        return LIB_PATH
    nvcc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    subprocess.run([nvcc if os.path.exists(nvcc) else "nvcc", "-O3", "-std=c++17",
                    "-gencode", "arch=compute_100a,code=sm_100a", "-Xcompiler", "-fPIC",
                    "-shared", "-fmad=false", _SRC, "-o", LIB_PATH], check=True)
    return LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(LIB_PATH)
        L.m2s_fill_normal.restype = ctypes.c_int
        L.m2s_fill_normal.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64,
                                      ctypes.c_int64, ctypes.c_double, ctypes.c_double,
                                      ctypes.c_void_p]
        _lib = L
    return _lib


def fill_normal(t, key: int, start: int = 0, mean: float = 0.0, std: float = 1.0) -> None:
    """Fill a contiguous float32 / bfloat16 CUDA tensor with elements
    start .. start+numel-1 of the ~N(mean, std) stream of ``key``."""
    import torch
    assert t.is_cuda and t.is_contiguous() and t.dtype in (torch.float32, torch.bfloat16)
    stream = torch.cuda.current_stream(t.device).cuda_stream
    rc = _load().m2s_fill_normal(t.data_ptr(), int(t.dtype == torch.bfloat16), t.numel(),
                                 key & ((1 << 64) - 1), start, mean, std, stream)
    if rc != 0:
        raise RuntimeError(f"m2s_fill_normal failed with CUDA error {rc}")
