"""Build and call the SM-holding test helper (tests/gpu_hold.cu).

Test infrastructure only: the library never uses it.  hold_sm() occupies one
SM with a 32-thread CTA that holds `smem_bytes` of shared memory for a
bounded number of clock cycles, on a given torch stream.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "gpu_hold.cu")
LIB = os.path.join(HERE, "libgpu_hold.so")
_lib = None


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call([os.environ.get("NVCC", "nvcc"), "-gencode", "arch=compute_100a,code=sm_100a",
                               "-O2", "-shared", "-Xcompiler", "-fPIC", "-o", tmp, SRC])
        os.replace(tmp, LIB)
    return LIB


def hold_sm(cycles: int, smem_bytes: int, done, stream) -> None:
    """done: an int32 CUDA tensor the kernel sets to 1 when it ends."""
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.gpu_hold_sm.restype = ctypes.c_int
        _lib.gpu_hold_sm.argtypes = [ctypes.c_longlong, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    rc = _lib.gpu_hold_sm(int(cycles), int(smem_bytes), ctypes.c_void_p(done.data_ptr()),
                          ctypes.c_void_p(stream.cuda_stream))
    if rc:
        raise RuntimeError(f"gpu_hold_sm failed with CUDA error {rc}")
