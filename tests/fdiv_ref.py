"""Builds and loads the test-only CUDA helper ``csrc/fdiv_ref.cu`` (IEEE
division by ``__fdiv_rn`` and a device-side draw of random operands) into
``tests/_build/``, with the same nvcc and sm_100a target as the library."""
from __future__ import annotations

import ctypes
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "fdiv_ref.cu")
OUT = os.path.join(HERE, "_build", "libfdiv_ref.so")


def build(force: bool = False) -> str:
    from bit_quantization_aware_b200 import build as pqbuild
    if not force and os.path.exists(OUT) and os.path.getmtime(OUT) >= os.path.getmtime(SRC):
        return OUT
    os.makedirs(os.path.dirname(OUT), exist_ok=True)
    tmp = OUT + f".{os.getpid()}.tmp"
    subprocess.check_call([pqbuild.nvcc(), *pqbuild.ARCH, "-O3", "-std=c++17",
                           "-Xcompiler", "-fPIC", "-shared", "-o", tmp, SRC])
    os.replace(tmp, OUT)
    return OUT


def load():
    L = ctypes.CDLL(build())
    i64, p = ctypes.c_int64, ctypes.c_void_p
    L.fdiv_ref.argtypes = [p, p, p, i64, i64, p]
    L.fdiv_ref.restype = ctypes.c_int
    L.fdiv_draw.argtypes = [p, i64, ctypes.c_uint64, ctypes.c_int, ctypes.c_int, p]
    L.fdiv_draw.restype = ctypes.c_int
    return L
