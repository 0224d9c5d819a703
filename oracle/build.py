"""Compile the C oracle (``conv_ref.c``) with gcc.  Test infrastructure only."""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "conv_ref.c")
OUT_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(OUT_DIR, "liboracle_conv.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """gcc -O2 -fopenmp -shared; rebuilt when the source is newer."""
    os.makedirs(OUT_DIR, exist_ok=True)
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
                               SRC, "-o", tmp])
        os.replace(tmp, LIB)
    return LIB


def load() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            _lib = ctypes.CDLL(build())
    return _lib
