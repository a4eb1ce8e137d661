"""Host SIMD W4A8 decode of the MoE layer: a timed CPU baseline (the page's
own decode method, integer multiply-adds over unpacked nibbles), built with
gcc for the machine it runs on.  Independent of the CUDA library and of the
oracle; the GPU library never loads it."""
import ctypes
import hashlib
import os
import subprocess
from typing import Optional

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "w4a8_simd.c")
CFLAGS = ["-O3", "-march=native", "-fPIC", "-shared", "-fopenmp", "-std=c11"]


def _cpu_tag() -> str:
    """Short hash of this CPU's feature flags: the library is built with
    -march=native, so a copy built on another machine is never reused."""
    flags = ""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("flags"):
                    flags = line
                    break
    except OSError:
        pass
    return hashlib.sha256(flags.encode()).hexdigest()[:12]


LIB = os.path.join(HERE, f"libw4a8_simd_{_cpu_tag()}.so")

_lib = None


class _Layer(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("H", "F", "E", "k", "S")] + \
               [(n, ctypes.c_void_p) for n in ("w_router", "bias", "w_gate", "w_up", "w_down",
                                                "sh_gate", "sh_up", "sh_down")]


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        subprocess.run(["gcc", *CFLAGS, SRC, "-o", LIB, "-lm"], check=True)
    return LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        lib.simd_moe_forward.argtypes = [P, P, ctypes.c_int64, P]
        lib.simd_moe_forward.restype = ctypes.c_int
        lib.simd_block_dots.argtypes = [P, P, ctypes.c_int64, P]
        lib.simd_threads.argtypes = [ctypes.c_int]
        lib.simd_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def set_threads(n: int = 0) -> int:
    return _load().simd_threads(int(n))


def block_dots(blocks: np.ndarray, qa: np.ndarray) -> np.ndarray:
    blocks = np.ascontiguousarray(blocks, np.uint8)
    qa = np.ascontiguousarray(qa, np.int8)
    n = blocks.shape[0]
    out = np.empty(n, np.int32)
    _load().simd_block_dots(_p(blocks), _p(qa), n, _p(out))
    return out


def moe_forward(layer, x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float32)
    keep = []

    def c(a, dt):
        if a is None:
            return None
        a = np.ascontiguousarray(a, dt)
        keep.append(a)
        return a

    S = 1 if layer.sh_gate is not None else 0
    L = _Layer(layer.hidden, layer.ffn, layer.n_experts, layer.top_k, S,
               _p(c(layer.w_router, np.float32)), _p(c(layer.router_bias, np.float32)),
               _p(c(layer.w_gate, np.uint8)), _p(c(layer.w_up, np.uint8)), _p(c(layer.w_down, np.uint8)),
               _p(c(layer.sh_gate, np.uint8)), _p(c(layer.sh_up, np.uint8)), _p(c(layer.sh_down, np.uint8)))
    y = np.empty_like(x)
    if _load().simd_moe_forward(ctypes.byref(L), _p(x), x.shape[0], _p(y)) != 0:
        raise ValueError("invalid layer shape")
    return y
