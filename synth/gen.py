"""Generator binding: draws seeded normals / integers through ``libsynth.so``."""
from __future__ import annotations

import ctypes
import os
import subprocess

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_SO = os.path.join(_HERE, "libsynth.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the generator into ``synth/libsynth.so`` with gcc."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-shared", "-fPIC", _SRC, "-o", _SO, "-lm", "-lpthread"]
        )
    return _SO


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u64, i64, i32, dbl = ctypes.c_uint64, ctypes.c_int64, ctypes.c_int32, ctypes.c_double
        vp = ctypes.c_void_p
        lib.synth_normal_f32.argtypes = [u64, u64, dbl, dbl, i64, i64, vp, ctypes.c_int]
        lib.synth_normal_bf16.argtypes = [u64, u64, dbl, dbl, i64, i64, vp, ctypes.c_int]
        lib.synth_uniform_int.argtypes = [u64, u64, i32, i64, i64, vp, ctypes.c_int]
        lib.synth_word.argtypes = [u64, u64, u64]
        lib.synth_word.restype = u64
        _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, min(64, os.cpu_count() or 1))


def normal(seed: int, tag: int, shape, std: float, dtype=torch.bfloat16, mean: float = 0.0,
           first: int = 0, threads: int | None = None) -> torch.Tensor:
    """CPU tensor of ``mean + std * N(0,1)`` draws #first.. of stream (seed, tag)."""
    lib = _load()
    n = 1
    for s in shape:
        n *= int(s)
    th = threads or default_threads()
    if dtype == torch.float32:
        out = torch.empty(n, dtype=torch.float32)
        lib.synth_normal_f32(seed, tag, mean, std, first, n, out.data_ptr(), th)
    elif dtype == torch.bfloat16:
        out = torch.empty(n, dtype=torch.int16)
        lib.synth_normal_bf16(seed, tag, mean, std, first, n, out.data_ptr(), th)
        out = out.view(torch.bfloat16)
    else:
        raise ValueError(f"unsupported dtype {dtype}")
    return out.view(*shape)


def uniform_int(seed: int, tag: int, n: int, value_range: int, first: int = 0,
                threads: int | None = None) -> torch.Tensor:
    """CPU int32 tensor: word #first+i of stream (seed, tag) modulo ``value_range``."""
    lib = _load()
    out = torch.empty(n, dtype=torch.int32)
    lib.synth_uniform_int(seed, tag, value_range, first, n, out.data_ptr(), threads or default_threads())
    return out


def word(seed: int, tag: int, i: int) -> int:
    """Raw 64-bit word #i of stream (seed, tag)."""
    return int(_load().synth_word(seed, tag, i))
