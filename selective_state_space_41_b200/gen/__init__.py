"""Seeded synthetic inputs (host side), shared by the tests, the benchmark and
the smoke check.  The arithmetic of the scan lives elsewhere: this module only
draws numbers (Philox4x32-10 + Box-Muller, see ``ssgen.c``) into host tensors.
"""
import ctypes
import os
import subprocess

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ssgen.c")
LIB = os.path.join(HERE, "libssgen.so")

NORMAL, UNIFORM = 0, 1
_F32, _BF16 = 0, 1

_lib = None


def build(force: bool = False) -> str:
    """Compile ``ssgen.c`` into ``libssgen.so`` (gcc, OpenMP, strict IEEE)."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
           SRC, "-o", LIB + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.ssgen_fill.restype = ctypes.c_int
        lib.ssgen_fill.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int64, ctypes.c_int,
                                   ctypes.c_double, ctypes.c_double, ctypes.c_int, ctypes.c_void_p,
                                   ctypes.c_int]
        lib.ssgen_philox4x32_10.restype = None
        lib.ssgen_philox4x32_10.argtypes = [ctypes.POINTER(ctypes.c_uint32)] * 3
        lib.ssgen_f32_to_bf16.restype = ctypes.c_uint16
        lib.ssgen_f32_to_bf16.argtypes = [ctypes.c_float]
        _lib = lib
    return _lib


def philox4x32_10(ctr, key):
    """One Philox4x32-10 block: four 32-bit counter words, two key words."""
    c = (ctypes.c_uint32 * 4)(*ctr)
    k = (ctypes.c_uint32 * 2)(*key)
    o = (ctypes.c_uint32 * 4)()
    _load().ssgen_philox4x32_10(c, k, o)
    return list(o)


def f32_to_bf16_bits(x: float) -> int:
    return int(_load().ssgen_f32_to_bf16(ctypes.c_float(x)))


def fill(shape, dtype, seed, stream, kind=NORMAL, p0=0.0, p1=1.0, pin=False, nthreads=0):
    """A new host tensor of ``shape`` filled with seeded draws.

    kind NORMAL: mean p0, std p1.  kind UNIFORM: [p0, p1).
    dtype torch.float32 or torch.bfloat16 (bf16 = RNE of the float32 draw).
    """
    if dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("generator writes float32 or bfloat16")
    t = torch.empty(shape, dtype=dtype, pin_memory=pin)
    n = t.numel()
    rc = _load().ssgen_fill(int(seed), int(stream), n, int(kind), float(p0), float(p1),
                            _F32 if dtype == torch.float32 else _BF16,
                            ctypes.c_void_p(t.data_ptr()) if n else None, int(nthreads))
    if rc != 0:
        raise RuntimeError("ssgen_fill rejected its arguments")
    return t
