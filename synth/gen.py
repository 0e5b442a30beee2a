"""Seeded, counter-based synthetic inputs shared by the oracle side and the CUDA side.

This module only draws numbers: it holds none of the method's arithmetic.  Every value
is a pure function of (base seed, tensor name, element index), so any slice can be
regenerated on its own and both sides of a parity test receive identical inputs.

Generator (published definitions, implemented here from them):
  * splitmix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number generators",
    OOPSLA 2014): state_i = key + (i + 1) * 0x9E3779B97F4A7C15, output = mix64(state_i).
  * per-tensor key = mix64(seed XOR fnv1a64(name)) (FNV-1a, 64-bit).
  * uniform in [0, 1): top 53 bits * 2^-53.
  * normal: Box-Muller on consecutive pairs (u1, u2) -> (r cos 2*pi*u2, r sin 2*pi*u2),
    r = sqrt(-2 ln(1 - u1)).
  * bf16: round-to-nearest-even of the float32 value.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

BASE_SEED = 20251030
_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22


def _mix64(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def fnv1a64(name: str) -> int:
    h = 0xCBF29CE484222325
    for byte in name.encode():
        h ^= byte
        h = (h * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
    return h


def stream_key(name: str, seed: int = BASE_SEED) -> np.uint64:
    with np.errstate(over="ignore"):
        return _mix64(np.array([(seed ^ fnv1a64(name)) & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64))[0]


def raw_u64(name: str, n: int, seed: int = BASE_SEED, offset: int = 0) -> np.ndarray:
    key = stream_key(name, seed)
    out = np.empty(n, dtype=np.uint64)
    with np.errstate(over="ignore"):
        for s in range(0, n, _CHUNK):
            e = min(n, s + _CHUNK)
            idx = np.arange(offset + s + 1, offset + e + 1, dtype=np.uint64)
            out[s:e] = _mix64(key + idx * _GAMMA)
    return out


def uniform(name: str, n: int, seed: int = BASE_SEED, offset: int = 0) -> np.ndarray:
    """float64 uniforms in [0, 1)."""
    return (raw_u64(name, n, seed, offset) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "_libgen.so")
_lib = None


def build_fast(force: bool = False) -> str:
    """Compile _gen.c (the same generator in C, OpenMP) into _libgen.so next to this file."""
    src = os.path.join(_HERE, "_gen.c")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        tmp = _LIB_PATH + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", tmp, src, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _fast():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build_fast())
        for fn, ptr_t in (("synth_normal_f32", ctypes.c_float), ("synth_normal_bf16", ctypes.c_uint16)):
            f = getattr(lib, fn)
            f.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.POINTER(ptr_t)]
            f.restype = None
        _lib = lib
    return _lib


def normal(name: str, shape, std: float = 1.0, seed: int = BASE_SEED) -> np.ndarray:
    """float32 N(0, std^2) of the given shape; same values as normal_reference."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)
    _fast().synth_normal_f32(int(stream_key(name, seed)), n, float(std),
                             out.ctypes.data_as(ctypes.POINTER(ctypes.c_float)))
    return out.reshape(shape)


def normal_reference(name: str, shape, std: float = 1.0, seed: int = BASE_SEED) -> np.ndarray:
    """float32 N(0, std^2) of the given shape (Box-Muller over element pairs), in numpy."""
    n = int(np.prod(shape))
    m = (n + 1) // 2
    out = np.empty(2 * m, dtype=np.float32)
    for s in range(0, m, _CHUNK):
        e = min(m, s + _CHUNK)
        u = uniform(name, 2 * (e - s), seed, offset=2 * s)
        u1, u2 = u[0::2], u[1::2]
        r = np.sqrt(-2.0 * np.log1p(-u1))
        ang = 2.0 * np.pi * u2
        blk = np.empty(2 * (e - s), dtype=np.float64)
        blk[0::2] = r * np.cos(ang)
        blk[1::2] = r * np.sin(ang)
        out[2 * s:2 * e] = (blk * std).astype(np.float32)
    return out[:n].reshape(shape)


def randint(name: str, n: int, lo: int, hi: int, seed: int = BASE_SEED) -> np.ndarray:
    """int64 uniform integers in [lo, hi] (inclusive), by multiply-shift of the top 32 bits."""
    span = hi - lo + 1
    top = (raw_u64(name, n, seed) >> np.uint64(32)).astype(np.uint64)
    return (lo + ((top * np.uint64(span)) >> np.uint64(32)).astype(np.int64)).astype(np.int64)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest-even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16(name: str, shape, std: float = 1.0, seed: int = BASE_SEED) -> np.ndarray:
    """bf16 bit patterns of a seeded normal tensor (bf16_bits of normal())."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    _fast().synth_normal_bf16(int(stream_key(name, seed)), n, float(std),
                              out.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16)))
    return out.reshape(shape)
