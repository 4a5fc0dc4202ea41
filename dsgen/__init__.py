"""Seeded synthetic inputs for token-sparse decode attention.

Shared by the CPU oracle, the GPU tests and the benchmark.  This module draws
inputs only; it holds none of the attention method's arithmetic.  All tensors
are returned as numpy ``uint16`` arrays of bf16 bit patterns, so that both
sides of a parity test start from identical bits.

The C source (``gen.c``) is compiled on first use with the host C compiler if
the shared object is missing or older than the source.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

from .configs import CONFIGS, ORDER, Workload, workload  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.c")
_LIB = os.path.join(_HERE, "libdsgen.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile gen.c into libdsgen.so next to it; returns the library path."""
    stale = not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fPIC", "-shared", "-Wall", "-o", tmp, _SRC, "-lm", "-lpthread"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            u64, i32 = ctypes.c_uint64, ctypes.c_int
            p16 = ctypes.POINTER(ctypes.c_uint16)
            p32 = ctypes.POINTER(ctypes.c_int32)
            dims = [u64] + [i32] * 8
            lib.dsgen_qkv.argtypes = dims + [p16, p16, p16, i32]
            lib.dsgen_q_slab.argtypes = dims + [i32, i32, p16]
            lib.dsgen_kv_slab.argtypes = dims + [i32, i32, i32, p16]
            lib.dsgen_channels.argtypes = [u64, i32, i32, i32, p32]
            lib.dsgen_perm_head.argtypes = [u64, i32, i32, p32]
            lib.dsgen_perm_head.restype = None
            lib.dsgen_hh_positions.argtypes = dims + [p32]
            lib.dsgen_q_calib.argtypes = [u64, i32, i32, i32, i32, i32, p16]
            _lib = lib
    return _lib


def _p16(a):
    if a is None:
        return None
    assert a.dtype == np.uint16 and a.flags.c_contiguous
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16))


def _p32(a):
    assert a.dtype == np.int32 and a.flags.c_contiguous
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def _dims(w: Workload):
    return (w.seed, w.B, w.Hq, w.Hkv, w.d, w.T, w.n_out, w.r if w.n_hh else 0, w.n_hh)


def qkv(w: Workload, want=("Q", "K", "V"), nthreads: int = 0):
    """Full Q [B,Hq,d], K and V [B,Hkv,T,d] (bf16 bits) for workload ``w``."""
    lib = _load()
    Q = np.empty((w.B, w.Hq, w.d), np.uint16) if "Q" in want else None
    K = np.empty((w.B, w.Hkv, w.T, w.d), np.uint16) if "K" in want else None
    V = np.empty((w.B, w.Hkv, w.T, w.d), np.uint16) if "V" in want else None
    rc = lib.dsgen_qkv(*_dims(w), _p16(Q), _p16(K), _p16(V), nthreads)
    if rc != 0:
        raise ValueError(f"dsgen_qkv rejected {w}")
    return Q, K, V


def q_slab(w: Workload, b: int, h: int) -> np.ndarray:
    """Q[b, h, :] alone (bit-identical to the full tensor's slab)."""
    out = np.empty((w.d,), np.uint16)
    if _load().dsgen_q_slab(*_dims(w), b, h, _p16(out)) != 0:
        raise ValueError("bad slab")
    return out


def kv_slab(w: Workload, which: str, b: int, g: int) -> np.ndarray:
    """K[b, g] or V[b, g] ([T, d]) alone (bit-identical to the full tensor's slab)."""
    out = np.empty((w.T, w.d), np.uint16)
    sel = {"K": 0, "V": 1}[which]
    if _load().dsgen_kv_slab(*_dims(w), sel, b, g, _p16(out)) != 0:
        raise ValueError("bad slab")
    return out


def q_calib(w: Workload, Nq: int) -> np.ndarray:
    """Calibration queries Qc [B,Hq,Nq,d] (bf16 bits): Nq extra queries per head,
    with the same outlier channels as Q, from a stream of their own."""
    out = np.empty((w.B, w.Hq, Nq, w.d), np.uint16)
    if _load().dsgen_q_calib(w.seed, w.B, w.Hq, w.d, w.n_out, Nq, _p16(out)) != 0:
        raise ValueError("bad calibration request")
    return out


def channels(w: Workload, r: int | None = None) -> np.ndarray:
    """C [Hq, r] int32: each query head's r label channels, ascending."""
    r = w.r if r is None else r
    C = np.empty((w.Hq, r), np.int32)
    if _load().dsgen_channels(w.seed, w.Hq, w.d, r, _p32(C)) != 0:
        raise ValueError("bad channel request")
    return C


def permutation(w: Workload, h: int) -> np.ndarray:
    """The channel permutation pi_h of query head h; its first n_out entries are outliers."""
    p = np.empty((w.d,), np.int32)
    _load().dsgen_perm_head(w.seed, h, w.d, _p32(p))
    return p


def outliers(w: Workload, h: int) -> np.ndarray:
    return np.sort(permutation(w, h)[: w.n_out])


def hh_positions(w: Workload) -> np.ndarray:
    """Heavy-hitter token positions [Hq, n_hh] (empty when the workload has none)."""
    pos = np.empty((w.Hq, w.n_hh), np.int32)
    if w.n_hh and _load().dsgen_hh_positions(*_dims(w), _p32(pos)) != 0:
        raise ValueError("bad heavy-hitter request")
    return pos


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even) and return the bits.

    Used by tests to build small hand-made inputs; NaN is not expected.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bias = 0x7FFF + ((u >> 16) & 1)
    return ((u + bias) >> 16).astype(np.uint16)
