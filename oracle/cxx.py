"""The C++ oracle (oracle/ds_oracle.cpp) -- TEST INFRASTRUCTURE ONLY.

The same functions, signatures and results as the numpy oracle: label,
score, top-k, attention, dense, merge and the whole step (O1-O5), and the
calibration, group-shared, block and hierarchical selections beside them,
computed in plain C++ (float64, std::sort, std::exp).  This module only
converts arrays and calls the library; every arithmetic step runs in
ds_oracle.cpp.  The library is built here with g++ on first use (or by
``build()``).

Only ``tests/`` and ``bench.py``'s CPU-baseline leg use it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ds_oracle.cpp")
_LIB = os.path.join(_HERE, "libds_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ds_oracle.cpp into libds_oracle.so next to it; returns the path."""
    stale = not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-fPIC", "-shared", "-std=c++17", "-Wall",
                               "-Wextra", "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            vp, i32, i64, f64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
            sig = {
                "dso_bf16_to_f64": [vp, i64, vp],
                "dso_to_f32": [vp, i64, vp],
                "dso_label": [vp, vp, i32, i32, i32, i32, i32, i32, vp],
                "dso_score": [vp, vp, vp, i32, i32, i32, i32, i32, vp],
                "dso_topk_f64": [vp, i64, i32, i32, vp],
                "dso_topk_f32": [vp, i64, i32, i32, vp],
                "dso_attend": [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f64, vp, vp, vp],
                "dso_dense": [vp, vp, vp, i32, i32, i32, i32, i32, f64, vp, vp],
                "dso_lse_merge": [vp, vp, i32, i32, vp, vp],
                "dso_attend_split": [vp, vp, vp, vp, i32, i32, f64, i32, vp, vp],
                "dso_calib_importance": [vp, vp, i32, i32, i32, i32, i32, i32, i32, vp],
                "dso_calib_select": [vp, i32, i32, i32, vp],
                "dso_group_score_f64": [vp, i32, i32, i32, i32, vp],
                "dso_group_score_f32": [vp, i32, i32, i32, i32, vp],
                "dso_group_attend": [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f64, vp,
                                     vp],
                "dso_block_score_f64": [vp, i64, i32, i32, vp],
                "dso_block_score_f32": [vp, i64, i32, i32, vp],
                "dso_block_tokens": [vp, i32, i32, i32, vp],
                "dso_block_attend": [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, f64,
                                     vp, vp],
                "dso_hier_topk_f64": [vp, i64, i32, i32, vp],
                "dso_hier_topk_f32": [vp, i64, i32, i32, vp],
                "dso_step_heads_mt": [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f64, i32,
                                      i32, vp, vp, vp, vp],
            }
            for name, args in sig.items():
                fn = getattr(lib, name)
                fn.argtypes = args
                fn.restype = (ctypes.c_int if name in ("dso_block_tokens", "dso_step_heads_mt")
                              else None)
            _lib = lib
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a):
    return ctypes.c_void_p(a.ctypes.data)


# ---------------------------------------------------------------------------

def bf16_to_f64(bits):
    b = _c(bits, np.uint16)
    out = np.empty(b.shape, np.float64)
    _load().dso_bf16_to_f64(_p(b), b.size, _p(out))
    return out


def to_f32(x):
    a = _c(x, np.float64)
    out = np.empty(a.shape, np.float32)
    _load().dso_to_f32(_p(a), a.size, _p(out))
    return out


def label(K, C, Hq: int):
    """label [B, Hq, T, r] from K [B, Hkv, T, d] and C [Hq, r]."""
    K = _c(K, np.uint16)
    C = _c(C, np.int32)
    B, Hkv, T, d = K.shape
    r = C.shape[1]
    out = np.empty((B, Hq, T, r), np.uint16)
    _load().dso_label(_p(K), _p(C), B, Hq, Hkv, T, d, r, _p(out))
    return out


def label_head(K_bg, C_h):
    K = _c(K_bg, np.uint16)
    return label(K[None, None], _c(C_h, np.int32)[None], 1)[0, 0]


def score(Q, C, lab):
    """s [B, Hq, T] float64 from Q [B, Hq, d], C [Hq, r], label [B, Hq, T, r]."""
    Q = _c(Q, np.uint16)
    C = _c(C, np.int32)
    lab = _c(lab, np.uint16)
    B, Hq, T, r = lab.shape
    out = np.empty((B, Hq, T), np.float64)
    _load().dso_score(_p(Q), _p(C), _p(lab), B, Hq, T, Q.shape[-1], r, _p(out))
    return out


def score_head(q_h, C_h, label_h):
    q = _c(q_h, np.uint16)
    return score(q[None, None], _c(C_h, np.int32)[None], _c(label_h, np.uint16)[None, None])[0, 0]


def topk(s, k: int):
    """idx [..., k] int32 for scores [..., T]; float32 scores are ordered as float32."""
    s = np.asarray(s)
    T = s.shape[-1]
    if not 1 <= k <= T:
        raise ValueError("need 1 <= k <= T")
    f32 = s.dtype == np.float32
    flat = _c(s.reshape(-1, T), np.float32 if f32 else np.float64)
    out = np.empty((flat.shape[0], k), np.int32)
    fn = _load().dso_topk_f32 if f32 else _load().dso_topk_f64
    fn(_p(flat), flat.shape[0], T, k, _p(out))
    return out.reshape(*s.shape[:-1], k)


def topk_head(s, k: int):
    return topk(np.asarray(s)[None], k)[0]


def attend(Q, K, V, idx, scale, weights: bool = False):
    """O [B, Hq, d], lse [B, Hq] (float64) for idx [B, Hq, k] (and w [B, Hq, k])."""
    Q = _c(Q, np.uint16)
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    idx = _c(idx, np.int32)
    B, Hq, d = Q.shape
    _, Hkv, T, _ = K.shape
    k = idx.shape[-1]
    O = np.empty((B, Hq, d), np.float64)
    L = np.empty((B, Hq), np.float64)
    w = np.empty((B, Hq, k), np.float64) if weights else None
    _load().dso_attend(_p(Q), _p(K), _p(V), _p(idx), B, Hq, Hkv, T, d, k, float(scale), _p(O),
                       _p(L), _p(w) if weights else None)
    return (O, L, w) if weights else (O, L)


def attend_head(q_h, K_bg, V_bg, idx, scale):
    """(o [d], lse, w [len(idx)]) of one query over the rows idx of K and V."""
    O, L, w = attend(_c(q_h, np.uint16)[None, None], _c(K_bg, np.uint16)[None, None],
                     _c(V_bg, np.uint16)[None, None], _c(idx, np.int32)[None, None], scale,
                     weights=True)
    return O[0, 0], float(L[0, 0]), w[0, 0]


def dense(Q, K, V, scale):
    Q = _c(Q, np.uint16)
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    B, Hq, d = Q.shape
    _, Hkv, T, _ = K.shape
    O = np.empty((B, Hq, d), np.float64)
    L = np.empty((B, Hq), np.float64)
    _load().dso_dense(_p(Q), _p(K), _p(V), B, Hq, Hkv, T, d, float(scale), _p(O), _p(L))
    return O, L


def lse_merge(outs, lses):
    outs = _c(outs, np.float64)
    lses = _c(lses, np.float64)
    n, d = outs.shape
    o = np.empty(d, np.float64)
    lse = np.empty(1, np.float64)
    _load().dso_lse_merge(_p(outs), _p(lses), n, d, _p(o), _p(lse))
    return o, float(lse[0])


def attend_split_head(q_h, K_bg, V_bg, idx, scale, n_chunks: int):
    q = _c(q_h, np.uint16)
    K = _c(K_bg, np.uint16)
    V = _c(V_bg, np.uint16)
    idx = _c(idx, np.int32)
    d = q.shape[0]
    o = np.empty(d, np.float64)
    lse = np.empty(1, np.float64)
    _load().dso_attend_split(_p(q), _p(K), _p(V), _p(idx), idx.shape[0], d, float(scale),
                             int(n_chunks), _p(o), _p(lse))
    return o, float(lse[0])


def sparse_step(Q, K, V, C, k: int, scale):
    """label -> score -> top-k on float32-rounded scores -> attention (each step in C++)."""
    Hq = np.asarray(Q).shape[1]
    lab = label(K, C, Hq)
    s64 = score(Q, C, lab)
    s32 = to_f32(s64)
    idx = topk(s32, k)
    O, L = attend(Q, K, V, idx, scale)
    return {"label": lab, "s64": s64, "s32": s32, "idx": idx, "O": O, "lse": L}


# ---- offline channel calibration -------------------------------------------------

def calibrate_importance(Qc, K, T: int, Hq: int):
    """I [Hq, d] float64 from Qc [B, Hq, Nq, d] and K [B, Hkv, T_cap, d] (tokens < T)."""
    Qc = _c(Qc, np.uint16)
    K = _c(K, np.uint16)
    B, _, Nq, d = Qc.shape
    _, Hkv, T_cap, _ = K.shape
    I = np.empty((Hq, d), np.float64)
    _load().dso_calib_importance(_p(Qc), _p(K), B, Hq, Hkv, Nq, T_cap, T, d, _p(I))
    return I


def calibrate_select(I, r: int):
    I = _c(I, np.float64)
    Hq, d = I.shape
    C = np.empty((Hq, r), np.int32)
    _load().dso_calib_select(_p(I), Hq, d, r, _p(C))
    return C


def calibrate(Qc, K, T: int, Hq: int, r: int):
    I = calibrate_importance(Qc, K, T, Hq)
    return calibrate_select(I, r), I


# ---- group-shared selection ------------------------------------------------------

def group_score(s, Hkv: int):
    """sg [B, Hkv, T] in the precision of s [B, Hq, T] (head order)."""
    s = np.asarray(s)
    f32 = s.dtype == np.float32
    s = _c(s, np.float32 if f32 else np.float64)
    B, Hq, T = s.shape
    sg = np.empty((B, Hkv, T), s.dtype)
    fn = _load().dso_group_score_f32 if f32 else _load().dso_group_score_f64
    fn(_p(s), B, Hq, Hkv, T, _p(sg))
    return sg


def group_attend(Q, K, V, idx_g, scale):
    Q = _c(Q, np.uint16)
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    idx_g = _c(idx_g, np.int32)
    B, Hq, d = Q.shape
    _, Hkv, T, _ = K.shape
    k = idx_g.shape[-1]
    O = np.empty((B, Hq, d), np.float64)
    L = np.empty((B, Hq), np.float64)
    _load().dso_group_attend(_p(Q), _p(K), _p(V), _p(idx_g), B, Hq, Hkv, T, d, k, float(scale),
                             _p(O), _p(L))
    return O, L


def group_sparse_step(Q, K, V, C, k: int, scale):
    Hq, Hkv = np.asarray(Q).shape[1], np.asarray(K).shape[1]
    lab = label(K, C, Hq)
    s64 = score(Q, C, lab)
    s32 = to_f32(s64)
    sg64 = group_score(s64, Hkv)
    sg32 = group_score(s32, Hkv)
    idx = topk(sg32, k)
    O, L = group_attend(Q, K, V, idx, scale)
    return {"label": lab, "s64": s64, "sg64": sg64, "sg32": sg32, "idx": idx, "O": O, "lse": L}


# ---- block-granular selection ----------------------------------------------------

def block_score(s, bs: int):
    s = np.asarray(s)
    f32 = s.dtype == np.float32
    T = s.shape[-1]
    flat = _c(s.reshape(-1, T), np.float32 if f32 else np.float64)
    nb = -(-T // bs)
    out = np.empty((flat.shape[0], nb), flat.dtype)
    fn = _load().dso_block_score_f32 if f32 else _load().dso_block_score_f64
    fn(_p(flat), flat.shape[0], T, bs, _p(out))
    return out.reshape(*s.shape[:-1], nb)


def block_tokens(bidx, bs: int, T: int):
    b = _c(bidx, np.int32)
    out = np.empty(b.size * bs, np.int32)
    n = _load().dso_block_tokens(_p(b), b.size, bs, T, _p(out))
    return out[:n].copy()


def block_sparse_step(Q, K, V, C, bs: int, kb: int, scale):
    Q = _c(Q, np.uint16)
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    B, Hq, d = Q.shape
    _, Hkv, T, _ = K.shape
    lab = label(K, C, Hq)
    s32 = to_f32(score(Q, C, lab))
    sb = block_score(s32, bs)
    bidx = topk(sb, kb)
    O = np.empty((B, Hq, d), np.float64)
    L = np.empty((B, Hq), np.float64)
    _load().dso_block_attend(_p(Q), _p(K), _p(V), _p(bidx), B, Hq, Hkv, T, d, kb, bs,
                             float(scale), _p(O), _p(L))
    return {"s32": s32, "sb": sb, "bidx": bidx, "O": O, "lse": L}


# ---- hierarchical top-k ------------------------------------------------------------

def hier_topk(s, k: int):
    s = np.asarray(s)
    T = s.shape[-1]
    if not 1 <= k <= T:
        raise ValueError("need 1 <= k <= T")
    f32 = s.dtype == np.float32
    flat = _c(s.reshape(-1, T), np.float32 if f32 else np.float64)
    out = np.empty((flat.shape[0], k), np.int32)
    fn = _load().dso_hier_topk_f32 if f32 else _load().dso_hier_topk_f64
    fn(_p(flat), flat.shape[0], T, k, _p(out))
    return out.reshape(*s.shape[:-1], k)


def hier_topk_head(s, k: int):
    return hier_topk(np.asarray(s)[None], k)[0]


# ---- the per-head step over host threads (CPU baseline) ---------------------------

def step_heads_mt(Qs, Cs, Ls, Ks, Vs, k: int, scale, sparse: bool = True,
                  dense: bool = False, nthreads: int = 0):
    """Per head i (query Qs[i] [d], channels Cs[i] [r], label rows Ls[i] [T, r], its
    KV head's rows Ks[i], Vs[i] [T, d]): the sparse step (score, float32 rounding,
    top-k, attention) and/or dense attention, the heads spread over nthreads host
    threads (0: every core).  Returns (O, lse, Od, lsed, threads used)."""
    Qs, Ks, Vs = (_c(a, np.uint16) for a in (Qs, Ks, Vs))
    Cs = _c(Cs, np.int32)
    n, T, d = Ks.shape
    r = Cs.shape[1]
    Ls = _c(Ls, np.uint16) if sparse else np.zeros((n, 1, r), np.uint16)
    O = np.empty((n, d), np.float64)
    lse = np.empty(n, np.float64)
    Od = np.empty((n, d), np.float64)
    lsed = np.empty(n, np.float64)
    mode = (1 if sparse else 0) | (2 if dense else 0)
    used = _load().dso_step_heads_mt(_p(Qs), _p(Cs), _p(Ls), _p(Ks), _p(Vs), n, T, d, r, int(k),
                                     float(scale), mode, int(nthreads), _p(O), _p(lse), _p(Od),
                                     _p(lsed))
    return O, lse, Od, lsed, int(used)
