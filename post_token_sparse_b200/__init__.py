"""Token-sparse (Double-Sparsity-style) decode attention on B200 (sm_100a).

Thin Python binding of ``libds.so`` (C ABI in ``include/ds.h``): argument
marshalling only.  Every step of the decode path runs in the library's CUDA
kernels; PyTorch supplies device memory and the current stream.  Importing
this package fails if the compiled library is missing -- there is no CPU or
PyTorch fallback.  Build it with ``python post_token_sparse_b200/build.py``.

Calls mirror the C ABI:

    label_append(K, C, label, t0, n)            label cache rows [t0, t0+n)
    score(Q, C, label, scores, T)               channel-sparse scores
    topk(scores, idx)                           per-row top-k, ascending
    score_topk(Q, C, label, idx, T, scores=None)  the two above in one launch
    sparse_decode(Q, K, V, idx, O, T, scale, lse=None, ws=None)
    decode(Q, K, V, O, T, scale, lse=None, ws=None)   dense reference
    decode_step(Q, K, V, C, label, idx, O, T, scale, append=True, lse=None, ws=None)
                                                the three steps above, fused

All tensors must be CUDA, contiguous, with the dtypes and shapes of
``include/ds.h``; the C library checks sizes and alignment and raises
``DsError`` with its status name on any failure.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libds.so")

DS_OK, DS_ERR_INVALID_ARG, DS_ERR_UNSUPPORTED, DS_ERR_WORKSPACE, DS_ERR_CUDA = range(5)
(OP_LABEL_APPEND, OP_SCORE, OP_TOPK, OP_SPARSE_DECODE, OP_DECODE, OP_SCORE_TOPK,
 OP_DECODE_STEP, OP_CALIBRATE, OP_GROUP_SPARSE_DECODE, OP_BLOCK_SPARSE_DECODE,
 OP_GROUP_DECODE_STEP) = range(11)
DEV_BAD_CHANNEL, DEV_BAD_INDEX, DEV_TIMEOUT = 1, 2, 4


class DsError(RuntimeError):
    def __init__(self, status: int, what: str):
        name = _lib.ds_status_string(status).decode()
        detail = ""
        if status == DS_ERR_CUDA:
            detail = ": " + _lib.ds_last_cuda_error().decode()
        super().__init__(f"{what} failed with {name}{detail}")
        self.status = status


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("d", ctypes.c_int32), ("T_cap", ctypes.c_int32), ("r", ctypes.c_int32)]

    def __repr__(self):
        return "Dims(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with "
                          "`python post_token_sparse_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, u32p = ctypes.c_void_p, ctypes.c_int32, ctypes.POINTER(ctypes.c_uint32)
    st = ctypes.c_int
    sig = {
        "ds_label_append": [vp, vp, vp, Dims, i32, i32, vp],
        "ds_score": [vp, vp, vp, vp, Dims, i32, vp],
        "ds_topk": [vp, vp, i32, i32, i32, vp, ctypes.c_size_t, vp],
        "ds_score_topk": [vp, vp, vp, vp, vp, Dims, i32, i32, vp, ctypes.c_size_t, vp],
        "ds_sparse_decode": [vp, vp, vp, vp, vp, vp, Dims, i32, i32, ctypes.c_float, vp,
                             ctypes.c_size_t, vp],
        "ds_decode": [vp, vp, vp, vp, vp, Dims, i32, ctypes.c_float, vp, ctypes.c_size_t, vp],
        "ds_device_status": [u32p, i32, vp],
        "ds_decode_step": [vp, vp, vp, vp, vp, vp, vp, vp, Dims, i32, i32, ctypes.c_float, i32,
                           vp, ctypes.c_size_t, vp],
        "ds_decode_step_kv": [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, Dims, i32, i32,
                              ctypes.c_float, vp, ctypes.c_size_t, vp],
        "ds_calibrate": [vp, i32, vp, Dims, i32, vp, vp, vp, ctypes.c_size_t, vp],
        "ds_group_score_topk": [vp, vp, vp, vp, vp, Dims, i32, i32, vp],
        "ds_group_decode_step": [vp, vp, vp, vp, vp, vp, vp, vp, vp, Dims, i32, i32,
                                 ctypes.c_float, i32, vp, ctypes.c_size_t, vp],
        "ds_block_score_topk": [vp, vp, vp, vp, vp, Dims, i32, i32, i32, vp],
        "ds_hier_score_topk": [vp, vp, vp, vp, Dims, i32, i32, vp],
        "ds_kv_append": [vp, vp, vp, vp, Dims, i32, vp],
        "ds_block_sparse_decode": [vp, vp, vp, vp, vp, vp, Dims, i32, i32, i32, ctypes.c_float,
                                   vp, ctypes.c_size_t, vp],
        "ds_group_sparse_decode": [vp, vp, vp, vp, vp, vp, Dims, i32, i32, ctypes.c_float, vp,
                                   ctypes.c_size_t, vp],
    }
    for name, args in sig.items():
        if not hasattr(lib, name):
            raise ImportError(f"{LIB_PATH} has no {name}: rebuild it with "
                              "`python post_token_sparse_b200/build.py --force`")
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = st
    lib.ds_workspace_size.argtypes = [i32, Dims, i32, i32]
    lib.ds_workspace_size.restype = ctypes.c_size_t
    lib.ds_status_string.argtypes = [st]
    lib.ds_status_string.restype = ctypes.c_char_p
    lib.ds_last_cuda_error.argtypes = []
    lib.ds_last_cuda_error.restype = ctypes.c_char_p
    lib.ds_kernel_launches.argtypes = []
    lib.ds_kernel_launches.restype = ctypes.c_uint64
    return lib


_lib = _load()


def lib():
    """The loaded ctypes library (for callers that want the raw C ABI)."""
    return _lib


# ---------------------------------------------------------------------------
# marshalling helpers

def _ptr(t: torch.Tensor | None, dtype=None, name="tensor", host_ok=False):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    # K and V (and a decode step's Q, O, lse) may also be pinned host tensors
    # (see include/ds.h); whether a host tensor is pinned and mapped is checked by
    # the library (DS_ERR_INVALID_ARG otherwise), once, on the decode path
    host_ok = host_ok or name in ("K", "V")
    if not t.is_cuda and not host_ok:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise TypeError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(device=None):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(status: int, what: str):
    if status != DS_OK:
        raise DsError(status, what)


def dims_of(Q: torch.Tensor, K: torch.Tensor, r: int) -> Dims:
    """Dims from Q [B,Hq,d] and K [B,Hkv,T_cap,d]."""
    B, Hq, d = Q.shape
    _, Hkv, T_cap, _ = K.shape
    return Dims(B, Hq, Hkv, d, T_cap, r)


def workspace_size(op: int, dims: Dims, T: int, k: int) -> int:
    return int(_lib.ds_workspace_size(op, dims, T, k))


def workspace(op: int, dims: Dims, T: int, k: int, device) -> torch.Tensor | None:
    """A zero-filled device buffer of the size ``op`` needs (None when it needs none).

    Calls leave the workspace zero-filled again, so one buffer serves any number
    of calls that do not overlap on the GPU."""
    n = workspace_size(op, dims, T, k)
    return torch.zeros(n, dtype=torch.uint8, device=device) if n else None


# ---------------------------------------------------------------------------
# the calls

def kv_append(K_new, V_new, K, V, t: int, stream_device=None):
    """K[:, :, t] = K_new and V[:, :, t] = V_new (K_new/V_new [B,Hkv,d] may be pinned host)."""
    B, Hkv, T_cap, d = K.shape
    dims = Dims(B, Hkv, Hkv, d, T_cap, 1)
    dev = stream_device if stream_device is not None else (
        K.device if K.is_cuda else torch.device("cuda", torch.cuda.current_device()))
    _check(_lib.ds_kv_append(_ptr(K_new, torch.bfloat16, "K"), _ptr(V_new, torch.bfloat16, "V"),
                             _ptr(K, torch.bfloat16, "K"), _ptr(V, torch.bfloat16, "V"), dims, t,
                             _stream(dev)), "ds_kv_append")


def label_append(K, C, label, t0: int, n: int):
    B, Hkv, T_cap, d = K.shape
    Hq, r = C.shape
    dims = Dims(B, Hq, Hkv, d, T_cap, r)
    _check(_lib.ds_label_append(_ptr(K, torch.bfloat16, "K"), _ptr(C, torch.int32, "C"),
                                _ptr(label, torch.bfloat16, "label"), dims, t0, n,
                                _stream(label.device)), "ds_label_append")


def score(Q, C, label, scores, T: int):
    B, Hq, d = Q.shape
    _, _, T_cap, r = label.shape
    dims = Dims(B, Hq, Hq, d, T_cap, r)  # the score step does not read K
    _check(_lib.ds_score(_ptr(Q, torch.bfloat16, "Q"), _ptr(C, torch.int32, "C"),
                         _ptr(label, torch.bfloat16, "label"), _ptr(scores, torch.float32,
                                                                     "scores"),
                         dims, T, _stream(Q.device)), "ds_score")


def topk(scores, idx, ws=None):
    """Top-k of each row of scores [BH, T] into idx [BH, k]; ws: the workspace of
    OP_TOPK (made here when not given)."""
    BH, T = scores.shape
    k = idx.shape[-1]
    if idx.numel() != BH * k:
        raise TypeError("idx must have BH*k elements")
    if ws is None:
        ws = workspace(OP_TOPK, Dims(1, BH, 1, 128, T, 1), T, k, scores.device)
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(_lib.ds_topk(_ptr(scores, torch.float32, "scores"), _ptr(idx, torch.int32, "idx"),
                        BH, T, k, _ptr(ws, None, "ws"), nbytes, _stream(scores.device)),
           "ds_topk")


def score_topk(Q, C, label, idx, T: int, scores=None, ws=None):
    """Top-k of the channel-sparse scores; ws: the workspace of OP_SCORE_TOPK (made
    here when None and the sizes use one)."""
    B, Hq, d = Q.shape
    _, _, T_cap, r = label.shape
    dims = Dims(B, Hq, Hq, d, T_cap, r)
    k = idx.shape[-1]
    if ws is None:
        ws = workspace(OP_SCORE_TOPK, dims, T, k, Q.device)
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(_lib.ds_score_topk(_ptr(Q, torch.bfloat16, "Q"), _ptr(C, torch.int32, "C"),
                              _ptr(label, torch.bfloat16, "label"),
                              _ptr(scores, torch.float32, "scores"),
                              _ptr(idx, torch.int32, "idx"), dims, T, k,
                              _ptr(ws, None, "ws"), nbytes, _stream(Q.device)),
           "ds_score_topk")


def sparse_decode(Q, K, V, idx, O, T: int, scale: float, lse=None, ws=None):
    dims = dims_of(Q, K, 1)
    k = idx.shape[-1]
    if ws is None:
        ws = workspace(OP_SPARSE_DECODE, dims, T, k, Q.device)
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(_lib.ds_sparse_decode(_ptr(Q, torch.bfloat16, "Q"), _ptr(K, torch.bfloat16, "K"),
                                 _ptr(V, torch.bfloat16, "V"), _ptr(idx, torch.int32, "idx"),
                                 _ptr(O, torch.float32, "O"), _ptr(lse, torch.float32, "lse"),
                                 dims, T, k, scale, _ptr(ws, None, "ws"), nbytes,
                                 _stream(Q.device)), "ds_sparse_decode")


def decode_step(Q, K, V, C, label, idx, O, T: int, scale: float, append: bool = True,
                lse=None, ws=None):
    """One decode step: label row of token T-1 (if append), top-k into idx, attention into O."""
    dims = dims_of(Q, K, C.shape[1])
    k = idx.shape[-1]
    if ws is None:
        ws = workspace(OP_DECODE_STEP, dims, T, k, label.device)
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(_lib.ds_decode_step(_ptr(Q, torch.bfloat16, "Q", True), _ptr(K, torch.bfloat16, "K"),
                               _ptr(V, torch.bfloat16, "V"), _ptr(C, torch.int32, "C"),
                               _ptr(label, torch.bfloat16, "label"),
                               _ptr(idx, torch.int32, "idx"), _ptr(O, torch.float32, "O", True),
                               _ptr(lse, torch.float32, "lse", True), dims, T, k, scale,
                               int(bool(append)), _ptr(ws, None, "ws"), nbytes,
                               _stream(label.device)), "ds_decode_step")


def decode_step_kv(Q, K_new, V_new, K, V, C, label, idx, O, T: int, scale: float, lse=None,
                   ws=None):
    """decode_step with the newest token's K/V rows handed over: K[:, :, T-1] = K_new,
    V[:, :, T-1] = V_new, then the step with append (K_new/V_new [B,Hkv,d] may be pinned host)."""
    dims = dims_of(Q, K, C.shape[1])
    k = idx.shape[-1]
    if ws is None:
        ws = workspace(OP_DECODE_STEP, dims, T, k, label.device)
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(_lib.ds_decode_step_kv(_ptr(Q, torch.bfloat16, "Q", True),
                                  _ptr(K_new, torch.bfloat16, "K_new", True),
                                  _ptr(V_new, torch.bfloat16, "V_new", True),
                                  _ptr(K, torch.bfloat16, "K"), _ptr(V, torch.bfloat16, "V"),
                                  _ptr(C, torch.int32, "C"), _ptr(label, torch.bfloat16, "label"),
                                  _ptr(idx, torch.int32, "idx"),
                                  _ptr(O, torch.float32, "O", True),
                                  _ptr(lse, torch.float32, "lse", True), dims, T, k, scale,
                                  _ptr(ws, None, "ws"), nbytes, _stream(label.device)),
           "ds_decode_step_kv")


def decode(Q, K, V, O, T: int, scale: float, lse=None, ws=None):
    dims = dims_of(Q, K, 1)
    if ws is None:
        ws = workspace(OP_DECODE, dims, T, T, Q.device)
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(_lib.ds_decode(_ptr(Q, torch.bfloat16, "Q"), _ptr(K, torch.bfloat16, "K"),
                          _ptr(V, torch.bfloat16, "V"), _ptr(O, torch.float32, "O"),
                          _ptr(lse, torch.float32, "lse"), dims, T, scale,
                          _ptr(ws, None, "ws"), nbytes, _stream(Q.device)), "ds_decode")


def group_score_topk(Q, C, label, group_scores, idx, T: int):
    """One selection per KV group: group_scores [B*Hkv, T] fp32, idx [B*Hkv, k]."""
    B, Hq, T_cap, r = label.shape
    Hkv = group_scores.shape[0] // B
    dims = Dims(B, Hq, Hkv, Q.shape[-1], T_cap, r)
    _check(_lib.ds_group_score_topk(_ptr(Q, torch.bfloat16, "Q"), _ptr(C, torch.int32, "C"),
                                    _ptr(label, torch.bfloat16, "label"),
                                    _ptr(group_scores, torch.float32, "group_scores"),
                                    _ptr(idx, torch.int32, "idx"), dims, T, idx.shape[-1],
                                    _stream(Q.device)), "ds_group_score_topk")


def group_decode_step(Q, K, V, C, label, group_scores, idx, O, T: int, scale: float,
                      append: bool = True, lse=None, ws=None):
    """Label row of token T-1 (if append), group-shared selection and attention, three
    launches: group_scores [B*Hkv, T], idx [B*Hkv, k], O [B, Hq, d]."""
    B, Hq, T_cap, r = label.shape
    Hkv = K.shape[1]
    dims = Dims(B, Hq, Hkv, Q.shape[-1], T_cap, r)
    k = idx.shape[-1]
    if ws is None:
        ws = workspace(OP_GROUP_DECODE_STEP, dims, T, k, Q.device)
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(_lib.ds_group_decode_step(
        _ptr(Q, torch.bfloat16, "Q"), _ptr(K, torch.bfloat16, "K"), _ptr(V, torch.bfloat16, "V"),
        _ptr(C, torch.int32, "C"), _ptr(label, torch.bfloat16, "label"),
        _ptr(group_scores, torch.float32, "group_scores"), _ptr(idx, torch.int32, "idx"),
        _ptr(O, torch.float32, "O"), _ptr(lse, torch.float32, "lse"), dims, T, k, scale,
        int(bool(append)), _ptr(ws, None, "ws"), nbytes, _stream(Q.device)),
        "ds_group_decode_step")


def group_sparse_decode(Q, K, V, idx, O, T: int, scale: float, lse=None, ws=None):
    """Attention of every query head over its KV group's kept tokens (idx [B*Hkv, k])."""
    dims = dims_of(Q, K, 1)
    k = idx.shape[-1]
    if ws is None:
        ws = workspace(OP_GROUP_SPARSE_DECODE, dims, T, k, Q.device)
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(_lib.ds_group_sparse_decode(_ptr(Q, torch.bfloat16, "Q"), _ptr(K, torch.bfloat16, "K"),
                                       _ptr(V, torch.bfloat16, "V"), _ptr(idx, torch.int32, "idx"),
                                       _ptr(O, torch.float32, "O"), _ptr(lse, torch.float32, "lse"),
                                       dims, T, k, scale, _ptr(ws, None, "ws"), nbytes,
                                       _stream(Q.device)), "ds_group_sparse_decode")


def block_score_topk(Q, C, label, block_scores, bidx, T: int, bs: int):
    """Block-granular selection: block_scores [B*Hq, ceil(T/bs)] fp32, bidx [B*Hq, kb]."""
    B, Hq, T_cap, r = label.shape
    dims = Dims(B, Hq, Hq, Q.shape[-1], T_cap, r)
    _check(_lib.ds_block_score_topk(_ptr(Q, torch.bfloat16, "Q"), _ptr(C, torch.int32, "C"),
                                    _ptr(label, torch.bfloat16, "label"),
                                    _ptr(block_scores, torch.float32, "block_scores"),
                                    _ptr(bidx, torch.int32, "bidx"), dims, T, bs, bidx.shape[-1],
                                    _stream(Q.device)), "ds_block_score_topk")


def block_sparse_decode(Q, K, V, bidx, O, T: int, bs: int, scale: float, lse=None, ws=None):
    """Attention of every query head over the tokens of its kept blocks."""
    dims = dims_of(Q, K, 1)
    kb = bidx.shape[-1]
    if ws is None:
        ws = workspace(OP_BLOCK_SPARSE_DECODE, dims, T, kb * bs, Q.device)
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(_lib.ds_block_sparse_decode(_ptr(Q, torch.bfloat16, "Q"), _ptr(K, torch.bfloat16, "K"),
                                       _ptr(V, torch.bfloat16, "V"), _ptr(bidx, torch.int32, "bidx"),
                                       _ptr(O, torch.float32, "O"), _ptr(lse, torch.float32, "lse"),
                                       dims, T, bs, kb, scale, _ptr(ws, None, "ws"), nbytes,
                                       _stream(Q.device)), "ds_block_sparse_decode")


def hier_score_topk(Q, C, label, idx, T: int):
    """Hierarchical (top-down) selection of k = idx.shape[-1] tokens per head."""
    B, Hq, T_cap, r = label.shape
    dims = Dims(B, Hq, Hq, Q.shape[-1], T_cap, r)
    _check(_lib.ds_hier_score_topk(_ptr(Q, torch.bfloat16, "Q"), _ptr(C, torch.int32, "C"),
                                   _ptr(label, torch.bfloat16, "label"),
                                   _ptr(idx, torch.int32, "idx"), dims, T, idx.shape[-1],
                                   _stream(Q.device)), "ds_hier_score_topk")


def calibrate(Qc, K, C, T: int, importance=None, ws=None):
    """Offline channel calibration: C [Hq, r] from calibration queries Qc
    [B,Hq,Nq,d] and keys K [B,Hkv,T_cap,d] (tokens < T); importance [Hq, d]
    fp32 optionally."""
    B, Hq, Nq, d = Qc.shape
    _, Hkv, T_cap, _ = K.shape
    dims = Dims(B, Hq, Hkv, d, T_cap, C.shape[1])
    if ws is None:
        ws = workspace(OP_CALIBRATE, dims, T, Nq, Qc.device)
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(_lib.ds_calibrate(_ptr(Qc, torch.bfloat16, "Qc"), Nq, _ptr(K, torch.bfloat16, "K"),
                             dims, T, _ptr(C, torch.int32, "C"),
                             _ptr(importance, torch.float32, "importance"),
                             _ptr(ws, None, "ws"), nbytes, _stream(Qc.device)), "ds_calibrate")


def device_status(clear: bool = True, device=None) -> int:
    """Status bits kernels set on the current device (DEV_BAD_CHANNEL, DEV_BAD_INDEX,
    DEV_TIMEOUT)."""
    bits = ctypes.c_uint32(0)
    _check(_lib.ds_device_status(ctypes.byref(bits), int(clear), _stream(device)),
           "ds_device_status")
    return int(bits.value)


def kernel_launches() -> int:
    """Kernels launched by libds.so in this process so far."""
    return int(_lib.ds_kernel_launches())


# ---------------------------------------------------------------------------
# sparse decode for callers that cannot allocate device memory

_lib.ds_sparse_decode_noalloc.argtypes = [ctypes.c_void_p] * 6 + [
    Dims, ctypes.c_int32, ctypes.c_int32, ctypes.c_float, ctypes.c_void_p]
_lib.ds_sparse_decode_noalloc.restype = ctypes.c_int
NOALLOC_SCRATCH_BYTES = 4 << 20


def sparse_decode_noalloc(Q, K, V, idx, O, T: int, scale: float, lse=None):
    """sparse_decode without a workspace: the split partials use a fixed array
    inside the library (NOALLOC_SCRATCH_BYTES per GPU).  For callers that must not
    allocate device memory on their decode path; see ds_sparse_decode_noalloc in
    include/ds.h for the sharing rule (calls that overlap on the GPU race)."""
    dims = dims_of(Q, K, 1)
    k = idx.shape[-1]
    _check(_lib.ds_sparse_decode_noalloc(
        _ptr(Q, torch.bfloat16, "Q"), _ptr(K, torch.bfloat16, "K"), _ptr(V, torch.bfloat16, "V"),
        _ptr(idx, torch.int32, "idx"), _ptr(O, torch.float32, "O"),
        _ptr(lse, torch.float32, "lse"), dims, T, k, scale, _stream(Q.device)),
        "ds_sparse_decode_noalloc")
