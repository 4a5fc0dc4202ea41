"""ds_sparse_decode_noalloc: sparse attention without a caller-supplied workspace.

Some callers of this library cannot allocate device memory on their decode
path -- a serving loop that reserved all of HBM at start-up, a latency-critical
loop that cannot afford cudaMalloc's implicit device synchronisation, or a
plug-in that only receives its input and output buffers.  This entry point
keeps its scratch (the split partials) in a fixed array inside the library.
The test calls it through the C ABI and checks it against ds_sparse_decode,
twice in a row (the second call finds the first call's leftovers in the shared
array), and checks that an oversized request is refused.  The file name sorts
last so a run that stops at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import dsgen
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

TOL = 1e-2  # the sparse-attention tolerance of the parity tests

if torch.cuda.is_available():
    import post_token_sparse_b200 as ds


def _raw_noalloc(Q, K, V, idx, O, lse, dims, T, k, scale):
    """The entry point called directly through the C ABI (ctypes), no binding."""
    lib = ds.lib()
    return lib.ds_sparse_decode_noalloc(
        ctypes.c_void_p(Q.data_ptr()), ctypes.c_void_p(K.data_ptr()),
        ctypes.c_void_p(V.data_ptr()), ctypes.c_void_p(idx.data_ptr()),
        ctypes.c_void_p(O.data_ptr()), ctypes.c_void_p(lse.data_ptr()), dims, T, k,
        ctypes.c_float(scale), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("B,Hq,Hkv,T,k", [
    (1, 4, 4, 50000, 20000),   # few heads, many rows: split partials in the scratch array
    (1, 8, 2, 9000, 4000),     # grouped KV heads, split
    (8, 32, 32, 2048, 100),    # short rows: no split, no scratch used
])
def test_noalloc_matches_workspace_path_twice(B, Hq, Hkv, T, k):
    w = dsgen.Workload("noalloc", B=B, Hq=Hq, Hkv=Hkv, T=T, r=8, k=k, n_out=8, seed=900 + T)
    inp = gu.Inputs(w)
    rng = np.random.default_rng(T + k)
    dims = ds.dims_of(inp.dQ, inp.dK, w.r)
    need = ds.workspace_size(ds.OP_SPARSE_DECODE, dims, T, k)
    assert need <= ds.NOALLOC_SCRATCH_BYTES
    assert (need == 0) == (k < 128)
    for call in range(2):
        idx_np = np.sort(np.stack([rng.choice(T, k, replace=False) for _ in range(B * Hq)]),
                         axis=1).astype(np.int32)
        idx = gu.dev_i32(idx_np)
        O_ref = torch.empty((B, Hq, w.d), dtype=torch.float32, device="cuda")
        L_ref = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
        ds.sparse_decode(inp.dQ, inp.dK, inp.dV, idx, O_ref, T, w.scale, lse=L_ref)
        O = torch.full((B, Hq, w.d), float("nan"), dtype=torch.float32, device="cuda")
        L = torch.full((B, Hq), float("nan"), dtype=torch.float32, device="cuda")
        st = _raw_noalloc(inp.dQ, inp.dK, inp.dV, idx, O, L, dims, T, k, w.scale)
        assert st == ds.DS_OK, ds.lib().ds_status_string(st)
        torch.cuda.synchronize()
        assert torch.isfinite(O).all() and torch.isfinite(L).all()
        assert (O - O_ref).abs().max().item() <= TOL, call
        assert ((L - L_ref).abs() <= 1e-3 * (1 + L_ref.abs())).all(), call
    inp.free()


def test_noalloc_refuses_requests_beyond_its_scratch():
    """One long head split many ways needs more partials than the fixed array holds."""
    B, Hq, T, k = 1, 4000, 4096, 4096
    dims = ds.Dims(B, Hq, Hq, 128, T, 8)
    need = ds.workspace_size(ds.OP_SPARSE_DECODE, dims, T, k)
    assert need > ds.NOALLOC_SCRATCH_BYTES
    small = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    n0 = ds.kernel_launches()
    lib = ds.lib()
    p = ctypes.c_void_p(small.data_ptr())
    st = lib.ds_sparse_decode_noalloc(p, p, p, p, p, None, dims, T, k, ctypes.c_float(0.1),
                                      None)
    assert st == ds.DS_ERR_WORKSPACE
    assert ds.kernel_launches() == n0
