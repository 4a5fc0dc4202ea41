"""ds_sparse_decode_noalloc: sparse attention without a caller-supplied workspace.

Some callers of this library cannot allocate device memory on their decode
path -- a serving loop that reserved all of HBM at start-up, a latency-critical
loop that cannot afford cudaMalloc's implicit device synchronisation, or a
plug-in that only receives its input and output buffers.  This entry point
keeps its scratch (arrival counters and partials) in a fixed array inside the
library.  The tests call it through the C ABI and check it against
ds_sparse_decode and against the oracle, twice in a row (the second call finds
the first call's leftovers in the shared array), and check the bound on the
scratch it can need.  The file name sorts last so a run that stops at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import dsgen
import oracle
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

TOL = 1e-2  # the sparse-attention tolerance of the parity tests

if torch.cuda.is_available():
    import post_token_sparse_b200 as ds


def _raw_noalloc(Q, K, V, idx, O, lse, dims, T, k, scale, stream=None):
    """The entry point called directly through the C ABI (ctypes), no binding."""
    lib = ds.lib()
    st = stream if stream is not None else torch.cuda.current_stream()
    return lib.ds_sparse_decode_noalloc(
        ctypes.c_void_p(Q.data_ptr()), ctypes.c_void_p(K.data_ptr()),
        ctypes.c_void_p(V.data_ptr()), ctypes.c_void_p(idx.data_ptr()),
        ctypes.c_void_p(O.data_ptr()), ctypes.c_void_p(lse.data_ptr()), dims, T, k,
        ctypes.c_float(scale), ctypes.c_void_p(st.cuda_stream))


@pytest.mark.parametrize("B,Hq,Hkv,T,k", [
    (1, 4, 4, 50000, 20000),   # few heads, many rows: partials in the scratch array
    (1, 8, 2, 9000, 4000),     # grouped KV heads, heads shared by warps
    (8, 32, 32, 2048, 12),     # short rows: whole heads per warp, no scratch used
    (32, 32, 32, 4096, 1000),  # many heads shared by warps
])
def test_noalloc_matches_workspace_path_and_oracle_twice(B, Hq, Hkv, T, k):
    w = dsgen.Workload("noalloc", B=B, Hq=Hq, Hkv=Hkv, T=T, r=8, k=k, n_out=8, seed=900 + T)
    inp = gu.Inputs(w)
    rng = np.random.default_rng(T + k)
    dims = ds.dims_of(inp.dQ, inp.dK, w.r)
    need = ds.workspace_size(ds.OP_SPARSE_DECODE, dims, T, k)
    assert need <= ds.NOALLOC_SCRATCH_BYTES
    heads = gu.sample_heads(B, Hq, 6, seed=T)
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
        # the oracle on sampled heads, on the same index set
        On, Ln = O.cpu().numpy(), L.cpu().numpy()
        for b, h in heads:
            g = h // w.G
            o, lse, _ = oracle.attend_head(inp.Q[b, h], inp.K[b, g], inp.V[b, g],
                                           idx_np[b * Hq + h], w.scale)
            assert np.abs(On[b, h] - o).max() <= TOL, (call, b, h)
            assert abs(Ln[b, h] - lse) <= 1e-3 * (1 + abs(lse)), (call, b, h)
    inp.free()


def test_noalloc_scratch_bounds_every_request():
    """The work plan never needs more partials than the fixed array holds: a head
    is shared by several warps only when there are fewer heads than warps in
    the grid, so the slots stay below the CTA count plus that.  Sizes beyond the
    library's limits are refused before any launch."""
    for B, Hq, T, k in [(1, 1, 1 << 20, 1 << 20), (1, 2367, 4096, 4096), (1, 2368, 4096, 4096),
                        (1, 2000, 1 << 20, 1 << 20), (64, 1000, 65536, 60000),
                        (1, 65535, 100, 100), (3, 1000, 7, 5)]:
        dims = ds.Dims(B, Hq, Hq, 128, T, 8)
        assert ds.workspace_size(ds.OP_SPARSE_DECODE, dims, T, k) <= ds.NOALLOC_SCRATCH_BYTES
    dims = ds.Dims(2, 40000, 40000, 128, 100, 8)  # B * Hq beyond the grid limits
    small = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    n0 = ds.kernel_launches()
    p = ctypes.c_void_p(small.data_ptr())
    st = ds.lib().ds_sparse_decode_noalloc(p, p, p, p, p, None, dims, 100, 10,
                                           ctypes.c_float(0.1), None)
    assert st == ds.DS_ERR_UNSUPPORTED
    assert ds.kernel_launches() == n0
