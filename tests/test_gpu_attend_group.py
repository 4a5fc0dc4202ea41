"""Group-by-group attention (k_attend_group): dense decode and group-shared sparse
decode when each KV head serves 2..8 query heads.

Every K/V row is read once per group and applied to all G heads on the tensor
cores, with the softmax weights split into a bf16 high part and a remainder.
The results are checked against the oracle (float64) at the dense and sparse
tolerances of the other parity tests, over edge cases of the work plan: a
single row, fewer rows than a 16-row step, ragged last steps, whole groups per
warp, groups split across the warps of one CTA and across many CTAs (the
two-level merge), G = 2..8 including odd G, G > 8 (the per-head kernel), and
repeated calls (bit-identical: the merge order does not depend on timing).
"""
import numpy as np
import pytest
import torch

import dsgen
import oracle
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

DENSE_TOL = 5e-3
SPARSE_TOL = 1e-2

if torch.cuda.is_available():
    import post_token_sparse_b200 as ds


def _lse_ok(got, ref):
    return np.all(np.abs(got - ref) <= 1e-3 * (1 + np.abs(ref)))


DENSE = [
    # name, B, Hq, Hkv, T, T_cap
    ("g2-T1", 1, 2, 1, 1, 1),
    ("g3-T15", 2, 6, 2, 15, 20),
    ("g8-T16", 1, 8, 1, 16, 16),
    ("g4-T17", 3, 12, 3, 17, 40),
    ("g5-T333-whole-groups", 1, 40, 8, 333, 400),
    ("g8-T5000-split", 2, 64, 8, 5000, 5003),
    ("g7-T2049", 1, 28, 4, 2049, 2100),
    ("g2-T70000-many-ctas", 1, 4, 2, 70000, 70000),
    ("g8-B1-Hkv1-T200000", 1, 8, 1, 200000, 200000),
    ("g16-per-head-kernel", 1, 16, 1, 3000, 3000),
]


@pytest.mark.parametrize("case", DENSE, ids=[c[0] for c in DENSE])
def test_group_dense_decode_matches_oracle(case):
    name, B, Hq, Hkv, T, T_cap = case
    w = dsgen.Workload(name, B=B, Hq=Hq, Hkv=Hkv, T=T_cap, r=8, k=1, n_out=8, seed=0x6D0 + T)
    inp = gu.Inputs(w)
    O = torch.full((B, Hq, w.d), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device="cuda")
    ds.decode(inp.dQ, inp.dK, inp.dV, O, T, w.scale, lse=lse)
    On, Ln = O.cpu().numpy(), lse.cpu().numpy()
    assert np.isfinite(On).all() and np.isfinite(Ln).all()
    if B * Hq * T <= 2_000_000:
        ref_O, ref_L = oracle.dense(inp.Q, inp.K[:, :, :T], inp.V[:, :, :T], w.scale)
        assert np.abs(On - ref_O).max() <= DENSE_TOL
        assert _lse_ok(Ln, ref_L)
    else:
        ids = np.arange(T, dtype=np.int32)
        for b, h in gu.sample_heads(B, Hq, 4, seed=T):
            g = h // w.G
            o, l, _ = oracle.attend_head(inp.Q[b, h], inp.K[b, g], inp.V[b, g], ids, w.scale)
            assert np.abs(On[b, h] - o).max() <= DENSE_TOL, (b, h)
            assert abs(Ln[b, h] - l) <= 1e-3 * (1 + abs(l)), (b, h)
    # a second call gives the same bits
    O2 = torch.empty_like(O)
    lse2 = torch.empty_like(lse)
    ds.decode(inp.dQ, inp.dK, inp.dV, O2, T, w.scale, lse=lse2)
    assert torch.equal(O, O2) and torch.equal(lse, lse2)
    assert ds.device_status() == 0
    inp.free()


SPARSE = [
    # name, B, Hq, Hkv, T, k
    ("g2-k1", 2, 4, 2, 100, 1),
    ("g4-k7", 1, 8, 2, 300, 7),
    ("g8-k16", 2, 16, 2, 1000, 16),
    ("g8-k33", 1, 8, 1, 5000, 33),
    ("g3-k1000", 2, 12, 4, 9000, 1000),
    ("g8-k4096-split", 1, 32, 4, 60000, 4096),
    ("g6-kT", 1, 12, 2, 3000, 3000),
]


@pytest.mark.parametrize("case", SPARSE, ids=[c[0] for c in SPARSE])
def test_group_sparse_decode_matches_oracle(case):
    name, B, Hq, Hkv, T, k = case
    w = dsgen.Workload(name, B=B, Hq=Hq, Hkv=Hkv, T=T, r=8, k=k, n_out=8, seed=0x65D + k)
    inp = gu.Inputs(w)
    rng = np.random.default_rng(T + k)
    I = np.sort(np.stack([rng.choice(T, k, replace=False) for _ in range(B * Hkv)]),
                axis=1).astype(np.int32)
    idx = gu.dev_i32(I)
    O = torch.full((B, Hq, w.d), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device="cuda")
    ds.group_sparse_decode(inp.dQ, inp.dK, inp.dV, idx, O, T, w.scale, lse=lse)
    ref_O, ref_L = oracle.group_attend(inp.Q, inp.K, inp.V, I.reshape(B, Hkv, k), w.scale)
    assert np.abs(O.cpu().numpy() - ref_O).max() <= SPARSE_TOL
    assert _lse_ok(lse.cpu().numpy(), ref_L)
    O2 = torch.empty_like(O)
    ds.group_sparse_decode(inp.dQ, inp.dK, inp.dV, idx, O2, T, w.scale)
    assert torch.equal(O, O2)
    assert ds.device_status() == 0
    inp.free()


def test_group_sparse_equals_dense_on_all_tokens():
    """k = T with ids 0..T-1: the sparse kernel reads the same rows in the same
    order as the dense one, so the results are bit-identical."""
    B, Hq, Hkv, T = 2, 16, 2, 20000
    w = dsgen.Workload("g-kT", B=B, Hq=Hq, Hkv=Hkv, T=T, r=8, k=T, n_out=8, seed=0x6E)
    inp = gu.Inputs(w)
    idx = gu.dev_i32(np.tile(np.arange(T, dtype=np.int32), (B * Hkv, 1)))
    O_s = torch.empty((B, Hq, w.d), dtype=torch.float32, device="cuda")
    O_d = torch.empty_like(O_s)
    L_s = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    L_d = torch.empty_like(L_s)
    ds.group_sparse_decode(inp.dQ, inp.dK, inp.dV, idx, O_s, T, w.scale, lse=L_s)
    ds.decode(inp.dQ, inp.dK, inp.dV, O_d, T, w.scale, lse=L_d)
    assert torch.equal(O_s, O_d) and torch.equal(L_s, L_d)
    inp.free()


def test_group_ids_out_of_range_are_flagged_not_read():
    """Token ids outside [0, T) set the status bit and are clamped (no fault)."""
    B, Hq, Hkv, T, k = 1, 8, 1, 500, 20
    w = dsgen.Workload("g-bad", B=B, Hq=Hq, Hkv=Hkv, T=T, r=8, k=k, n_out=8, seed=3)
    inp = gu.Inputs(w)
    I = np.arange(k, dtype=np.int32)[None].copy()
    I[0, 5] = T + 7
    I[0, 9] = -3
    ds.device_status(clear=True)
    O = torch.empty((B, Hq, w.d), dtype=torch.float32, device="cuda")
    ds.group_sparse_decode(inp.dQ, inp.dK, inp.dV, gu.dev_i32(I), O, T, w.scale)
    torch.cuda.synchronize()
    assert ds.device_status(clear=True) & 2
    assert torch.isfinite(O).all()
    inp.free()


def test_group_full_gqa_workload_dense_sampled():
    """The full grouped workload (B 16, 64 query heads on 8 KV heads, T 16384),
    dense, on sampled heads."""
    w = dsgen.workload("gqa-B16-Hq64-Hkv8-T16K")
    inp = gu.Inputs(w)
    O = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    ds.decode(inp.dQ, inp.dK, inp.dV, O, w.T, w.scale, lse=lse)
    On, Ln = O.cpu().numpy(), lse.cpu().numpy()
    ids = np.arange(w.T, dtype=np.int32)
    for b, h in gu.sample_heads(w.B, w.Hq, 6, seed=11):
        g = h // w.G
        o, l, _ = oracle.attend_head(inp.Q[b, h], inp.K[b, g], inp.V[b, g], ids, w.scale)
        assert np.abs(On[b, h] - o).max() <= DENSE_TOL, (b, h)
        assert abs(Ln[b, h] - l) <= 1e-3 * (1 + abs(l)), (b, h)
    inp.free()
