"""Group-shared selection (ds_group_score_topk + ds_group_sparse_decode) against
the oracle's group step.

* Group scores: bit-identical to the float32 sum, in head order, of the
  per-head scores ds_score returns (same operations); within the float32
  error bound of the oracle's float64 group score.
* Selection: exactly the oracle's top-k of the GPU's own group scores; every
  kept token's float64 group score within tolerance of the k-th largest.
* Attention: every query head over its group's set, against the oracle on
  that set (max abs error 1e-2, as the per-head path).
"""
import numpy as np
import pytest
import torch

import dsgen
import oracle
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import post_token_sparse_b200 as ds

CASES = [
    # name, B, Hq, Hkv, T, T_cap, r, k
    ("gqa-small", 2, 8, 2, 1000, 1003, 16, 37),
    ("one-head-per-group", 1, 4, 4, 500, 512, 8, 20),
    ("g8-r32", 1, 16, 2, 5000, 5000, 32, 300),
    ("g4-r128-ragged", 1, 8, 2, 777, 800, 128, 77),
    ("long-cluster", 1, 4, 1, 40000, 40000, 8, 2500),
    ("k-equals-T", 1, 4, 2, 96, 96, 16, 96),
    ("g8-r128", 1, 16, 2, 9000, 9000, 128, 500),
    ("g2-r8-T32768", 1, 4, 2, 32768, 32768, 8, 4000),
    ("g4-k1-ragged", 2, 8, 2, 4097, 4100, 16, 1),
    ("g3-kT", 1, 6, 2, 6000, 6000, 16, 6000),
]


def _run(w, inp, T, k):
    B, Hq, Hkv = w.B, w.Hq, w.Hkv
    label = torch.empty((B, Hq, w.T, inp.r), dtype=torch.bfloat16, device="cuda")
    ds.label_append(inp.dK, inp.dC, label, 0, T)
    sg = torch.empty((B * Hkv, T), dtype=torch.float32, device="cuda")
    idx = torch.full((B * Hkv, k), -1, dtype=torch.int32, device="cuda")
    ds.group_score_topk(inp.dQ, inp.dC, label, sg, idx, T)
    O = torch.empty((B, Hq, w.d), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    ds.group_sparse_decode(inp.dQ, inp.dK, inp.dV, idx, O, T, w.scale, lse=lse)
    # per-head scores for the bit-identity check
    s = torch.empty((B * Hq, T), dtype=torch.float32, device="cuda")
    ds.score(inp.dQ, inp.dC, label, s, T)
    torch.cuda.synchronize()
    return label, sg, idx, O, lse, s


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_group_step_matches_oracle(case):
    name, B, Hq, Hkv, T, T_cap, r, k = case
    w = dsgen.Workload(name, B=B, Hq=Hq, Hkv=Hkv, T=T_cap, r=r, k=k, n_out=min(16, r),
                       seed=0x6A0 + T)
    inp = gu.Inputs(w, r=r)
    label, sg, idx, O, lse, s = _run(w, inp, T, k)
    G = Hq // Hkv
    S = s.cpu().numpy().reshape(B, Hq, T)
    SG = sg.cpu().numpy().reshape(B, Hkv, T)
    # bit-identical to the float32 head-order sum of the per-head scores
    assert np.array_equal(SG, oracle.group_score(S, Hkv))
    # selection: the oracle's rule on the GPU's own group scores
    I = idx.cpu().numpy().reshape(B, Hkv, k)
    assert np.array_equal(I, oracle.topk(SG, k))
    # against the float64 group score
    lab = oracle.label(inp.K[:, :, :T], inp.C, Hq)
    s64 = oracle.score(inp.Q, inp.C, lab)
    sg64 = oracle.group_score(s64, Hkv)
    for b in range(B):
        for g in range(Hkv):
            bound = np.zeros(T)
            for h in range(g * G, g * G + G):
                qc = oracle.bf16_to_f64(inp.Q[b, h])[inp.C[h]]
                bound += gu.score_error_bound(qc, oracle.bf16_to_f64(lab[b, h])) + \
                    G * 2.0 ** -23 * np.abs(s64[b, h])
            assert np.all(np.abs(SG[b, g] - sg64[b, g]) <= bound)
            kth = np.sort(sg64[b, g])[::-1][k - 1]
            assert np.all(sg64[b, g][I[b, g]] >= kth - 2 * bound.max())
    # attention over the group's set
    ref_O, ref_L = oracle.group_attend(inp.Q, inp.K[:, :, :T], inp.V[:, :, :T], I, w.scale)
    assert np.abs(O.cpu().numpy() - ref_O).max() <= 1e-2
    L = lse.cpu().numpy()
    assert np.all(np.abs(L - ref_L) <= 1e-3 * (1 + np.abs(ref_L)))
    assert ds.device_status() == 0
    inp.free()


def test_one_head_per_group_is_the_per_head_path():
    w = dsgen.Workload("g1", B=2, Hq=4, Hkv=4, T=3000, r=16, k=100, n_out=16, seed=0x6A1)
    inp = gu.Inputs(w)
    label, sg, idx, O, lse, s = _run(w, inp, w.T, w.k)
    idx_h = torch.empty((w.B * w.Hq, w.k), dtype=torch.int32, device="cuda")
    ds.score_topk(inp.dQ, inp.dC, label, idx_h, w.T)
    O_h = torch.empty_like(O)
    ds.sparse_decode(inp.dQ, inp.dK, inp.dV, idx_h, O_h, w.T, w.scale)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx_h)
    assert torch.equal(O, O_h)  # same kernel, same rows, same order
    inp.free()


def test_group_full_workload_sampled():
    w = dsgen.workload("gqa-B16-Hq64-Hkv8-T16K")
    inp = gu.Inputs(w)
    label, sg, idx, O, lse, s = _run(w, inp, w.T, w.k)
    G = w.G
    SG = sg.cpu().numpy().reshape(w.B, w.Hkv, w.T)
    S = s.cpu().numpy().reshape(w.B, w.Hq, w.T)
    assert np.array_equal(SG, oracle.group_score(S, w.Hkv))
    I = idx.cpu().numpy().reshape(w.B, w.Hkv, w.k)
    On = O.cpu().numpy()
    rng = np.random.default_rng(5)
    for b, g in [(0, 0), (w.B - 1, w.Hkv - 1), (int(rng.integers(w.B)), int(rng.integers(w.Hkv)))]:
        assert np.array_equal(I[b, g], oracle.topk_head(SG[b, g], w.k))
        for h in (g * G, g * G + G - 1):
            o, _, _ = oracle.attend_head(inp.Q[b, h], inp.K[b, g], inp.V[b, g], I[b, g], w.scale)
            assert np.abs(On[b, h] - o).max() <= 1e-2
    inp.free()



STEP_CASES = [
    # name, B, Hq, Hkv, T, T_cap, r, k, append
    ("g4-r16", 2, 8, 2, 1000, 1003, 16, 37, True),
    ("g8-r32", 1, 16, 2, 5000, 5000, 32, 300, True),
    ("g8-r8-T1", 1, 8, 1, 1, 4, 8, 1, True),
    ("g2-r128-no-append", 1, 4, 2, 777, 800, 128, 77, False),
    ("g1-per-head", 2, 4, 4, 3000, 3000, 16, 100, True),
    ("g16-per-head-kernel", 1, 16, 1, 2000, 2000, 8, 64, True),
    ("g8-r16-T16384", 2, 16, 2, 16384, 16384, 16, 1024, True),
]


@pytest.mark.parametrize("case", STEP_CASES, ids=[c[0] for c in STEP_CASES])
def test_group_decode_step_equals_the_three_calls(case):
    """ds_group_decode_step (the group-score kernel appends token T-1's label rows)
    gives bit for bit the label cache, group scores, index set, O and lse of
    ds_label_append + ds_group_score_topk + ds_group_sparse_decode."""
    name, B, Hq, Hkv, T, T_cap, r, k, append = case
    w = dsgen.Workload(name, B=B, Hq=Hq, Hkv=Hkv, T=T_cap, r=r, k=k, n_out=min(16, r),
                       seed=0x6D5 + T)
    inp = gu.Inputs(w, r=r)
    label = torch.zeros((B, Hq, T_cap, r), dtype=torch.bfloat16, device="cuda")
    n0 = T - 1 if append else T
    if n0 > 0:
        ds.label_append(inp.dK, inp.dC, label, 0, n0)
    label_sep = label.clone()
    if append:
        ds.label_append(inp.dK, inp.dC, label_sep, T - 1, 1)
    sg_sep = torch.empty((B * Hkv, T), dtype=torch.float32, device="cuda")
    idx_sep = torch.empty((B * Hkv, k), dtype=torch.int32, device="cuda")
    ds.group_score_topk(inp.dQ, inp.dC, label_sep, sg_sep, idx_sep, T)
    O_sep = torch.empty((B, Hq, w.d), dtype=torch.float32, device="cuda")
    L_sep = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    ds.group_sparse_decode(inp.dQ, inp.dK, inp.dV, idx_sep, O_sep, T, w.scale, lse=L_sep)
    sg = torch.full_like(sg_sep, float("nan"))
    idx = torch.full_like(idx_sep, -1)
    O = torch.full_like(O_sep, float("nan"))
    L = torch.full_like(L_sep, float("nan"))
    ds.group_decode_step(inp.dQ, inp.dK, inp.dV, inp.dC, label, sg, idx, O, T, w.scale,
                         append=append, lse=L)
    torch.cuda.synchronize()
    assert torch.equal(label, label_sep)
    assert torch.equal(sg, sg_sep)
    assert torch.equal(idx, idx_sep)
    assert torch.equal(O, O_sep) and torch.equal(L, L_sep)
    got_label = gu.host_bits(label)[:, :, :T]
    assert np.array_equal(got_label, oracle.label(inp.K[:, :, :T], inp.C, Hq))
    assert ds.device_status() == 0
    inp.free()
