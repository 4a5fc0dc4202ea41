"""Hierarchical top-k (ds_hier_score_topk) against the oracle's search.

The search's decisions are taken on the fp32 scores, so the oracle runs on the
scores ds_score gives (same operations as the kernel): the kept set must be
bit-identical.  With k = T it is every token.  Attention over the kept set is
then checked like the per-head path.
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
    ("T1000-k37", 2, 4, 2, 1000, 1003, 16, 37),
    ("T4096-k256-r8", 1, 4, 4, 4096, 4096, 8, 256),
    ("T777-k100-r128", 1, 2, 2, 777, 800, 128, 100),
    ("T20000-k2048-r32", 1, 2, 2, 20000, 20000, 32, 2048),
    ("k-equals-T", 1, 2, 2, 300, 300, 16, 300),
    ("k1", 1, 2, 2, 513, 513, 64, 1),
    ("T2-k1", 1, 2, 2, 2, 2, 8, 1),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_hier_matches_oracle(case):
    name, B, Hq, Hkv, T, T_cap, r, k = case
    w = dsgen.Workload(name, B=B, Hq=Hq, Hkv=Hkv, T=T_cap, r=r, k=k, n_out=min(16, r),
                       seed=0x41E + T)
    inp = gu.Inputs(w, r=r)
    label = torch.empty((B, Hq, T_cap, r), dtype=torch.bfloat16, device="cuda")
    ds.label_append(inp.dK, inp.dC, label, 0, T)
    BH = B * Hq
    idx = torch.full((BH, k), -1, dtype=torch.int32, device="cuda")
    ds.hier_score_topk(inp.dQ, inp.dC, label, idx, T)
    s = torch.empty((BH, T), dtype=torch.float32, device="cuda")
    ds.score(inp.dQ, inp.dC, label, s, T)
    O = torch.empty((B, Hq, w.d), dtype=torch.float32, device="cuda")
    ds.sparse_decode(inp.dQ, inp.dK, inp.dV, idx, O, T, w.scale)
    torch.cuda.synchronize()
    I = idx.cpu().numpy()
    assert np.array_equal(I, oracle.hier_topk(s.cpu().numpy(), k))
    if k == T:
        assert np.array_equal(I, np.tile(np.arange(T, dtype=np.int32), (BH, 1)))
    ref_O, _ = oracle.attend(inp.Q, inp.K[:, :, :T], inp.V[:, :, :T], I.reshape(B, Hq, k),
                             w.scale)
    assert np.abs(O.cpu().numpy() - ref_O).max() <= 1e-2
    assert ds.device_status() == 0
    inp.free()


def test_hier_full_workload_sampled():
    w = dsgen.workload("llama2-7b-B8-H32-T4K")
    inp = gu.Inputs(w)
    label = torch.empty((w.B, w.Hq, w.T, w.r), dtype=torch.bfloat16, device="cuda")
    ds.label_append(inp.dK, inp.dC, label, 0, w.T)
    BH = w.B * w.Hq
    idx = torch.empty((BH, w.k), dtype=torch.int32, device="cuda")
    ds.hier_score_topk(inp.dQ, inp.dC, label, idx, w.T)
    s = torch.empty((BH, w.T), dtype=torch.float32, device="cuda")
    ds.score(inp.dQ, inp.dC, label, s, w.T)
    torch.cuda.synchronize()
    I, S = idx.cpu().numpy(), s.cpu().numpy()
    for row in gu.sample_heads(w.B, w.Hq, 12, seed=9):
        r_ = row[0] * w.Hq + row[1]
        assert np.array_equal(I[r_], oracle.hier_topk_head(S[r_], w.k))
    inp.free()
