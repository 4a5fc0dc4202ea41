"""Block-granular selection (ds_block_score_topk + ds_block_sparse_decode)
against the oracle's block step.

* Block scores: bit-identical to the oracle's block maxima of the positive
  parts of the GPU's own per-token scores (ds_score; a max does not round).
* Selection: exactly the oracle's top-kb of the GPU's block scores; every kept
  block's float64 block score within tolerance of the kb-th largest.
* Attention: every head over its blocks' tokens (clipped to T), against the
  oracle on those tokens (max abs error 1e-2).
* bs = 1 keeps the top-k of the positive-clamped scores.
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
    # name, B, Hq, Hkv, T, T_cap, r, bs, kb
    ("bs64", 2, 4, 4, 4096, 4096, 16, 64, 4),
    ("bs64-short-last-block", 1, 4, 2, 1000, 1003, 8, 64, 16),   # 16 = every block
    ("bs16-r32", 1, 4, 4, 3000, 3072, 32, 16, 20),
    ("bs8-r128", 1, 2, 2, 777, 800, 128, 8, 13),
    ("bs32-r64-gqa", 2, 8, 2, 2500, 2500, 64, 32, 9),
    ("bs2-r8", 1, 2, 2, 129, 129, 8, 2, 65),
    ("long", 1, 4, 4, 40000, 40000, 8, 64, 40),
]


def _run(w, inp, T, bs, kb):
    BH = w.B * w.Hq
    label = torch.empty((w.B, w.Hq, w.T, inp.r), dtype=torch.bfloat16, device="cuda")
    ds.label_append(inp.dK, inp.dC, label, 0, T)
    nblk = -(-T // bs)
    sb = torch.empty((BH, nblk), dtype=torch.float32, device="cuda")
    bidx = torch.full((BH, kb), -1, dtype=torch.int32, device="cuda")
    ds.block_score_topk(inp.dQ, inp.dC, label, sb, bidx, T, bs)
    O = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    ds.block_sparse_decode(inp.dQ, inp.dK, inp.dV, bidx, O, T, bs, w.scale, lse=lse)
    s = torch.empty((BH, T), dtype=torch.float32, device="cuda")
    ds.score(inp.dQ, inp.dC, label, s, T)
    torch.cuda.synchronize()
    return sb, bidx, O, lse, s


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_block_step_matches_oracle(case):
    name, B, Hq, Hkv, T, T_cap, r, bs, kb = case
    w = dsgen.Workload(name, B=B, Hq=Hq, Hkv=Hkv, T=T_cap, r=r, k=1, n_out=min(16, r),
                       seed=0xB10 + T)
    inp = gu.Inputs(w, r=r)
    sb, bidx, O, lse, s = _run(w, inp, T, bs, kb)
    S = s.cpu().numpy().reshape(B, Hq, T)
    SB = sb.cpu().numpy().reshape(B, Hq, -1)
    assert np.array_equal(SB, oracle.block_score(S, bs))
    I = bidx.cpu().numpy().reshape(B, Hq, kb)
    assert np.array_equal(I, oracle.topk(SB, kb))
    lab = oracle.label(inp.K[:, :, :T], inp.C, Hq)
    s64 = oracle.score(inp.Q, inp.C, lab)
    sb64 = oracle.block_score(s64, bs)
    On, L = O.cpu().numpy(), lse.cpu().numpy()
    for b in range(B):
        for h in range(Hq):
            kth = np.sort(sb64[b, h])[::-1][kb - 1]
            assert np.all(sb64[b, h][I[b, h]] >= kth - 1e-3 * (abs(kth) + 1))
            g = h // (Hq // Hkv)
            toks = oracle.block_tokens(I[b, h], bs, T)
            o, l, _ = oracle.attend_head(inp.Q[b, h], inp.K[b, g], inp.V[b, g], toks, w.scale)
            assert np.abs(On[b, h] - o).max() <= 1e-2
            assert abs(L[b, h] - l) <= 1e-3 * (1 + abs(l))
    assert ds.device_status() == 0
    inp.free()


def test_block_size_one_is_topk_of_clamped_scores():
    w = dsgen.Workload("bs1", B=1, Hq=4, Hkv=4, T=2000, r=16, k=1, n_out=16, seed=0xB11)
    inp = gu.Inputs(w)
    kb = 150
    sb, bidx, O, lse, s = _run(w, inp, w.T, 1, kb)
    S = s.cpu().numpy()
    assert np.array_equal(bidx.cpu().numpy(), oracle.topk(np.maximum(S, 0), kb))
    inp.free()
