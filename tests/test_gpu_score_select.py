"""The one-launch selection with a workspace (4096 < T <= 32768) against the
oracle, bit for bit.

ds_score_topk runs it for these sizes when given a workspace (the binding makes
one).  Its index set must be the oracle's top-k of the GPU's own fp32 scores
(ds_score computes them in the same order), with ties to the lower token index;
with a score buffer, the scores it writes must be ds_score's bit for bit; and
the same call without a workspace (the other selection paths) must agree.
Tie-heavy inputs force the slower resolutions: a bracket that misses, a
boundary bin resolved through its list, and one recomputed in place.
"""
import ctypes

import numpy as np
import pytest
import torch

import dsgen
import oracle
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import post_token_sparse_b200 as ds


def _run(B, Hq, Hkv, T, r, k, seed, kmod=None, zero_q=False):
    w = dsgen.Workload("pipe", B=B, Hq=Hq, Hkv=Hkv, T=T, r=r, k=k, n_out=min(16, r), seed=seed)
    inp = gu.Inputs(w, with_v=False)
    if kmod is not None:  # K rows repeat with period kmod: few distinct scores per head
        src = inp.dK[:, :, :kmod, :].clone()
        reps = -(-T // kmod)
        inp.dK[:] = src.repeat(1, 1, reps, 1)[:, :, :T, :]
    if zero_q:
        inp.dQ.zero_()
    BH = B * Hq
    label = torch.zeros((B, Hq, T, r), dtype=torch.bfloat16, device="cuda")
    ds.label_append(inp.dK, inp.dC, label, 0, T)
    scores = torch.empty((BH, T), dtype=torch.float32, device="cuda")
    ds.score(inp.dQ, inp.dC, label, scores, T)
    idx = torch.full((BH, k), -1, dtype=torch.int32, device="cuda")
    ds.score_topk(inp.dQ, inp.dC, label, idx, T)
    s2 = torch.full((BH, T), float("nan"), dtype=torch.float32, device="cuda")
    idx2 = torch.full((BH, k), -1, dtype=torch.int32, device="cuda")
    ds.score_topk(inp.dQ, inp.dC, label, idx2, T, scores=s2)
    # the same call without a workspace: the other selection paths
    idx3 = torch.full((BH, k), -1, dtype=torch.int32, device="cuda")
    dims = ds.Dims(B, Hq, Hq, 128, T, r)
    st = ds.lib().ds_score_topk(
        ctypes.c_void_p(inp.dQ.data_ptr()), ctypes.c_void_p(inp.dC.data_ptr()),
        ctypes.c_void_p(label.data_ptr()), None, ctypes.c_void_p(idx3.data_ptr()), dims, T, k,
        None, 0, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == ds.DS_OK
    torch.cuda.synchronize()
    assert ds.workspace_size(ds.OP_SCORE_TOPK, dims, T, k) > 0
    assert torch.equal(s2.view(torch.int32), scores.view(torch.int32))
    assert torch.equal(idx2, idx)
    assert torch.equal(idx3, idx)
    S = scores.cpu().numpy()
    I = idx.cpu().numpy()
    for row in range(BH):
        want = oracle.topk_head(S[row], k)
        assert np.array_equal(I[row], want), row
    inp.free()


@pytest.mark.parametrize("B,Hq,Hkv,T,r,k", [
    (16, 32, 32, 8192, 8, 1),       # k = 1
    (16, 32, 32, 8192, 8, 8192),    # k = T: every token
    (15, 32, 32, 6000, 16, 777),    # T not a multiple of 32
    (4, 128, 128, 32768, 32, 2048), # the largest T
    (16, 32, 32, 32768, 64, 100),
    (8, 64, 8, 12000, 16, 1000),    # grouped KV heads
    (4, 128, 128, 20000, 128, 5000),
    (16, 32, 32, 4097, 8, 256),     # the smallest T
    (1, 3, 3, 30000, 8, 3000),      # few heads
])
def test_score_select_topk_bit_exact(B, Hq, Hkv, T, r, k):
    _run(B, Hq, Hkv, T, r, k, seed=0x51E + T + k)


@pytest.mark.parametrize("T,k,kmod", [
    (8192, 3000, 7),      # ~1170 tokens per score value: the boundary bin through the list
    (32768, 5000, 5),     # ~6550 per value: the boundary bin recomputed in place
    (20000, 1, 3),
    (32768, 20000, 2),
])
def test_score_select_few_distinct_scores(T, k, kmod):
    _run(16, 32, 32, T, 16, k, seed=0x7E5 + T, kmod=kmod)


def test_score_select_all_scores_equal():
    """Q = 0: every score is +0 (or -0, equal to it): the first k tokens."""
    _run(16, 32, 32, 10000, 8, 4321, seed=99, zero_q=True)


@pytest.mark.parametrize("BH,T,k,mode", [(6, 4097, 1, "normal"), (5, 16384, 1024, "ints"),
                                         (3, 16384, 8192, "normal"), (4, 12000, 11999, "ints"),
                                         (2, 9000, 700, "zero"), (4, 16384, 1024, "wide"),
                                         (3, 16000, 300, "wide")])
def test_topk_over_scores_one_launch_equals_plain(BH, T, k, mode):
    """ds_topk with a workspace (tiles of written scores into key prefixes, the
    row's last tile selects) gives the index set of the call without one, and
    the oracle's rule on the same scores (ties to the lower index)."""
    import ctypes
    rng = np.random.default_rng(T + k)
    if mode == "ints":
        S = rng.integers(-20, 21, size=(BH, T)).astype(np.float32)
    elif mode == "zero":
        S = np.zeros((BH, T), np.float32)
        S[:, ::7] = -0.0
    elif mode == "wide":
        # magnitudes over ~80 binades: the bracket spans far more than 256
        # 16-bit key prefixes (the two-level search for the boundary bin)
        S = (rng.choice([-1.0, 1.0], size=(BH, T)) *
             np.exp(rng.uniform(-28, 28, size=(BH, T)))).astype(np.float32)
    else:
        S = (rng.standard_normal((BH, T)) * 40).astype(np.float32)
    sc = torch.from_numpy(S).cuda()
    i_ws = torch.full((BH, k), -1, dtype=torch.int32, device="cuda")
    ds.topk(sc, i_ws)  # the binding makes the workspace
    ws_bytes = ds.workspace_size(ds.OP_TOPK, ds.Dims(1, BH, 1, 128, T, 1), T, k)
    assert ws_bytes > 0
    i_plain = torch.full_like(i_ws, -1)
    st = ds.lib().ds_topk(ctypes.c_void_p(sc.data_ptr()), ctypes.c_void_p(i_plain.data_ptr()),
                          BH, T, k, None, 0,
                          ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == ds.DS_OK
    torch.cuda.synchronize()
    assert torch.equal(i_ws, i_plain)
    I = i_ws.cpu().numpy()
    for b in range(BH):
        assert np.array_equal(I[b], oracle.topk_head(S[b], k)), b
