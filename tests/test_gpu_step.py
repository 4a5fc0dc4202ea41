"""ds_decode_step: the whole decode step in one call, against the three-call path and the oracle.

The index set must equal the one the separate calls produce (the same
selection code and the same fp32 scores); the label row of the newest token
must be the oracle's; O is checked against the oracle on the GPU's own set
(1e-2, as for ds_sparse_decode) and against the three-call path's O (the
summation order of the attention may differ, so only to fp32 rounding).
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
    # (name, B, Hq, Hkv, T, T_cap, r, k)     fused unless noted
    ("mha-T1-r8", 1, 2, 2, 1, 1, 8, 1),
    ("mha-T100-r16", 2, 3, 3, 100, 120, 16, 7),
    ("gqa-T1000-r16", 2, 8, 2, 1000, 1003, 16, 37),
    ("mha-T4097-r32", 1, 4, 4, 4097, 4100, 32, 300),
    ("mha-T3000-r64-kT", 1, 2, 2, 3000, 3000, 64, 3000),
    ("mha-T2500-r128", 1, 2, 2, 2500, 2600, 128, 777),
    ("mha-T20000-r8", 2, 4, 4, 20000, 20000, 8, 1250),
    ("mha-T40000-r8-fallback", 1, 2, 2, 40000, 40000, 8, 10000),   # k > 8192
    ("mha-T300000-r8-fallback", 1, 1, 1, 300000, 300000, 8, 4000),  # needs a cluster
]


def _run(case, append):
    name, B, Hq, Hkv, T, T_cap, r, k = case
    w = dsgen.Workload(name, B=B, Hq=Hq, Hkv=Hkv, T=T_cap, r=r, k=k, n_out=min(8, r),
                       seed=0x5EED + T)
    inp = gu.Inputs(w, r=r)
    BH = B * Hq
    # label cache up to T-1 (or T when the step does not append); row T-1 stale
    label = torch.zeros((B, Hq, T_cap, r), dtype=torch.bfloat16, device="cuda")
    n0 = T - 1 if append else T
    if n0 > 0:
        ds.label_append(inp.dK, inp.dC, label, 0, n0)
    label_sep = label.clone()
    # the three calls
    if append:
        ds.label_append(inp.dK, inp.dC, label_sep, T - 1, 1)
    idx_sep = torch.empty((BH, k), dtype=torch.int32, device="cuda")
    ds.score_topk(inp.dQ, inp.dC, label_sep, idx_sep, T)
    O_sep = torch.empty((B, Hq, w.d), dtype=torch.float32, device="cuda")
    ds.sparse_decode(inp.dQ, inp.dK, inp.dV, idx_sep, O_sep, T, w.scale)
    # the fused step
    idx = torch.full((BH, k), -1, dtype=torch.int32, device="cuda")
    O = torch.empty((B, Hq, w.d), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    ds.decode_step(inp.dQ, inp.dK, inp.dV, inp.dC, label, idx, O, T, w.scale, append=append,
                   lse=lse)
    torch.cuda.synchronize()
    return w, inp, T, label, label_sep, idx, idx_sep, O, O_sep, lse


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("append", [True, False])
def test_decode_step_matches_three_calls_and_oracle(case, append):
    w, inp, T, label, label_sep, idx, idx_sep, O, O_sep, lse = _run(case, append)
    assert torch.equal(idx, idx_sep)
    got_label = gu.host_bits(label)[:, :, :T]
    assert np.array_equal(got_label, oracle.label(inp.K[:, :, :T], inp.C, w.Hq))
    assert (O - O_sep).abs().max().item() <= 1e-5
    I = idx.cpu().numpy().reshape(w.B, w.Hq, w.k)
    ref_O, ref_L = oracle.attend(inp.Q, inp.K, inp.V, I, w.scale)
    assert np.abs(O.cpu().numpy() - ref_O).max() <= 1e-2
    L = lse.cpu().numpy()
    assert np.all(np.abs(L - ref_L) <= 1e-3 * (1 + np.abs(ref_L)))
    assert ds.device_status() == 0


def test_decode_step_workspace_only_for_the_fallback():
    d_fused = ds.Dims(8, 32, 32, 128, 4096, 16)
    assert ds.workspace_size(ds.OP_DECODE_STEP, d_fused, 4096, 256) == 0
    d_long = ds.Dims(1, 32, 32, 128, 262144, 8)
    assert ds.workspace_size(ds.OP_DECODE_STEP, d_long, 262144, 16384) > 0


@pytest.mark.parametrize("name", ["llama2-7b-B8-H32-T4K", "sweep-B32-H32-T32K-r8-k2048",
                                  "gqa-B16-Hq64-Hkv8-T16K"])
def test_decode_step_full_workload_sampled_heads(name):
    w = dsgen.workload(name)
    inp = gu.Inputs(w)
    BH = w.B * w.Hq
    label = torch.empty((w.B, w.Hq, w.T, w.r), dtype=torch.bfloat16, device="cuda")
    ds.label_append(inp.dK, inp.dC, label, 0, w.T - 1)
    idx = torch.empty((BH, w.k), dtype=torch.int32, device="cuda")
    O = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    ds.decode_step(inp.dQ, inp.dK, inp.dV, inp.dC, label, idx, O, w.T, w.scale, append=True)
    torch.cuda.synchronize()
    I = idx.cpu().numpy().reshape(w.B, w.Hq, w.k)
    On = O.cpu().numpy()
    for b, h in gu.sample_heads(w.B, w.Hq, 10, seed=3):
        g = h // w.G
        lab = oracle.label_head(inp.K[b, g], inp.C[h])
        s64 = oracle.score_head(inp.Q[b, h], inp.C[h], lab)
        sel = I[b, h]
        assert len(np.unique(sel)) == w.k and np.all(np.diff(sel) > 0)
        s_k = np.sort(s64)[::-1][w.k - 1]
        assert np.all(s64[sel] >= s_k - 1e-3 * (abs(s_k) + 1))
        o, _, _ = oracle.attend_head(inp.Q[b, h], inp.K[b, g], inp.V[b, g], sel, w.scale)
        assert np.abs(On[b, h] - o).max() <= 1e-2
    inp.free()


KV_CASES = [
    # (name, B, Hq, Hkv, T, T_cap, r, k)
    ("mha-T100-r16", 2, 3, 3, 100, 120, 16, 7),
    ("gqa-T1000-r16", 2, 8, 2, 1000, 1003, 16, 37),    # four CTAs share each new row
    ("mha-T1-r8", 1, 2, 2, 1, 1, 8, 1),                 # the new token is the only one
    ("mha-T4097-r32", 1, 4, 4, 4097, 4100, 32, 300),
    ("mha-T2500-r128-kT", 1, 2, 2, 2500, 2600, 128, 2500),  # every token kept
    ("mha-T40000-r8-fallback", 1, 2, 2, 40000, 40000, 8, 10000),
]


@pytest.mark.parametrize("host", [False, True], ids=["device", "host-io"])
@pytest.mark.parametrize("case", KV_CASES, ids=[c[0] for c in KV_CASES])
def test_decode_step_kv_equals_kv_append_then_step(case, host):
    """ds_decode_step_kv is ds_kv_append(T-1) followed by ds_decode_step with append:
    the same caches, label cache and index set bit for bit, the same O to fp32
    rounding.  The new rows differ from what the caches held at T-1, so a row not
    stored, or token T-1 attended from the stale cache row, shows."""
    name, B, Hq, Hkv, T, T_cap, r, k = case
    w = dsgen.Workload(name, B=B, Hq=Hq, Hkv=Hkv, T=T_cap, r=r, k=k, n_out=min(8, r),
                       seed=0x5EED + 7 * T)
    inp = gu.Inputs(w, r=r)
    g = torch.Generator(device="cpu").manual_seed(T)
    kn = (3 * torch.randn((B, Hkv, w.d), generator=g)).to(torch.bfloat16)
    vn = torch.randn((B, Hkv, w.d), generator=g).to(torch.bfloat16)
    label = torch.zeros((B, Hq, T_cap, r), dtype=torch.bfloat16, device="cuda")
    if T > 1:
        ds.label_append(inp.dK, inp.dC, label, 0, T - 1)
    BH = B * Hq
    # the separate calls
    K1, V1, L1 = inp.dK.clone(), inp.dV.clone(), label.clone()
    ds.kv_append(kn.cuda(), vn.cuda(), K1, V1, T - 1)
    idx1 = torch.empty((BH, k), dtype=torch.int32, device="cuda")
    O1 = torch.empty((B, Hq, w.d), dtype=torch.float32, device="cuda")
    ds.decode_step(inp.dQ, K1, V1, inp.dC, L1, idx1, O1, T, w.scale, append=True)
    # the one call
    K2, V2, L2 = inp.dK.clone(), inp.dV.clone(), label.clone()
    idx2 = torch.full((BH, k), -1, dtype=torch.int32, device="cuda")
    if host:
        q, kn2, vn2 = inp.dQ.cpu().pin_memory(), kn.pin_memory(), vn.pin_memory()
        O2 = torch.empty((B, Hq, w.d), dtype=torch.float32).pin_memory()
        lse2 = torch.empty((B, Hq), dtype=torch.float32).pin_memory()
    else:
        q, kn2, vn2 = inp.dQ, kn.cuda(), vn.cuda()
        O2 = torch.empty((B, Hq, w.d), dtype=torch.float32, device="cuda")
        lse2 = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    ds.decode_step_kv(q, kn2, vn2, K2, V2, inp.dC, L2, idx2, O2, T, w.scale, lse=lse2)
    torch.cuda.synchronize()
    assert torch.equal(K2.view(torch.int16), K1.view(torch.int16))
    assert torch.equal(V2.view(torch.int16), V1.view(torch.int16))
    assert torch.equal(L2.view(torch.int16), L1.view(torch.int16))
    assert torch.equal(idx2, idx1)
    assert (O2.cuda() - O1).abs().max().item() <= 1e-5
    # and the oracle on the appended caches
    Kh = gu.host_bits(K1)
    Vh = gu.host_bits(V1)
    I = idx2.cpu().numpy().reshape(B, Hq, k)
    ref_O, ref_L = oracle.attend(inp.Q, Kh, Vh, I, w.scale)
    assert np.abs(O2.cpu().numpy() - ref_O).max() <= 1e-2
    L = lse2.cpu().numpy()
    assert np.all(np.abs(L - ref_L) <= 1e-3 * (1 + np.abs(ref_L)))
    assert ds.device_status() == 0


@pytest.mark.parametrize("T,k,mode", [(4096, 256, "ints"), (4096, 4096, "ints"), (3000, 2999, "ints"),
                                      (37, 5, "ints"), (4096, 1000, "zero_q"), (1, 1, "zero_q"),
                                      (2049, 700, "ints")])
def test_decode_step_whole_head_ties(T, k, mode):
    """Heads of at most 4096 tokens are selected in the step kernel from keys held
    in shared memory.  Scores with many ties (a query of ones over labels in
    {-1, 0, 1}: integer scores; or a zero query: every score 0) must give the
    same index set as ds_score_topk and as the oracle's rule (ties to the lower
    index) applied to the scores ds_score returns."""
    B, Hq, r = 2, 4, 16
    w = dsgen.Workload("ties", B=B, Hq=Hq, Hkv=Hq, T=T, r=r, k=k, n_out=8, seed=0x71E + T)
    inp = gu.Inputs(w, r=r)
    rng = np.random.default_rng(T + k)
    lab = rng.integers(-1, 2, size=(B, Hq, T, r)).astype(np.float32)
    label = torch.from_numpy(lab).to(torch.bfloat16).cuda()
    Q = torch.zeros_like(inp.dQ) if mode == "zero_q" else torch.ones_like(inp.dQ)
    idx = torch.full((B * Hq, k), -1, dtype=torch.int32, device="cuda")
    O = torch.empty((B, Hq, w.d), dtype=torch.float32, device="cuda")
    ds.decode_step(Q, inp.dK, inp.dV, inp.dC, label, idx, O, T, w.scale, append=False)
    idx_sep = torch.empty_like(idx)
    ds.score_topk(Q, inp.dC, label, idx_sep, T)
    s = torch.empty((B * Hq, T), dtype=torch.float32, device="cuda")
    ds.score(Q, inp.dC, label, s, T)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx_sep)
    S = s.cpu().numpy()
    I = idx.cpu().numpy()
    for bh in range(B * Hq):
        assert np.array_equal(I[bh], oracle.topk_head(S[bh], k)), bh
    if mode == "zero_q":
        assert np.array_equal(I, np.tile(np.arange(k, dtype=np.int32), (B * Hq, 1)))
    assert ds.device_status() == 0
    inp.free()
