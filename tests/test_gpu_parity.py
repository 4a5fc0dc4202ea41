"""GPU parity: every call of the C ABI against the CPU oracle, element by element.

Tolerances:
  label            bit-exact (a copy)
  scores           |gpu - exact| <= gamma_{r-1} * sum_j |q_j label_j| (fp32
                   recursive-summation bound; products of bf16 are exact)
  top-k            bit-exact index set on the oracle's fp32 scores
  selection        every GPU-selected index has an exact score within
                   1e-3 * (|s_k| + 1) of the exact k-th score
  sparse O         max abs error <= 1e-2, on the GPU's own index set
  dense O          max abs error <= 5e-3
  lse              |gpu - oracle| <= 1e-3 * (1 + |lse|)
"""
import math

import numpy as np
import pytest
import torch

import dsgen
import oracle
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import post_token_sparse_b200 as ds

SPARSE_TOL = 1e-2
DENSE_TOL = 5e-3


def _lse_ok(gpu, ref):
    return np.all(np.abs(gpu - ref) <= 1e-3 * (1 + np.abs(ref)))


@pytest.fixture(autouse=True)
def _clear_status():
    if torch.cuda.is_available():
        ds.device_status(clear=True)
    yield


SMALL = [
    # (name, B, Hq, Hkv, T, T_cap, r, k)
    ("mha-T1", 1, 2, 2, 1, 1, 8, 1),
    ("mha-T7-r1", 1, 3, 3, 7, 9, 1, 3),
    ("mha-T63", 2, 4, 4, 63, 64, 8, 5),
    ("mha-T65-r5", 1, 4, 4, 65, 70, 5, 64),
    ("gqa-T1000-r16", 2, 8, 2, 1000, 1003, 16, 37),
    ("mha-T4097-r32", 1, 4, 4, 4097, 4100, 32, 300),
    ("mha-T3000-r64", 1, 2, 2, 3000, 3000, 64, 3000),
    ("mha-T2500-r128", 1, 2, 2, 2500, 2600, 128, 777),
    ("gqa-T5000-r24", 1, 8, 1, 5000, 5000, 24, 1000),
]


def _small(name, B, Hq, Hkv, T, T_cap, r, k):
    w = dsgen.Workload(name, B=B, Hq=Hq, Hkv=Hkv, T=T_cap, r=r, k=k, n_out=min(8, r),
                       seed=0xABC0 + T)
    return gu.Inputs(w, r=r), T


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_label_append_bit_exact(case):
    inp, T = _small(*case)
    w = inp.w
    sentinel = 0x7E7E
    label = torch.full((w.B, w.Hq, w.T, inp.r), sentinel, dtype=torch.int16, device="cuda")
    label = label.view(torch.bfloat16)
    # prompt in two pieces, then one token
    cut = max(1, T // 3)
    ds.label_append(inp.dK, inp.dC, label, 0, cut)
    if T - cut > 1:
        ds.label_append(inp.dK, inp.dC, label, cut, T - cut - 1)
    if T > cut:
        ds.label_append(inp.dK, inp.dC, label, T - 1, 1)
    got = gu.host_bits(label)
    ref = oracle.label(inp.K, inp.C, w.Hq)
    assert np.array_equal(got[:, :, :T], ref[:, :, :T])
    assert np.all(got[:, :, T:] == sentinel)  # rows beyond T untouched
    assert ds.device_status() == 0


def _label_dev(inp, T):
    w = inp.w
    label = torch.zeros((w.B, w.Hq, w.T, inp.r), dtype=torch.bfloat16, device="cuda")
    ds.label_append(inp.dK, inp.dC, label, 0, T)
    return label


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_score_within_fp32_bound(case):
    inp, T = _small(*case)
    w = inp.w
    label = _label_dev(inp, T)
    scores = torch.empty((w.B * w.Hq, T), dtype=torch.float32, device="cuda")
    ds.score(inp.dQ, inp.dC, label, scores, T)
    got = scores.cpu().numpy().reshape(w.B, w.Hq, T)
    lab = oracle.label(inp.K[:, :, :T], inp.C, w.Hq)
    s64 = oracle.score(inp.Q, inp.C, lab)
    for b in range(w.B):
        for h in range(w.Hq):
            qc = oracle.bf16_to_f64(inp.Q[b, h][inp.C[h]])
            bound = gu.score_error_bound(qc, oracle.bf16_to_f64(lab[b, h]))
            assert np.all(np.abs(got[b, h] - s64[b, h]) <= bound), (b, h)


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_score_topk_fused_equals_unfused(case):
    inp, T = _small(*case)
    w = inp.w
    BH = w.B * w.Hq
    label = _label_dev(inp, T)
    s_sep = torch.empty((BH, T), dtype=torch.float32, device="cuda")
    ds.score(inp.dQ, inp.dC, label, s_sep, T)
    i_sep = torch.empty((BH, w.k), dtype=torch.int32, device="cuda")
    ds.topk(s_sep, i_sep)
    s_fus = torch.empty((BH, T), dtype=torch.float32, device="cuda")
    i_fus = torch.empty((BH, w.k), dtype=torch.int32, device="cuda")
    ds.score_topk(inp.dQ, inp.dC, label, i_fus, T, scores=s_fus)
    i_fus2 = torch.empty((BH, w.k), dtype=torch.int32, device="cuda")
    if inp.r in (8, 16, 32, 64, 128):
        ds.score_topk(inp.dQ, inp.dC, label, i_fus2, T)  # without writing scores
    else:
        i_fus2.copy_(i_fus)
    assert torch.equal(s_sep, s_fus)
    assert torch.equal(i_sep, i_fus) and torch.equal(i_fus, i_fus2)
    # the GPU's set is the exact top-k of the GPU's own fp32 scores
    ref = oracle.topk(s_sep.cpu().numpy(), w.k)
    assert np.array_equal(i_sep.cpu().numpy(), ref)


def _check_topk(scores: np.ndarray, k: int):
    s32 = np.ascontiguousarray(scores, dtype=np.float32)
    d_s = gu.dev_f32(s32)
    idx = torch.empty((s32.shape[0], k), dtype=torch.int32, device="cuda")
    ds.topk(d_s, idx)
    got = idx.cpu().numpy()
    ref = oracle.topk(s32, k)
    bad = np.nonzero(~np.all(got == ref, axis=1))[0]
    assert bad.size == 0, f"rows {bad[:5]} differ"


TOPK_SHAPES = [(1, 1, 1), (3, 7, 2), (5, 64, 64), (2, 65, 10), (1, 4096, 256), (7, 1000, 999),
               (1, 786432, 49152), (4, 32768, 32768), (40, 40000, 1000),
               (1, 40961, 5000), (2, 100000, 6250), (64, 100000, 100), (1, 262144, 16384),
               (1, 655360, 40960), (300, 32768, 2048)]


@pytest.mark.parametrize("BH,T,k", TOPK_SHAPES, ids=[f"BH{a}-T{b}-k{c}" for a, b, c in
                                                   TOPK_SHAPES])
def test_topk_bit_exact_random(BH, T, k):
    rng = np.random.default_rng(T * 31 + k)
    _check_topk(rng.standard_normal((BH, T)) * 100, k)


@pytest.mark.parametrize("T,k", [(100, 17), (5000, 2500), (100000, 30000), (262144, 1)])
def test_topk_ties_and_signed_zeros(T, k):
    rng = np.random.default_rng(T + k)
    s = rng.integers(-4, 5, (3, T)).astype(np.float32)
    s[rng.random((3, T)) < 0.2] = -0.0
    s[0, rng.integers(0, T, 5)] = np.inf
    s[1, rng.integers(0, T, 5)] = -np.inf
    s[2] = 0.0  # a row of +0 ...
    s[2, ::3] = -0.0  # ... mixed with -0: all equal, so the first k win
    _check_topk(s, k)
    # all equal
    _check_topk(np.full((2, T), 3.25, np.float32), k)


def test_topk_golden():
    import json, os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "topk_worked.json")))
    s = np.array([[float(x) for x in g["scores"]]], np.float32)
    d_s = gu.dev_f32(s)
    for k, exp in g["expected"].items():
        idx = torch.empty((1, int(k)), dtype=torch.int32, device="cuda")
        ds.topk(d_s, idx)
        assert idx.cpu().numpy()[0].tolist() == exp


def _attend_check(inp, T, idx_np, O, lse, tol):
    w = inp.w
    ref_O, ref_L = oracle.attend(inp.Q, inp.K, inp.V, idx_np, w.scale)
    err = np.abs(O.cpu().numpy() - ref_O).max()
    assert err <= tol, err
    assert _lse_ok(lse.cpu().numpy(), ref_L)
    return err


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_sparse_decode_matches_oracle(case):
    inp, T = _small(*case)
    w = inp.w
    BH = w.B * w.Hq
    label = _label_dev(inp, T)
    idx = torch.empty((BH, w.k), dtype=torch.int32, device="cuda")
    scores = torch.empty((BH, T), dtype=torch.float32, device="cuda")
    ds.score_topk(inp.dQ, inp.dC, label, idx, T, scores=scores)
    O = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    ds.sparse_decode(inp.dQ, inp.dK, inp.dV, idx, O, T, w.scale, lse=lse)
    idx_np = idx.cpu().numpy().reshape(w.B, w.Hq, w.k)
    _attend_check(inp, T, idx_np, O, lse, SPARSE_TOL)
    assert ds.device_status() == 0


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_dense_decode_matches_oracle(case):
    inp, T = _small(*case)
    w = inp.w
    O = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    ds.decode(inp.dQ, inp.dK, inp.dV, O, T, w.scale, lse=lse)
    ref_O, ref_L = oracle.dense(inp.Q, inp.K[:, :, :T], inp.V[:, :, :T], w.scale)
    assert np.abs(O.cpu().numpy() - ref_O).max() <= DENSE_TOL
    assert _lse_ok(lse.cpu().numpy(), ref_L)


@pytest.mark.parametrize("B,Hq,Hkv,T,k", [(1, 1, 1, 50000, 50000), (1, 2, 1, 20000, 3000),
                                         (1, 1, 1, 9000, 1), (1, 4, 4, 300, 300)])
def test_sparse_decode_split_paths(B, Hq, Hkv, T, k):
    """Few heads, many rows: the rows are split across CTAs and LSE-merged."""
    w = dsgen.Workload("split", B=B, Hq=Hq, Hkv=Hkv, T=T, r=8, k=k, n_out=8, seed=77 + T)
    inp = gu.Inputs(w)
    rng = np.random.default_rng(T)
    idx_np = np.sort(np.stack([rng.choice(T, k, replace=False) for _ in range(B * Hq)]),
                     axis=1).astype(np.int32)
    idx = gu.dev_i32(idx_np)
    O = torch.empty((B, Hq, w.d), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    ds.sparse_decode(inp.dQ, inp.dK, inp.dV, idx, O, T, w.scale, lse=lse)
    _attend_check(inp, T, idx_np.reshape(B, Hq, k), O, lse, SPARSE_TOL)
    O2 = torch.empty_like(O)
    ds.decode(inp.dQ, inp.dK, inp.dV, O2, T, w.scale)
    ref_O, _ = oracle.dense(inp.Q, inp.K, inp.V, w.scale)
    assert np.abs(O2.cpu().numpy() - ref_O).max() <= DENSE_TOL


def test_attend_golden_worked_example():
    """The hand-derived example, embedded in d = 128 with zero padding."""
    import json, os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "attend_worked.json")))
    d = 128
    q = np.zeros((1, 1, d), np.float32)
    q[0, 0, :4] = g["q"]
    K = np.zeros((1, 1, 4, d), np.float32)
    K[0, 0, :, :4] = g["K"]
    V = np.zeros((1, 1, 4, d), np.float32)
    V[0, 0, :, :4] = g["V"]
    dq, dK, dV = (gu.dev_bf16(dsgen.bf16_bits_from_f32(a)) for a in (q, K, V))
    idx = gu.dev_i32(np.array([g["idx"]], np.int32))
    O = torch.empty((1, 1, d), dtype=torch.float32, device="cuda")
    lse = torch.empty((1, 1), dtype=torch.float32, device="cuda")
    ds.sparse_decode(dq, dK, dV, idx, O, 4, math.log(2.0), lse=lse)
    want = np.zeros(d)
    want[:4] = g["o"]
    assert np.abs(O.cpu().numpy()[0, 0] - want).max() < 1e-5
    assert abs(lse.item() - math.log(7.0)) < 1e-5


def test_full_channels_all_tokens_equals_dense():
    """r = d and k = T through the whole sparse pipeline equals dense attention."""
    w = dsgen.Workload("rd-kT", B=2, Hq=4, Hkv=4, T=3000, r=128, k=3000, n_out=16, seed=5)
    inp = gu.Inputs(w, r=128)
    BH = w.B * w.Hq
    label = _label_dev(inp, w.T)
    idx = torch.empty((BH, w.T), dtype=torch.int32, device="cuda")
    ds.score_topk(inp.dQ, inp.dC, label, idx, w.T)
    assert torch.equal(idx, torch.arange(w.T, dtype=torch.int32, device="cuda").expand(BH, -1))
    O_s = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    O_d = torch.empty_like(O_s)
    ds.sparse_decode(inp.dQ, inp.dK, inp.dV, idx, O_s, w.T, w.scale)
    ds.decode(inp.dQ, inp.dK, inp.dV, O_d, w.T, w.scale)
    assert (O_s - O_d).abs().max().item() < 1e-5
    ref_O, _ = oracle.dense(inp.Q, inp.K, inp.V, w.scale)
    assert np.abs(O_d.cpu().numpy() - ref_O).max() <= DENSE_TOL


def test_out_of_range_inputs_are_flagged_not_faulted():
    w = dsgen.Workload("bad", B=1, Hq=2, Hkv=2, T=100, r=8, k=4, n_out=8, seed=9)
    inp = gu.Inputs(w)
    C_bad = inp.C.copy()
    C_bad[0, 0] = 200
    label = torch.zeros((1, 2, 100, 8), dtype=torch.bfloat16, device="cuda")
    ds.label_append(inp.dK, gu.dev_i32(C_bad), label, 0, 100)
    assert ds.device_status() & ds.DEV_BAD_CHANNEL
    idx = gu.dev_i32(np.array([[0, 5, 99, 1000], [-3, 1, 2, 3]], np.int32))
    O = torch.empty((1, 2, 128), dtype=torch.float32, device="cuda")
    ds.sparse_decode(inp.dQ, inp.dK, inp.dV, idx, O, 100, w.scale)
    assert ds.device_status() & ds.DEV_BAD_INDEX
    assert torch.isfinite(O).all()
    assert ds.device_status() == 0  # cleared by the previous read


def test_errors_on_device_launch_nothing():
    w = dsgen.Workload("err", B=1, Hq=1, Hkv=1, T=50000, r=8, k=100, n_out=8, seed=3)
    inp = gu.Inputs(w)
    O = torch.empty((1, 1, 128), dtype=torch.float32, device="cuda")
    n0 = ds.kernel_launches()
    with pytest.raises(ds.DsError) as e:
        ds.decode(inp.dQ, inp.dK, inp.dV, O, 50000, w.scale,
                  ws=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert e.value.status == ds.DS_ERR_WORKSPACE
    with pytest.raises(ds.DsError):
        ds.topk(torch.empty((1, 10), device="cuda"), torch.empty((1, 11), dtype=torch.int32,
                                                                 device="cuda"))
    assert ds.kernel_launches() == n0


# ---------------------------------------------------------------------------
# the named workloads at full size, sampled heads checked one by one

FULL = ["tiny-B1-H4-T1K", "llama2-7b-B8-H32-T4K", "gqa-B16-Hq64-Hkv8-T16K",
        "long-B1-H32-T256K"] + [n for n in dsgen.ORDER if n.startswith("sweep")]

# the inputs of the last workload set, kept while the next test uses the same
# set (the nine sweep cells share one)
_INPUTS = {}


def _inputs(w):
    key = (w.seed, w.B, w.Hq, w.Hkv, w.T)
    if key not in _INPUTS:
        for old in _INPUTS.values():
            old.free()
        _INPUTS.clear()
        _INPUTS[key] = gu.Inputs(w)
    inp = _INPUTS[key]
    inp.C = dsgen.channels(w, w.r)
    inp.dC = gu.dev_i32(inp.C)
    inp.r = w.r
    return inp


def _full_step(name):
    w = dsgen.workload(name)
    inp = _inputs(w)
    BH = w.B * w.Hq
    label = _label_dev(inp, w.T)
    scores = torch.empty((BH, w.T), dtype=torch.float32, device="cuda")
    ds.score(inp.dQ, inp.dC, label, scores, w.T)
    idx = torch.empty((BH, w.k), dtype=torch.int32, device="cuda")
    ds.score_topk(inp.dQ, inp.dC, label, idx, w.T)
    O = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    ds.sparse_decode(inp.dQ, inp.dK, inp.dV, idx, O, w.T, w.scale, lse=lse)
    Od = torch.empty_like(O)
    lsed = torch.empty_like(lse)
    ds.decode(inp.dQ, inp.dK, inp.dV, Od, w.T, w.scale, lse=lsed)
    # the decode step in the launch configuration the benchmark times (label row
    # of the newest token appended, selection, attention)
    idx_st = torch.empty_like(idx)
    O_st = torch.empty_like(O)
    ds.decode_step(inp.dQ, inp.dK, inp.dV, inp.dC, label, idx_st, O_st, w.T, w.scale,
                   append=True)
    torch.cuda.synchronize()
    assert torch.equal(idx_st, idx)
    assert (O_st - O).abs().max().item() <= 1e-5
    del label
    return w, inp, scores, idx, O, lse, Od, lsed


@pytest.mark.parametrize("name", FULL)
def test_full_workload_sampled_heads(name):
    """Every named workload at full size: scores, bit-exact top-k, selection and
    attention on sampled heads against the numpy oracle, and on four of them
    against the C++ oracle as well; dense attention on the first cell of each
    input set."""
    import oracle.cxx as cxx

    w, inp, scores, idx, O, lse, Od, lsed = _full_step(name)
    n_sample = w.B * w.Hq if w.B * w.Hq <= 64 else 12
    heads = gu.sample_heads(w.B, w.Hq, n_sample, seed=1)
    S = scores.cpu().numpy().reshape(w.B, w.Hq, w.T)
    I = idx.cpu().numpy().reshape(w.B, w.Hq, w.k)
    On, Ln, Odn, Ldn = (t.cpu().numpy() for t in (O, lse, Od, lsed))
    worst = {"sparse": 0.0, "dense": 0.0}
    with_dense = not name.startswith("sweep") or name.endswith("r8-k512")
    for i, (b, h) in enumerate(heads):
        g = h // w.G
        Kbg, Vbg = inp.K[b, g], inp.V[b, g]
        lab = oracle.label_head(Kbg, inp.C[h])
        s64 = oracle.score_head(inp.Q[b, h], inp.C[h], lab)
        s32 = oracle.to_f32(s64)
        # scores within the fp32 bound
        qc = oracle.bf16_to_f64(inp.Q[b, h][inp.C[h]])
        assert np.all(np.abs(S[b, h] - s64) <= gu.score_error_bound(qc, oracle.bf16_to_f64(lab)))
        # bit-exact top-k on the oracle's fp32 scores
        it = torch.empty((1, w.k), dtype=torch.int32, device="cuda")
        ds.topk(gu.dev_f32(s32[None]), it)
        assert np.array_equal(it.cpu().numpy()[0], oracle.topk_head(s32, w.k))
        # selection tolerance of the GPU's own set against exact scores
        sel = I[b, h]
        assert len(np.unique(sel)) == w.k and np.all(np.diff(sel) > 0)
        assert sel[0] >= 0 and sel[-1] < w.T
        s_k = np.sort(s64)[::-1][w.k - 1]
        assert np.all(s64[sel] >= s_k - 1e-3 * (abs(s_k) + 1))
        # attention on the GPU's set, and dense
        o, l, _ = oracle.attend_head(inp.Q[b, h], Kbg, Vbg, sel, w.scale)
        e = np.abs(On[b, h] - o).max()
        worst["sparse"] = max(worst["sparse"], e)
        assert e <= SPARSE_TOL and abs(Ln[b, h] - l) <= 1e-3 * (1 + abs(l))
        if with_dense or i < 2:
            od, ld, _ = oracle.attend_head(inp.Q[b, h], Kbg, Vbg, np.arange(w.T), w.scale)
            e = np.abs(Odn[b, h] - od).max()
            worst["dense"] = max(worst["dense"], e)
            assert e <= DENSE_TOL and abs(Ldn[b, h] - ld) <= 1e-3 * (1 + abs(ld))
        if i < 4:
            # the C++ oracle: label bits, its fp32 scores' top-k, selection, O
            labx = cxx.label_head(Kbg, inp.C[h])
            assert np.array_equal(labx, lab)
            sx = cxx.score_head(inp.Q[b, h], inp.C[h], labx)
            ds.topk(gu.dev_f32(cxx.to_f32(sx)[None]), it)
            assert np.array_equal(it.cpu().numpy()[0], cxx.topk_head(cxx.to_f32(sx), w.k))
            sxk = np.sort(sx)[::-1][w.k - 1]
            assert np.all(sx[sel] >= sxk - 1e-3 * (abs(sxk) + 1))
            ox, lx, _ = cxx.attend_head(inp.Q[b, h], Kbg, Vbg, sel, w.scale)
            assert np.abs(On[b, h] - ox).max() <= SPARSE_TOL
            assert abs(Ln[b, h] - lx) <= 1e-3 * (1 + abs(lx))
    if w.n_hh:
        pos = dsgen.hh_positions(w)
        for h in range(w.Hq):
            assert set(pos[h].tolist()) <= set(I[0, h].tolist())
    print(f"{name}: max abs err sparse {worst['sparse']:.3g} dense {worst['dense']:.3g}")
    if not name.startswith("sweep"):
        for old in _INPUTS.values():
            old.free()
        _INPUTS.clear()


def test_full_sweep_every_channel_every_token_equals_dense():
    """The sweep's r = d, k = T cell at full size (B32 H32 T32K): the whole sparse
    pipeline with every channel and every token keeps every token and equals
    dense attention; dense matches the oracle on sampled heads."""
    base = dsgen.workload("sweep-B32-H32-T32K-r8-k512")
    w = base.with_(name="sweep-B32-H32-T32K-r128-kT", r=base.d, k=base.T)
    inp = _inputs(w)  # the sweep's input set (kept from the cells above)
    BH = w.B * w.Hq
    label = _label_dev(inp, w.T)
    idx = torch.empty((BH, w.T), dtype=torch.int32, device="cuda")
    ds.score_topk(inp.dQ, inp.dC, label, idx, w.T)
    assert torch.equal(idx, torch.arange(w.T, dtype=torch.int32, device="cuda").expand(BH, -1))
    idx.fill_(-1)
    O_s = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    ds.decode_step(inp.dQ, inp.dK, inp.dV, inp.dC, label, idx, O_s, w.T, w.scale, append=True)
    assert torch.equal(idx, torch.arange(w.T, dtype=torch.int32, device="cuda").expand(BH, -1))
    del label
    O_d = torch.empty_like(O_s)
    ds.decode(inp.dQ, inp.dK, inp.dV, O_d, w.T, w.scale)
    torch.cuda.synchronize()
    assert (O_s - O_d).abs().max().item() < 1e-5
    Odn = O_d.cpu().numpy()
    for b, h in gu.sample_heads(w.B, w.Hq, 6, seed=3):
        od, _, _ = oracle.attend_head(inp.Q[b, h], inp.K[b, h], inp.V[b, h], np.arange(w.T),
                                      w.scale)
        assert np.abs(Odn[b, h] - od).max() <= DENSE_TOL
    for old in _INPUTS.values():
        old.free()
    _INPUTS.clear()


@pytest.mark.parametrize("B,H,T,k", [(1, 2, 5000, 1234), (2, 3, 70000, 20000)])
def test_score_topk_all_scores_tied(B, H, T, k):
    """Every K row identical: all scores tie, the first k tokens must be kept.

    Exercises the path where one CTA has more candidates than it can list and
    recomputes their exact keys from the label cache."""
    w = dsgen.Workload("tied", B=B, Hq=H, Hkv=H, T=T, r=16, k=k, n_out=16, seed=4242)
    inp = gu.Inputs(w, with_v=False)
    inp.dK[:] = inp.dK[:, :, :1, :]
    label = _label_dev(inp, T)
    idx = torch.empty((B * H, k), dtype=torch.int32, device="cuda")
    ds.score_topk(inp.dQ, inp.dC, label, idx, T)
    want = torch.arange(k, dtype=torch.int32, device="cuda").expand(B * H, -1)
    assert torch.equal(idx, want)


def _sampled_tokens(T):
    """Tokens the top-k draws its bracketing sample from (128 blocks of 32)."""
    q = T // 32
    starts = [(b * q // 128) * 32 for b in range(128)]
    return np.concatenate([np.arange(s, s + 32) for s in starts])


@pytest.mark.parametrize("k", [50000, 49999, 1, 99999])
def test_topk_bracket_overflow_falls_back_exactly(k):
    """Two-valued scores: the sample bracket holds every token, the candidate lists
    overflow and the exact refinement path must produce the exact top-k."""
    T = 100000
    rng = np.random.default_rng(k)
    s = np.where(rng.random((2, T)) < 0.5, 1.0, -1.0).astype(np.float32)
    _check_topk(s, k)


@pytest.mark.parametrize("k", [1000, 4096, 10000])
def test_topk_bracket_miss_falls_back_exactly(k):
    """The sampled blocks score higher than every other token, so the sample
    misplaces the k-th key; the result must still be exact."""
    T = 100000
    rng = np.random.default_rng(k + 7)
    s = rng.standard_normal((2, T)).astype(np.float32)
    s[:, _sampled_tokens(T)] = 100.0
    _check_topk(s, k)
