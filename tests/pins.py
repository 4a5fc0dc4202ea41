"""Pins of the CPU oracle: checks against facts that do not come from the oracle.

Each pin takes the oracle module as an argument so that the same checks can be
run against deliberately broken copies of it (tests/test_oracle_mutations.py):
a plausible slip anywhere in the oracle -- a dropped term, a wrong sign or
index, a transposed operand -- must make at least one pin fail.

What pins what:
  bf16 decoding       known IEEE bit patterns
  label gather        identity / permutation cases; per-element brute force;
                      the query-head -> KV-head map on marked KV heads
  score               one-hot queries (a lookup); brute-force dot products;
                      agreement with the attention logits at r = d
  top-k               a characterisation of the (score desc, index asc)
                      order checked pair by pair; Python's sorted(); ties,
                      -0/+0, +-inf; the hand-derived worked example
  attention           torch scaled_dot_product_attention in float64;
                      closed forms (q = 0, k = 1, identical keys, weights
                      exactly 3/4 and 1/4); sum of weights; convexity;
                      torch.logsumexp for the LSE; the worked example
  merge               split invariance against the unsplit result
  whole step          r = d, k = T equals dense attention
  group selection     brute-force sums over the heads of each group; one
                      head per group is the per-head path; identical heads
                      keep the per-head set; group attention equals per-head
                      attention on the broadcast set
  block selection     brute-force block maxima of the positive parts, short
                      last block; bs = 1 is top-k of the clamped scores;
                      blocks' tokens contiguous and clipped; the step equals
                      attention over the blocks' tokens
  hierarchical top-k  the hand-derived worked example (tests/golden/
                      hier_worked.json, odd lengths included); k = T and
                      scores falling with position and constant scores
                      give the exact top-k
  calibration         brute-force mean over (query, token) pairs; the
                      query-head -> KV-head map on marked KV heads; ties to
                      the lower channel; channel-permutation equivariance;
                      recovery of the generator's seeded outlier channels
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

import dsgen

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _bits(x):
    return dsgen.bf16_bits_from_f32(np.asarray(x, dtype=np.float32))


def _rand_bits(rng, shape, scale=1.0):
    return _bits(rng.standard_normal(shape) * scale)


def _f(bits):
    """Decode bf16 bits here, independently of the oracle's decoder."""
    out = np.empty(np.shape(bits), np.float64)
    flat = np.asarray(bits, np.uint16).reshape(-1)
    o = out.reshape(-1)
    for i, b in enumerate(flat):
        sign = -1.0 if b & 0x8000 else 1.0
        e = (int(b) >> 7) & 0xFF
        m = int(b) & 0x7F
        if e == 0:
            o[i] = sign * m * 2.0 ** -133
        elif e == 0xFF:
            o[i] = sign * math.inf if m == 0 else math.nan
        else:
            o[i] = sign * (1 + m / 128.0) * 2.0 ** (e - 127)
    return out


def _load(name):
    with open(os.path.join(GOLDEN, name)) as fh:
        return json.load(fh)


def _num(x):
    return {"ln2": math.log(2.0), "ln7": math.log(7.0)}.get(x, None) if isinstance(x, str) \
        and x.startswith("ln") else float(x)


# ---------------------------------------------------------------------------

def pin_bf16(orc):
    cases = {0x3F80: 1.0, 0xC000: -2.0, 0x3E80: 0.25, 0x4049: 3.140625, 0x0000: 0.0,
             0x0001: 2.0 ** -133, 0x7F7F: 3.3895313892515355e38, 0x7F80: math.inf,
             0xFF80: -math.inf, 0xBF00: -0.5}
    got = orc.bf16_to_f64(np.array(list(cases), np.uint16))
    assert np.array_equal(got, np.array(list(cases.values()))), got
    neg0 = orc.bf16_to_f64(np.array([0x8000], np.uint16))[0]
    assert neg0 == 0.0 and math.copysign(1.0, neg0) < 0
    rng = np.random.default_rng(1)
    b = _rand_bits(rng, (257,), 5.0)
    assert np.array_equal(orc.bf16_to_f64(b), _f(b))


def pin_label(orc):
    rng = np.random.default_rng(2)
    T, d = 9, 16
    K = _rand_bits(rng, (T, d))
    assert np.array_equal(orc.label_head(K, np.arange(d)), K)
    perm = rng.permutation(d)[:5]
    lab = orc.label_head(K, np.sort(perm))
    for t in range(T):
        for j, c in enumerate(np.sort(perm)):
            assert lab[t, j] == K[t, c]
    # grouped KV heads: query heads 0,1 -> KV 0; 2,3 -> KV 1; 4,5 -> KV 2
    B, Hq, Hkv = 2, 6, 3
    KK = np.empty((B, Hkv, T, d), np.uint16)
    for b in range(B):
        for g in range(Hkv):
            KK[b, g] = _bits(np.full((T, d), 10 * b + g + 1))
    C = np.tile(np.arange(3, dtype=np.int32), (Hq, 1))
    L = orc.label(KK, C, Hq)
    for b in range(B):
        for h in range(Hq):
            assert np.all(_f(L[b, h]) == 10 * b + h // 2 + 1), (b, h)


def pin_score(orc):
    rng = np.random.default_rng(3)
    T, d, r = 11, 8, 3
    K = _rand_bits(rng, (T, d), 3.0)
    C = np.array([1, 4, 6], np.int32)
    lab = orc.label_head(K, C)
    # one-hot queries pick out one label column exactly
    for j, c in enumerate(C):
        q = np.zeros(d, np.float32)
        q[c] = 1.0
        assert np.array_equal(orc.score_head(_bits(q), C, lab), _f(lab[:, j]))
    # a unit on a non-label channel contributes nothing
    q = np.zeros(d, np.float32)
    q[0] = 1.0
    assert np.all(orc.score_head(_bits(q), C, lab) == 0.0)
    # brute-force dot products over the label channels
    q = _rand_bits(rng, (d,), 2.0)
    s = orc.score_head(q, C, lab)
    qf, Kf = _f(q), _f(K)
    for t in range(T):
        ref = sum(qf[c] * Kf[t, c] for c in C)
        assert abs(s[t] - ref) <= 1e-12 * (1 + abs(ref))
    # at r = d the score is the attention logit divided by its scale
    Cfull = np.arange(d, dtype=np.int32)
    sfull = orc.score_head(q, Cfull, orc.label_head(K, Cfull))
    scale = 0.37
    _, lse, w = orc.attend_head(q, K, K, np.arange(T), scale)
    assert np.allclose(np.log(w), scale * sfull - lse, atol=1e-10)


def _check_topk_characterisation(s, k, idx):
    T = len(s)
    idx = list(map(int, idx))
    assert len(idx) == k and len(set(idx)) == k
    assert idx == sorted(idx) and all(0 <= i < T for i in idx)
    sel = set(idx)
    for i in sel:
        for j in range(T):
            if j in sel:
                continue
            assert s[i] > s[j] or (s[i] == s[j] and i < j), (i, j, s[i], s[j])


def pin_topk(orc):
    rng = np.random.default_rng(4)
    for T in (1, 2, 7, 33, 64):
        for _ in range(4):
            s = rng.integers(-3, 4, T).astype(np.float64)  # many ties
            s[rng.random(T) < 0.1] = -0.0
            if T > 3:
                s[rng.integers(0, T)] = math.inf
                s[rng.integers(0, T)] = -math.inf
            for k in sorted({1, max(1, T // 3), T}):
                idx = orc.topk_head(s, k)
                _check_topk_characterisation(s, k, idx)
                ref = sorted(sorted(range(T), key=lambda t: (-s[t], t))[:k])
                assert list(idx) == ref
    # all-equal scores keep the first k tokens
    assert list(orc.topk_head(np.full(50, 2.5), 7)) == list(range(7))
    # +0 and -0 tie, so the lower index wins either way round
    assert list(orc.topk_head(np.array([0.0, -0.0]), 1)) == [0]
    assert list(orc.topk_head(np.array([-0.0, 0.0]), 1)) == [0]
    g = _load("topk_worked.json")
    s = np.array([float(x) for x in g["scores"]])
    for k, exp in g["expected"].items():
        assert list(orc.topk_head(s, int(k))) == exp, (k, exp)
    # batched wrapper keeps the leading shape and matches per-row calls
    S = rng.standard_normal((2, 3, 40))
    I = orc.topk(S, 5)
    assert I.shape == (2, 3, 5)
    for a in range(2):
        for b in range(3):
            assert np.array_equal(I[a, b], orc.topk_head(S[a, b], 5))


def _sdpa(q, Kr, Vr, scale):
    qt = torch.from_numpy(q)[None, None, None, :]
    Kt = torch.from_numpy(Kr)[None, None]
    Vt = torch.from_numpy(Vr)[None, None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, scale=scale)
    return o[0, 0, 0].numpy()


def pin_attend(orc):
    rng = np.random.default_rng(5)
    T, d = 40, 16
    q = _rand_bits(rng, (d,), 1.5)
    K = _rand_bits(rng, (T, d), 1.5)
    V = _rand_bits(rng, (T, d))
    idx = np.sort(rng.choice(T, 13, replace=False))
    scale = 1 / math.sqrt(d)
    o, lse, w = orc.attend_head(q, K, V, idx, scale)
    ref = _sdpa(_f(q), _f(K)[idx], _f(V)[idx], scale)
    assert np.allclose(o, ref, atol=1e-12, rtol=1e-12)
    logits = torch.from_numpy(_f(K)[idx] @ _f(q)) * scale
    assert abs(lse - torch.logsumexp(logits, 0).item()) < 1e-12
    assert abs(w.sum() - 1.0) < 1e-12 and np.all(w >= 0)
    Vr = _f(V)[idx]
    assert np.all(o >= Vr.min(0) - 1e-12) and np.all(o <= Vr.max(0) + 1e-12)
    # order of the selected rows does not matter
    o2, lse2, _ = orc.attend_head(q, K, V, idx[::-1].copy(), scale)
    assert np.allclose(o, o2, atol=1e-13) and abs(lse - lse2) < 1e-12
    # q = 0: plain mean of the selected V rows; lse = log k
    o0, lse0, _ = orc.attend_head(np.zeros(d, np.uint16), K, V, idx, scale)
    assert np.allclose(o0, Vr.mean(0), atol=1e-13)
    assert abs(lse0 - math.log(len(idx))) < 1e-12
    # k = 1: that row of V exactly, lse = its logit
    o1, lse1, _ = orc.attend_head(q, K, V, idx[:1], scale)
    assert np.array_equal(o1, Vr[0])
    assert abs(lse1 - scale * float(_f(K)[idx[0]] @ _f(q))) < 1e-12
    # identical keys: the mean of V whatever q is
    Ksame = np.tile(K[:1], (T, 1))
    os_, _, _ = orc.attend_head(q, Ksame, V, idx, scale)
    assert np.allclose(os_, Vr.mean(0), atol=1e-12)
    # two tokens, logit gap ln 3: weights exactly 3/4 and 1/4
    e0 = np.zeros(d, np.float32)
    e0[2] = 1.0
    K2 = _bits(np.stack([2.0 * e0, np.zeros(d, np.float32)]))
    V2 = _bits(np.stack([np.full(d, 4.0, np.float32), np.zeros(d, np.float32)]))
    o3, _, w3 = orc.attend_head(_bits(e0), K2, V2, np.array([0, 1]), math.log(3.0) / 2.0)
    assert np.allclose(w3, [0.75, 0.25], atol=1e-15)
    assert np.allclose(o3, 3.0, atol=1e-14)
    # the hand-derived worked example
    g = _load("attend_worked.json")
    og, lg, _ = orc.attend_head(_bits(g["q"]), _bits(g["K"]), _bits(g["V"]),
                                np.array(g["idx"]), _num(g["scale"]))
    assert np.allclose(og, g["o"], atol=1e-14) and abs(lg - _num(g["lse"])) < 1e-14


def pin_merge(orc):
    rng = np.random.default_rng(6)
    T, d = 90, 16
    q = _rand_bits(rng, (d,), 2.0)
    K = _rand_bits(rng, (T, d), 2.0)
    V = _rand_bits(rng, (T, d))
    idx = np.sort(rng.choice(T, 61, replace=False))
    o, lse, _ = orc.attend_head(q, K, V, idx, 0.3)
    for n in (1, 2, 3, 7, 61):
        om, lm = orc.attend_split_head(q, K, V, idx, 0.3, n)
        assert np.allclose(om, o, atol=1e-12) and abs(lm - lse) < 1e-12, n
    # a single part merges to itself
    om, lm = orc.lse_merge([o], [lse])
    assert np.allclose(om, o, atol=1e-15) and abs(lm - lse) < 1e-15


def pin_dense(orc):
    rng = np.random.default_rng(7)
    B, Hq, Hkv, T, d = 2, 4, 2, 24, 16
    Q = _rand_bits(rng, (B, Hq, d), 2.0)
    K = _rand_bits(rng, (B, Hkv, T, d), 2.0)
    V = _rand_bits(rng, (B, Hkv, T, d))
    O, L = orc.dense(Q, K, V, 0.25)
    for b in range(B):
        for h in range(Hq):
            g = h // 2
            ref = _sdpa(_f(Q[b, h]), _f(K[b, g]), _f(V[b, g]), 0.25)
            assert np.allclose(O[b, h], ref, atol=1e-12), (b, h)
            lg = torch.logsumexp(torch.from_numpy(_f(K[b, g]) @ _f(Q[b, h])) * 0.25, 0)
            assert abs(L[b, h] - lg.item()) < 1e-12


def pin_full_channels_all_tokens(orc):
    """r = d and k = T: the sparse step is dense attention."""
    rng = np.random.default_rng(8)
    B, Hq, Hkv, T, d = 1, 4, 4, 50, 16
    Q = _rand_bits(rng, (B, Hq, d), 2.0)
    K = _rand_bits(rng, (B, Hkv, T, d), 2.0)
    V = _rand_bits(rng, (B, Hkv, T, d))
    C = np.tile(np.arange(d, dtype=np.int32), (Hq, 1))
    st = orc.sparse_step(Q, K, V, C, T, 0.25)
    O, L = orc.dense(Q, K, V, 0.25)
    assert np.array_equal(st["idx"], np.broadcast_to(np.arange(T), (B, Hq, T)))
    assert np.allclose(st["O"], O, atol=1e-13) and np.allclose(st["lse"], L, atol=1e-13)


def pin_worked_score(orc):
    g = _load("score_worked.json")
    K, q, C = _bits(g["K"]), _bits(g["q"]), np.array(g["C"], np.int32)
    lab = orc.label_head(K, C)
    assert np.array_equal(lab, _bits(g["label"]))
    s = orc.score_head(q, C, lab)
    assert np.array_equal(s, np.array(g["scores"], np.float64))
    assert list(orc.topk_head(s, 2)) == g["top2"]
    assert list(orc.topk_head(s, 1)) == g["top1"]


def pin_f32_rounding(orc):
    # nearest-even: 1 + 2^-24 is a tie between 1 and 1 + 2^-23 and goes to 1
    x = np.array([1.0 + 2.0 ** -24, 1.0 + 3 * 2.0 ** -24, -1.0 - 2.0 ** -25, 2.0 ** 130])
    with np.errstate(over="ignore"):
        got = orc.to_f32(x)
    assert got.dtype == np.float32
    assert got[0] == np.float32(1.0)
    assert got[1] == np.float32(1.0 + 2.0 ** -22)
    assert got[2] == np.float32(-1.0)
    assert np.isinf(got[3])


# ---------------------------------------------------------------------------
# offline channel calibration

def pin_calib_bruteforce(orc):
    rng = np.random.default_rng(41)
    B, Hq, Hkv, Nq, T, Tcap, d = 2, 4, 2, 3, 5, 7, 8
    Qc = _rand_bits(rng, (B, Hq, Nq, d), 2.0)
    K = _rand_bits(rng, (B, Hkv, Tcap, d), 1.5)
    I = orc.calibrate_importance(Qc, K, T, Hq)
    qf, kf = _f(Qc), _f(K)
    for h in range(Hq):
        g = h // (Hq // Hkv)
        for c in range(d):
            tot = 0.0
            for b in range(B):
                for n in range(Nq):
                    for t in range(T):
                        tot += abs(qf[b, h, n, c] * kf[b, g, t, c])
            ref = tot / (B * Nq * T)
            assert abs(I[h, c] - ref) <= 1e-12 * (1 + ref), (h, c, I[h, c], ref)


def pin_calib_groups_and_order(orc):
    # KV head g is large only on channel 5 + g: query head h picks 5 + g(h)
    B, Hq, Hkv, Nq, T, d = 1, 6, 3, 2, 4, 16
    Qc = _bits(np.ones((B, Hq, Nq, d)))
    K = np.empty((B, Hkv, T, d), np.uint16)
    for g in range(Hkv):
        x = np.full((T, d), 0.5)
        x[:, 5 + g] = -4.0  # magnitude counts, not sign
        K[0, g] = _bits(x)
    C, I = orc.calibrate(Qc, K, T, Hq, 1)
    for h in range(Hq):
        assert C[h, 0] == 5 + h // 2, (h, C[h])
        assert I[h, 5 + h // 2] == 4.0 and I[h, 0] == 0.5
    # r = 3: the large channel plus ties at 0.5 broken toward the lowest channels
    C3, _ = orc.calibrate(Qc, K, T, Hq, 3)
    for h in range(Hq):
        assert list(C3[h]) == [0, 1, 5 + h // 2], (h, C3[h])
    # all equal: channels 0..r-1, ascending
    Ce, _ = orc.calibrate(Qc, _bits(np.ones((B, Hkv, T, d))), T, Hq, 4)
    assert np.array_equal(Ce, np.tile(np.arange(4, dtype=np.int32), (Hq, 1)))
    # explicit selection order: descending importance, ascending output
    Isel = np.array([[0.1, 3.0, 2.0, 3.0, -1.0, 2.5]])
    assert list(orc.calibrate_select(Isel, 3)[0]) == [1, 3, 5]
    assert list(orc.calibrate_select(Isel, 4)[0]) == [1, 2, 3, 5]


def pin_calib_permutation(orc):
    rng = np.random.default_rng(43)
    B, Hq, Hkv, Nq, T, d = 2, 2, 1, 4, 9, 12
    Qc = _rand_bits(rng, (B, Hq, Nq, d))
    K = _rand_bits(rng, (B, Hkv, T, d))
    perm = rng.permutation(d)
    I = orc.calibrate_importance(Qc, K, T, Hq)
    Ip = orc.calibrate_importance(Qc[..., perm], K[..., perm], T, Hq)
    assert np.allclose(Ip, I[:, perm], rtol=1e-13, atol=0)
    # tokens past T are ignored
    K2 = K.copy()
    K2[:, :, T - 1] = _bits(np.full(d, 100.0))
    assert not np.allclose(orc.calibrate_importance(Qc, K2, T, Hq), I)
    assert np.allclose(orc.calibrate_importance(Qc, K2, T - 1, Hq),
                       orc.calibrate_importance(Qc, K, T - 1, Hq))


def pin_calib_recovers_outliers(orc):
    # generator property: Q and K are scaled x6 on each head's n_out outlier
    # channels, so those channels carry the largest |q_c k_c|
    w = dsgen.Workload("calib-pin", B=2, Hq=4, Hkv=2, T=256, r=8, k=16, n_out=8, seed=0xCA11)
    _, K, _ = dsgen.qkv(w, want=("K",))
    Qc = dsgen.q_calib(w, 16)
    C, _ = orc.calibrate(Qc, K, w.T, w.Hq, w.n_out)
    for h in range(w.Hq):
        assert np.array_equal(C[h], dsgen.outliers(w, h)), (h, C[h], dsgen.outliers(w, h))


# ---------------------------------------------------------------------------
# group-shared selection

def pin_group_score(orc):
    rng = np.random.default_rng(51)
    B, Hq, Hkv, T = 2, 6, 2, 7
    s = rng.standard_normal((B, Hq, T))
    sg = orc.group_score(s, Hkv)
    for b in range(B):
        for g in range(Hkv):
            for t in range(T):
                ref = s[b, 3 * g, t] + s[b, 3 * g + 1, t] + s[b, 3 * g + 2, t]
                assert sg[b, g, t] == ref  # same addition order, exact
    # float32 input is summed in float32 (round after each addition)
    s32 = np.array([[[1.0], [2.0 ** -24], [2.0 ** -24]]], np.float32)
    assert orc.group_score(s32, 1)[0, 0, 0] == np.float32(1.0)
    # one head per group: the per-head scores unchanged
    assert np.array_equal(orc.group_score(s, Hq), s)


def pin_group_step(orc):
    rng = np.random.default_rng(52)
    B, Hkv, G, T, d, r, k = 1, 2, 3, 40, 16, 4, 6
    Hq = Hkv * G
    Q = _rand_bits(rng, (B, Hq, d))
    K = _rand_bits(rng, (B, Hkv, T, d))
    V = _rand_bits(rng, (B, Hkv, T, d))
    C = np.sort(np.stack([rng.permutation(d)[:r] for _ in range(Hq)]), axis=1).astype(np.int32)
    scale = 0.25
    res = orc.group_sparse_step(Q, K, V, C, k, scale)
    # brute force: group scores from explicit dot products, then a full sort
    qf, kf = _f(Q), _f(K)
    for g in range(Hkv):
        sg = [sum(sum(qf[0, h, c] * kf[0, g, t, c] for c in C[h]) for h in range(g * G, g * G + G))
              for t in range(T)]
        assert np.allclose(res["sg64"][0, g], sg, rtol=1e-12, atol=1e-12)
        order = sorted(range(T), key=lambda t: (-float(res["sg32"][0, g, t]), t))[:k]
        assert list(res["idx"][0, g]) == sorted(order)
        # every head of the group attends over the group's set
        for h in range(g * G, g * G + G):
            o, lse, _ = orc.attend_head(Q[0, h], K[0, g], V[0, g], res["idx"][0, g], scale)
            assert np.allclose(res["O"][0, h], o) and abs(res["lse"][0, h] - lse) < 1e-12
    # one query head per KV head: the per-head step
    Q1, C1 = Q[:, :Hkv], C[:Hkv]
    one = orc.group_sparse_step(Q1, K, V, C1, k, scale)
    per = orc.sparse_step(Q1, K, V, C1, k, scale)
    assert np.array_equal(one["idx"], per["idx"]) and np.allclose(one["O"], per["O"])
    # G identical heads: the group keeps the single head's set
    Qr = np.repeat(Q1, G, axis=1)
    Cr = np.repeat(C1, G, axis=0)
    rep = orc.group_sparse_step(Qr, K, V, Cr, k, scale)
    sg64 = rep["sg64"]
    for g in range(Hkv):
        want = sorted(sorted(range(T), key=lambda t: (-per["s64"][0, g, t], t))[:k])
        got = list(rep["idx"][0, g])
        # equal up to float32 near-ties of the single head's scores
        if got != want:
            kth = np.sort(sg64[0, g])[::-1][k - 1]
            assert all(sg64[0, g, t] >= kth - 1e-6 * (abs(kth) + 1) for t in got)


# ---------------------------------------------------------------------------
# block-granular selection

def pin_block_score(orc):
    s = np.array([[-1.0, 3.0, -2.0, 0.5, -0.25, -4.0, 7.0, -1.0, 2.0, -3.0]])
    # bs = 4: blocks [-1,3,-2,.5] [-.25,-4,7,-1] [2,-3] (short); negative-only block -> 0
    assert np.array_equal(orc.block_score(s, 4), [[3.0, 7.0, 2.0]])
    assert np.array_equal(orc.block_score(np.array([[-1.0, -2.0, -0.5]]), 2), [[0.0, 0.0]])
    rng = np.random.default_rng(61)
    x = rng.standard_normal((3, 37))
    for bs in (1, 2, 5, 8, 37, 64):
        got = orc.block_score(x, bs)
        for i in range(3):
            ref = [max(0.0, max(x[i, j:j + bs])) for j in range(0, 37, bs)]
            assert list(got[i]) == ref, (bs, i)
    # bs = 1: the positive-clamped scores themselves
    assert np.array_equal(orc.block_score(x, 1), np.maximum(x, 0))


def pin_block_tokens_and_step(orc):
    assert list(orc.block_tokens(np.array([2, 0]), 4, 10)) == [0, 1, 2, 3, 8, 9]
    assert list(orc.block_tokens(np.array([1]), 3, 5)) == [3, 4]
    rng = np.random.default_rng(62)
    B, Hq, Hkv, T, d, r = 1, 2, 1, 50, 16, 4
    Q = _rand_bits(rng, (B, Hq, d))
    K = _rand_bits(rng, (B, Hkv, T, d))
    V = _rand_bits(rng, (B, Hkv, T, d))
    C = np.sort(np.stack([rng.permutation(d)[:r] for _ in range(Hq)]), axis=1).astype(np.int32)
    scale = 0.3
    bs, kb = 8, 3
    res = orc.block_sparse_step(Q, K, V, C, bs, kb, scale)
    qf, kf = _f(Q), _f(K)
    for h in range(Hq):
        s = [np.float32(sum(qf[0, h, c] * kf[0, 0, t, c] for c in C[h])) for t in range(T)]
        blocks = [max(0.0, max(float(v) for v in s[j:j + bs])) for j in range(0, T, bs)]
        order = sorted(range(len(blocks)), key=lambda j: (-blocks[j], j))[:kb]
        assert list(res["bidx"][0, h]) == sorted(order)
        toks = [t for j in sorted(order) for t in range(j * bs, min(j * bs + bs, T))]
        o, lse, _ = orc.attend_head(Q[0, h], K[0, 0], V[0, 0], np.array(toks), scale)
        assert np.allclose(res["O"][0, h], o) and abs(res["lse"][0, h] - lse) < 1e-12
    # bs = 1 selects the top-k of the positive-clamped float32 scores
    one = orc.block_sparse_step(Q, K, V, C, 1, 5, scale)
    assert np.array_equal(one["bidx"], orc.topk(np.maximum(one["s32"], 0), 5))


# ---------------------------------------------------------------------------
# hierarchical top-k

def pin_hier_topk(orc):
    g = _load("hier_worked.json")
    s = np.array(g["scores"])
    for k, want in g["expected"].items():
        assert list(orc.hier_topk_head(s, int(k))) == want, (k, orc.hier_topk_head(s, int(k)))
    for case in ("odd", "uneven"):
        assert list(orc.hier_topk_head(np.array(g[case]["scores"]), g[case]["k"])) == \
            g[case]["expected"], case
    rng = np.random.default_rng(71)
    for T, k in [(1, 1), (13, 13), (64, 5), (100, 7), (257, 16)]:
        x = rng.standard_normal(T)
        # exhaustive search (k = T): every token
        if k == T:
            assert list(orc.hier_topk_head(x, k)) == list(range(T))
        # scores falling with position: each part's first token is its best
        dec = -np.arange(T, dtype=np.float64) + 0.01 * (T - np.arange(T)) ** 0.5
        assert list(orc.hier_topk_head(dec, k)) == list(range(k))
        # all equal: ties to the lower start narrow onto the first k tokens, the
        # exact top-k's answer too
        assert list(orc.hier_topk_head(np.zeros(T), k)) == list(range(k))
        got = orc.hier_topk_head(x, k)
        assert len(set(got)) == k and all(0 <= t < T for t in got) and list(got) == sorted(got)


# the pins of steps O1-O5 and the merge: also run against the C++ oracle
CORE_PINS = [pin_bf16, pin_label, pin_score, pin_topk, pin_attend, pin_merge, pin_dense,
             pin_full_channels_all_tokens, pin_worked_score, pin_f32_rounding]

PINS = [pin_bf16, pin_label, pin_score, pin_topk, pin_attend, pin_merge, pin_dense,
        pin_full_channels_all_tokens, pin_worked_score, pin_f32_rounding,
        pin_calib_bruteforce, pin_calib_groups_and_order, pin_calib_permutation,
        pin_calib_recovers_outliers, pin_group_score, pin_group_step, pin_block_score,
        pin_block_tokens_and_step, pin_hier_topk]
