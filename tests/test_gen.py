"""The seeded input generator: determinism, slabs, workload structure."""
import numpy as np
import pytest

import dsgen
import oracle


def _f(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


SMALL = dsgen.Workload("unit-B2-Hq4-Hkv2-T300", B=2, Hq=4, Hkv=2, T=300, r=8, k=20, n_out=8,
                       seed=123)


def test_deterministic_and_seeded():
    a = dsgen.qkv(SMALL)
    b = dsgen.qkv(SMALL, nthreads=1)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    c = dsgen.qkv(SMALL.with_(seed=124))
    assert not np.array_equal(a[1], c[1])


def test_slabs_match_full_tensors():
    Q, K, V = dsgen.qkv(SMALL)
    for b in range(SMALL.B):
        for h in range(SMALL.Hq):
            assert np.array_equal(dsgen.q_slab(SMALL, b, h), Q[b, h])
        for g in range(SMALL.Hkv):
            assert np.array_equal(dsgen.kv_slab(SMALL, "K", b, g), K[b, g])
            assert np.array_equal(dsgen.kv_slab(SMALL, "V", b, g), V[b, g])


def test_channels_are_sorted_prefixes_of_the_permutation():
    for r in (1, 8, 16, 128):
        C = dsgen.channels(SMALL, r)
        assert C.shape == (SMALL.Hq, r)
        for h in range(SMALL.Hq):
            p = dsgen.permutation(SMALL, h)
            assert sorted(p.tolist()) == list(range(SMALL.d))
            assert np.array_equal(C[h], np.sort(p[:r]))


def test_outlier_channels_scaled_by_six():
    w = SMALL.with_(T=4000)
    Q, K, V = dsgen.qkv(w)
    for g in range(w.Hkv):
        out = set()
        for h in range(g * w.G, (g + 1) * w.G):
            out |= set(dsgen.outliers(w, h).tolist())
        Kf = _f(K[:, g]).reshape(-1, w.d)
        sd = Kf.std(0)
        for c in range(w.d):
            want = 6.0 if c in out else 1.0
            assert abs(sd[c] / want - 1.0) < 0.05, (g, c, sd[c])
    Vf = _f(V).reshape(-1, w.d)
    assert abs(Vf.std() - 1.0) < 0.02 and abs(Vf.mean()) < 0.02


def test_heavy_hitters_are_all_selected():
    """Reduced long-context workload: every heavy-hitter token is in the top T/16."""
    w = dsgen.Workload("hh-B1-H4-T16K", B=1, Hq=4, Hkv=4, T=16384, r=8, k=1024, n_out=8,
                       n_hh=round(0.005 * 16384), seed=dsgen.workload("long-B1-H32-T256K").seed)
    Q, K, _ = dsgen.qkv(w, want=("Q", "K"))
    C = dsgen.channels(w)
    pos = dsgen.hh_positions(w)
    assert pos.shape == (w.Hq, w.n_hh)
    lab = oracle.label(K, C, w.Hq)
    s = oracle.score(Q, C, lab)
    idx = oracle.topk(oracle.to_f32(s), w.k)
    for h in range(w.Hq):
        assert len(set(pos[h].tolist())) == w.n_hh
        assert set(pos[h].tolist()) <= set(idx[0, h].tolist()), h
        # the heavy-hitter rows score 6*sqrt(r)*||q_C||
        qc = _f(Q[0, h])[C[h]]
        want = 6 * np.sqrt(w.r) * np.linalg.norm(qc)
        assert np.allclose(s[0, h, pos[h]], want, rtol=2e-2)


def test_bf16_rounding_helper():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0], np.float32)
    bits = dsgen.bf16_bits_from_f32(x)
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to even -> 1
    assert bits.tolist() == [0x3F80, 0x3F80, 0x3F82, 0xC020, 0x0000]


def test_bad_dims_rejected():
    with pytest.raises(ValueError):
        dsgen.qkv(SMALL.with_(Hkv=3))
