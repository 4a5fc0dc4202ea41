"""The C++ oracle (oracle/ds_oracle.cpp), no GPU needed.

1. Every pin of the numpy oracle, run against the C++ one: bf16 decoding,
   label gather, score, top-k order and worked examples, attention against
   torch's scaled_dot_product_attention and closed forms, merge invariance,
   dense, r = d with k = T; calibration, group-shared, block and hierarchical
   selection.
2. Planted slips in a copy of the C++ source (compiled into a temporary
   directory): each must make at least one pin fail.
3. Agreement with the numpy oracle on seeded workloads (MHA and grouped KV
   heads, tie-heavy scores): the two implementations share no code.
"""
import importlib.util
import os
import shutil

import numpy as np
import pytest

import dsgen
import oracle
import oracle.cxx as cxx
from tests import pins


@pytest.mark.parametrize("pin", pins.PINS, ids=lambda p: p.__name__)
def test_cxx_pin(pin):
    pin(cxx)


# (name, original text, mutated text) in ds_oracle.cpp
MUTATIONS = [
    ("bf16 shift", "static_cast<uint32_t>(bits) << 16", "static_cast<uint32_t>(bits) << 15"),
    ("label without the gather", "Kbg[static_cast<int64_t>(t) * d + C[h * r + j]]",
     "Kbg[static_cast<int64_t>(t) * d + j]"),
    ("query head to KV head map", "(static_cast<int64_t>(b) * Hkv + h / G) * T * d;\n      uint16_t*",
     "(static_cast<int64_t>(b) * Hkv + h % Hkv) * T * d;\n      uint16_t*"),
    ("score uses leading channels of q", "bf16_value(q[C[h * r + j]])", "bf16_value(q[j])"),
    ("top-k smallest", "return s[a] > s[b];", "return s[a] < s[b];"),
    ("ties to the higher index", "    return a < b;\n  });", "    return a > b;\n  });"),
    ("top-k not ascending", "  std::sort(order.begin(), order.begin() + k);\n", ""),
    ("scale dropped", "l[i] = scale * dot;", "l[i] = dot;"),
    ("softmax sign", "l[i] = std::exp(l[i] - m);", "l[i] = std::exp(m - l[i]);"),
    ("softmax not normalised", "const double wi = l[i] / z;", "const double wi = l[i];"),
    ("lse without max", "*lse = m + std::log(z);", "*lse = std::log(z);"),
    ("V rows misaligned with K rows", "V + static_cast<int64_t>(idx[i]) * d",
     "V + static_cast<int64_t>(idx[(i + 1) % n]) * d"),
    ("merge weights inverted", "const double a = std::exp(lses[i] - M);",
     "const double a = std::exp(M - lses[i]);"),
    ("dense drops the last token", "all[i] = static_cast<int32_t>(i % T);",
     "all[i] = static_cast<int32_t>(std::min<size_t>(i % T, T - 2));"),
    ("f32 rounding dropped", "out[i] = static_cast<float>(in[i]);",
     "out[i] = static_cast<float>(in[i] * (1.0 + 1e-7));"),
    ("calibration without magnitudes", "acc += std::fabs(bf16_value(K[row * d + c]));",
     "acc += bf16_value(K[row * d + c]);"),
    ("calibration reads past T", "for (int t = 0; t < T; ++t) {\n          const int64_t row",
     "for (int t = 0; t < T_cap; ++t) {\n          const int64_t row"),
    ("calibration sums q and k", "I[h * d + c] += qsum[c] * kg[c];",
     "I[h * d + c] += qsum[c] + kg[c];"),
    ("calibration ignores importance", "dso_topk_f64(I, Hq, d, r, C);",
     "for (int i = 0; i < Hq * r; ++i) C[i] = i % r;"),
    ("group score in the wrong group", "sg[(static_cast<int64_t>(b) * Hkv + h / G) * T + t] +=",
     "sg[(static_cast<int64_t>(b) * Hkv + h % Hkv) * T + t] +="),
    ("group attention on the wrong group",
     "const int64_t bg = static_cast<int64_t>(b) * Hkv + h / G;",
     "const int64_t bg = static_cast<int64_t>(b) * Hkv + h % Hkv;"),
    ("block score keeps negatives", "      S m = 0;\n", "      S m = s[i * T + j * bs];\n"),
    ("block tokens off by one", "for (int t = j * bs; t < std::min((j + 1) * bs, T); ++t) out",
     "for (int t = j * bs + 1; t < std::min((j + 1) * bs, T); ++t) out"),
    ("hierarchy halves the other way", "const int m = p.first + (p.second - p.first + 1) / 2;",
     "const int m = p.first + (p.second - p.first) / 2;"),
    ("hierarchy ties to the higher start", "return a.first < b.first;",
     "return a.first > b.first;"),
    ("hierarchy keeps the worst parts", "return s[a.first] > s[b.first];",
     "return s[a.first] < s[b.first];"),
    ("hierarchy scores parts by their last token",
     "if (s[a.first] != s[b.first]) return s[a.first] > s[b.first];",
     "if (s[a.second - 1] != s[b.second - 1]) return s[a.second - 1] > s[b.second - 1];"),
]


def _variant(tmp_path, name, old, new):
    src = open(cxx._SRC).read()
    assert src.count(old) >= 1, name
    d = tmp_path / name.replace(" ", "_")
    d.mkdir()
    (d / "ds_oracle.cpp").write_text(src.replace(old, new, 1))
    shutil.copy(os.path.join(os.path.dirname(cxx.__file__), "cxx.py"), d / "cxx.py")
    spec = importlib.util.spec_from_file_location(f"cxx_mut_{len(os.listdir(tmp_path))}",
                                                  d / "cxx.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("mut", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_cxx_pins_catch_planted_slip(tmp_path, mut):
    mod = _variant(tmp_path, *mut)
    failed = []
    for pin in pins.PINS:
        try:
            with np.errstate(all="ignore"):
                pin(mod)
        except Exception:  # noqa: BLE001  (an assertion, or a bad value further on)
            failed.append(pin.__name__)
    assert failed, f"no pin caught: {mut[0]}"


@pytest.mark.parametrize("shape", [(2, 4, 4, 300, 16, 20), (2, 8, 2, 257, 8, 33),
                                   (1, 4, 1, 64, 32, 64)])
def test_cxx_agrees_with_numpy_oracle(shape):
    B, Hq, Hkv, T, r, k = shape
    w = dsgen.Workload("cross", B=B, Hq=Hq, Hkv=Hkv, T=T, r=r, k=k, n_out=min(8, r),
                       seed=0xC0DE + T)
    Q, K, V = dsgen.qkv(w)
    C = dsgen.channels(w, r)
    a = oracle.sparse_step(Q, K, V, C, k, w.scale)
    b = cxx.sparse_step(Q, K, V, C, k, w.scale)
    assert np.array_equal(a["label"], b["label"])
    assert np.allclose(a["s64"], b["s64"], rtol=1e-13, atol=1e-12)
    # the two fp32 roundings agree wherever the fp64 scores do to the last bit
    same = a["s64"] == b["s64"]
    assert np.array_equal(a["s32"][same], b["s32"][same])
    assert np.array_equal(oracle.topk(b["s32"], k), b["idx"])
    assert np.allclose(a["O"], b["O"], atol=1e-12) and np.allclose(a["lse"], b["lse"], atol=1e-12)
    Od, Ld = cxx.dense(Q, K, V, w.scale)
    Odn, Ldn = oracle.dense(Q, K, V, w.scale)
    assert np.allclose(Od, Odn, atol=1e-12) and np.allclose(Ld, Ldn, atol=1e-12)


def test_cxx_topk_on_ties_agrees_with_numpy_oracle():
    rng = np.random.default_rng(11)
    for T in (1, 5, 64, 1000):
        s = rng.integers(-2, 3, (3, T)).astype(np.float32)
        s[rng.random((3, T)) < 0.2] = -0.0
        for k in sorted({1, max(1, T // 7), T}):
            assert np.array_equal(cxx.topk(s, k), oracle.topk(s, k))
            assert np.array_equal(cxx.topk(s.astype(np.float64), k),
                                  oracle.topk(s.astype(np.float64), k))


def test_cxx_rows_beside_the_path_agree_with_numpy_oracle():
    w = dsgen.Workload("cross-next", B=2, Hq=8, Hkv=2, T=300, r=16, k=24, n_out=8,
                       seed=0xC0DF)
    Q, K, V = dsgen.qkv(w)
    C = dsgen.channels(w, 16)
    Qc = dsgen.q_calib(w, 5)
    Ca, Ia = oracle.calibrate(Qc, K, 290, w.Hq, 8)
    Cb, Ib = cxx.calibrate(Qc, K, 290, w.Hq, 8)
    assert np.array_equal(Ca, Cb) and np.allclose(Ia, Ib, rtol=1e-13, atol=0)
    a = oracle.group_sparse_step(Q, K, V, C, w.k, w.scale)
    b = cxx.group_sparse_step(Q, K, V, C, w.k, w.scale)
    assert np.array_equal(a["sg32"], b["sg32"]) and np.array_equal(a["idx"], b["idx"])
    assert np.allclose(a["sg64"], b["sg64"], rtol=1e-13, atol=1e-12)
    assert np.allclose(a["O"], b["O"], atol=1e-12) and np.allclose(a["lse"], b["lse"], atol=1e-12)
    for bs, kb in ((64, 2), (7, 5), (1, 9)):
        a = oracle.block_sparse_step(Q, K, V, C, bs, kb, w.scale)
        b = cxx.block_sparse_step(Q, K, V, C, bs, kb, w.scale)
        assert np.array_equal(a["sb"], b["sb"]) and np.array_equal(a["bidx"], b["bidx"])
        assert np.allclose(a["O"], b["O"], atol=1e-12)
    s32 = cxx.sparse_step(Q, K, V, C, w.k, w.scale)["s32"]
    for k in (1, 5, 24, 300):
        assert np.array_equal(oracle.hier_topk(s32, k), cxx.hier_topk(s32, k))


def test_threaded_step_equals_the_per_head_oracle():
    """The C++ oracle's multi-threaded driver (the CPU baseline) gives, head by
    head, the numpy oracle's sparse step and dense attention."""
    import dsgen
    w = dsgen.Workload("mt", B=2, Hq=6, Hkv=2, T=700, r=8, k=37, n_out=8, seed=321)
    Q, K, V = dsgen.qkv(w)
    C = dsgen.channels(w)
    heads = [(b, h) for b in range(w.B) for h in range(w.Hq)]
    Qs = np.stack([Q[b, h] for b, h in heads])
    Ks = np.stack([K[b, h // w.G] for b, h in heads])
    Vs = np.stack([V[b, h // w.G] for b, h in heads])
    Cs = np.stack([C[h] for _, h in heads])
    Ls = np.stack([oracle.label_head(Ks[i], Cs[i]) for i in range(len(heads))])
    O, L, Od, Ld, used = cxx.step_heads_mt(Qs, Cs, Ls, Ks, Vs, w.k, w.scale, dense=True,
                                           nthreads=3)
    assert used == 3
    for i in range(len(heads)):
        s = oracle.to_f32(oracle.score_head(Qs[i], Cs[i], Ls[i]))
        o, l, _ = oracle.attend_head(Qs[i], Ks[i], Vs[i], oracle.topk_head(s, w.k), w.scale)
        assert np.abs(O[i] - o).max() <= 1e-12 and abs(L[i] - l) <= 1e-12
        od, ld, _ = oracle.attend_head(Qs[i], Ks[i], Vs[i], np.arange(w.T), w.scale)
        assert np.abs(Od[i] - od).max() <= 1e-12 and abs(Ld[i] - ld) <= 1e-12
    # sparse only, all cores
    O2, L2, _, _, used2 = cxx.step_heads_mt(Qs, Cs, Ls, Ks, Vs, w.k, w.scale)
    assert used2 >= 1 and np.array_equal(O2, O) and np.array_equal(L2, L)
