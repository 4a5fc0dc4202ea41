"""Plant plausible mistakes in a copy of the oracle and check the pins catch each.

Every mutation edits the oracle's source text in memory (the file on disk is
untouched), loads it as a separate module and runs all pins against it: at
least one pin must fail.  This is the evidence that the pins constrain every
step of the oracle, not just that the oracle agrees with itself.
"""
import importlib.util
import types

import pytest

import oracle.ds_oracle as real
from tests import pins

SRC_PATH = real.__file__

# (name, original text, mutated text)
MUTATIONS = [
    ("bf16 shift", "<< 16).view(np.float32)", "<< 15).view(np.float32)"),
    ("f32 rounding dropped", "np.asarray(x, dtype=np.float64).astype(np.float32)",
     "np.asarray(x, dtype=np.float64)"),
    ("label wrong axis", "np.asarray(K_bg)[:, np.asarray(C_h, dtype=np.int64)]",
     "np.asarray(K_bg)[:, np.arange(len(C_h))]"),
    ("query head to KV head map", "return h // (Hq // Hkv)", "return h % Hkv"),
    ("score uses leading channels of q", "np.asarray(q_h)[np.asarray(C_h, dtype=np.int64)]",
     "np.asarray(q_h)[: len(C_h)]"),
    ("score sign", "return bf16_to_f64(label_h) @ qc", "return -(bf16_to_f64(label_h) @ qc)"),
    ("top-k smallest", "np.lexsort((np.arange(T), -s))", "np.lexsort((np.arange(T), s))"),
    ("ties to higher index", "np.lexsort((np.arange(T), -s))", "np.lexsort((-np.arange(T), -s))"),
    ("top-k not ascending", "return np.sort(order[:k]).astype(np.int32)",
     "return order[:k].astype(np.int32)"),
    ("top-k off by one", "return np.sort(order[:k]).astype(np.int32)",
     "return np.sort(order[1:k + 1]).astype(np.int32)"),
    ("scale dropped", "logits = (Kr @ q) * scale", "logits = (Kr @ q)"),
    ("scale squared", "logits = (Kr @ q) * scale", "logits = (Kr @ q) * scale * scale"),
    ("V gathered from K", "Vr = bf16_to_f64(np.asarray(V_bg)[idx])",
     "Vr = bf16_to_f64(np.asarray(K_bg)[idx])"),
    ("softmax sign", "e = np.exp(logits - m)", "e = np.exp(m - logits)"),
    ("softmax not normalised", "w = e / z", "w = e"),
    ("lse without max", "return w @ Vr, m + math.log(z), w", "return w @ Vr, math.log(z), w"),
    ("V rows misaligned with K rows", "Vr = bf16_to_f64(np.asarray(V_bg)[idx])",
     "Vr = bf16_to_f64(np.asarray(V_bg)[idx[::-1]])"),
    ("merge weights unnormalised", "return (a[:, None] * outs).sum(0) / a.sum(), M + math.log(a.sum())",
     "return (a[:, None] * outs).sum(0), M + math.log(a.sum())"),
    ("merge lse drops max", "return (a[:, None] * outs).sum(0) / a.sum(), M + math.log(a.sum())",
     "return (a[:, None] * outs).sum(0) / a.sum(), math.log(a.sum())"),
    ("dense drops last token", "idx = np.broadcast_to(np.arange(T, dtype=np.int32), (B, Hq, T))",
     "idx = np.broadcast_to(np.arange(T - 1, dtype=np.int32), (B, Hq, T - 1))"),
    ("step selects on float64 scores with wrong k", "idx = topk(s32, k)", "idx = topk(s32, max(1, k - 1))"),
    ("calibration without magnitudes", "qsum = np.abs(bf16_to_f64(Qc[b, h])).sum(axis=0)",
     "qsum = bf16_to_f64(Qc[b, h]).sum(axis=0)"),
    ("calibration keys without magnitudes", "ksum = [np.abs(bf16_to_f64(K[b, g, :T])).sum(axis=0)",
     "ksum = [bf16_to_f64(K[b, g, :T]).sum(axis=0)"),
    ("calibration reads past T", "ksum = [np.abs(bf16_to_f64(K[b, g, :T])).sum(axis=0)",
     "ksum = [np.abs(bf16_to_f64(K[b, g])).sum(axis=0)"),
    ("calibration sums q and k instead of the product", "I[h] += qsum * ksum[group_of(h, Hq, Hkv)]",
     "I[h] += qsum + ksum[group_of(h, Hq, Hkv)]"),
    ("calibration pairs the wrong KV head", "I[h] += qsum * ksum[group_of(h, Hq, Hkv)]",
     "I[h] += qsum * ksum[h % Hkv]"),
    ("calibration mean over the wrong count", "return I / (B * Nq * T)", "return I / (Nq * T)"),
    ("calibration picks the smallest", "order = np.lexsort((np.arange(d), -np.asarray(I[h], np.float64)))",
     "order = np.lexsort((np.arange(d), np.asarray(I[h], np.float64)))"),
    ("calibration ties to the higher channel",
     "order = np.lexsort((np.arange(d), -np.asarray(I[h], np.float64)))",
     "order = np.lexsort((-np.arange(d), -np.asarray(I[h], np.float64)))"),
    ("calibration output unsorted", "C[h] = np.sort(order[:r])", "C[h] = order[:r]"),
    ("group score takes the wrong group", "sg[:, group_of(h, Hq, Hkv)] += s[:, h]",
     "sg[:, h % Hkv] += s[:, h]"),
    ("group score keeps the last head only", "sg[:, group_of(h, Hq, Hkv)] += s[:, h]",
     "sg[:, group_of(h, Hq, Hkv)] = s[:, h]"),
    ("group score in float64 for the float32 pipeline",
     "sg = np.zeros((B, Hkv, T), dtype=s.dtype)", "sg = np.zeros((B, Hkv, T))"),
    ("group attention uses the first group's set", "idx[:, h] = idx_g[:, group_of(h, Hq, Hkv)]",
     "idx[:, h] = idx_g[:, 0]"),
    ("group step selects on the first heads' own scores", "idx = topk(sg32, k)",
     "idx = topk(s32[:, :Hkv], k)"),
    ("block score keeps negative scores",
     "out[..., j] = np.maximum(s[..., j * bs:min((j + 1) * bs, T)], 0).max(axis=-1)",
     "out[..., j] = s[..., j * bs:min((j + 1) * bs, T)].max(axis=-1)"),
    ("block score sums instead of max",
     "out[..., j] = np.maximum(s[..., j * bs:min((j + 1) * bs, T)], 0).max(axis=-1)",
     "out[..., j] = np.maximum(s[..., j * bs:min((j + 1) * bs, T)], 0).sum(axis=-1)"),
    ("block score drops the short last block", "nb = -(-T // bs)", "nb = T // bs"),
    ("block tokens off by one", "for t in range(j * bs, min((j + 1) * bs, T))]",
     "for t in range(j * bs + 1, min((j + 1) * bs + 1, T))]"),
    ("block tokens not clipped", "for t in range(j * bs, min((j + 1) * bs, T))]",
     "for t in range((j * bs), (j + 1) * bs)]"),
    ("block step selects on tokens, not blocks", "bidx = topk(sb, kb)", "bidx = topk(s32, kb)"),
    ("hierarchy halves the other way", "m = b + (e - b + 1) // 2", "m = b + (e - b) // 2"),
    ("hierarchy scores parts by their last token",
     "children.sort(key=lambda c: (-s[c[0]], c[0]))", "children.sort(key=lambda c: (-s[c[1] - 1], c[0]))"),
    ("hierarchy ties to the higher start",
     "children.sort(key=lambda c: (-s[c[0]], c[0]))", "children.sort(key=lambda c: (-s[c[0]], -c[0]))"),
    ("hierarchy keeps the worst parts",
     "children.sort(key=lambda c: (-s[c[0]], c[0]))", "children.sort(key=lambda c: (s[c[0]], c[0]))"),
    ("hierarchy starts from unequal parts", "parts = [((i * T) // k, ((i + 1) * T) // k) for i in range(k)]",
     "parts = [(i * (T // k), (i + 1) * (T // k) if i < k - 1 else T) for i in range(k)]"),
]


def _mutant(orig, new):
    src = open(SRC_PATH).read()
    assert src.count(orig) == 1, f"mutation anchor not unique: {orig!r}"
    mod = types.ModuleType("oracle_mutant")
    mod.__file__ = SRC_PATH
    exec(compile(src.replace(orig, new), SRC_PATH, "exec"), mod.__dict__)
    return mod


def test_unmutated_copy_passes():
    src = open(SRC_PATH).read()
    mod = types.ModuleType("oracle_copy")
    exec(compile(src, SRC_PATH, "exec"), mod.__dict__)
    for pin in pins.PINS:
        pin(mod)


@pytest.mark.parametrize("name,orig,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_mutation_is_caught(name, orig, new):
    mod = _mutant(orig, new)
    failed = []
    for pin in pins.PINS:
        try:
            pin(mod)
        except Exception:  # noqa: BLE001 - any failure counts as caught
            failed.append(pin.__name__)
    assert failed, f"no pin caught the mutation '{name}'"
