"""Plain, slow, double-precision oracle of Double-Sparsity-style decode attention.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline leg, never by the product path.

What is computed, and where it comes from
-----------------------------------------
Source page: "Post-Training Sparse Attention with Double Sparsity"
(arXiv 2408.07092).

* Token sparsity -- self-attention is computed over the important tokens only
  (Abstract; Key points 2).
* Channel sparsity -- a few important feature channels, fixed offline by
  calibration, are used to identify the important tokens (Abstract;
  Method details: Core idea; Method details: Technical framework).
* Token selection keeps the tokens with the higher activation under those
  channels (Method details: Key design).
* The 1/16 token and 1/16 channel ratios are the reported operating point
  (Abstract; Experimental highlights).

The page gives no formulas.  The concrete steps below are the plainest reading
of those statements, with these choices where the page is silent:

  label   label[b,h,t,j] = K[b, g(h), t, C[h,j]]   (exact copy of bf16 bits;
          g(h) = h // (Hq/Hkv) for grouped KV heads; one label cache per
          query head)
  score   s[b,h,t] = sum_j q[b,h,C[h,j]] * label[b,h,t,j]      (unscaled)
  top-k   the k tokens with the largest score; ties go to the lower token
          index; -0 and +0 compare equal; output in ascending token order
  attend  l_i = (q . K_i) / sqrt(d) over the selected rows i; w = softmax(l);
          o = sum_i w_i V_i; lse = log sum_i exp(l_i)
  dense   attend with every token selected
  merge   the key set split into chunks, each chunk's (o_c, lse_c) combined by
          log-sum-exp weights -- the standard split-softmax identity.

Inputs are bf16 bit patterns (numpy uint16); every arithmetic step runs in
float64 on the exact decoded values.  ``s32`` (float64 scores rounded to
float32, nearest-even) is what the bit-exact top-k parity check feeds to the
GPU top-k.

Offline channel calibration (the step before the path).  The page says the
channel pattern is static, so it is fixed offline (Method details: Core idea;
Technical framework), and leaves the criterion open (Key design: "unknown").
The reading taken here, the plainest one:

  importance  I[h,c] = mean over the pairs (calibration query n, cached token t)
              of the same sequence b of |q[b,h,n,c] * k[b,g(h),t,c]|, the
              magnitude of channel c's share of the attention logit
  selection   the r channels with the largest I[h,c]; ties go to the lower
              channel; output ascending

Group-shared selection (grouped KV heads).  The page's token sparsity keeps
the important tokens of the attention (Abstract; Key points 2); with grouped
KV heads the G query heads of a group read the same K/V rows, so one
selection per group lets each row be read once for all of them.  The page
does not define a group score; the reading taken here:

  group score  sg[b,g,t] = sum over the query heads h of group g of s[b,h,t]
               (the per-head approximate scores; head order h = gG .. gG+G-1)
  group top-k  the k tokens of largest sg, with the per-head top-k's order
  attention    every query head of the group attends over the group's set

Block-granular selection (page "Jenga: Enhancing LLM Long-Context Fine-tuning
with Contextual Token Sparsity", Core method 1: Information-driven Token
Elimination; Observation 2 gives the default block of 64 tokens).  There a
token's informativeness sums only the positive attention scores it receives,
a block's informativeness is the largest of its tokens', and blocks are kept
against a threshold tuned per layer on a model.  For one decode query, with no
model to tune a threshold on, the reading taken is:

  token        I[t] = max(s[t], 0) (s the approximate score above)
  block        Ib[j] = max over t in [j*bs, min((j+1)*bs, T)) of I[t]
  selection    a fixed count: the kb blocks of largest Ib, ties to the lower
               block (the decode analogue of the top-k above); the kept tokens
               are every token of those blocks (clipped to T), ascending
  attention    as above, over the kept tokens

Hierarchical top-k (page "A Training-free Sub-quadratic Cost Transformer
Model Serving Framework With Hierarchically Pruned Attention", Core idea:
attention locality, nearby tokens score alike; Technical framework: a
hierarchy of tokens searched tree-like for each query's important keys).  The
page leaves the hierarchy and the search open (its examples, k-means and
binary search, are the summary's guesses); the reading taken here is a
binary hierarchy of contiguous ranges searched top-down:

  start        k parts of [0, T): part i is [floor(iT/k), floor((i+1)T/k))
  level        every part of more than one token is halved (the first half
               takes the extra token); each part is scored by the approximate
               score of its first token; the k best parts stay (score
               descending, start ascending)
  end          after ceil(log2 of the longest start part) levels every part
               is one token: the k kept tokens, ascending

It reads about 2k·log2(T/k) label rows instead of T, and equals the exact
top-k when the search is exhaustive (k = T) or the scores fall with position.

Pins (see tests/test_oracle_pins.py): bf16 decoding against known bit
patterns; label gather against the identity/permutation cases and a
per-element brute force; score against one-hot queries and the attention
logits; top-k against a characterisation of the (score desc, index asc)
order by exhaustive pair checks and against Python's sort; attention against
torch's scaled_dot_product_attention in float64, closed forms (q = 0, k = 1,
identical keys, a two-token case with weight exactly 3/4), weights summing to
one and convexity; merge against the unsplit result; the r = d, k = T case
against dense attention; hand-derived worked examples in tests/golden/.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "bf16_to_f64", "label_head", "label", "score_head", "score", "to_f32",
    "topk_head", "topk", "attend_head", "attend", "dense", "lse_merge",
    "attend_split_head", "sparse_step", "group_of",
    "calibrate_importance", "calibrate_select", "calibrate",
    "group_score", "group_attend", "group_sparse_step",
    "block_score", "block_tokens", "block_sparse_step",
    "hier_topk_head", "hier_topk",
]


# ---------------------------------------------------------------------------
# number format

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns: the bits are the top half of a float32."""
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_f32(x: np.ndarray) -> np.ndarray:
    """float64 -> float32, round to nearest even (IEEE default)."""
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def group_of(h: int, Hq: int, Hkv: int) -> int:
    """KV head read by query head h when Hq/Hkv query heads share one KV head."""
    return h // (Hq // Hkv)


# ---------------------------------------------------------------------------
# label cache (channel sparsity: the calibrated channels of K, kept contiguous)

def label_head(K_bg: np.ndarray, C_h: np.ndarray) -> np.ndarray:
    """label[t, j] = K[t, C_h[j]] for one (batch, query head); bf16 bits copied.

    Double Sparsity page, Method details: Core idea -- the static channel
    pattern (C_h) is what identifies the important tokens.
    """
    return np.ascontiguousarray(np.asarray(K_bg)[:, np.asarray(C_h, dtype=np.int64)])


def label(K: np.ndarray, C: np.ndarray, Hq: int) -> np.ndarray:
    """label [B, Hq, T, r] from K [B, Hkv, T, d] and C [Hq, r]."""
    B, Hkv, T, _ = K.shape
    r = C.shape[1]
    out = np.empty((B, Hq, T, r), np.uint16)
    for b in range(B):
        for h in range(Hq):
            out[b, h] = label_head(K[b, group_of(h, Hq, Hkv)], C[h])
    return out


# ---------------------------------------------------------------------------
# approximate score (channel-sparse q . k)

def score_head(q_h: np.ndarray, C_h: np.ndarray, label_h: np.ndarray) -> np.ndarray:
    """s[t] = sum_j q[C_h[j]] * label[t, j], in float64 (unscaled).

    Double Sparsity page, Method details: Core idea and Key design -- tokens
    are judged by their activation under the calibrated channels only.
    """
    qc = bf16_to_f64(np.asarray(q_h)[np.asarray(C_h, dtype=np.int64)])
    return bf16_to_f64(label_h) @ qc


def score(Q: np.ndarray, C: np.ndarray, lab: np.ndarray) -> np.ndarray:
    """s [B, Hq, T] float64 from Q [B, Hq, d], C [Hq, r], label [B, Hq, T, r]."""
    B, Hq, T, _ = lab.shape
    s = np.empty((B, Hq, T), np.float64)
    for b in range(B):
        for h in range(Hq):
            s[b, h] = score_head(Q[b, h], C[h], lab[b, h])
    return s


# ---------------------------------------------------------------------------
# token selection

def topk_head(s: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest scores; ties to the lower index; ascending output.

    Double Sparsity page, Method details: Key design -- keep the tokens with
    the higher (approximate) activation.  The order is the total order
    (score descending, index ascending); -0.0 and +0.0 compare equal as
    floating-point values.  NaN scores are outside the contract.
    """
    s = np.asarray(s)
    T = s.shape[0]
    if not 1 <= k <= T:
        raise ValueError("need 1 <= k <= T")
    # lexsort: the last key is the primary one.
    order = np.lexsort((np.arange(T), -s))
    return np.sort(order[:k]).astype(np.int32)


def topk(s: np.ndarray, k: int) -> np.ndarray:
    """idx [..., k] int32 for scores [..., T]."""
    lead = s.shape[:-1]
    flat = s.reshape(-1, s.shape[-1])
    out = np.empty((flat.shape[0], k), np.int32)
    for i in range(flat.shape[0]):
        out[i] = topk_head(flat[i], k)
    return out.reshape(*lead, k)


# ---------------------------------------------------------------------------
# exact softmax attention over the selected tokens

def attend_head(q_h, K_bg, V_bg, idx, scale):
    """Softmax attention of one query over the rows ``idx`` of K and V.

    Double Sparsity page, Abstract / Key points 2 -- self-attention computed
    with the important tokens only.  Returns (o [d], lse, w [len(idx)]), all
    float64: l_i = scale * q . K_i, w = softmax(l), o = sum_i w_i V_i,
    lse = log sum_i exp(l_i).
    """
    idx = np.asarray(idx, dtype=np.int64)
    q = bf16_to_f64(q_h)
    Kr = bf16_to_f64(np.asarray(K_bg)[idx])
    Vr = bf16_to_f64(np.asarray(V_bg)[idx])
    logits = (Kr @ q) * scale
    m = logits.max()
    e = np.exp(logits - m)
    z = e.sum()
    w = e / z
    return w @ Vr, m + math.log(z), w


def attend(Q, K, V, idx, scale):
    """O [B, Hq, d], lse [B, Hq] (float64) for idx [B, Hq, k]."""
    B, Hq, d = Q.shape
    Hkv = K.shape[1]
    O = np.empty((B, Hq, d), np.float64)
    L = np.empty((B, Hq), np.float64)
    for b in range(B):
        for h in range(Hq):
            g = group_of(h, Hq, Hkv)
            O[b, h], L[b, h], _ = attend_head(Q[b, h], K[b, g], V[b, g], idx[b, h], scale)
    return O, L


def dense(Q, K, V, scale):
    """Dense decode attention: every one of the T cached tokens selected."""
    B, Hq, _ = Q.shape
    T = K.shape[2]
    idx = np.broadcast_to(np.arange(T, dtype=np.int32), (B, Hq, T))
    return attend(Q, K, V, idx, scale)


def lse_merge(outs, lses):
    """Combine per-chunk results (o_c, lse_c) of one query into (o, lse).

    Softmax over a union of disjoint key chunks: with M = max_c lse_c,
    o = sum_c exp(lse_c - M) o_c / sum_c exp(lse_c - M) and
    lse = M + log sum_c exp(lse_c - M).
    """
    lses = np.asarray(lses, dtype=np.float64)
    outs = np.asarray(outs, dtype=np.float64)
    M = lses.max()
    a = np.exp(lses - M)
    return (a[:, None] * outs).sum(0) / a.sum(), M + math.log(a.sum())


def attend_split_head(q_h, K_bg, V_bg, idx, scale, n_chunks):
    """attend_head over ``idx`` cut into ``n_chunks`` consecutive chunks, then merged."""
    parts = [c for c in np.array_split(np.asarray(idx), n_chunks) if len(c)]
    res = [attend_head(q_h, K_bg, V_bg, c, scale) for c in parts]
    return lse_merge([r[0] for r in res], [r[1] for r in res])


# ---------------------------------------------------------------------------
# the whole decode step

def sparse_step(Q, K, V, C, k, scale):
    """label -> score -> top-k on float32-rounded scores -> attention.

    Returns a dict with the label cache, float64 and float32 scores, the index
    set and the attention output (float64).
    """
    Hq = Q.shape[1]
    lab = label(K, C, Hq)
    s64 = score(Q, C, lab)
    s32 = to_f32(s64)
    idx = topk(s32, k)
    O, L = attend(Q, K, V, idx, scale)
    return {"label": lab, "s64": s64, "s32": s32, "idx": idx, "O": O, "lse": L}


# ---- offline channel calibration -------------------------------------------------

def calibrate_importance(Qc: np.ndarray, K: np.ndarray, T: int, Hq: int) -> np.ndarray:
    """I[h, c] = 1/(B*Nq*T) * sum_b sum_n sum_t |q[b,h,n,c] * k[b,g(h),t,c]|.

    Qc [B,Hq,Nq,d] calibration queries and K [B,Hkv,T_cap,d] keys (bf16 bits);
    tokens 0..T-1.  |q k| = |q| |k|, so for each sequence b the double sum over
    (n, t) is the product of the two single sums.  Returns [Hq, d] float64.
    """
    B, _, Nq, d = Qc.shape
    Hkv = K.shape[1]
    I = np.zeros((Hq, d))
    for b in range(B):
        ksum = [np.abs(bf16_to_f64(K[b, g, :T])).sum(axis=0) for g in range(Hkv)]
        for h in range(Hq):
            qsum = np.abs(bf16_to_f64(Qc[b, h])).sum(axis=0)
            I[h] += qsum * ksum[group_of(h, Hq, Hkv)]
    return I / (B * Nq * T)


def calibrate_select(I: np.ndarray, r: int) -> np.ndarray:
    """C [Hq, r]: per head the r channels of largest importance, ties to the
    lower channel, in ascending channel order."""
    Hq, d = I.shape
    C = np.empty((Hq, r), np.int32)
    for h in range(Hq):
        order = np.lexsort((np.arange(d), -np.asarray(I[h], np.float64)))
        C[h] = np.sort(order[:r])
    return C


def calibrate(Qc: np.ndarray, K: np.ndarray, T: int, Hq: int, r: int):
    """(C [Hq, r] int32, I [Hq, d] float64) for a calibration set."""
    I = calibrate_importance(Qc, K, T, Hq)
    return calibrate_select(I, r), I


# ---- group-shared selection ------------------------------------------------------

def group_score(s: np.ndarray, Hkv: int) -> np.ndarray:
    """sg [B, Hkv, T]: the sum of the per-head scores s [B, Hq, T] over the
    query heads of each KV group, added in head order."""
    B, Hq, T = s.shape
    G = Hq // Hkv
    sg = np.zeros((B, Hkv, T), dtype=s.dtype)
    for h in range(Hq):
        sg[:, group_of(h, Hq, Hkv)] += s[:, h]
    return sg


def group_attend(Q, K, V, idx_g, scale):
    """O [B, Hq, d], lse [B, Hq]: query head h attends over its group's set
    idx_g [B, Hkv, k]."""
    B, Hq, _ = Q.shape
    Hkv = K.shape[1]
    idx = np.empty((B, Hq, idx_g.shape[-1]), np.int32)
    for h in range(Hq):
        idx[:, h] = idx_g[:, group_of(h, Hq, Hkv)]
    return attend(Q, K, V, idx, scale)


def group_sparse_step(Q, K, V, C, k, scale):
    """label -> per-head scores -> group scores -> group top-k -> attention.

    The group scores are summed from the float32-rounded per-head scores in
    float32 (sg32, what a float32 pipeline selects on) and in float64 (sg64).
    """
    Hq, Hkv = Q.shape[1], K.shape[1]
    lab = label(K, C, Hq)
    s64 = score(Q, C, lab)
    s32 = to_f32(s64)
    sg64 = group_score(s64, Hkv)
    sg32 = group_score(s32.astype(np.float32), Hkv)
    idx = topk(sg32, k)
    O, L = group_attend(Q, K, V, idx, scale)
    return {"label": lab, "s64": s64, "sg64": sg64, "sg32": sg32, "idx": idx, "O": O, "lse": L}


# ---- block-granular selection ----------------------------------------------------

def block_score(s: np.ndarray, bs: int) -> np.ndarray:
    """Ib [..., ceil(T/bs)]: per block of bs consecutive tokens, the largest
    positive part max(s_t, 0) of its tokens' scores (the last block may be short)."""
    s = np.asarray(s)
    T = s.shape[-1]
    nb = -(-T // bs)
    out = np.empty(s.shape[:-1] + (nb,), dtype=s.dtype)
    for j in range(nb):
        out[..., j] = np.maximum(s[..., j * bs:min((j + 1) * bs, T)], 0).max(axis=-1)
    return out


def block_tokens(bidx: np.ndarray, bs: int, T: int) -> np.ndarray:
    """Ascending token indices of the blocks ``bidx`` (one head), clipped to T."""
    toks = [t for j in sorted(int(x) for x in bidx) for t in range(j * bs, min((j + 1) * bs, T))]
    return np.asarray(toks, dtype=np.int32)


def block_sparse_step(Q, K, V, C, bs, kb, scale):
    """label -> scores -> block scores (on the float32-rounded scores) -> top-kb
    blocks -> attention of each head over its blocks' tokens."""
    B, Hq, _ = Q.shape
    Hkv = K.shape[1]
    T = K.shape[2]
    lab = label(K, C, Hq)
    s64 = score(Q, C, lab)
    s32 = to_f32(s64)
    sb = block_score(s32, bs)
    bidx = topk(sb, kb)
    O = np.empty((B, Hq, Q.shape[2]))
    L = np.empty((B, Hq))
    for b in range(B):
        for h in range(Hq):
            g = group_of(h, Hq, Hkv)
            toks = block_tokens(bidx[b, h], bs, T)
            O[b, h], L[b, h], _ = attend_head(Q[b, h], K[b, g], V[b, g], toks, scale)
    return {"s32": s32, "sb": sb, "bidx": bidx, "O": O, "lse": L}


# ---- hierarchical top-k ------------------------------------------------------------

def hier_topk_head(s: np.ndarray, k: int) -> np.ndarray:
    """The k tokens the top-down search over contiguous ranges keeps (ascending)."""
    s = np.asarray(s)
    T = s.shape[0]
    if not 1 <= k <= T:
        raise ValueError("need 1 <= k <= T")
    parts = [((i * T) // k, ((i + 1) * T) // k) for i in range(k)]
    while any(e - b > 1 for b, e in parts):
        children = []
        for b, e in parts:
            if e - b > 1:
                m = b + (e - b + 1) // 2
                children += [(b, m), (m, e)]
            else:
                children.append((b, e))
        children.sort(key=lambda c: (-s[c[0]], c[0]))  # first token's score, then start
        parts = sorted(children[:k])
    return np.array([b for b, _ in parts], np.int32)


def hier_topk(s: np.ndarray, k: int) -> np.ndarray:
    """idx [..., k] int32 for scores [..., T]."""
    lead = s.shape[:-1]
    flat = s.reshape(-1, s.shape[-1])
    out = np.empty((flat.shape[0], k), np.int32)
    for i in range(flat.shape[0]):
        out[i] = hier_topk_head(flat[i], k)
    return out.reshape(*lead, k)
