"""The routed-MoE layer, written out per token and per rank.

Test infrastructure (see oracle/__init__.py).

The pages fix the structure ([paperlens] "MoEは扉を開けると同時に、別の扉を閉める",
paper §1: a layer holds E experts and each token passes through k << E of
them; [wiki] "FreeToken：エッジネイティブMoEセットアップガイドと比較": the router
turns on a few of hundreds of feed-forward experts per token) but not the
router function or the expert form. The readings taken here:

* logits s = x W_r^T + b, accumulated in fp64 and rounded once to fp32;
* top-k on the fp32 logits, larger first, equal logits -> lower expert index;
* weights = softmax over the k chosen logits (the same as a full softmax
  renormalised over the chosen; convex weights);
* expert = SwiGLU without biases: h = silu(W_gate x) * (W_up x), Y = W_down h,
  silu(g) = g / (1 + exp(-g));
* y[t] = sum over ranks j = 0..k-1 of w[t, j] * Y_j, in rank order.

The cache never changes the result ([paperlens] "設計: 2階建てのエキスパート記憶",
paper §3.3; [techfeed] "帯域適応型実行（q*ポリシー）": the partial sums are
added with no change to routing and no approximation), so nothing here knows
about slots.

Pins (tests/test_oracle_moe.py): a dense evaluation of all E experts masked
to the top-k weights; k = 1 (output = one expert, weight exactly 1); k = E
(torch.softmax mixture); identical experts (output = that expert); all-tie
logits (ids 0..k-1, output 0); duplicate router rows (lower index wins);
structured weights with a closed-form SwiGLU output; silu against
torch.nn.functional.silu; top-k against numpy's stable lexsort on random
logits with planted ties; the permutation against its defining sort;
layer_forward_grouped against layer_forward.
"""
from __future__ import annotations

import numpy as np


def router_logits(x: np.ndarray, w_router: np.ndarray, bias=None) -> np.ndarray:
    """s[t, e] = sum_i x[t, i] W_r[e, i] + b[e] (or b[t, e]), fp64, then fp32.

    x [T, d], w_router [E, d] (any float dtype, read exactly), bias None,
    [E] or [T, E]. Returns float32 [T, E]."""
    s = np.asarray(x, np.float64) @ np.asarray(w_router, np.float64).T
    if bias is not None:
        s = s + np.asarray(bias, np.float64)
    return s.astype(np.float32)


def select_topk(s32: np.ndarray, k: int) -> np.ndarray:
    """ids [T, k] int32: the k largest logits per token, in rank order
    (larger logit first; equal logits -> lower expert index first)."""
    T, E = s32.shape
    ids = np.empty((T, k), dtype=np.int32)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(s32[t, e]), e))
        ids[t] = order[:k]
    return ids


def topk_weights(s32: np.ndarray, ids: np.ndarray) -> np.ndarray:
    """w [T, k] float64: softmax over the chosen logits of each token."""
    T, k = ids.shape
    w = np.empty((T, k), dtype=np.float64)
    for t in range(T):
        z = s32[t, ids[t]].astype(np.float64)
        ez = np.exp(z - z.max())
        w[t] = ez / ez.sum()
    return w


def route(x, w_router, bias, k):
    """Router of one layer: (ids [T, k] int32, w [T, k] fp64, s32 [T, E])."""
    s32 = router_logits(x, w_router, bias)
    ids = select_topk(s32, k)
    return ids, topk_weights(s32, ids), s32


def topk_gap(s32: np.ndarray, k: int) -> np.ndarray:
    """Per token: (k-th largest logit) - ((k+1)-th largest), fp32 values in
    fp64 (inf when k == E). Used to reject near-tie inputs."""
    T, E = s32.shape
    if k >= E:
        return np.full(T, np.inf)
    srt = -np.sort(-s32.astype(np.float64), axis=1)
    return srt[:, k - 1] - srt[:, k]


def permutation(ids: np.ndarray, E: int):
    """Token -> expert grouping of the flattened routing ids [T*k]:
    counts [E], offsets [E+1] (exclusive scan), perm [T*k] (sorted position ->
    flat index t*k+j, ordered by expert then by flat index), inv = perm^-1."""
    flat = ids.reshape(-1).astype(np.int64)
    counts = np.zeros(E, dtype=np.int32)
    for e in flat:
        counts[e] += 1
    offsets = np.zeros(E + 1, dtype=np.int32)
    for e in range(E):
        offsets[e + 1] = offsets[e] + counts[e]
    fill = offsets[:-1].copy()
    perm = np.empty(flat.size, dtype=np.int32)
    for i, e in enumerate(flat):  # flat order = (token, rank) order: stable
        perm[fill[e]] = i
        fill[e] += 1
    inv = np.empty_like(perm)
    inv[perm] = np.arange(flat.size, dtype=np.int32)
    return counts, offsets, perm, inv


def silu(g: np.ndarray) -> np.ndarray:
    return g / (1.0 + np.exp(-g))


def expert_ffn(w_gate: np.ndarray, w_up: np.ndarray, w_down: np.ndarray, xt: np.ndarray) -> np.ndarray:
    """SwiGLU expert on one token: W_down (silu(W_gate x) * (W_up x)), fp64."""
    xt = np.asarray(xt, np.float64)
    g = w_gate @ xt
    u = w_up @ xt
    return w_down @ (silu(g) * u)


def layer_forward(x, w_router, bias, k, expert_weights, tokens=None):
    """One MoE layer, per token and per rank.

    x [T, d]; w_router [E, d]; bias None / [E] / [T, E]; expert_weights(e) ->
    (W_gate, W_up, W_down) float64. tokens: optional subset of token indices
    to evaluate (the routing of each token only needs its own row).
    Returns (y [len(tokens), d] fp64, ids, w) for those tokens."""
    x = np.asarray(x, np.float64)
    T = x.shape[0]
    tok = np.arange(T) if tokens is None else np.asarray(tokens)
    b = bias
    if bias is not None and np.ndim(bias) == 2:
        b = np.asarray(bias)[tok]
    ids, w, _ = route(x[tok], w_router, b, k)
    cache = {}
    y = np.zeros((len(tok), x.shape[1]), dtype=np.float64)
    for n, t in enumerate(tok):
        acc = np.zeros(x.shape[1], dtype=np.float64)
        for j in range(k):
            e = int(ids[n, j])
            if e not in cache:
                cache[e] = expert_weights(e)
            acc = acc + w[n, j] * expert_ffn(*cache[e], x[t])
        y[n] = acc
    return y, ids, w


def layer_forward_grouped(x, w_router, bias, k, expert_weights, tokens=None):
    """The same layer as layer_forward, evaluated expert by expert: each
    chosen expert is applied once to the matrix whose columns are the tokens
    routed to it (expert_ffn on a [d, n] argument is n independent columns),
    then every token adds its k outputs with its weights in rank order. Every
    output element is the same fp64 expression as in layer_forward; only the
    order in which the experts are visited differs, so large layers (thousands
    of tokens over hundreds of experts) decode each expert's weights once.

    Arguments and result as layer_forward."""
    return layer_forward_batches([(x, w_router, bias, tokens)], k, expert_weights)[0]


def layer_forward_batches(batches, k, expert_weights):
    """layer_forward_grouped over several batches of one layer's experts at
    once, so that each expert's weights are decoded once for all of them:
    batches is a list of (x, w_router, bias, tokens); returns one
    (y, ids, w) per batch, each as layer_forward would."""
    routed = []
    for x, w_router, bias, tokens in batches:
        x = np.asarray(x, np.float64)
        tok = np.arange(x.shape[0]) if tokens is None else np.asarray(tokens)
        b = bias
        if bias is not None and np.ndim(bias) == 2:
            b = np.asarray(bias)[tok]
        ids, w, _ = route(x[tok], w_router, b, k)
        out = np.zeros((len(tok), k, x.shape[1]), dtype=np.float64)  # expert output of (token, rank)
        routed.append((x, tok, ids, w, out))
    experts = np.unique(np.concatenate([r[2].ravel() for r in routed])) if routed else []
    for e in experts:
        wg, wu, wd = expert_weights(int(e))
        for x, tok, ids, _, out in routed:
            rows, ranks = np.nonzero(ids == e)
            if rows.size:
                out[rows, ranks] = expert_ffn(wg, wu, wd, x[tok[rows]].T).T
    res = []
    for x, tok, ids, w, out in routed:
        y = np.zeros((len(tok), x.shape[1]), dtype=np.float64)
        for j in range(k):
            y = y + w[:, j:j + 1] * out[:, j]
        res.append((y, ids, w))
    return res
