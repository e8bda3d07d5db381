"""Pins of oracle/moe.py against things other than itself: a dense
brute-force evaluation built from library routines, closed forms and
special cases of the routed-MoE layer."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import moe


def _experts(E, d, d_ff, rng, scale=0.3):
    return [(rng.normal(0, scale, (d_ff, d)), rng.normal(0, scale, (d_ff, d)), rng.normal(0, scale, (d, d_ff)))
            for _ in range(E)]


def dense_masked(x, wr, b, k, W):
    """All E experts on every token (batched), weighted by a probability
    vector that is the softmax of the chosen logits and 0 elsewhere. Built from
    numpy lexsort, torch.softmax, torch einsum and torch silu only."""
    xt = torch.tensor(x, dtype=torch.float64)
    s = (xt @ torch.tensor(wr, dtype=torch.float64).T)
    if b is not None:
        s = s + torch.tensor(b, dtype=torch.float64)
    s32 = s.to(torch.float32).to(torch.float64)
    T, E = s32.shape
    mask = torch.zeros(T, E, dtype=torch.bool)
    for t in range(T):
        order = np.lexsort((np.arange(E), -s32[t].numpy()))
        mask[t, torch.tensor(order[:k])] = True
    p = torch.softmax(s32.masked_fill(~mask, float("-inf")), dim=1)
    Wg = torch.tensor(np.stack([w[0] for w in W]))
    Wu = torch.tensor(np.stack([w[1] for w in W]))
    Wd = torch.tensor(np.stack([w[2] for w in W]))
    g = torch.einsum("efd,td->tef", Wg, xt)
    u = torch.einsum("efd,td->tef", Wu, xt)
    Y = torch.einsum("edf,tef->ted", Wd, F.silu(g) * u)
    return torch.einsum("te,ted->td", p, Y).numpy(), mask.numpy()


@pytest.mark.parametrize("E,k,T,d,d_ff", [(8, 2, 16, 64, 128), (6, 3, 5, 16, 24), (4, 4, 3, 8, 8), (9, 1, 7, 12, 20)])
def test_layer_matches_dense_bruteforce(E, k, T, d, d_ff):
    rng = np.random.default_rng(E * 100 + k)
    x = rng.normal(0, 1, (T, d))
    wr = rng.normal(0, 0.5, (E, d))
    b = rng.normal(0, 0.1, E)
    W = _experts(E, d, d_ff, rng)
    y, ids, w = moe.layer_forward(x, wr, b, k, lambda e: W[e])
    yd, mask = dense_masked(x, wr, b, k, W)
    rms = np.sqrt(np.mean(yd ** 2))
    assert np.max(np.abs(y - yd)) <= 1e-9 * max(rms, 1e-30)
    for t in range(T):
        assert set(ids[t].tolist()) == set(np.nonzero(mask[t])[0].tolist())


def test_k1_is_one_expert_with_weight_exactly_one():
    rng = np.random.default_rng(1)
    E, d, d_ff, T = 5, 10, 14, 6
    x = rng.normal(0, 1, (T, d)); wr = rng.normal(0, 1, (E, d))
    W = _experts(E, d, d_ff, rng)
    y, ids, w = moe.layer_forward(x, wr, None, 1, lambda e: W[e])
    assert np.all(w == 1.0)
    for t in range(T):
        e = int(np.argmax((x[t] @ wr.T).astype(np.float32)))
        assert ids[t, 0] == e
        g = W[e][0] @ x[t]; u = W[e][1] @ x[t]
        ref = W[e][2] @ (F.silu(torch.tensor(g)).numpy() * u)
        np.testing.assert_allclose(y[t], ref, rtol=1e-12, atol=1e-14)


def test_k_equals_E_is_full_softmax_mixture():
    rng = np.random.default_rng(2)
    E, d, d_ff, T = 4, 6, 10, 5
    x = rng.normal(0, 1, (T, d)); wr = rng.normal(0, 1, (E, d))
    _, ids, w = moe.layer_forward(x, wr, None, E, lambda e: _experts(1, d, d_ff, np.random.default_rng(e))[0])
    s32 = (x @ wr.T).astype(np.float32).astype(np.float64)
    p = torch.softmax(torch.tensor(s32), dim=1).numpy()
    for t in range(T):
        np.testing.assert_allclose(w[t], p[t, ids[t]], rtol=1e-13)
        assert sorted(ids[t].tolist()) == list(range(E))


def test_identical_experts_give_that_expert():
    rng = np.random.default_rng(3)
    E, k, d, d_ff, T = 7, 3, 9, 11, 4
    W1 = _experts(1, d, d_ff, rng)[0]
    x = rng.normal(0, 1, (T, d)); wr = rng.normal(0, 1, (E, d))
    y, _, w = moe.layer_forward(x, wr, None, k, lambda e: W1)
    assert np.all(w >= 0)
    np.testing.assert_allclose(w.sum(1), 1.0, rtol=0, atol=1e-15)
    for t in range(T):
        ref = moe.expert_ffn(*W1, x[t])
        np.testing.assert_allclose(y[t], ref, rtol=1e-12, atol=1e-14)


def test_all_ties_pick_lowest_indices_and_zero_output():
    E, k, d, d_ff, T = 8, 3, 6, 7, 4
    rng = np.random.default_rng(4)
    W = _experts(E, d, d_ff, rng)
    x = np.zeros((T, d))
    y, ids, w = moe.layer_forward(x, rng.normal(0, 1, (E, d)), np.zeros(E), k, lambda e: W[e])
    assert np.all(ids == np.arange(k))
    np.testing.assert_allclose(w, 1.0 / k, rtol=1e-15)
    assert np.all(y == 0.0)


def test_duplicate_router_rows_prefer_lower_index():
    rng = np.random.default_rng(5)
    E, d = 10, 12
    wr = rng.normal(0, 1, (E, d))
    x = rng.normal(0, 1, (20, d))
    wr[7] = wr[2]
    s = moe.router_logits(x, wr, None)
    ids = moe.select_topk(s, 1)
    for t in range(20):
        if int(np.argmax(s[t])) in (2, 7):
            assert ids[t, 0] == 2
    # force rows 2 and 7 to be the two best: both chosen, 2 first
    b = np.zeros(E); b[2] = b[7] = 100.0
    ids2 = moe.select_topk(moe.router_logits(x, wr, b), 2)
    assert np.all(ids2 == [2, 7])


def test_topk_against_lexsort_with_planted_ties():
    rng = np.random.default_rng(6)
    T, E, k = 50, 32, 6
    s = rng.integers(-4, 5, size=(T, E)).astype(np.float32)  # many ties
    ids = moe.select_topk(s, k)
    for t in range(T):
        ref = np.lexsort((np.arange(E), -s[t]))[:k]
        assert ids[t].tolist() == ref.tolist()


def test_structured_weights_closed_form():
    # d = d_ff = n; W_gate = a * P (P[i, p(i)] = 1), W_up = diag(D), W_down = Q
    # (Q[i, q(i)] = 1): y_i = silu(a x_{p(q(i))}) * D_{q(i)} * x_{q(i)}.
    # A transposed or swapped operand gives a different index pattern.
    n, a = 9, 0.7
    rng = np.random.default_rng(7)
    p, q = rng.permutation(n), rng.permutation(n)
    P = np.zeros((n, n)); P[np.arange(n), p] = 1.0
    Q = np.zeros((n, n)); Q[np.arange(n), q] = 1.0
    D = rng.uniform(0.5, 2.0, n)
    x = rng.normal(0, 1, n)
    y = moe.expert_ffn(a * P, np.diag(D), Q, x)
    ref = np.array([a * x[p[q[i]]] / (1 + np.exp(-a * x[p[q[i]]])) * D[q[i]] * x[q[i]] for i in range(n)])
    np.testing.assert_allclose(y, ref, rtol=1e-14, atol=1e-15)


def test_silu_matches_torch():
    g = np.linspace(-30, 30, 1001)
    np.testing.assert_allclose(moe.silu(g), F.silu(torch.tensor(g)).numpy(), rtol=1e-14, atol=1e-300)


def test_permutation_is_stable_sort_by_expert():
    rng = np.random.default_rng(8)
    T, E, k = 37, 11, 3
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offsets, perm, inv = moe.permutation(ids, E)
    flat = ids.reshape(-1)
    np.testing.assert_array_equal(counts, np.bincount(flat, minlength=E))
    np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=E))]))
    np.testing.assert_array_equal(perm, np.argsort(flat, kind="stable"))
    np.testing.assert_array_equal(inv[perm], np.arange(T * k))
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.all(flat[seg] == e) and np.all(np.diff(seg) > 0)


def test_empty_batch():
    counts, offsets, perm, inv = moe.permutation(np.zeros((0, 2), np.int32), 4)
    assert counts.sum() == 0 and offsets.tolist() == [0] * 5 and perm.size == 0
    y, ids, w = moe.layer_forward(np.zeros((0, 4)), np.ones((3, 4)), None, 2, lambda e: None)
    assert y.shape == (0, 4)


def test_router_logits_round_once_to_fp32():
    rng = np.random.default_rng(9)
    x = rng.normal(0, 1, (4, 300)); wr = rng.normal(0, 1, (5, 300)); b = rng.normal(0, 1, 5)
    s = moe.router_logits(x, wr, b)
    assert s.dtype == np.float32
    exact = np.array([[sum(x[t, i] * wr[e, i] for i in range(300)) + b[e] for e in range(5)] for t in range(4)])
    np.testing.assert_array_equal(s, exact.astype(np.float32))


@pytest.mark.parametrize("E,k,T,d,d_ff,per_token", [(8, 2, 16, 64, 128, False), (6, 3, 40, 16, 24, True),
                                                    (9, 1, 7, 12, 20, False), (5, 5, 3, 8, 8, True)])
def test_grouped_layer_matches_dense_bruteforce_and_per_token(E, k, T, d, d_ff, per_token):
    """The expert-by-expert evaluation against the dense masked brute force
    and the per-token layer, on full batches and on token subsets (with a
    per-token bias, the subset's bias rows are taken)."""
    rng = np.random.default_rng(7 * E + k)
    x = rng.normal(0, 1, (T, d))
    wr = rng.normal(0, 0.5, (E, d))
    b = rng.normal(0, 0.1, (T, E) if per_token else E)
    W = _experts(E, d, d_ff, rng)
    y, ids, w = moe.layer_forward_grouped(x, wr, b, k, lambda e: W[e])
    yd, _ = dense_masked(x, wr, b if not per_token else None, k, W) if not per_token else (None, None)
    y1, ids1, w1 = moe.layer_forward(x, wr, b, k, lambda e: W[e])
    rms = np.sqrt(np.mean(y1 ** 2))
    np.testing.assert_array_equal(ids, ids1)
    np.testing.assert_array_equal(w, w1)
    assert np.max(np.abs(y - y1)) <= 1e-12 * rms
    if yd is not None:
        assert np.max(np.abs(y - yd)) <= 1e-9 * rms
    sub = np.array([T - 1, 0, T // 2])
    ys, _, _ = moe.layer_forward_grouped(x, wr, b, k, lambda e: W[e], tokens=sub)
    assert np.max(np.abs(ys - y1[sub])) <= 1e-12 * rms


def test_batches_match_each_batch_alone():
    """Several batches through one expert pass: each result equals the
    per-token layer on that batch (different routers, biases and subsets)."""
    rng = np.random.default_rng(11)
    E, k, d, d_ff = 7, 3, 16, 24
    W = _experts(E, d, d_ff, rng)
    batches = []
    for T, per_token, sub in ((9, False, None), (4, True, [3, 1]), (1, False, None)):
        x = rng.normal(0, 1, (T, d))
        wr = rng.normal(0, 0.5, (E, d))
        b = rng.normal(0, 0.1, (T, E) if per_token else E)
        batches.append((x, wr, b, sub))
    res = moe.layer_forward_batches(batches, k, lambda e: W[e])
    for (x, wr, b, sub), (y, ids, w) in zip(batches, res):
        y1, ids1, w1 = moe.layer_forward(x, wr, b, k, lambda e: W[e], tokens=sub)
        np.testing.assert_array_equal(ids, ids1)
        assert np.max(np.abs(y - y1)) <= 1e-12 * np.sqrt(np.mean(y1 ** 2))


def test_half_bf16_step_of_the_parity_check():
    """The slack the parity check gives a bf16 output is half the bf16
    spacing: a value rounded to bf16 is within it, one twice as far is not."""
    import sys
    sys.path.insert(0, __import__("os").path.dirname(__file__))
    from parity import half_ulp_bf16
    rng = np.random.default_rng(3)
    v = rng.normal(0, 10, 10000)
    r = torch.tensor(v, dtype=torch.float64).to(torch.bfloat16).to(torch.float64).numpy()
    h = half_ulp_bf16(v)
    assert np.all(np.abs(r - v) <= h)
    assert np.all(half_ulp_bf16(np.array([1.0, 1.5, 2.0 - 1e-9])) == np.array([2 ** -8, 2 ** -8, 2 ** -7]))
    assert half_ulp_bf16(np.array([0.0]))[0] == 0.0
