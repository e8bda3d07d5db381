"""Pins of oracle/ep.py, the expert-parallel layer: the one-device layer
(itself pinned to a dense brute force), brute-force owner counts, the
exchange's round trip and the cache's partition of lookups."""
import numpy as np
import pytest

from oracle import cache as ocache
from oracle import ep, moe
from test_oracle_moe import _experts, dense_masked


def _setup(E, k, d, d_ff, Ts, seed):
    rng = np.random.default_rng(seed)
    wr = rng.normal(0, 0.5, (E, d))
    W = _experts(E, d, d_ff, rng)
    xs = [rng.normal(0, 1, (T, d)) for T in Ts]
    bs = [rng.normal(0, 0.3, E) for _ in Ts]
    return wr, W, xs, bs


@pytest.mark.parametrize("G,Ts", [(1, [7]), (2, [5, 3]), (2, [0, 4]), (4, [1, 0, 6, 2]), (8, [3, 1, 1, 0, 2, 5, 1, 4])])
def test_ep_equals_one_device_layer(G, Ts):
    E, k, d, d_ff = 8, 3, 12, 20
    wr, W, xs, bs = _setup(E, k, d, d_ff, Ts, 10 * G + len(Ts))
    out = ep.ep_layer_forward(xs, wr, bs, k, lambda e: W[e], G)
    for s in range(G):
        if Ts[s] == 0:
            assert out["y"][s].shape == (0, d)
            continue
        y1, ids1, w1 = moe.layer_forward(xs[s], wr, bs[s], k, lambda e: W[e])
        assert np.array_equal(out["y"][s], y1)  # same rows, same sum order: exact
        assert np.array_equal(out["ids"][s], ids1)
        yd, _ = dense_masked(xs[s], wr, bs[s], k, W)
        assert np.max(np.abs(out["y"][s] - yd)) <= 1e-9 * np.sqrt(np.mean(yd ** 2))


def test_send_counts_brute_force():
    E, k, d, d_ff, G = 16, 4, 6, 8, 4
    Ts = [9, 0, 5, 13]
    wr, W, xs, bs = _setup(E, k, d, d_ff, Ts, 3)
    out = ep.ep_layer_forward(xs, wr, bs, k, lambda e: W[e], G)
    sc = out["send_counts"]
    for s in range(G):
        for o in range(G):
            n = sum(1 for e in out["ids"][s].reshape(-1) if e // (E // G) == o)
            assert sc[s, o] == n
        assert sc[s].sum() == Ts[s] * k


def test_dispatch_order_groups_owners_then_experts():
    rng = np.random.default_rng(5)
    E, G, T, k = 12, 3, 10, 4
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    sc, order, eids = ep.dispatch_plan(ids, E, G)
    flat = ids.reshape(-1)
    assert sorted(order.tolist()) == list(range(T * k))
    assert np.array_equal(eids, flat[order])
    # (expert, flat index) ascending, the defining sort of the permutation
    keys = [(int(flat[i]), int(i)) for i in order]
    assert keys == sorted(keys)
    lo = 0
    for o in range(G):
        blk = eids[lo:lo + sc[o]]
        assert all(e // (E // G) == o for e in blk)
        lo += sc[o]


def test_all_to_all_round_trip():
    rng = np.random.default_rng(7)
    G = 4
    counts = [rng.integers(0, 4, G) for _ in range(G)]
    send = [np.array([(s, i) for i in range(int(c.sum()))]).reshape(-1, 2) for s, c in enumerate(counts)]
    recv = ep.all_to_all(send, counts)
    for o in range(G):
        # o gets, from each s in order, s's rows sum(counts[s][:o]) .. + counts[s][o]
        want = [(s, i) for s in range(G)
                for i in range(int(counts[s][:o].sum()), int(counts[s][:o].sum() + counts[s][o]))]
        assert [tuple(r) for r in recv[o]] == want
    back_counts = [[counts[s][o] for s in range(G)] for o in range(G)]
    back = ep.all_to_all(recv, back_counts)
    for s in range(G):
        assert np.array_equal(back[s].reshape(-1, 2), send[s].reshape(-1, 2))


def test_owner_caches_partition_the_one_device_lookups():
    E, k, d, d_ff, G, L = 8, 2, 6, 8, 2, 3
    Ts = [4, 3]
    rng = np.random.default_rng(11)
    wr = [rng.normal(0, 0.5, (E, d)) for _ in range(L)]
    W = _experts(E, d, d_ff, rng)
    caches = [ocache.ExpertCache(L, E // G, 3, 52700, 77300) for _ in range(G)]
    for step in range(4):
        for layer in range(L):
            xs = [rng.normal(0, 1, (T, d)) for T in Ts]
            out = ep.ep_layer_forward(xs, wr[layer], None, k, lambda e: W[e], G, caches, layer)
            routed = sorted({int(e) for s in range(G) for e in out["ids"][s].reshape(-1)})
            got = []
            for o, rec in enumerate(out["records"]):
                got += [o * (E // G) + e for (_, e, _) in rec["lookups"]]
                assert all(lay == layer for (lay, _, _) in rec["lookups"])
            assert sorted(got) == routed


def test_g1_cache_record_is_the_one_device_record():
    E, k, d, d_ff, L = 8, 2, 6, 8, 2
    rng = np.random.default_rng(13)
    wr = rng.normal(0, 0.5, (E, d))
    W = _experts(E, d, d_ff, rng)
    a = [ocache.ExpertCache(L, E, 3, 11800, 47500)]
    b = ocache.ExpertCache(L, E, 3, 11800, 47500)
    for step in range(6):
        for layer in range(L):
            x = rng.normal(0, 1, (5, d))
            out = ep.ep_layer_forward([x], wr, None, k, lambda e: W[e], 1, a, layer)
            _, ids, _ = moe.layer_forward(x, wr, None, k, lambda e: W[e])
            counts = np.bincount(ids.reshape(-1), minlength=E)
            assert out["records"][0] == b.forward(layer, ocache.DECODE, counts)
    assert a[0].n == b.n and a[0].contents() == b.contents()


def test_full_share_caches_have_only_compulsory_misses():
    """With room for its whole share and B_P = B_H (every miss staged), an
    owner misses only on first touches."""
    E, k, d, d_ff, G, L = 8, 3, 6, 8, 4, 2
    rng = np.random.default_rng(17)
    wr = rng.normal(0, 0.5, (E, d))
    W = _experts(E, d, d_ff, rng)
    caches = [ocache.ExpertCache(L, E // G, L * E // G, 1, 1) for _ in range(G)]
    seen = set()
    for step in range(5):
        for layer in range(L):
            xs = [rng.normal(0, 1, (2, d)) for _ in range(G)]
            out = ep.ep_layer_forward(xs, wr, None, k, lambda e: W[e], G, caches, layer)
            for s in range(G):
                seen |= {(layer, int(e)) for e in out["ids"][s].reshape(-1)}
    assert sum(c.n["misses"] for c in caches) == len(seen)
    assert sum(c.n["streamed"] for c in caches) == 0


def test_ep_compare_g1_equals_replicas_and_runs():
    """The expert-parallel simulation: with one device both arms are the same
    cache on the same stream; with several it runs and counts sensibly."""
    from oracle import ep_compare
    rows = ep_compare.run(steps=4, gs=(1, 2), fracs=(0.10,))
    g1 = rows[0]
    assert g1[0] == 1 and g1[3] == g1[4] and g1[5] == g1[6]
    g2 = rows[1]
    assert 0 < g2[3] <= 1 and 0 < g2[4] <= 1 and g2[5] > 0 and g2[6] > 0
