"""Expert parallelism over G devices: the routed-MoE layer with its experts
split among owners, written out as the exchange that split implies.

Test infrastructure (see oracle/__init__.py).

The pages serve one GPU. They note that in a datacenter a fast interconnect
such as NVLink hides the cost of moving experts between devices while on a
consumer machine the PCIe link is the bottleneck ([ainew] "UC バークレーと
MIT、MoE モデルを一般ハードウェアで動かす推論エンジン「FreeToken」公開",
opening paragraph), and that a miss costs a move over the bus ([wiki]
"FreeToken：エッジネイティブMoEセットアップガイドと比較", the paragraph on
cache misses). Splitting the experts among G devices gives each device its
own host link for its own misses. How the split is made is not on the pages;
the readings taken here:

* G divides E; device r owns experts [r E/G, (r+1) E/G) of every layer, with
  its own slot cache over those (layer, expert) keys, its own share of the
  host pool and its own B_P : B_H;
* the router is replicated: each device routes its own tokens;
* dispatch: device s sends owner o the rows (t, j) of its tokens routed to
  o's experts, in the order of its own expert permutation (expert ascending,
  then flat index t*k + j ascending); owner blocks are therefore contiguous
  in that order;
* owner o receives the blocks of devices 0..G-1, in that order, one after the
  other, and computes every row's expert output; its cache looks the unique
  experts among the received rows up once per layer call, with the
  one-device rules on local expert ids e - o E/G;
* the outputs return in the order they came, and device s combines
  y[t] = sum_j w[t, j] Y[t, j] in rank order.

Every returned row is the same function of the same inputs as on one device
and the combine adds in the same order, so y equals the one-device layer
exactly; the cache still changes only where weights are read from.

Pins (tests/test_oracle_ep.py): y equal to `moe.layer_forward` for G in
1, 2, 4, 8 with ragged and empty token counts; the send counts against a
brute-force count of owners; the exchange's round trip restoring every row;
the owners' lookups partitioning the one-device lookups; G = 1 giving the
one-device cache record; only compulsory misses when every owner's cache
holds its whole share.
"""
from __future__ import annotations

import numpy as np

from . import cache as ocache
from . import moe


def owner_of(e: int, E: int, G: int) -> int:
    """The device that owns expert e when E experts are split in G blocks."""
    return e // (E // G)


def dispatch_plan(ids: np.ndarray, E: int, G: int):
    """Rows one device sends, for its routing ids [T, k].

    Returns (send_counts [G] int64, order [T*k] int32, eids [T*k] int32):
    order[i] is the flat index t*k + j of the i-th row sent, eids[i] its
    expert; owner o's rows are order[sum(send_counts[:o]) : ...]."""
    assert E % G == 0, "G must divide E"
    _, offsets, perm, _ = moe.permutation(ids, E)
    flat = ids.reshape(-1)
    send_counts = np.zeros(G, dtype=np.int64)
    for o in range(G):
        lo, hi = o * (E // G), (o + 1) * (E // G)
        send_counts[o] = offsets[hi] - offsets[lo]
    order = perm.astype(np.int32)
    eids = flat[order].astype(np.int32)
    return send_counts, order, eids


def all_to_all(send, send_counts):
    """The exchange: send[s] is device s's rows (first axis), split by
    send_counts[s] among devices 0..G-1. Returns recv[o] = the blocks that
    devices 0..G-1 sent to o, concatenated in device order."""
    G = len(send)
    recv = []
    for o in range(G):
        parts = []
        for s in range(G):
            lo = int(np.sum(send_counts[s][:o]))
            parts.append(send[s][lo:lo + int(send_counts[s][o])])
        recv.append(np.concatenate(parts, axis=0))
    return recv


def ep_layer_forward(xs, w_router, biases, k, expert_weights, G, caches=None, layer=0,
                     mode=ocache.DECODE):
    """One MoE layer on G devices.

    xs: list of G token blocks [T_s, d] (T_s may be 0); biases: None or a list
    of G (None / [E] / [T_s, E]); expert_weights(e) -> (W_gate, W_up, W_down).
    caches: optional list of G ExpertCache(L, E/G, C_r, ...) of the owners.
    Returns dict(y=[G arrays [T_s, d] fp64], ids, w, send_counts [G, G],
    records=[G cache records or None])."""
    E = np.asarray(w_router).shape[0]
    d = np.asarray(xs[0]).shape[1]
    Eg = E // G
    ids_l, w_l, order_l, send_x, send_e, counts = [], [], [], [], [], []
    for s in range(G):
        x = np.asarray(xs[s], np.float64)
        T = x.shape[0]
        if T:
            b = None if biases is None else biases[s]
            ids, w, _ = moe.route(x, w_router, b, k)
        else:
            ids, w = np.zeros((0, k), np.int32), np.zeros((0, k))
        sc, order, eids = dispatch_plan(ids, E, G)
        ids_l.append(ids)
        w_l.append(w)
        order_l.append(order)
        counts.append(sc)
        send_x.append(x[order // k] if T else np.zeros((0, d)))
        send_e.append(eids)
    recv_x = all_to_all(send_x, counts)
    recv_e = all_to_all(send_e, counts)
    recv_counts = [[counts[s][o] for s in range(G)] for o in range(G)]

    weights = {}
    recv_y, records = [], []
    for o in range(G):
        n = recv_x[o].shape[0]
        assert all(owner_of(int(e), E, G) == o for e in recv_e[o])
        rec = None
        if caches is not None:
            local = np.zeros(Eg, dtype=np.int64)
            for e in recv_e[o]:
                local[int(e) - o * Eg] += 1
            rec = caches[o].forward(layer, mode, local)
        records.append(rec)
        y = np.zeros((n, d), dtype=np.float64)
        for i in range(n):
            e = int(recv_e[o][i])
            if e not in weights:
                weights[e] = expert_weights(e)
            y[i] = moe.expert_ffn(*weights[e], recv_x[o][i])
        recv_y.append(y)
    back = all_to_all(recv_y, recv_counts)  # the return trip: owners -> sources

    ys = []
    for s in range(G):
        T = np.asarray(xs[s]).shape[0]
        Y = np.zeros((T * k, d), dtype=np.float64)
        Y[order_l[s]] = back[s]  # row i of the block came from flat index order[i]
        y = np.zeros((T, d), dtype=np.float64)
        for t in range(T):
            acc = np.zeros(d, dtype=np.float64)
            for j in range(k):
                acc = acc + w_l[s][t, j] * Y[t * k + j]
            y[t] = acc
        ys.append(y)
    return dict(y=ys, ids=ids_l, w=w_l, send_counts=np.array(counts), records=records)
