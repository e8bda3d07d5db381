"""The expert-parallel exchange of sparse_moe_expert_topk_b200.ep on two gloo
ranks (one process per rank, as torchrun starts them), with the compute
steps taken by the oracle on the CPU: the layer's result on each rank must
equal the one-device oracle layer exactly, and each owner's cache record the
oracle's G-device simulation."""
import json
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
E, K, D, DFF, L, G = 8, 3, 12, 16, 3, 2
STEPS = 3
TOKENS = [[3, 2], [0, 4], [5, 1]]  # per step, tokens of rank 0 and rank 1 (rank 0 empty at step 1)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _model():
    rng = np.random.default_rng(2026)
    wr = [rng.normal(0, 0.5, (E, D)) for _ in range(L)]
    W = [[(rng.normal(0, 0.3, (DFF, D)), rng.normal(0, 0.3, (DFF, D)), rng.normal(0, 0.3, (D, DFF)))
          for _ in range(E)] for _ in range(L)]
    return wr, W


def _tokens(step, layer, rank):
    rng = np.random.default_rng([step, layer, rank])
    return rng.normal(0, 1, (TOKENS[step][rank], D))


class OracleOps:
    """The compute steps on the CPU, in fp64, from the oracle."""

    def __init__(self, rank, wr, W):
        from oracle import cache as ocache
        self.rank, self.wr, self.W = rank, wr, W
        self.cache = ocache.ExpertCache(L, E // G, 2, 52700, 77300)
        self.records = []

    def dispatch(self, layer, x, bias):
        import torch
        from oracle import ep, moe
        xn = x.numpy()
        T = xn.shape[0]
        if T:
            ids, w, _ = moe.route(xn, self.wr[layer], bias, K)
        else:
            ids, w = np.zeros((0, K), np.int32), np.zeros((0, K))
        sc, order, eids = ep.dispatch_plan(ids, E, G)
        rows = torch.from_numpy(xn[order // K].copy()) if T else torch.zeros((0, D), dtype=torch.float64)
        return rows, torch.from_numpy(eids.astype(np.int64)), sc.tolist(), (order, w, T)

    def experts(self, layer, mode, rows, eids):
        import torch
        from oracle import moe
        n0 = self.rank * (E // G)
        local = np.zeros(E // G, dtype=np.int64)
        for e in eids.tolist():
            assert n0 <= e < n0 + E // G
            local[e - n0] += 1
        self.records.append(self.cache.forward(layer, mode, local))
        out = np.zeros((rows.shape[0], D))
        for i, e in enumerate(eids.tolist()):
            out[i] = moe.expert_ffn(*self.W[layer][e], rows[i].numpy())
        return torch.from_numpy(out)

    def combine(self, back, state):
        import torch
        order, w, T = state
        Y = np.zeros((T * K, D))
        Y[order] = back.numpy()
        y = np.zeros((T, D))
        for t in range(T):
            for j in range(K):
                y[t] = y[t] + w[t, j] * Y[t * K + j]
        return torch.from_numpy(y)


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist
    from sparse_moe_expert_topk_b200.ep import ExpertParallelLayer
    from oracle import moe
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    wr, W = _model()
    ops = OracleOps(rank, wr, W)
    layer_fn = ExpertParallelLayer(ops, E)
    res = {"owned": list(layer_fn.owned), "exact": [], "records": []}
    for step in range(STEPS):
        for layer in range(L):
            x = _tokens(step, layer, rank)
            y = layer_fn.forward(layer, 0, torch.from_numpy(x))
            if x.shape[0]:
                y1, _, _ = moe.layer_forward(x, wr[layer], None, K, lambda e: W[layer][e])
                res["exact"].append(bool(np.array_equal(y.numpy(), y1)))
            else:
                res["exact"].append(tuple(y.shape) == (0, D))
    res["records"] = [[list(map(list, r["lookups"])), r["m"], r["qstar"], r["qstage"]] for r in ops.records]
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


def test_expert_parallel_layer_on_two_gloo_ranks(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(G, port, str(tmp_path)), nprocs=G, start_method="spawn")
    got = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(G)]

    from oracle import cache as ocache
    from oracle import ep
    wr, W = _model()
    caches = [ocache.ExpertCache(L, E // G, 2, 52700, 77300) for _ in range(G)]
    want = [[] for _ in range(G)]
    for step in range(STEPS):
        for layer in range(L):
            xs = [_tokens(step, layer, r) for r in range(G)]
            out = ep.ep_layer_forward(xs, wr[layer], None, K, lambda e: W[layer][e], G, caches, layer)
            for r in range(G):
                rec = out["records"][r]
                want[r].append([list(map(list, rec["lookups"])), rec["m"], rec["qstar"], rec["qstage"]])
    for r in range(G):
        assert got[r]["owned"] == list(range(r * E // G, (r + 1) * E // G))
        assert all(got[r]["exact"]), got[r]["exact"]
        assert got[r]["records"] == want[r]


def test_owned_experts_blocks():
    from sparse_moe_expert_topk_b200.ep import owned_experts
    assert [list(owned_experts(8, 4, r)) for r in range(4)] == [[0, 1], [2, 3], [4, 5], [6, 7]]
    assert list(owned_experts(256, 1, 0)) == list(range(256))
    with pytest.raises(ValueError):
        owned_experts(256, 3, 0)


def test_dispatch_counts_are_checked_before_any_exchange():
    """A dispatch whose counts do not cover its rows is refused on the host,
    before the first collective (one gloo rank in this process)."""
    import datetime

    import torch
    import torch.distributed as dist
    from sparse_moe_expert_topk_b200.ep import ExpertParallelLayer

    class BadOps:
        def dispatch(self, layer, x, bias):
            return x, torch.zeros(x.shape[0], dtype=torch.int64), [x.shape[0] + 1], None

    store = dist.HashStore()
    dist.init_process_group("gloo", store=store, rank=0, world_size=1, timeout=datetime.timedelta(seconds=30))
    try:
        layer = ExpertParallelLayer(BadOps(), 4)
        with pytest.raises(ValueError):
            layer.forward(0, 0, torch.zeros((3, 2), dtype=torch.float64))
    finally:
        dist.destroy_process_group()


class _SmallOwnerOps(OracleOps):
    """OracleOps whose owner on rank 1 takes at most two rows per call."""

    def __init__(self, rank, wr, W):
        super().__init__(rank, wr, W)
        self.max_rows = 2 if rank == 1 else 10 ** 6


def _rank_small_owner(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist
    from sparse_moe_expert_topk_b200.ep import ExpertParallelLayer
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    wr, W = _model()
    layer_fn = ExpertParallelLayer(_SmallOwnerOps(rank, wr, W), E)
    res = {}
    try:
        layer_fn.forward(0, 0, torch.from_numpy(_tokens(0, 0, rank)))  # 3 + 2 tokens, k = 3: 15 rows
        res["raised"] = False
    except ValueError as e:
        res["raised"] = "owner cannot take" in str(e)
    # both ranks are still in step: a later collective completes
    t = torch.ones(1)
    dist.all_reduce(t)
    res["after"] = float(t.item())
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"small{rank}.json"), "w") as f:
        json.dump(res, f)


def test_owner_capacity_is_agreed_before_rows_move(tmp_path):
    """One owner too small for what it is sent: every rank raises the same
    error before the row exchange, and no rank is left waiting (a collective
    after the failed call completes on both)."""
    port = _free_port()
    mp.start_processes(_rank_small_owner, args=(G, port, str(tmp_path)), nprocs=G, start_method="spawn")
    got = [json.load(open(tmp_path / f"small{r}.json")) for r in range(G)]
    assert all(g["raised"] for g in got), got
    assert all(g["after"] == G for g in got), got
