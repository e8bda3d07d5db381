"""GPU parity of the expert-parallel layer through the C ABI.

G devices' shares of the experts are held by G contexts on one GPU (each with
E/G local experts, its own pool, slots and LRU); the exchange between them is
done with tensor copies in the order the all-to-alls of
sparse_moe_expert_topk_b200.ep produce (blocks of sources 0..G-1 per owner,
then the return trip). Against the oracle (oracle/ep.py, oracle/moe.py):
routing ids, the pack order, the rows per owner, the inverse order and each
owner's lookup record bit-exact; the layer's outputs within the BF16
tolerance. The module layer (ExpertParallelLayer with CudaEpOps) on a
one-rank NCCL group gives the one-device forward's outputs bit for bit."""
import numpy as np
import pytest
import torch

import ftgen
import sparse_moe_expert_topk_b200 as ft
from oracle import cache as ocache
from oracle import ep as oep
from oracle import moe as omoe
from parity import ExpertWeights, check_close, gap_hidden, to_np

pytestmark = pytest.mark.gpu


class Owners:
    """G contexts, context o holding global experts [o E/G, (o+1) E/G)."""

    def __init__(self, wl, G, slots, max_rows):
        from ftgen.ctx import Harness
        self.wl, self.G, self.Eg = wl, G, wl.E // G
        self.h = [Harness(wl, cache_slots=slots, max_tokens=max_rows, expert_base=o * self.Eg, n_experts=self.Eg)
                  for o in range(G)]
        self.ws = [ExpertWeights(h, keep=8) for h in self.h]
        self.oc = [ocache.ExpertCache(1, self.Eg, slots, wl.bp_mbps, wl.bh_mbps) for _ in range(G)]
        self.routers = self.h[0].routers  # the full [E, d] routers (same seeds on every context)
        self.dev = self.h[0].dev

    def weights(self, layer, e):
        return self.ws[e // self.Eg](layer, e % self.Eg)

    def close(self):
        for h in self.h:
            h.close()


def _pack(ow, x, bias):
    """Route and pack one source's tokens with the library."""
    wl, dev = ow.wl, ow.dev
    T, k = x.shape[0], wl.k
    x = x.to(dev)
    b = None if bias is None else torch.as_tensor(bias, dtype=torch.float32).to(dev)
    ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    if T:
        ft.ft_route_topk_static(x, ow.routers[0], b, 0, T, wl.E, wl.d, k, wl.wtype, ids, w, None)
    n = T * k
    scratch = torch.empty(ft.ft_ep_pack_scratch_bytes(T, k, wl.E), dtype=torch.uint8, device=dev)
    rows = torch.empty((n, wl.d), dtype=x.dtype, device=dev)
    eids = torch.empty(n, dtype=torch.int32, device=dev)
    counts = torch.empty(ow.G, dtype=torch.int64, device=dev)
    inv = torch.empty(n, dtype=torch.int32, device=dev)
    bad = torch.empty(1, dtype=torch.int32, device=dev)
    ft.ft_ep_pack(ids, T, k, wl.E, ow.G, x, wl.d, wl.wtype, rows, eids, counts, inv, bad, scratch, None)
    torch.cuda.synchronize()
    assert bad.item() == 0
    return dict(x=x, ids=ids, w=w, rows=rows, eids=eids, counts=counts.tolist(), inv=inv, T=T)


def _layer(ow, xs, bias, mode=ft.FT_DECODE, check_y=True, sample=None):
    """One expert-parallel layer call over the sources xs; checks everything
    against the oracle and returns the outputs."""
    wl, G, k = ow.wl, ow.G, ow.wl.k
    src = [_pack(ow, x, bias) for x in xs]
    router = ow.routers[0].float().cpu().numpy()
    for s, p in enumerate(src):
        if p["T"] == 0:
            assert p["counts"] == [0] * G
            continue
        xn = xs[s].float().numpy()
        ids_ref, _, _ = omoe.route(xn, router, bias, k)
        np.testing.assert_array_equal(p["ids"].cpu().numpy(), ids_ref)
        sc, order, eids = oep.dispatch_plan(ids_ref, wl.E, G)
        assert p["counts"] == sc.tolist()
        np.testing.assert_array_equal(p["eids"].cpu().numpy(), eids)
        _, _, _, inv = omoe.permutation(ids_ref, wl.E)
        np.testing.assert_array_equal(p["inv"].cpu().numpy(), inv)
        np.testing.assert_array_equal(p["rows"].cpu().float().numpy(), xn[order // k])
    # the exchange: owner o receives the blocks of sources 0..G-1 in order
    offs = [np.concatenate([[0], np.cumsum(p["counts"])]) for p in src]
    outs = []
    for o in range(G):
        rows = torch.cat([p["rows"][offs[s][o]:offs[s][o + 1]] for s, p in enumerate(src)])
        eids = torch.cat([p["eids"][offs[s][o]:offs[s][o + 1]] for s, p in enumerate(src)])
        n = rows.shape[0]
        out = torch.empty((n, wl.d), dtype=torch.float32, device=ow.dev)
        ft.ft_moe_expert_rows(ow.h[o].ctx, 0, mode, rows, eids, o * ow.Eg, n, out)
        outs.append(out)
        local = np.bincount(eids.cpu().numpy() - o * ow.Eg, minlength=ow.Eg) if n else np.zeros(ow.Eg, np.int64)
        rec = ow.oc[o].forward(0, ocache.DECODE if mode == ft.FT_DECODE else ocache.PREFILL, local)
        if n:
            r = ft.ft_moe_last_route(ow.h[o].ctx, ow.Eg, n)
            assert r["lookup_e"].tolist() == [e for (_, e, _) in rec["lookups"]]
            assert r["lookup_kind"].tolist() == [kk for (_, _, kk) in rec["lookups"]]
    # the return trip and the combine at each source
    ys = []
    for s, p in enumerate(src):
        back = torch.cat([outs[o][sum(src[q]["counts"][o] for q in range(s)):
                                  sum(src[q]["counts"][o] for q in range(s + 1))] for o in range(G)])
        y = torch.empty((p["T"], wl.d), dtype=p["x"].dtype, device=ow.dev)
        ft.ft_ep_combine(back, p["w"], p["inv"], p["T"], k, wl.d, wl.wtype, y, None)
        ys.append(y)
    torch.cuda.synchronize()
    if check_y:
        for s, x in enumerate(xs):
            if x.shape[0] == 0:
                continue
            tok = np.arange(x.shape[0]) if sample is None else sample[: x.shape[0]]
            y_ref, _, _ = omoe.layer_forward(x.float().numpy(), router, bias, k, lambda e: ow.weights(0, e),
                                             tokens=tok)
            check_close(to_np(ys[s])[tok], y_ref, wl.wtype, f"source {s}")
    return ys


def _check_counters(ow):
    for o in range(ow.G):
        st = ow.h[o].stats()
        for key in ("lookups", "hits", "misses", "staged", "streamed"):
            assert st[key] == ow.oc[o].n[key], (o, key)
        assert st["device_error"] == 0
        key_of, stamp = ft.ft_moe_cache_contents(ow.h[o].ctx, ow.h[o].C)
        assert key_of.tolist() == ow.oc[o].key_of and stamp.tolist() == ow.oc[o].stamp


@pytest.mark.parametrize("G", [2, 4])
def test_ep_decode_bf16(cuda_ok, G):
    wl = ftgen.workload("decode_bf16")
    bias = ftgen.zipf_log_bias(wl.E, 1.1, wl.seed("zipf"))
    Ts = [1, 4, 16, 0][:G] if G == 4 else [16, 1]
    ow = Owners(wl, G, slots=96 // G, max_rows=sum(Ts) * wl.k)
    try:
        for step in range(12):
            xs = [gap_hidden(wl, T, wl.seed("ep", G, s, step), ow.routers[0], bias) if T else
                  torch.zeros((0, wl.d), dtype=torch.bfloat16) for s, T in enumerate(Ts)]
            _layer(ow, xs, bias, check_y=(step % 4 == 1))
        _check_counters(ow)
    finally:
        ow.close()


def test_ep_prefill_bf16_full_layer(cuda_ok):
    """Owners with room for two layers of their share take the prefill path
    (whole layer resident, tcgen05 GEMM); rows from two sources of 300 tokens."""
    wl = ftgen.workload("prefill_bf16")
    G, Ts = 2, [300, 300]
    ow = Owners(wl, G, slots=2 * wl.E // G, max_rows=sum(Ts) * wl.k)
    try:
        xs = [gap_hidden(wl, T, wl.seed("ep_prefill", s), ow.routers[0], None) for s, T in enumerate(Ts)]
        sample = np.array([0, 1, 2, 77, 150, 299])
        _layer(ow, xs, None, mode=ft.FT_PREFILL, sample=sample)
    finally:
        ow.close()


def test_ep_layer_module_on_one_nccl_rank(cuda_ok):
    """ExpertParallelLayer with CudaEpOps on a one-rank NCCL group: the owner
    holds every expert, the all-to-alls are local, and the layer must agree
    with the one-device forward of a context over the same pool and router:
    the same cache counters, and the same output bytes (at up to 32 tokens
    both route with the same logits code, every expert row is computed by the
    same GEMV with the same K order, and both combine in rank order)."""
    import datetime
    import os

    import torch.distributed as dist
    from ftgen.ctx import Harness
    from sparse_moe_expert_topk_b200.ep import CudaEpOps, ExpertParallelLayer

    wl = ftgen.workload("decode_bf16")
    bias = ftgen.zipf_log_bias(wl.E, 1.1, wl.seed("zipf"))
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", "29561")
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    one = Harness(wl, cache_slots=48, max_tokens=16)
    own = Harness(wl, cache_slots=48, max_tokens=16 * wl.k, expert_base=0, n_experts=wl.E, fill=True)
    try:
        ops = CudaEpOps(own.ctx, own.routers, wl.E, wl.k, wl.d, wl.wtype, stream=own.stream, max_rows=16 * wl.k)
        layer = ExpertParallelLayer(ops, wl.E)
        b = torch.as_tensor(bias, dtype=torch.float32).to(own.dev)
        for step, T in enumerate([1, 4, 16, 16, 4, 1]):
            x = gap_hidden(wl, T, wl.seed("ep_one", step), own.routers[0], bias).to(own.dev)
            y_ep = layer.forward(0, ft.FT_DECODE, x, b)
            y_one = one.forward(0, x, b)
            torch.cuda.synchronize()
            check_close(to_np(y_ep), to_np(y_one).astype(np.float64), wl.wtype, f"step {step}")
            assert torch.equal(y_ep.view(torch.int16), y_one.view(torch.int16)), f"step {step}"
        s_one, s_own = one.stats(), own.stats()
        for key in ("lookups", "hits", "misses", "staged", "streamed"):
            assert s_one[key] == s_own[key], key
    finally:
        one.close()
        own.close()
        dist.destroy_process_group()
