"""GPU parity of the elastic slot pool (ft_moe_resize_cache) against the
oracle's resize rule: which entries survive, where they land, their stamps,
the LRU sequence after the resize, and outputs computed from moved slots."""
import numpy as np
import pytest
import torch

import ftgen
import sparse_moe_expert_topk_b200 as ft
from oracle import moe as omoe
from oracle.cache import DECODE, PREFILL
from parity import ExpertWeights, check_close, gap_hidden, gpu_route, oracle_cache, to_np

pytestmark = pytest.mark.gpu

WL = ftgen.Workload("resize_small", L=3, E=32, k=4, d=1024, d_ff=512, wtype=ftgen.W_BF16, cache_slots=40,
                    bp_mbps=52700, bh_mbps=77300)


def _call(h, oc, W, layer, mode, x, bias, check_y):
    wl = h.wl
    T = x.shape[0]
    b = None if bias is None else torch.as_tensor(bias).to(h.dev)
    y = h.forward(layer, x.to(h.dev), b, mode=mode)
    torch.cuda.synchronize()
    xn = x.float().numpy()
    wr = h.routers[layer].float().cpu().numpy()
    ids_ref, _, _ = omoe.route(xn, wr, bias, wl.k)
    counts = omoe.permutation(ids_ref, wl.E)[0]
    rec = oc.forward(layer, PREFILL if mode == ft.FT_PREFILL else DECODE, counts)
    r = gpu_route(h, T)
    assert r["lookup_e"].tolist() == [e for (_, e, _) in rec["lookups"]]
    assert r["lookup_kind"].tolist() == [k for (_, _, k) in rec["lookups"]]
    assert (r["m"], r["qstar"], r["qstage"]) == (rec["m"], rec["qstar"], rec["qstage"])
    if check_y:
        y_ref, _, _ = omoe.layer_forward(xn, wr, bias, wl.k, lambda e: W(layer, e))
        check_close(to_np(y), y_ref, wl.wtype, f"layer {layer}")


def _resize(h, oc, n):
    ft.ft_moe_resize_cache(h.ctx, n)
    oc.resize(n)
    h.C = n
    key_of, stamp = ft.ft_moe_cache_contents(h.ctx, n)
    assert key_of.tolist() == oc.key_of
    assert stamp.tolist() == oc.stamp


def test_resize_schedule_decode_and_prefill(cuda_ok):
    """Decode at batch 4 with a Zipf bias, the pool resized 40 -> 12 -> 96
    (every expert of every layer) -> 64 (prefill double buffer on, tcgen05
    path) -> 0 (everything streamed) -> 20, with outputs checked right after
    each resize, when hits are read from slots that moved."""
    wl = WL
    zb = ftgen.zipf_log_bias(wl.E, 1.1, wl.seed("zipf"))
    with _harness(max_tokens=256) as h:
        oc = oracle_cache(h)
        W = ExpertWeights(h, keep=96)
        step = 0

        def decode(n_steps, check_first=True):
            nonlocal step
            for i in range(n_steps):
                for l in range(wl.L):
                    x = gap_hidden(wl, 4, wl.seed("dec", step, l), h.routers[l], zb)
                    _call(h, oc, W, l, ft.FT_DECODE, x, zb, check_y=check_first and i == 0)
                step += 1

        decode(4)
        for n in (12, 96):
            _resize(h, oc, n)
            decode(3)
        _resize(h, oc, 64)
        for l in range(wl.L):
            x = gap_hidden(wl, 200, wl.seed("pf", l), h.routers[l], None)
            _call(h, oc, W, l, ft.FT_PREFILL, x, None, check_y=(l == 1))
        decode(2)
        _resize(h, oc, 0)
        decode(2)
        assert h.stats()["device_error"] == 0
        _resize(h, oc, 20)
        decode(3)
        st = h.stats()
        for k in ("lookups", "hits", "misses", "staged", "streamed"):
            assert st[k] == oc.n[k], k
        assert st["device_error"] == 0


def test_resize_failure_leaves_context_unchanged(cuda_ok, monkeypatch):
    """An allocation failure (injected on the host) returns FT_ENOMEM and the
    cache keeps its size, contents and behaviour; range errors are FT_EINVAL."""
    wl = WL
    with _harness(max_tokens=16) as h:
        oc = oracle_cache(h)
        W = ExpertWeights(h, keep=8)
        for s in range(3):
            for l in range(wl.L):
                x = gap_hidden(wl, 4, wl.seed("f", s, l), h.routers[l], None)
                _call(h, oc, W, l, ft.FT_DECODE, x, None, check_y=False)
        before = ft.ft_moe_cache_contents(h.ctx, h.C)
        monkeypatch.setenv("FT_FAULT", "resize_alloc")
        with pytest.raises(ft.FtError) as ei:
            ft.ft_moe_resize_cache(h.ctx, 10)
        assert ei.value.status == ft.FT_ENOMEM
        monkeypatch.delenv("FT_FAULT")
        for bad in (-1, wl.L * wl.E + 1):
            with pytest.raises(ft.FtError) as ei:
                ft.ft_moe_resize_cache(h.ctx, bad)
            assert ei.value.status == ft.FT_EINVAL
        after = ft.ft_moe_cache_contents(h.ctx, h.C)
        assert before[0].tolist() == after[0].tolist() and before[1].tolist() == after[1].tolist()
        x = gap_hidden(wl, 4, wl.seed("f", 9, 0), h.routers[0], None)
        _call(h, oc, W, 0, ft.FT_DECODE, x, None, check_y=True)


def _harness(**kw):
    from ftgen.ctx import Harness
    return Harness(WL, **kw)
