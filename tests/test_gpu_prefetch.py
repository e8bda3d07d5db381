"""GPU parity of the decode prefetch (ft_moe_set_prefetch) against the
oracle's prefetch mode: after each decode lookup the next layer's experts of
its last call are staged; the lookup record, q*, the cache contents and
stamps after every call, the counters and sampled outputs must match."""
import dataclasses

import numpy as np
import pytest
import torch

import ftgen
import sparse_moe_expert_topk_b200 as ft
from oracle import moe as omoe
from oracle.cache import DECODE
from parity import ExpertWeights, check_close, gap_hidden, gpu_route, oracle_cache, to_np

pytestmark = pytest.mark.gpu

WL = ftgen.Workload("prefetch_small", L=3, E=32, k=4, d=1024, d_ff=512, wtype=ftgen.W_BF16, cache_slots=24,
                    bp_mbps=52700, bh_mbps=77300)


def _harness(wl, **kw):
    from ftgen.ctx import Harness
    return Harness(wl, **kw)


@pytest.mark.parametrize("L", [3, 1])
def test_prefetch_matches_oracle(cuda_ok, L):
    wl = dataclasses.replace(WL, L=L, cache_slots=24 if L == 3 else 10)
    B, steps = 2, 10
    with _harness(wl, max_tokens=B) as h:
        oc = oracle_cache(h)
        oc.prefetch_on = True
        ft.ft_moe_set_prefetch(h.ctx, 1)
        W = ExpertWeights(h, keep=64)
        traces = [ftgen.markov_trace(steps, B, wl.E, wl.k, 0.8, 1.1, wl.seed("pf-trace", l)) for l in range(L)]
        zb = [ftgen.zipf_log_bias(wl.E, 1.1, wl.seed("pf-pi", l)) for l in range(L)]
        for st in range(steps):
            for l in range(L):
                bias = ftgen.trace_bias(traces[l][st], zb[l], 8.0)
                x = gap_hidden(wl, B, wl.seed("pf-x", st, l), h.routers[l], bias)
                y = h.forward(l, x.to(h.dev), torch.as_tensor(bias).to(h.dev))
                torch.cuda.synchronize()
                xn = x.float().numpy()
                wr = h.routers[l].float().cpu().numpy()
                ids_ref, _, _ = omoe.route(xn, wr, bias, wl.k)
                counts = omoe.permutation(ids_ref, wl.E)[0]
                rec = oc.forward(l, DECODE, counts)
                r = gpu_route(h, B)
                assert r["lookup_e"].tolist() == [e for (_, e, _) in rec["lookups"]], (st, l)
                assert r["lookup_kind"].tolist() == [k for (_, _, k) in rec["lookups"]], (st, l)
                assert (r["m"], r["qstar"], r["qstage"]) == (rec["m"], rec["qstar"], rec["qstage"])
                key_of, stamp = ft.ft_moe_cache_contents(h.ctx, h.C)
                assert key_of.tolist() == oc.key_of, (st, l)
                assert stamp.tolist() == oc.stamp, (st, l)
                if st % 3 == 2:
                    y_ref, _, _ = omoe.layer_forward(xn, wr, bias, wl.k, lambda e: W(l, e))
                    check_close(to_np(y), y_ref, wl.wtype, f"step {st} layer {l}")
        stt = h.stats()
        for k in ("lookups", "hits", "misses", "staged", "streamed", "prefetched"):
            assert stt[k] == oc.n[k], k
        assert stt["prefetched"] > 0 and stt["device_error"] == 0
