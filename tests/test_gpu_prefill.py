"""GPU parity of the prefill path through the C ABI: whole-layer loads with
the next layer copied in behind (layer-ahead double buffer in the shared slot
pool), the tcgen05 grouped GEMM with the fused SwiGLU epilogue, the on-demand
fallback when two layers do not fit, and decode after prefill."""
import dataclasses

import numpy as np
import pytest
import torch

import ftgen
import sparse_moe_expert_topk_b200 as ft
from oracle import moe as omoe
from oracle.cache import DECODE, PREFILL
from parity import ExpertWeights, check_close, check_route_weights, gap_hidden, gpu_route, oracle_cache, to_np

pytestmark = pytest.mark.gpu


def _harness(wl, **kw):
    from ftgen.ctx import Harness
    return Harness(wl, **kw)


def _call(h, oc, W, layer, mode, x, bias, sample=None):
    wl = h.wl
    T = x.shape[0]
    b = None if bias is None else torch.as_tensor(bias).to(h.dev)
    y, ids, w = h.forward(layer, x.to(h.dev), b, mode=mode, want_route=True)
    torch.cuda.synchronize()
    xn = x.float().numpy()
    wr = h.routers[layer].float().cpu().numpy()
    ids_ref, w_ref, _ = omoe.route(xn, wr, bias, wl.k)
    np.testing.assert_array_equal(ids.cpu().numpy(), ids_ref)
    check_route_weights(w.cpu().numpy(), w_ref, xn, wr, f"layer {layer}")
    counts, offsets, perm, inv = omoe.permutation(ids_ref, wl.E)
    r = gpu_route(h, T)
    np.testing.assert_array_equal(r["perm"], perm)
    np.testing.assert_array_equal(r["inv"], inv)
    rec = oc.forward(layer, PREFILL if mode == ft.FT_PREFILL else DECODE, counts)
    assert r["lookup_e"].tolist() == [e for (_, e, _) in rec["lookups"]]
    assert r["lookup_kind"].tolist() == [k for (_, _, k) in rec["lookups"]]
    assert r["n_lookup_cur"] == rec["n_cur"]
    assert (r["m"], r["qstar"], r["qstage"]) == (rec["m"], rec["qstar"], rec["qstage"])
    if sample is not None:
        toks = np.asarray(sample)
        y_ref, _, _ = omoe.layer_forward(xn, wr, bias, wl.k, lambda e: W(layer, e), tokens=toks)
        check_close(to_np(y)[toks], y_ref, wl.wtype, f"layer {layer} tokens {toks[:4]}...")
    return y


def _check_state(h, oc):
    key_of, stamp = ft.ft_moe_cache_contents(h.ctx, h.C)
    assert key_of.tolist() == oc.key_of
    assert stamp.tolist() == oc.stamp
    st = h.stats()
    for k in ("lookups", "hits", "misses", "staged", "streamed", "layer_calls"):
        assert st[k] == oc.n[k], k
    assert st["device_error"] == 0


def test_prefill_bf16_full_layer_T4096(cuda_ok):
    """Single-layer BF16 prefill: T=4096, near-uniform routing (b = 0), every
    expert starts on the host, C = 2E. Routing, permutation and the load
    record bit-exact; outputs of sampled tokens within 2e-2 rms."""
    wl = ftgen.workload("prefill_bf16")
    T = 4096
    with _harness(wl, max_tokens=T) as h:
        oc = oracle_cache(h)
        W = ExpertWeights(h, keep=4)
        x = gap_hidden(wl, T, wl.seed("x", 0), h.routers[0], None)
        rng = np.random.default_rng(0)
        sample = np.sort(np.concatenate([[0, 1, T - 1], rng.choice(T, 9, replace=False)]))
        y = _call(h, oc, W, 0, ft.FT_PREFILL, x, None, sample=sample)
        assert torch.isfinite(y.float()).all()
        # hot: the layer is resident now, a second pass is all hits
        x2 = gap_hidden(wl, T, wl.seed("x", 1), h.routers[0], None)
        _call(h, oc, W, 0, ft.FT_PREFILL, x2, None, sample=sample[:4])
        _check_state(h, oc)
        st = h.stats()
        assert st["misses"] == wl.E and st["hits"] == wl.E


SMALL = ftgen.Workload("prefill_small", L=3, E=32, k=4, d=1024, d_ff=512, wtype=ftgen.W_BF16, cache_slots=64)


@pytest.mark.parametrize("T", [200, 613])
def test_multilayer_prefill_double_buffer_then_decode(cuda_ok, T):
    """3 layers, C = 2E: each prefill call computes layer l and loads l+1;
    then decode steps run on the warm cache (LRU shared by all layers)."""
    wl = SMALL
    with _harness(wl, max_tokens=T) as h:
        oc = oracle_cache(h)
        W = ExpertWeights(h, keep=40)
        for l in range(wl.L):
            x = gap_hidden(wl, T, wl.seed("pf", T, l), h.routers[l], None)
            _call(h, oc, W, l, ft.FT_PREFILL, x, None, sample=[0, 5, T // 2, T - 1])
        for step in range(6):
            for l in range(wl.L):
                x = gap_hidden(wl, 3, wl.seed("dec", T, step, l), h.routers[l], None)
                _call(h, oc, W, l, ft.FT_DECODE, x, None, sample=[0, 1, 2] if step == 2 else None)
        # a second prefill pass, after decode reset the layer-ahead state
        for l in range(wl.L):
            x = gap_hidden(wl, T, wl.seed("pf2", T, l), h.routers[l], None)
            _call(h, oc, W, l, ft.FT_PREFILL, x, None, sample=[1] if l == 1 else None)
        _check_state(h, oc)


def test_prefill_experts_spanning_several_token_tiles(cuda_ok):
    """Skewed prefill (Zipf log-bias on the logits): the heaviest experts get
    several hundred tokens each, more than one 256-token MMA tile, with a
    ragged last tile. Outputs of tokens routed to the heaviest expert, its
    first and last included, within 2e-2 rms."""
    wl = SMALL
    T = 2400
    with _harness(wl, max_tokens=T) as h:
        oc = oracle_cache(h)
        W = ExpertWeights(h, keep=40)
        bias = ftgen.zipf_log_bias(wl.E, 1.1, wl.seed("skew"))
        x = gap_hidden(wl, T, wl.seed("skew-x"), h.routers[0], bias)
        ids_ref, _, _ = omoe.route(x.float().numpy(), h.routers[0].float().cpu().numpy(), bias, wl.k)
        counts = np.bincount(ids_ref.ravel(), minlength=wl.E)
        heavy = int(np.argmax(counts))
        assert counts[heavy] > 256
        toks = np.nonzero((ids_ref == heavy).any(axis=1))[0]
        sample = np.unique(np.concatenate([toks[:2], toks[255:258], toks[-2:]]))
        _call(h, oc, W, 0, ft.FT_PREFILL, x, bias, sample=sample)
        _check_state(h, oc)


def test_prefill_fallback_when_two_layers_do_not_fit(cuda_ok):
    """C < 2E: prefill follows the decode rules (q* split, streamed misses)."""
    wl = dataclasses.replace(SMALL, name="prefill_fallback", cache_slots=40, bp_mbps=11800, bh_mbps=47500)
    T = 96
    with _harness(wl, max_tokens=T) as h:
        oc = oracle_cache(h)
        W = ExpertWeights(h, keep=40)
        for l in range(wl.L):
            x = gap_hidden(wl, T, wl.seed("fb", l), h.routers[l], None)
            _call(h, oc, W, l, ft.FT_PREFILL, x, None, sample=[0, T - 1])
        _check_state(h, oc)
        assert h.stats()["streamed"] > 0


NVFP4_SMALL = ftgen.Workload("mixed_small", L=3, E=32, k=4, d=1024, d_ff=512, wtype=ftgen.W_NVFP4, cache_slots=64,
                             bp_mbps=11800, bh_mbps=47500)


def test_nvfp4_prefill_then_batched_decode(cuda_ok):
    """Mixed-workload sequence at reduced size: NVFP4 prefill of every layer
    (double buffer, C = 2E), then decode at batch 1..8 with Markov routing
    biases on the shared cache, at the 11.8:47.5 profile."""
    wl = NVFP4_SMALL
    T = 300
    with _harness(wl, max_tokens=T) as h:
        oc = oracle_cache(h)
        W = ExpertWeights(h, keep=40)
        for l in range(wl.L):
            x = gap_hidden(wl, T, wl.seed("pf", l), h.routers[l], None)
            _call(h, oc, W, l, ft.FT_PREFILL, x, None, sample=[0, 7, T - 1])
        steps = 5
        traces = [ftgen.markov_trace(steps, 8, wl.E, wl.k, 0.8, 1.1, wl.seed("tr", l)) for l in range(wl.L)]
        zb = [ftgen.zipf_log_bias(wl.E, 1.1, wl.seed("pi", l)) for l in range(wl.L)]
        for st in range(steps):
            B = (1, 2, 4, 8, 8)[st]
            for l in range(wl.L):
                bias = ftgen.trace_bias(traces[l][st][:B], zb[l], 8.0)
                x = gap_hidden(wl, B, wl.seed("dec", st, l), h.routers[l], bias)
                _call(h, oc, W, l, ft.FT_DECODE, x, bias, sample=list(range(B)) if st in (1, 4) else None)
        _check_state(h, oc)
