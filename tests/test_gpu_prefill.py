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
from parity import (ExpertWeights, PrefetchWeights, check_close, check_route_weights, gap_hidden, gpu_route,
                    oracle_cache, to_np)

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
    if sample is not None:  # "all": every token
        toks = None if isinstance(sample, str) else np.asarray(sample)
        y_ref, _, _ = omoe.layer_forward_grouped(xn, wr, bias, wl.k, lambda e: W(layer, e), tokens=toks)
        yg = to_np(y) if toks is None else to_np(y)[toks]
        check_close(yg, y_ref, wl.wtype, f"layer {layer} ({len(y_ref)} tokens)")
    return y


def _check_outputs(h, layer, calls, what=""):
    """Outputs of several calls of one layer against the expert-by-expert
    oracle, each expert decoded once: calls = [(y_gpu, x, bias, tokens)],
    tokens None for every token."""
    wl = h.wl
    wr = h.routers[layer].float().cpu().numpy()
    W = PrefetchWeights(h, layer)
    try:
        res = omoe.layer_forward_batches([(x.float().numpy(), wr, bias, tok) for (_, x, bias, tok) in calls], wl.k, W)
    finally:
        W.close()
    for i, ((y, x, bias, tok), (y_ref, _, _)) in enumerate(zip(calls, res)):
        yg = to_np(y) if tok is None else to_np(y)[np.asarray(tok)]
        check_close(yg, y_ref, wl.wtype, f"{what} call {i} ({len(y_ref)} tokens)")


def _check_state(h, oc):
    key_of, stamp = ft.ft_moe_cache_contents(h.ctx, h.C)
    assert key_of.tolist() == oc.key_of
    assert stamp.tolist() == oc.stamp
    st = h.stats()
    for k in ("lookups", "hits", "misses", "staged", "streamed", "layer_calls"):
        assert st[k] == oc.n[k], k
    assert st["device_error"] == 0


def _expert_sample(ids, E, k, T, n_experts=8, tile=256):
    """Tokens routed to a sample of experts: the first and the last expert,
    the heaviest and the lightest ones, and experts whose token count leaves
    a ragged last MMA tile; every token routed to one of them."""
    counts = np.bincount(ids.ravel(), minlength=E)
    active = np.nonzero(counts)[0]
    pick = {int(active[0]), int(active[-1]), int(np.argmax(counts)), int(active[np.argmin(counts[active])])}
    ragged = [int(e) for e in active if counts[e] % 16 and int(e) not in pick]
    rng = np.random.default_rng(E + T)
    for e in rng.permutation(ragged)[: max(0, n_experts - len(pick))]:
        pick.add(int(e))
    toks = np.nonzero(np.isin(ids, sorted(pick)).any(axis=1))[0]
    return sorted(pick), toks


def test_prefill_bf16_full_layer_T4096(cuda_ok):
    """Single-layer BF16 prefill: T=4096, near-uniform routing (b = 0), every
    expert starts on the host, C = 2E. Routing, permutation and the load
    record bit-exact; the outputs of every token of the cold call, and of
    every token routed to eight sampled experts in the hot call, within
    2e-2 rms."""
    wl = ftgen.workload("prefill_bf16")
    T = 4096
    with _harness(wl, max_tokens=T) as h:
        oc = oracle_cache(h)
        x = gap_hidden(wl, T, wl.seed("x", 0), h.routers[0], None)
        y = _call(h, oc, None, 0, ft.FT_PREFILL, x, None)
        assert torch.isfinite(y.float()).all()
        # hot: the layer is resident now, a second pass is all hits
        x2 = gap_hidden(wl, T, wl.seed("x", 1), h.routers[0], None)
        y2 = _call(h, oc, None, 0, ft.FT_PREFILL, x2, None)
        _check_state(h, oc)
        st = h.stats()
        assert st["misses"] == wl.E and st["hits"] == wl.E
        ids2, _, _ = omoe.route(x2.float().numpy(), h.routers[0].float().cpu().numpy(), None, wl.k)
        picked, toks = _expert_sample(ids2, wl.E, wl.k, T)
        assert 0 in picked and wl.E - 1 in picked and len(picked) >= 8
        _check_outputs(h, 0, [(y, x, None, None), (y2, x2, None, toks)], "T=4096")


def test_prefill_bf16_hot_T16384(cuda_ok):
    """The tensor-bound point: T = 16384 tokens (about 384 per expert, two
    256-token MMA tiles each, the second ragged) on a resident layer.
    Routing bit-exact; outputs of every token routed to eight sampled experts
    (first, last, heaviest, lightest, ragged) within 2e-2 rms."""
    wl = ftgen.workload("prefill_bf16")
    T = 16384
    with _harness(wl, max_tokens=T) as h:
        oc = oracle_cache(h)
        x0 = gap_hidden(wl, 512, wl.seed("warm", 0), h.routers[0], None)
        _call(h, oc, None, 0, ft.FT_PREFILL, x0, None)  # loads the whole layer
        x = gap_hidden(wl, T, wl.seed("x16k", 0), h.routers[0], None)
        y = _call(h, oc, None, 0, ft.FT_PREFILL, x, None)
        _check_state(h, oc)
        assert h.stats()["misses"] == wl.E
        ids, _, _ = omoe.route(x.float().numpy(), h.routers[0].float().cpu().numpy(), None, wl.k)
        counts = np.bincount(ids.ravel(), minlength=wl.E)
        assert (counts > 256).sum() > 0
        picked, toks = _expert_sample(ids, wl.E, wl.k, T)
        _check_outputs(h, 0, [(y, x, None, toks)], "T=16384")


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
            _call(h, oc, W, l, ft.FT_PREFILL, x, None, sample="all")
        for step in range(6):
            for l in range(wl.L):
                x = gap_hidden(wl, 3, wl.seed("dec", T, step, l), h.routers[l], None)
                _call(h, oc, W, l, ft.FT_DECODE, x, None, sample="all")
        # a second prefill pass, after decode reset the layer-ahead state
        for l in range(wl.L):
            x = gap_hidden(wl, T, wl.seed("pf2", T, l), h.routers[l], None)
            _call(h, oc, W, l, ft.FT_PREFILL, x, None, sample="all")
        _check_state(h, oc)


def test_prefill_experts_spanning_several_token_tiles(cuda_ok):
    """Skewed prefill (Zipf log-bias on the logits): the heaviest experts get
    several hundred tokens each, more than one 256-token MMA tile, with a
    ragged last tile. Outputs of every token within 2e-2 rms."""
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
        _call(h, oc, W, 0, ft.FT_PREFILL, x, bias, sample="all")
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
            _call(h, oc, W, l, ft.FT_PREFILL, x, None, sample="all")
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
            _call(h, oc, W, l, ft.FT_PREFILL, x, None, sample="all")
        steps = 5
        traces = [ftgen.markov_trace(steps, 8, wl.E, wl.k, 0.8, 1.1, wl.seed("tr", l)) for l in range(wl.L)]
        zb = [ftgen.zipf_log_bias(wl.E, 1.1, wl.seed("pi", l)) for l in range(wl.L)]
        for st in range(steps):
            B = (1, 2, 4, 8, 8)[st]
            for l in range(wl.L):
                bias = ftgen.trace_bias(traces[l][st][:B], zb[l], 8.0)
                x = gap_hidden(wl, B, wl.seed("dec", st, l), h.routers[l], bias)
                _call(h, oc, W, l, ft.FT_DECODE, x, bias, sample="all")
        _check_state(h, oc)


def test_nvfp4_prefill_full_shape(cuda_ok):
    """The mixed workload's prefill at full layer shape (NVFP4, E = 256,
    top-6, d = 4096, d_ff = 1536), two layers with the layer-ahead double
    buffer (C = 2E), T = 1024 near-uniformly routed tokens per layer. Routing
    and the load record bit-exact; every token's output within 4e-2 rms."""
    base = ftgen.workload("mixed_nvfp4")
    wl = dataclasses.replace(base, name="nvfp4_prefill_full", L=2, cache_slots=2 * base.E)
    T = 1024
    with _harness(wl, max_tokens=T) as h:
        oc = oracle_cache(h)
        for l in range(wl.L):
            x = gap_hidden(wl, T, wl.seed("pf", l), h.routers[l], None)
            y = _call(h, oc, None, l, ft.FT_PREFILL, x, None)
            _check_outputs(h, l, [(y, x, None, None)], f"layer {l}")
        _check_state(h, oc)
        assert h.stats()["misses"] == wl.L * wl.E
