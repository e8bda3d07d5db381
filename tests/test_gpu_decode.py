"""GPU parity of the decode path through the C ABI against the oracle:
routing ids, permutation, LRU hit/staged/streamed sequence and q* bit-exact;
layer outputs within the stated tolerance."""
import numpy as np
import pytest
import torch

import ftgen
import sparse_moe_expert_topk_b200 as ft
from oracle import moe as omoe
from oracle.cache import DECODE
from parity import (ExpertWeights, ParallelExpertWeights, check_close, check_route_weights, gap_hidden, gpu_route,
                    oracle_cache, to_np)

pytestmark = pytest.mark.gpu


def _harness(wl, **kw):
    from ftgen.ctx import Harness
    return Harness(wl, **kw)


def _run_and_check(h, oc, W, layer, x, bias, check_y=True, mode=ft.FT_DECODE):
    wl = h.wl
    T = x.shape[0]
    y, ids, w = h.forward(layer, x.to(h.dev), None if bias is None else torch.as_tensor(bias).to(h.dev),
                          mode=mode, want_route=True)
    torch.cuda.synchronize()
    xn = x.float().numpy()
    ids_ref, w_ref, _ = omoe.route(xn, h.routers[layer].float().cpu().numpy(), bias, wl.k)
    np.testing.assert_array_equal(ids.cpu().numpy(), ids_ref)
    check_route_weights(w.cpu().numpy(), w_ref, xn, h.routers[layer].float().cpu().numpy(), f"layer {layer}")
    counts, offsets, perm, inv = omoe.permutation(ids_ref, wl.E)
    r = gpu_route(h, T)
    np.testing.assert_array_equal(r["counts"], counts)
    np.testing.assert_array_equal(r["offsets"], offsets)
    np.testing.assert_array_equal(r["perm"], perm)
    np.testing.assert_array_equal(r["inv"], inv)
    rec = oc.forward(layer, DECODE if mode == ft.FT_DECODE else 1, counts)
    assert r["lookup_e"].tolist() == [e for (_, e, _) in rec["lookups"]]
    assert r["lookup_kind"].tolist() == [k for (_, _, k) in rec["lookups"]]
    assert r["n_lookup_cur"] == rec["n_cur"]
    if mode == ft.FT_DECODE:
        assert (r["m"], r["qstar"], r["qstage"]) == (rec["m"], rec["qstar"], rec["qstage"])
    rel = None
    if check_y:
        if hasattr(W, "need"):
            W.need(layer, np.unique(ids_ref))
        y_ref, _, _ = omoe.layer_forward_grouped(xn, h.routers[layer].float().cpu().numpy(), bias, wl.k,
                                                 lambda e: W(layer, e))
        rel = check_close(to_np(y), y_ref, wl.wtype, f"layer {layer}")
    return y, rel


def _check_cache_state(h, oc):
    key_of, stamp = ft.ft_moe_cache_contents(h.ctx, h.C)
    assert key_of.tolist() == oc.key_of
    assert stamp.tolist() == oc.stamp
    st = h.stats()
    for k in ("lookups", "hits", "misses", "staged", "streamed", "layer_calls"):
        assert st[k] == oc.n[k], k
    assert st["device_error"] == 0


def test_tiny_f32_layer(cuda_ok):
    wl = ftgen.workload("tiny_f32")
    with _harness(wl, gen_device="cpu") as h:
        oc = oracle_cache(h)
        W = ExpertWeights(h)
        for step in range(6):  # a few calls so the 4-slot cache evicts
            x = gap_hidden(wl, 16, wl.seed("x", step), h.routers[0], None)
            _, rel = _run_and_check(h, oc, W, 0, x, None)
            assert rel <= 1e-4
        _check_cache_state(h, oc)


@pytest.mark.parametrize("T", [1, 4, 16])
def test_decode_bf16_64_steps(cuda_ok, T):
    """The decode trace of the default workload at batch 1, 4 and 16: routing,
    permutation, the lookup record and q* of every call bit-exact, and every
    call's outputs within 2e-2 rms."""
    wl = ftgen.workload("decode_bf16")
    bias = ftgen.zipf_log_bias(wl.E, 1.1, wl.seed("zipf"))
    with _harness(wl, max_tokens=16) as h:
        oc = oracle_cache(h)
        W = ParallelExpertWeights(h, keep=64)
        for step in range(wl.steps):
            x = gap_hidden(wl, T, wl.seed("x", T, step), h.routers[0], bias)
            _run_and_check(h, oc, W, 0, x, bias, check_y=True)
        W.close()
        _check_cache_state(h, oc)
        st = h.stats()
        assert st["misses"] > 0 and st["hits"] > 0 and st["staged"] > 0 and st["streamed"] > 0
        # device time of the calls and of their staging copies, through the ABI
        assert st["ms_compute"] > 0 and st["ms_copy"] > 0
        ft.ft_moe_reset_cache(h.ctx)
        st = h.stats()
        assert st["ms_compute"] == 0 and st["ms_copy"] == 0


def test_outputs_independent_of_cache_state(cuda_ok):
    """Same inputs under all-cold (C=0, everything streamed), q*=0, q*=m and
    a warm cache: bit-identical outputs."""
    wl = ftgen.workload("decode_bf16")
    bias = ftgen.zipf_log_bias(wl.E, 1.1, wl.seed("zipf"))
    xs = None
    outs = {}
    for name, C, bp, bh, warm in (("cold", 0, 1, 1, 0), ("q0", 94, 0, 77300, 0), ("qm", 94, 77300, 77300, 0),
                                  ("warm", 256, 52700, 77300, 3)):
        with _harness(wl, cache_slots=C, max_tokens=16) as h:
            ft.ft_set_bandwidths(h.ctx, bp, bh)
            if xs is None:
                xs = [gap_hidden(wl, 16, wl.seed("inv", i), h.routers[0], bias) for i in range(3)]
            b = torch.as_tensor(bias).to(h.dev)
            for _ in range(warm):
                for x in xs:
                    h.forward(0, x.to(h.dev), b)
            outs[name] = [h.forward(0, x.to(h.dev), b).cpu() for x in xs]
            torch.cuda.synchronize()
    for name in ("q0", "qm", "warm"):
        for a, b in zip(outs["cold"], outs[name]):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16)), name


@pytest.mark.parametrize("T", [0, 3, 13])
def test_ragged_and_empty_batches(cuda_ok, T):
    wl = ftgen.workload("decode_bf16")
    with _harness(wl, max_tokens=16) as h:
        oc = oracle_cache(h)
        W = ExpertWeights(h, keep=8)
        if T == 0:
            x = torch.zeros(0, wl.d, dtype=torch.bfloat16)
            h.forward(0, x.to(h.dev))
            assert h.stats()["lookups"] == 0
            return
        for step in range(3):
            x = gap_hidden(wl, T, wl.seed("ragged", T, step), h.routers[0], None)
            _run_and_check(h, oc, W, 0, x, None)
        _check_cache_state(h, oc)


def test_nvfp4_multilayer_trace(cuda_ok):
    """43-layer NVFP4 workload shape, reduced to 4 layers and 24 steps, with
    the Markov routing trace realised as a per-token bias; shared LRU; every
    call's outputs checked."""
    base = ftgen.workload("trace_nvfp4")
    L, steps = 4, 24
    import dataclasses
    wl = dataclasses.replace(base, L=L, cache_slots=int(0.37 * L * base.E))
    with _harness(wl, max_tokens=4) as h:
        oc = oracle_cache(h)
        W = ParallelExpertWeights(h, keep=96)
        traces = [ftgen.markov_trace(steps, 1, wl.E, wl.k, 0.8, 1.1, wl.seed("trace", l)) for l in range(L)]
        zb = [ftgen.zipf_log_bias(wl.E, 1.1, wl.seed("pi", l)) for l in range(L)]
        for step in range(steps):
            for l in range(L):
                bias = ftgen.trace_bias(traces[l][step], zb[l], 8.0)
                x = gap_hidden(wl, 1, wl.seed("x", step, l), h.routers[l], bias)
                _run_and_check(h, oc, W, l, x, bias, check_y=True)
        _check_cache_state(h, oc)


def test_nvfp4_shape_off_the_tensor_core_path(cuda_ok):
    """NVFP4 with d and d_ff multiples of 64 but not of 256 (d = 320,
    d_ff = 192): the experts run on the SIMT GEMV instead of the tensor-core
    one; same parity bar, decode at batch 1..5 on a small shared cache."""
    wl = ftgen.Workload("nvfp4_odd", L=2, E=16, k=2, d=320, d_ff=192, wtype=ftgen.W_NVFP4, cache_slots=6,
                        bp_mbps=52700, bh_mbps=77300)
    with _harness(wl, max_tokens=5) as h:
        oc = oracle_cache(h)
        W = ExpertWeights(h, keep=32)
        for step in range(6):
            for l in range(wl.L):
                T = 1 + (step + l) % 5
                x = gap_hidden(wl, T, wl.seed("odd", step, l), h.routers[l], None)
                _run_and_check(h, oc, W, l, x, None)
        _check_cache_state(h, oc)


def test_error_paths(cuda_ok):
    wl = ftgen.workload("tiny_f32")
    with _harness(wl, gen_device="cpu") as h:
        x = torch.zeros(4, wl.d, device=h.dev)
        y = torch.zeros_like(x)
        with pytest.raises(ft.FtError) as ei:
            ft.ft_moe_layer_forward(h.ctx, 1, ft.FT_DECODE, x, 4, None, 0, y)
        assert ei.value.status == ft.FT_EINVAL
        with pytest.raises(ft.FtError):
            ft.ft_moe_layer_forward(h.ctx, 0, ft.FT_DECODE, x, 17, None, 0, y)  # T > max_tokens
        with pytest.raises(ft.FtError):
            ft.ft_moe_layer_forward(h.ctx, 0, 7, x, 4, None, 0, y)
        with pytest.raises(ft.FtError):
            ft.ft_set_bandwidths(h.ctx, 1, 0)
        assert h.stats()["device_error"] == 0


@pytest.mark.parametrize("scale", [2.0 ** 15, 1.0, 2.0 ** -20])
def test_nvfp4_activation_range(cuda_ok, scale):
    """NVFP4 experts run f16 tensor-core MMAs; activations of any magnitude
    must come through: x * 2^15 makes |h| ~ 1e9, far above the f16 maximum
    65504, and x * 2^-20 makes |h| ~ 1e-12, below the smallest f16 subnormal
    (powers of two, so the bf16 inputs keep the top-k gap exactly).
    Decode at batch 1..5 through all three classes (hit, staged, streamed) on
    a small cache; routing bit-exact and outputs within 4e-2 rms of the
    oracle."""
    wl = ftgen.Workload("nvfp4_range", L=1, E=16, k=4, d=1024, d_ff=512, wtype=ftgen.W_NVFP4, cache_slots=6,
                        bp_mbps=52700, bh_mbps=77300)
    with _harness(wl, max_tokens=5) as h:
        oc = oracle_cache(h)
        W = ExpertWeights(h, keep=16)
        for step in range(8):
            T = 1 + step % 5
            x = gap_hidden(wl, T, wl.seed("range", step), h.routers[0], None)
            x = (x.float() * scale).to(torch.bfloat16)
            y, _ = _run_and_check(h, oc, W, 0, x, None)
            assert torch.isfinite(y.float()).all()
        _check_cache_state(h, oc)
        st = h.stats()
        assert st["hits"] > 0 and st["staged"] > 0 and st["streamed"] > 0


def test_host_buffer_call_matches_device_call(cuda_ok):
    """ft_moe_layer_forward_host (host x and y, copied by the library on the
    compute stream) gives the device-pointer call's output bytes, from pinned
    and from pageable host memory, and the same cache record."""
    import dataclasses
    wl = dataclasses.replace(ftgen.workload("decode_bf16"), name="host_call", E=64, cache_slots=24)
    bias = ftgen.zipf_log_bias(wl.E, 1.1, wl.seed("zipf"))
    with _harness(wl, max_tokens=16) as a, _harness(wl, max_tokens=16) as b:
        bd = torch.as_tensor(bias).to(a.dev)
        for step, T in enumerate((1, 4, 16, 3)):
            x = gap_hidden(wl, T, wl.seed("host", step), a.routers[0], bias)
            y_dev = a.forward(0, x.to(a.dev), bd)
            xh = x.pin_memory() if step % 2 == 0 else x.clone()
            yh = torch.empty_like(x)
            yh = yh.pin_memory() if step % 2 == 0 else yh
            ft.ft_moe_layer_forward_host(b.ctx, 0, ft.FT_DECODE, xh, T, bd, 0, yh)
            torch.cuda.synchronize()
            assert torch.equal(y_dev.cpu().view(torch.int16), yh.view(torch.int16)), step
        sa, sb = a.stats(), b.stats()
        for k in ("lookups", "hits", "misses", "staged", "streamed"):
            assert sa[k] == sb[k], k
        with pytest.raises(ft.FtError):
            x = torch.zeros(17, wl.d, dtype=torch.bfloat16)
            ft.ft_moe_layer_forward_host(b.ctx, 0, ft.FT_DECODE, x, 17, None, 0, torch.empty_like(x))


@pytest.mark.parametrize("wname", ["decode_bf16", "trace_nvfp4"])
def test_decode_against_the_cpp_oracle(cuda_ok, wname):
    """The plain C++ oracle (one thread per token, the layer's fp32 roundings)
    and its LRU simulator, against the library on decode calls at batch 1..16:
    ids bit-exact, the lookup record, m, q* and q_stage identical to the C++
    cache's, outputs within the BF16 / NVFP4 tolerance."""
    import dataclasses
    from oracle import cpp as ocpp
    base = ftgen.workload(wname)
    wl = dataclasses.replace(base, name=f"cpp_{wname}", L=2, E=64, cache_slots=20)
    with _harness(wl, max_tokens=16) as h:
        cc = ocpp.Cache(wl.L, wl.E, wl.cache_slots, wl.bp_mbps, wl.bh_mbps)
        zb = ftgen.zipf_log_bias(wl.E, 1.1, wl.seed("zipf"))
        for step in range(10):
            for l in range(wl.L):
                T = (1, 4, 16, 3, 8)[(step + l) % 5]
                x = gap_hidden(wl, T, wl.seed("cpp", step, l), h.routers[l], zb)
                y, ids, _ = h.forward(l, x.to(h.dev), torch.as_tensor(zb).to(h.dev), want_route=True)
                torch.cuda.synchronize()
                blobs = [h.blob(l, e) for e in range(wl.E)]
                ts = np.array([h.tscales[(l, e)] for e in range(wl.E)]) if wl.wtype == ftgen.W_NVFP4 else None
                y_c, ids_c, _ = ocpp.layer_forward(x.float().numpy(), h.routers[l].float().cpu().numpy(), zb, wl.k,
                                                   blobs, wl.wtype, wl.d, wl.d_ff, ts)
                np.testing.assert_array_equal(ids.cpu().numpy(), ids_c)
                check_close(to_np(y), y_c.astype(np.float64), wl.wtype, f"step {step} layer {l}")
                rec = cc.forward(l, 0, np.bincount(ids_c.ravel(), minlength=wl.E))
                r = gpu_route(h, T)
                assert r["lookup_e"].tolist() == [e for (_, e, _) in rec["lookups"]]
                assert r["lookup_kind"].tolist() == [k for (_, _, k) in rec["lookups"]]
                assert (r["m"], r["qstar"], r["qstage"]) == (rec["m"], rec["qstar"], rec["qstage"])
        key_of, stamp = ft.ft_moe_cache_contents(h.ctx, h.C)
        assert (key_of.tolist(), stamp.tolist()) == cc.contents()
        cnt, st = cc.counters(), h.stats()
        for k in ("lookups", "hits", "misses", "staged", "streamed"):
            assert st[k] == cnt[k], k
        cc.close()
