"""Exact ties in the router, on the GPU, bit-exact against the oracle.

The top-k decision takes the larger fp32 logit first and, between equal
logits, the lower expert index (the C ABI's reading; the pages do not give a
router). Two inputs tie exactly on any summation engine: x = 0 with b = 0
(every logit is a signed zero, so every expert ties and the ids must be
0..k-1, the weights 1/k and the output exactly 0), and a router whose rows
repeat (equal rows give equal fp32 sums, so of each pair the lower index must
be taken first). Both run at T = 1, 16 (the fused decode routing kernel),
33 and 300 (the separate router and top-k kernels), through
ft_moe_layer_forward and through the allocation-free ft_route_topk_static.
"""
import numpy as np
import pytest
import torch

import ftgen
import sparse_moe_expert_topk_b200 as ft
from oracle import moe as omoe
from parity import GAP, check_close, check_route_weights, ExpertWeights, to_np

pytestmark = pytest.mark.gpu

# k odd, so the k-th pick splits a pair of equal logits in the duplicate test
WL = ftgen.Workload("ties", L=1, E=64, k=5, d=1024, d_ff=512, wtype=ftgen.W_BF16, cache_slots=24)
TS = (1, 16, 33, 300)
SHIFT = 37  # row e + SHIFT repeats row e: the pair sits at different positions of any 16-row tile


def _harness(wl, **kw):
    from ftgen.ctx import Harness
    return Harness(wl, **kw)


def _static(h, x, wr, bias, T):
    ids = torch.full((T, WL.k), -1, dtype=torch.int32, device=h.dev)
    w = torch.full((T, WL.k), -1.0, dtype=torch.float32, device=h.dev)
    ft.ft_route_topk_static(x, wr, bias, 0, T, WL.E, WL.d, WL.k, WL.wtype, ids, w, h.stream)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("T", TS)
def test_all_logits_tie_at_zero(cuda_ok, T):
    with _harness(WL, max_tokens=max(TS)) as h:
        x = torch.zeros(T, WL.d, dtype=torch.bfloat16, device=h.dev)
        b = torch.zeros(WL.E, dtype=torch.float32, device=h.dev)
        xn = x.float().cpu().numpy()
        ids_ref, w_ref, _ = omoe.route(xn, h.routers[0].float().cpu().numpy(), np.zeros(WL.E), WL.k)
        assert (ids_ref == np.arange(WL.k)).all()
        for bias in (None, b):
            y, ids, w = h.forward(0, x, bias, want_route=True)
            torch.cuda.synchronize()
            np.testing.assert_array_equal(ids.cpu().numpy(), ids_ref)
            np.testing.assert_array_equal(w.cpu().numpy(), np.full((T, WL.k), 1.0 / WL.k, np.float32))
            assert (y.float() == 0).all()
            s_ids, s_w = _static(h, x, h.routers[0], bias, T)
            np.testing.assert_array_equal(s_ids, ids_ref)
            np.testing.assert_array_equal(s_w, np.full((T, WL.k), 1.0 / WL.k, np.float32))
        assert h.stats()["device_error"] == 0


def _dup_router(wr):
    """Rows SHIFT.. E-1 repeat rows 0.. E-1-SHIFT."""
    w = wr.clone()
    n = WL.E - SHIFT
    w[SHIFT:] = wr[:n]
    return w


def _gap_x(T, seed, wr_np):
    """x whose distinct logits keep a 1e-3 gap between the last distinct value
    the top-k reaches and the next one, and between every pair of distinct
    values it ranks (so that only the exact duplicates tie)."""
    x = ftgen.hidden(T, WL.d, WL.wtype, seed)
    att = np.zeros(T, np.int64)
    uniq = wr_np[:SHIFT]  # every row of the router is one of these
    for _ in range(200):
        s = omoe.router_logits(x.float().numpy(), uniq, None).astype(np.float64)
        srt = -np.sort(-s, axis=1)
        bad = np.nonzero((srt[:, :WL.k] - srt[:, 1:WL.k + 1]).min(axis=1) < GAP)[0]
        if bad.size == 0:
            return x
        for t in bad:
            att[t] += 1
            x[t] = ftgen.hidden_row(WL.d, WL.wtype, seed, int(t), int(att[t]))
    raise RuntimeError("no gap")


@pytest.mark.parametrize("T", TS)
def test_duplicate_router_rows_prefer_lower_index(cuda_ok, T):
    from ftgen.ctx import Harness
    with Harness(WL, max_tokens=max(TS)) as h:
        wr = _dup_router(h.routers[0])
        ft.ft_moe_set_router(h.ctx, 0, wr)
        wr_np = wr.float().cpu().numpy()
        x = _gap_x(T, WL.seed("dup", T), wr_np)
        xn = x.float().numpy()
        ids_ref, w_ref, s32 = omoe.route(xn, wr_np, None, WL.k)
        # every token's picks contain at least one duplicated pair, lower index first
        dup_pairs = 0
        for t in range(T):
            pos = {int(e): j for j, e in enumerate(ids_ref[t])}
            for e, j in pos.items():
                if e < WL.E - SHIFT and e + SHIFT in pos:
                    assert j < pos[e + SHIFT]
                    dup_pairs += 1
        assert dup_pairs >= T
        xd = x.to(h.dev)
        y, ids, w = h.forward(0, xd, None, want_route=True)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(ids.cpu().numpy(), ids_ref)
        check_route_weights(w.cpu().numpy(), w_ref, xn, wr_np, f"T={T}")
        # the two weights of a duplicated pair are equal bit for bit
        wg = w.cpu().numpy()
        for t in range(T):
            for j, e in enumerate(ids_ref[t]):
                if e >= SHIFT:
                    jj = np.nonzero(ids_ref[t] == e - SHIFT)[0]
                    if jj.size:
                        assert wg[t, j] == wg[t, jj[0]]
        W = ExpertWeights(h, keep=64)
        toks = np.arange(T) if T <= 33 else np.unique(np.r_[0, 1, T // 2, T - 1])
        y_ref, _, _ = omoe.layer_forward(xn, wr_np, None, WL.k, lambda e: W(0, e), tokens=toks)
        check_close(to_np(y)[toks], y_ref, WL.wtype, f"T={T}")
        s_ids, s_w = _static(h, xd, wr, None, T)
        np.testing.assert_array_equal(s_ids, ids_ref)
        check_route_weights(s_w, w_ref, xn, wr_np, f"static T={T}")
        assert h.stats()["device_error"] == 0
