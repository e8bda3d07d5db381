"""The allocation-free router entry point (ft_route_topk_static), through the
C ABI, against the oracle and against the routing outputs of
ft_moe_layer_forward.

ft_route_topk_static is for callers that cannot call cudaMalloc where they
route -- a serving loop whose memory manager already gave all free HBM to the
KV cache and the expert slots, or code that must avoid cudaMalloc's implicit
device synchronisation mid-step. Its scratch is a fixed device array in the
library, shared by every call, so every call of a sequence must give the same
result as the normal entry point. Batches of up to 32 tokens take the small-
batch logits kernel (the one the fused decode routing uses), larger ones the
tensor-core router kernel. This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import ftgen
import sparse_moe_expert_topk_b200 as ft
from oracle import moe as omoe
from parity import check_route_weights, gap_hidden

pytestmark = pytest.mark.gpu

WL = ftgen.Workload("no_alloc", L=1, E=64, k=4, d=1024, d_ff=512, wtype=ftgen.W_BF16, cache_slots=16)


def _static(x, wr, b, T, stream, dev):
    ids = torch.full((T, WL.k), -1, dtype=torch.int32, device=dev)
    w = torch.full((T, WL.k), -1.0, dtype=torch.float32, device=dev)
    ft.ft_route_topk_static(x, wr, b, 0, T, WL.E, WL.d, WL.k, WL.wtype, ids, w, stream)
    return ids, w


def test_static_router_matches_oracle_and_layer_forward(cuda_ok):
    """Calls in a row at T = 1, 4, 16, 32 (small-batch kernel), 33 and 300
    (tensor-core router), with and without a bias: ids bit-exact against the
    oracle and against ft_moe_layer_forward's routing outputs; weights within
    the derived fp32 bound of the oracle's, and bit-equal to the forward's
    where both use the same logits kernel (decode at T <= 32, T > 32)."""
    from ftgen.ctx import Harness
    with Harness(WL, max_tokens=300) as h:
        wr = h.routers[0]
        wr_np = wr.float().cpu().numpy()
        zipf = ftgen.zipf_log_bias(WL.E, 1.1, WL.seed("zipf"))
        bias = torch.as_tensor(zipf).to(h.dev)
        for call, T in enumerate((1, 4, 16, 32, 33, 300, 1, 300)):
            b_np = zipf if call % 2 == 0 else None
            b = bias if call % 2 == 0 else None
            x = gap_hidden(WL, T, WL.seed("x", call), wr, b_np)
            xd = x.to(h.dev)
            _, ids_f, w_f = h.forward(0, xd, b, want_route=True)
            ids, w = _static(xd, wr, b, T, h.stream, h.dev)
            torch.cuda.synchronize()
            xn = x.float().numpy()
            ids_ref, w_ref, _ = omoe.route(xn, wr_np, b_np, WL.k)
            np.testing.assert_array_equal(ids.cpu().numpy(), ids_ref)
            np.testing.assert_array_equal(ids.cpu().numpy(), ids_f.cpu().numpy())
            check_route_weights(w.cpu().numpy(), w_ref, xn, wr_np, f"call {call} T={T}")
            np.testing.assert_array_equal(w.cpu().numpy(), w_f.cpu().numpy())
        assert h.stats()["device_error"] == 0


def test_static_router_rejects_oversize(cuda_ok):
    T = ft.FT_ROUTE_STATIC_MAX_TOKENS + 1
    x = torch.zeros(T, 64, dtype=torch.bfloat16, device="cuda")
    wr = torch.zeros(8, 64, dtype=torch.bfloat16, device="cuda")
    ids = torch.zeros(T, 2, dtype=torch.int32, device="cuda")
    w = torch.zeros(T, 2, dtype=torch.float32, device="cuda")
    with pytest.raises(ft.FtError) as ei:
        ft.ft_route_topk_static(x, wr, None, 0, T, 8, 64, 2, ft.FT_W_BF16, ids, w, None)
    assert ei.value.status == ft.FT_EINVAL
