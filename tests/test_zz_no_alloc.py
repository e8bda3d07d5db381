"""The allocation-free router entry point (ft_route_topk_static) against the
routing outputs of ft_moe_layer_forward, through the C ABI.

ft_route_topk_static is for callers that cannot call cudaMalloc where they
route -- a serving loop whose memory manager already gave all free HBM to the
KV cache and the expert slots, or code that must avoid cudaMalloc's implicit
device synchronisation mid-step. Its scratch is a fixed device array in the
library, shared by every call, so two calls in a row must each give the same
result as the normal entry point. This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import ftgen
import sparse_moe_expert_topk_b200 as ft
from parity import check_route_weights

pytestmark = pytest.mark.gpu

WL = ftgen.Workload("no_alloc", L=1, E=64, k=4, d=1024, d_ff=512, wtype=ftgen.W_BF16, cache_slots=16)


def test_static_router_matches_layer_forward_twice(cuda_ok):
    from ftgen.ctx import Harness
    with Harness(WL, max_tokens=300) as h:
        wr = h.routers[0]
        bias = torch.as_tensor(ftgen.zipf_log_bias(WL.E, 1.1, WL.seed("zipf"))).to(h.dev)
        for call, T in enumerate((300, 37)):  # two calls in a row, different sizes and inputs
            x = ftgen.hidden(T, WL.d, WL.wtype, WL.seed("x", call)).to(h.dev)
            b = bias if call == 0 else None
            _, ids_ref, w_ref = h.forward(0, x, b, want_route=True)
            ids = torch.full((T, WL.k), -1, dtype=torch.int32, device=h.dev)
            w = torch.full((T, WL.k), -1.0, dtype=torch.float32, device=h.dev)
            ft.ft_route_topk_static(x, wr, b, 0, T, WL.E, WL.d, WL.k, WL.wtype, ids, w, h.stream)
            torch.cuda.synchronize()
            np.testing.assert_array_equal(ids.cpu().numpy(), ids_ref.cpu().numpy())
            check_route_weights(w.cpu().numpy(), w_ref.cpu().numpy(), x.float().cpu().numpy(), wr.float().cpu().numpy(), f"call {call}")


def test_static_router_rejects_oversize(cuda_ok):
    T = ft.FT_ROUTE_STATIC_MAX_TOKENS + 1
    x = torch.zeros(T, 64, dtype=torch.bfloat16, device="cuda")
    wr = torch.zeros(8, 64, dtype=torch.bfloat16, device="cuda")
    ids = torch.zeros(T, 2, dtype=torch.int32, device="cuda")
    w = torch.zeros(T, 2, dtype=torch.float32, device="cuda")
    with pytest.raises(ft.FtError) as ei:
        ft.ft_route_topk_static(x, wr, None, 0, T, 8, 64, 2, ft.FT_W_BF16, ids, w, None)
    assert ei.value.status == ft.FT_EINVAL
