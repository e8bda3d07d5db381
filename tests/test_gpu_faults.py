"""Host-injected failures through the C ABI (FT_FAULT; nothing faults on the
GPU): allocation failures at init return FT_ENOMEM and leak nothing; a
staging copy that fails or a host wait that times out in the middle of a
decode call returns its status, stays latched for later calls, and a cache
reset brings the context back to outputs that match the oracle."""
import numpy as np
import pytest
import torch

import ftgen
import sparse_moe_expert_topk_b200 as ft
from oracle import moe as omoe
from parity import ExpertWeights, check_close, gap_hidden, to_np

pytestmark = pytest.mark.gpu

WL = ftgen.Workload("fault_small", L=2, E=32, k=4, d=1024, d_ff=512, wtype=ftgen.W_BF16, cache_slots=16,
                    bp_mbps=52700, bh_mbps=77300)


def _harness(**kw):
    from ftgen.ctx import Harness
    return Harness(WL, **kw)


@pytest.mark.parametrize("what", ["pool_alloc", "slot_alloc"])
def test_init_allocation_failure(cuda_ok, monkeypatch, what):
    free0 = torch.cuda.mem_get_info()[0]
    monkeypatch.setenv("FT_FAULT", what)
    with pytest.raises(ft.FtError) as ei:
        _harness(max_tokens=8)
    assert ei.value.status == ft.FT_ENOMEM
    monkeypatch.delenv("FT_FAULT")
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] >= free0 - (64 << 20)  # the failed init left nothing behind


@pytest.mark.parametrize("what,status", [("memcpy", ft.FT_ECUDA), ("poll_timeout", ft.FT_ETIMEOUT)])
def test_failure_mid_forward_latches_and_recovers(cuda_ok, monkeypatch, what, status):
    wl = WL
    with _harness(max_tokens=8) as h:
        W = ExpertWeights(h, keep=8)
        x = gap_hidden(wl, 4, wl.seed("fault", what), h.routers[0], None)
        monkeypatch.setenv("FT_FAULT", what)
        with pytest.raises(ft.FtError) as ei:  # cold cache: the call stages misses
            h.forward(0, x.to(h.dev))
        assert ei.value.status == status
        monkeypatch.delenv("FT_FAULT")
        with pytest.raises(ft.FtError) as ei:  # latched until the cache is reset
            h.forward(0, x.to(h.dev))
        assert ei.value.status == status
        ft.ft_moe_reset_cache(h.ctx)
        y = h.forward(0, x.to(h.dev))
        torch.cuda.synchronize()
        xn = x.float().numpy()
        y_ref, _, _ = omoe.layer_forward(xn, h.routers[0].float().cpu().numpy(), None, wl.k, lambda e: W(0, e))
        check_close(to_np(y), y_ref, wl.wtype, what)
        assert h.stats()["device_error"] == 0
