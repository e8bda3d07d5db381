"""Set up a library context for a synthetic workload.

Glue between the seeded generator (ftgen) and the C ABI binding: creates the
context, fills the pinned host pool with generated expert blobs, uploads
seeded router weights, sets NVFP4 tensor scales and the B_P:B_H profile.
Holds none of the layer's arithmetic and does not import the oracle.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

import ftgen
import sparse_moe_expert_topk_b200 as ft


def host_view(addr: int, nbytes: int) -> torch.Tensor:
    """uint8 CPU tensor aliasing library-owned pinned memory."""
    buf = (ctypes.c_uint8 * nbytes).from_address(addr)
    return torch.frombuffer(buf, dtype=torch.uint8)


class Harness:
    """A context plus the tensors it points at (router weights, streams).

    With n_experts set, the context holds only the global experts
    expert_base .. expert_base + n_experts - 1 of every layer (one device's
    share of an expert-parallel layer), as its local experts 0..n_experts-1,
    and routes nothing; self.routers still holds the full [E, d] routers."""

    def __init__(self, wl: ftgen.Workload, L=None, cache_slots=None, max_tokens=None, gen_device="cuda",
                 device=0, fill=True, expert_base=0, n_experts=None):
        self.wl = wl
        self.E = wl.E if n_experts is None else n_experts
        self.expert_base = expert_base
        self.L = wl.L if L is None else L
        self.C = wl.cache_slots if cache_slots is None else cache_slots
        self.max_tokens = max(wl.batches) if max_tokens is None else max_tokens
        self.dev = torch.device("cuda", device)
        self.gen_device = gen_device
        self.cfg = ft.make_config(self.L, self.E, wl.k, wl.d, wl.d_ff, wl.wtype, self.C, self.max_tokens, device)
        self.slot_bytes = ft.ft_moe_slot_bytes(self.cfg)
        assert self.slot_bytes == wl.slot_bytes
        self.stream = torch.cuda.current_stream(self.dev)
        self.copy_stream = torch.cuda.Stream(self.dev)
        self.ctx = ft.ft_moe_init(self.cfg, self.stream, self.copy_stream)
        self.routers = []
        for l in range(self.L):
            w = ftgen.router_weight(wl.E, wl.d, wl.wtype, wl.seed("router", l)).to(self.dev)
            self.routers.append(w)
            if n_experts is None:
                ft.ft_moe_set_router(self.ctx, l, w)
        self.tscales = {}
        if fill:
            self.fill_pool()
        ft.ft_set_bandwidths(self.ctx, wl.bp_mbps, wl.bh_mbps)

    # --- expert pool --------------------------------------------------------
    def layer_view(self, layer: int) -> torch.Tensor:
        base = ft.ft_moe_expert_ptr(self.ctx, layer, 0)
        return host_view(base, self.E * self.slot_bytes)

    def blob(self, layer: int, e: int) -> np.ndarray:
        """numpy view of one pinned blob (read by the oracle)."""
        p = ft.ft_moe_expert_ptr(self.ctx, layer, e)
        return np.ctypeslib.as_array((ctypes.c_uint8 * self.slot_bytes).from_address(p))

    def fill_pool(self):
        wl = self.wl
        for l in range(self.L):
            view = self.layer_view(l)
            for e in range(self.E):
                g = self.expert_base + e  # global expert id: the blob is the same on any device
                b = ftgen.expert_blob(wl.d, wl.d_ff, wl.wtype, wl.seed("expert", l, g), device=self.gen_device)
                view[e * self.slot_bytes:(e + 1) * self.slot_bytes].copy_(b)
                if wl.wtype == ftgen.W_NVFP4:
                    ts = ftgen.tensor_scales(wl.seed("tscale", l, g))
                    self.tscales[(l, e)] = ts
                    ft.ft_moe_set_tensor_scales(self.ctx, l, e, ts)
        torch.cuda.synchronize(self.dev)

    # --- calls --------------------------------------------------------------
    def forward(self, layer, x, bias=None, mode=ft.FT_DECODE, want_route=False):
        T = x.shape[0]
        y = torch.empty_like(x)
        ids = torch.empty(T, self.wl.k, dtype=torch.int32, device=self.dev) if want_route else None
        w = torch.empty(T, self.wl.k, dtype=torch.float32, device=self.dev) if want_route else None
        bpt = 1 if (bias is not None and bias.dim() == 2) else 0
        ft.ft_moe_layer_forward(self.ctx, layer, mode, x, T, bias, bpt, y, ids, w)
        return (y, ids, w) if want_route else y

    def stats(self):
        return ft.ft_cache_stats(self.ctx)

    def close(self):
        if self.ctx is not None:
            ft.ft_moe_destroy(self.ctx)
            self.ctx = None

    def __enter__(self):
        return self

    def __exit__(self, *a):
        self.close()
