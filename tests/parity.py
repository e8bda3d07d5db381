"""Helpers for the GPU parity tests: seeded inputs with a guaranteed top-k
gap, and an oracle replay of a sequence of layer calls over the same pinned
expert blobs the library reads."""
from __future__ import annotations

from collections import OrderedDict

import numpy as np
import torch

import ftgen
from oracle import cache as ocache
from oracle import formats as ofmt
from oracle import moe as omoe

GAP = 1e-3  # minimum gap between consecutive logits among each token's k+1 largest


def rank_gaps(s32, k):
    """Per token, the smallest gap between consecutive logits among its k+1
    largest: the k-th vs (k+1)-th gap decides which experts are chosen, the
    others their rank order (inf where E = k)."""
    srt = -np.sort(-np.asarray(s32, np.float64), axis=1)
    m = min(k + 1, srt.shape[1])
    if m < 2:
        return np.full(srt.shape[0], np.inf)
    return (srt[:, :m - 1] - srt[:, 1:m]).min(axis=1)


def gap_hidden(wl, T, seed, w_router, bias, max_rounds=60):
    """x [T, d] from ftgen whose top-k is decided with a margin: for every
    token the k+1 largest logits are at least GAP apart from each other, so
    that the chosen experts and their rank order are the same whatever order
    a dot product is summed in (tokens that fall short are redrawn with the
    next attempt number)."""
    attempts = np.zeros(T, dtype=np.int64)
    x = ftgen.hidden(T, wl.d, wl.wtype, seed)
    wr = w_router.float().cpu().numpy()
    for _ in range(max_rounds):
        s32 = omoe.router_logits(x.float().numpy(), wr, bias)
        bad = np.nonzero(rank_gaps(s32, wl.k) < GAP)[0]
        if bad.size == 0:
            return x
        for t in bad:
            attempts[t] += 1
            x[t] = ftgen.hidden_row(wl.d, wl.wtype, seed, int(t), int(attempts[t]))
    raise RuntimeError("could not enforce the top-k gap")


class ExpertWeights:
    """fp64 expert matrices decoded by the oracle from the pinned pool blobs,
    with a small LRU of decoded experts."""

    def __init__(self, harness, keep=24):
        self.h = harness
        self.keep = keep
        self.cache = OrderedDict()

    def __call__(self, layer, e):
        key = (layer, e)
        if key in self.cache:
            self.cache.move_to_end(key)
            return self.cache[key]
        wl = self.h.wl
        ts = self.h.tscales.get(key)
        w = ofmt.unpack_expert(self.h.blob(layer, e).copy(), wl.d, wl.d_ff, wl.wtype, ts)
        self.cache[key] = w
        if len(self.cache) > self.keep:
            self.cache.popitem(last=False)
        return w


def tol_for(wtype):
    """max |gpu - oracle| allowed, as a fraction of rms(oracle)."""
    return {ftgen.W_F32: 1e-4, ftgen.W_BF16: 2e-2, ftgen.W_NVFP4: 4e-2}[wtype]


def half_ulp_bf16(v):
    """Half the bf16 spacing at |v| (taken one bf16 step above |v|, so that a
    value rounded up into the next binade is covered); 0 where v is 0."""
    a = np.abs(np.asarray(v, np.float64)) * (1.0 + 2.0 ** -7)
    out = np.zeros_like(a)
    nz = a > 0
    out[nz] = 2.0 ** (np.floor(np.log2(a[nz])) - 8)
    return out


def check_close(y_gpu, y_ref, wtype, what=""):
    """Layer outputs against the oracle: max |gpu - oracle| <= tol * rms(oracle)
    element by element, where the output type is bf16 (BF16 and NVFP4 experts)
    plus half a bf16 step of the oracle's value: the layer's output is bf16 by
    definition, and its own rounding of an element at five standard
    deviations already reaches 2% of rms, whatever the arithmetic before it."""
    y_gpu = np.asarray(y_gpu, np.float64)
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    if not y_ref.size:
        return 0.0
    d = np.abs(y_gpu - y_ref)
    slack = half_ulp_bf16(y_ref) if wtype != ftgen.W_F32 else 0.0
    bad = d > tol_for(wtype) * rms + slack
    i = int(np.argmax(d - slack))
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements off; worst |d| {d.flat[i]:.3e} > {tol_for(wtype)} * "
                           f"rms {rms:.3e} + half bf16 step {np.broadcast_to(slack, d.shape).flat[i]:.3e}")
    return float(np.max(d)) / rms if rms > 0 else 0.0


def check_route_weights(w_gpu, w_ref, x, w_router, what=""):
    """Top-k softmax weights against the oracle's.

    A logit is an fp32 dot product of length d. Whatever order the kernel
    sums in (one FMA chain, or tensor-core k-groups), its rounding error stays
    within the probabilistic bound sqrt(d) * u * sum_i |x_i W_ei|, u = 2^-24.
    A weight exp(s_j - s_max) / sum is off, relative to itself, by at most
    twice its token's largest logit error. That bound, per token, is the
    tolerance; the selected ids are checked bit-exact separately."""
    w_gpu = np.asarray(w_gpu, np.float64)
    w_ref = np.asarray(w_ref, np.float64)
    xa = np.abs(np.asarray(x, np.float64))
    wa = np.abs(np.asarray(w_router, np.float64))
    d = xa.shape[1]
    bound = 2.0 * np.sqrt(d) * 2.0 ** -24 * (xa @ wa.T).max(axis=1)
    err = np.abs(w_gpu - w_ref)
    lim = bound[:, None] * w_ref + 1e-7
    bad = np.argwhere(err > lim)
    assert bad.size == 0, (f"{what}: {len(bad)} weights off, first (t, j) = {tuple(bad[0])}: "
                           f"|d| {err[tuple(bad[0])]:.3e} > {lim[tuple(bad[0])]:.3e}")


def gpu_route(harness, T):
    import sparse_moe_expert_topk_b200 as ft
    return ft.ft_moe_last_route(harness.ctx, harness.wl.E, T * harness.wl.k)


def expected_record(rec, E):
    """Oracle cache record -> (lookup experts, kinds) in lookup order."""
    es = [e for (_, e, _) in rec["lookups"]]
    ks = [k for (_, _, k) in rec["lookups"]]
    return es, ks


def oracle_cache(harness):
    wl = harness.wl
    return ocache.ExpertCache(harness.L, wl.E, harness.C, wl.bp_mbps, wl.bh_mbps)


def to_np(t):
    return t.detach().float().cpu().numpy()


class PrefetchWeights:
    """Expert weights of one layer decoded by the oracle ahead of use, in
    ascending expert order, on a few threads (the grouped oracle visits the
    experts in ascending order and each is decoded once). Keeps only the
    experts of the window in memory."""

    def __init__(self, harness, layer, workers=8, window=12):
        from concurrent.futures import ThreadPoolExecutor
        self.h, self.layer, self.window = harness, layer, window
        self.pool = ThreadPoolExecutor(max_workers=workers)
        self.fut = {}

    def _decode(self, e):
        wl = self.h.wl
        ts = self.h.tscales.get((self.layer, e))
        return ofmt.unpack_expert(self.h.blob(self.layer, e).copy(), wl.d, wl.d_ff, wl.wtype, ts)

    def __call__(self, e):
        for n in range(e, min(self.h.E, e + self.window)):
            if n not in self.fut:
                self.fut[n] = self.pool.submit(self._decode, n)
        w = self.fut.pop(e).result()
        for n in [n for n in self.fut if n < e]:
            self.fut.pop(n).cancel()
        return w

    def close(self):
        self.pool.shutdown(wait=True, cancel_futures=True)
        self.fut.clear()


class ParallelExpertWeights:
    """fp64 expert matrices decoded by the oracle on a few threads, with an
    LRU of `keep` decoded experts: `need(layer, experts)` decodes the missing
    ones of a call at once, then the object is called like ExpertWeights."""

    def __init__(self, harness, keep=64, workers=8):
        from concurrent.futures import ThreadPoolExecutor
        self.h = harness
        self.keep = keep
        self.cache = OrderedDict()
        self.pool = ThreadPoolExecutor(max_workers=workers)

    def _decode(self, layer, e):
        wl = self.h.wl
        ts = self.h.tscales.get((layer, e))
        return ofmt.unpack_expert(self.h.blob(layer, e).copy(), wl.d, wl.d_ff, wl.wtype, ts)

    def need(self, layer, experts):
        missing = [int(e) for e in experts if (layer, int(e)) not in self.cache]
        for e, w in zip(missing, self.pool.map(lambda e: self._decode(layer, e), missing)):
            self.cache[(layer, e)] = w
        for e in experts:
            self.cache.move_to_end((layer, int(e)))
        while len(self.cache) > max(self.keep, len(experts)):
            self.cache.popitem(last=False)

    def __call__(self, layer, e):
        key = (layer, int(e))
        if key not in self.cache:
            self.need(layer, [e])
        return self.cache[key]

    def close(self):
        self.pool.shutdown(wait=True)
        self.cache.clear()
