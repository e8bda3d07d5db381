"""Python side of the plain C++ oracle (oracle/moe_oracle.cpp).

Test infrastructure (see oracle/__init__.py). Compiles the C++ file with the
host compiler into oracle/libmoe_oracle.so on first use (or from
__graft_entry__.build()) and calls it through ctypes. The C++ oracle computes
the layer per token, one std::thread per token, and simulates the shared LRU
cache; it is pinned against the numpy oracle (itself pinned to the dense
brute force and the pages' q* profiles) in tests/test_oracle_cpp.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_DIR = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_DIR, "moe_oracle.cpp")
LIB = os.path.join(_DIR, "libmoe_oracle.so")
_lib = None


def build() -> str:
    """Compile the oracle if the library is missing or older than its source."""
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        cxx = os.environ.get("CXX", "g++")
        subprocess.run([cxx, "-O2", "-std=c++17", "-shared", "-fPIC", "-pthread", "-o", LIB, SRC], check=True)
    return LIB


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P, I, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        L.fto_layer_forward.argtypes = [P, I, I, I, I, I, P, P, I, P, I, P, I, P, P, P]
        L.fto_layer_forward.restype = I
        L.fto_route.argtypes = [P, I, I, I, I, P, P, I, P, P]
        L.fto_route.restype = I
        L.fto_weight.argtypes = [P, I, I, I, P, I, ctypes.c_long, ctypes.c_long]
        L.fto_weight.restype = D
        L.fto_e2m1.argtypes = [I]
        L.fto_e2m1.restype = D
        L.fto_e4m3.argtypes = [I]
        L.fto_e4m3.restype = D
        L.fto_cache_new.argtypes = [I, I, ctypes.c_long, ctypes.c_uint, ctypes.c_uint]
        L.fto_cache_new.restype = P
        L.fto_cache_free.argtypes = [P]
        L.fto_cache_free.restype = None
        L.fto_cache_forward.argtypes = [P, I, I, P, P, P, P] + [ctypes.POINTER(I)] * 5
        L.fto_cache_forward.restype = I
        L.fto_cache_counters.argtypes = [P, P]
        L.fto_cache_counters.restype = None
        L.fto_cache_contents.argtypes = [P, P, P]
        L.fto_cache_contents.restype = None
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def layer_forward(x, w_router, bias, k, blobs, wtype, d, d_ff, tscales=None, threads=None):
    """The layer on T tokens, one thread per token (at most `threads` at once,
    default: as many as the machine has cores). x [T, d], w_router [E, d]
    (exact values of the bf16 / fp32 data), bias None / [E] / [T, E];
    blobs: one uint8 slot blob per expert; tscales [E, 3] for NVFP4.
    Returns (y [T, d] float32, ids [T, k] int32, w [T, k] float64)."""
    x = np.ascontiguousarray(x, np.float64)
    wr = np.ascontiguousarray(w_router, np.float64)
    T, E = x.shape[0], wr.shape[0]
    b = None if bias is None else np.ascontiguousarray(bias, np.float64)
    per_token = 1 if (b is not None and b.ndim == 2) else 0
    keep = [np.ascontiguousarray(bl).view(np.uint8) for bl in blobs]
    ptrs = (ctypes.c_void_p * E)(*[bl.ctypes.data for bl in keep])
    ts = None if tscales is None else np.ascontiguousarray(tscales, np.float32).reshape(E, 3)
    y = np.zeros((T, d), np.float32)
    ids = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float64)
    n = threads or os.cpu_count() or 1
    r = lib().fto_layer_forward(_p(x), T, d, d_ff, E, k, _p(wr), _p(b), per_token, ptrs, wtype, _p(ts), n, _p(y),
                                _p(ids), _p(w))
    if r != 0:
        raise ValueError("fto_layer_forward: bad argument")
    return y, ids, w


def route(x, w_router, bias, k):
    """Router only: (ids [T, k] int32, w [T, k] float64)."""
    x = np.ascontiguousarray(x, np.float64)
    wr = np.ascontiguousarray(w_router, np.float64)
    T, E = x.shape[0], wr.shape[0]
    b = None if bias is None else np.ascontiguousarray(bias, np.float64)
    per_token = 1 if (b is not None and b.ndim == 2) else 0
    ids = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float64)
    if lib().fto_route(_p(x), T, x.shape[1], E, k, _p(wr), _p(b), per_token, _p(ids), _p(w)) != 0:
        raise ValueError("fto_route: bad argument")
    return ids, w


def weight(blob, wtype, d, d_ff, tscale, m, r, c) -> float:
    bl = np.ascontiguousarray(blob).view(np.uint8)
    ts = None if tscale is None else np.ascontiguousarray(tscale, np.float32)
    return lib().fto_weight(_p(bl), wtype, d, d_ff, _p(ts), m, r, c)


def e2m1(code: int) -> float:
    return lib().fto_e2m1(code)


def e4m3(code: int) -> float:
    return lib().fto_e4m3(code)


class Cache:
    """The C++ shared LRU simulator (decode and prefill calls)."""

    def __init__(self, L, E, C, bp_mbps, bh_mbps):
        self.L, self.E, self.C = L, E, C
        self.h = lib().fto_cache_new(L, E, C, bp_mbps, bh_mbps)
        if not self.h:
            raise ValueError("fto_cache_new: bad argument")

    def forward(self, layer, mode, counts):
        """Record of one layer call: lookups [(layer, e, kind)], n_cur, m, qstar, qstage."""
        counts = np.ascontiguousarray(counts, np.int32)
        n = 2 * self.E
        ll, le, lk = np.zeros(n, np.int32), np.zeros(n, np.int32), np.zeros(n, np.int32)
        out = [ctypes.c_int() for _ in range(5)]
        r = lib().fto_cache_forward(self.h, layer, mode, _p(counts), _p(ll), _p(le), _p(lk),
                                    *[ctypes.byref(o) for o in out])
        if r != 0:
            raise RuntimeError("fto_cache_forward: no unpinned slot")
        nl, ncur, m, q, qs = (o.value for o in out)
        return dict(lookups=[(int(ll[i]), int(le[i]), int(lk[i])) for i in range(nl)], n_cur=ncur, m=m, qstar=q,
                    qstage=qs)

    def counters(self):
        out = np.zeros(6, np.uint64)
        lib().fto_cache_counters(self.h, _p(out))
        return dict(zip(("lookups", "hits", "misses", "staged", "streamed", "layer_calls"), (int(v) for v in out)))

    def contents(self):
        key_of = np.zeros(max(self.C, 1), np.int64)
        stamp = np.zeros(max(self.C, 1), np.uint64)
        lib().fto_cache_contents(self.h, _p(key_of), _p(stamp))
        return key_of[:self.C].tolist(), [int(s) for s in stamp[:self.C]]

    def close(self):
        if self.h:
            lib().fto_cache_free(self.h)
            self.h = None

    def __del__(self):
        self.close()
