"""Python binding of libft_moe.so (include/ft_moe.h): argument marshalling only.

Every step of a layer call runs in the library's CUDA kernels; this module
loads the shared library, declares the C signatures, converts torch tensors
and streams to raw pointers and turns non-zero ft_status codes into FtError.
It never falls back to a Python or CPU implementation: if the library is
missing, loading fails loudly.

Names follow the C ABI: ft_moe_init, ft_moe_layer_forward, ft_cache_stats,
ft_set_bandwidths, ... (see include/ft_moe.h for arguments, layouts,
ownership and errors).
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libft_moe.so")

FT_OK, FT_EINVAL, FT_ENOMEM, FT_ECUDA, FT_ETIMEOUT, FT_ESTATE, FT_EUNSUPPORTED = range(7)
FT_W_F32, FT_W_BF16, FT_W_NVFP4 = 0, 1, 2
FT_DECODE, FT_PREFILL = 0, 1
KIND_HIT, KIND_STAGED, KIND_STREAMED = 0, 1, 2

# Every symbol include/ft_moe.h declares.
EXPORTS = (
    "ft_moe_slot_bytes", "ft_moe_init", "ft_moe_destroy", "ft_moe_expert_ptr", "ft_moe_set_tensor_scales",
    "ft_moe_set_router", "ft_moe_layer_forward", "ft_moe_layer_forward_host", "ft_cache_stats", "ft_set_bandwidths", "ft_moe_reset_cache",
    "ft_moe_resize_cache", "ft_moe_set_prefetch", "ft_moe_last_route", "ft_moe_cache_contents", "ft_moe_probe_link", "ft_moe_profile", "ft_moe_profile_read",
    "ft_route_topk_static", "ft_moe_expert_rows", "ft_ep_pack_scratch_bytes", "ft_ep_pack", "ft_ep_combine",
    "ft_status_str",
)
FT_ROUTE_STATIC_MAX_TOKENS = 1024


class FtConfig(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("n_experts", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("d_model", ctypes.c_int32), ("d_ff", ctypes.c_int32), ("wtype", ctypes.c_int32),
                ("cache_slots", ctypes.c_int64), ("max_tokens", ctypes.c_int32), ("device", ctypes.c_int32)]


class FtStats(ctypes.Structure):
    _fields_ = [("layer_calls", ctypes.c_uint64), ("lookups", ctypes.c_uint64), ("hits", ctypes.c_uint64),
                ("misses", ctypes.c_uint64), ("staged", ctypes.c_uint64), ("streamed", ctypes.c_uint64),
                ("bytes_h2d", ctypes.c_uint64), ("bytes_zero_copy", ctypes.c_uint64),
                ("last_m", ctypes.c_int32), ("last_qstar", ctypes.c_int32), ("last_qstage", ctypes.c_int32),
                ("device_error", ctypes.c_int32), ("kernel_launches", ctypes.c_uint64), ("prefetched", ctypes.c_uint64),
                ("ms_compute", ctypes.c_double), ("ms_copy", ctypes.c_double)]

    def as_dict(self):
        return {k: getattr(self, k) for k, _ in self._fields_}


class FtKernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_uint64), ("ms", ctypes.c_double),
                ("bytes", ctypes.c_double), ("flops", ctypes.c_double)]


class FtError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {status_str(status)} ({status})")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (raises OSError if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise OSError(f"{LIB_PATH} is missing: run `python -m sparse_moe_expert_topk_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, I64, U32, U64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32, ctypes.c_uint64
        pI32, pF = ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_float)
        sig = {
            "ft_moe_slot_bytes": [ctypes.POINTER(FtConfig), ctypes.POINTER(U64)],
            "ft_moe_init": [ctypes.POINTER(FtConfig), P, P, ctypes.POINTER(P)],
            "ft_moe_expert_ptr": [P, I32, I32, ctypes.POINTER(P)],
            "ft_moe_set_tensor_scales": [P, I32, I32, pF],
            "ft_moe_set_router": [P, I32, P],
            "ft_moe_layer_forward": [P, I32, I32, P, I32, P, I32, P, P, P],
            "ft_moe_layer_forward_host": [P, I32, I32, P, I32, P, I32, P],
            "ft_cache_stats": [P, ctypes.POINTER(FtStats)],
            "ft_set_bandwidths": [P, U32, U32],
            "ft_moe_reset_cache": [P],
            "ft_moe_resize_cache": [P, ctypes.c_int64],
            "ft_moe_set_prefetch": [P, I32],
            "ft_moe_last_route": [P] + [P] * 11,
            "ft_moe_cache_contents": [P, P, P],
            "ft_moe_probe_link": [P, U64, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)],
            "ft_moe_profile": [P, I32],
            "ft_moe_profile_read": [P, ctypes.POINTER(FtKernelTime), I32, ctypes.POINTER(I32), I32],
            "ft_route_topk_static": [P, P, P, I32, I32, I32, I32, I32, I32, P, P, P],
            "ft_moe_expert_rows": [P, I32, I32, P, P, I32, I32, P],
            "ft_ep_pack_scratch_bytes": [I32, I32, I32, ctypes.POINTER(U64)],
            "ft_ep_pack": [P, I32, I32, I32, I32, P, I32, I32, P, P, P, P, P, P, U64, P],
            "ft_ep_combine": [P, P, P, I32, I32, I32, I32, P, P],
        }
        for name, args in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        L.ft_moe_destroy.argtypes = [P]
        L.ft_moe_destroy.restype = None
        L.ft_status_str.argtypes = [ctypes.c_int]
        L.ft_status_str.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_str(s: int) -> str:
    return lib().ft_status_str(int(s)).decode()


def _check(fn, status):
    if status != FT_OK:
        raise FtError(fn, status)


def _ptr(t):
    """Raw address of a tensor (None -> NULL)."""
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(s):
    if s is None:
        return None
    return ctypes.c_void_p(s.cuda_stream if hasattr(s, "cuda_stream") else int(s))


def make_config(n_layers, n_experts, top_k, d_model, d_ff, wtype, cache_slots, max_tokens, device=0) -> FtConfig:
    return FtConfig(n_layers, n_experts, top_k, d_model, d_ff, wtype, cache_slots, max_tokens, device)


def ft_moe_slot_bytes(cfg: FtConfig) -> int:
    out = ctypes.c_uint64()
    _check("ft_moe_slot_bytes", lib().ft_moe_slot_bytes(ctypes.byref(cfg), ctypes.byref(out)))
    return out.value


def ft_moe_init(cfg: FtConfig, compute_stream, copy_stream) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check("ft_moe_init", lib().ft_moe_init(ctypes.byref(cfg), _stream(compute_stream), _stream(copy_stream),
                                            ctypes.byref(h)))
    return h


def ft_moe_destroy(ctx):
    lib().ft_moe_destroy(ctx)


def ft_moe_expert_ptr(ctx, layer, expert) -> int:
    p = ctypes.c_void_p()
    _check("ft_moe_expert_ptr", lib().ft_moe_expert_ptr(ctx, layer, expert, ctypes.byref(p)))
    return p.value


def ft_moe_set_tensor_scales(ctx, layer, expert, scales):
    arr = (ctypes.c_float * 3)(*[float(v) for v in scales])
    _check("ft_moe_set_tensor_scales", lib().ft_moe_set_tensor_scales(ctx, layer, expert, arr))


def ft_moe_set_router(ctx, layer, w_router):
    _check("ft_moe_set_router", lib().ft_moe_set_router(ctx, layer, _ptr(w_router)))


def ft_moe_layer_forward(ctx, layer, mode, x, T, bias, bias_per_token, y, ids=None, w=None):
    _check("ft_moe_layer_forward",
           lib().ft_moe_layer_forward(ctx, layer, mode, _ptr(x), T, _ptr(bias), bias_per_token, _ptr(y),
                                      _ptr(ids), _ptr(w)))


def ft_moe_layer_forward_host(ctx, layer, mode, x_host, T, bias, bias_per_token, y_host):
    """The layer on host tensors (pinned for asynchronous copies): x_host in,
    y_host out, both copied by the library on the compute stream."""
    _check("ft_moe_layer_forward_host",
           lib().ft_moe_layer_forward_host(ctx, layer, mode, _ptr(x_host), T, _ptr(bias), bias_per_token,
                                           _ptr(y_host)))


def ft_cache_stats(ctx) -> dict:
    s = FtStats()
    _check("ft_cache_stats", lib().ft_cache_stats(ctx, ctypes.byref(s)))
    return s.as_dict()


def ft_set_bandwidths(ctx, bp_mbps, bh_mbps):
    _check("ft_set_bandwidths", lib().ft_set_bandwidths(ctx, int(bp_mbps), int(bh_mbps)))


def ft_moe_reset_cache(ctx):
    _check("ft_moe_reset_cache", lib().ft_moe_reset_cache(ctx))


def ft_moe_resize_cache(ctx, new_slots):
    _check("ft_moe_resize_cache", lib().ft_moe_resize_cache(ctx, int(new_slots)))


def ft_moe_set_prefetch(ctx, enable):
    _check("ft_moe_set_prefetch", lib().ft_moe_set_prefetch(ctx, 1 if enable else 0))


def ft_moe_last_route(ctx, E, Tk):
    """Host copies of the last call's routing and lookup record (numpy)."""
    import numpy as np
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    perm = np.zeros(max(Tk, 1), np.int32)
    inv = np.zeros(max(Tk, 1), np.int32)
    le = np.zeros(2 * 512, np.int32)
    lk = np.zeros(2 * 512, np.int32)
    sc = [ctypes.c_int32() for _ in range(5)]
    ptr = lambda a: a.ctypes.data_as(ctypes.c_void_p)  # noqa: E731
    _check("ft_moe_last_route",
           lib().ft_moe_last_route(ctx, ptr(counts), ptr(offsets), ptr(perm), ptr(inv), ptr(le), ptr(lk),
                                   *[ctypes.byref(v) for v in sc]))
    n_lookup, n_cur, m, qstar, qstage = (v.value for v in sc)
    return dict(counts=counts, offsets=offsets, perm=perm[:Tk], inv=inv[:Tk], lookup_e=le[:n_lookup],
                lookup_kind=lk[:n_lookup], n_lookup=n_lookup, n_lookup_cur=n_cur, m=m, qstar=qstar, qstage=qstage)


def ft_moe_cache_contents(ctx, C):
    import numpy as np
    key_of = np.zeros(max(C, 1), np.int32)
    stamp = np.zeros(max(C, 1), np.uint64)
    _check("ft_moe_cache_contents", lib().ft_moe_cache_contents(ctx, key_of.ctypes.data_as(ctypes.c_void_p),
                                                                stamp.ctypes.data_as(ctypes.c_void_p)))
    return key_of[:C], stamp[:C]


def ft_moe_probe_link(ctx, nbytes):
    h2d, zc = ctypes.c_double(), ctypes.c_double()
    _check("ft_moe_probe_link", lib().ft_moe_probe_link(ctx, nbytes, ctypes.byref(h2d), ctypes.byref(zc)))
    return h2d.value, zc.value


def ft_moe_profile(ctx, enable: bool):
    _check("ft_moe_profile", lib().ft_moe_profile(ctx, 1 if enable else 0))


def ft_moe_profile_read(ctx, reset=True) -> dict:
    """{kernel name: {launches, ms, bytes, flops}} (synchronises)."""
    cap = 32
    arr = (FtKernelTime * cap)()
    n = ctypes.c_int32()
    _check("ft_moe_profile_read", lib().ft_moe_profile_read(ctx, arr, cap, ctypes.byref(n), 1 if reset else 0))
    return {arr[i].name.decode(): dict(launches=arr[i].launches, ms=arr[i].ms, bytes=arr[i].bytes,
                                       flops=arr[i].flops) for i in range(min(n.value, cap))}


def ft_route_topk_static(x, w_router, bias, bias_per_token, T, n_experts, d_model, top_k, wtype, ids, w, stream):
    """Router + top-k with no allocation (scratch in a static device array)."""
    _check("ft_route_topk_static",
           lib().ft_route_topk_static(_ptr(x), _ptr(w_router), _ptr(bias), bias_per_token, T, n_experts, d_model,
                                      top_k, wtype, _ptr(ids), _ptr(w), _stream(stream)))


def ft_moe_expert_rows(ctx, layer, mode, rows, eids, expert_base, n, out):
    """Owner side of the expert-parallel layer: rows routed to this context's
    experts (global ids eids, local id = eid - expert_base) -> fp32 outputs."""
    _check("ft_moe_expert_rows",
           lib().ft_moe_expert_rows(ctx, layer, mode, _ptr(rows), _ptr(eids), expert_base, n, _ptr(out)))


def ft_ep_pack_scratch_bytes(T, top_k, n_experts) -> int:
    out = ctypes.c_uint64()
    _check("ft_ep_pack_scratch_bytes", lib().ft_ep_pack_scratch_bytes(T, top_k, n_experts, ctypes.byref(out)))
    return out.value


def ft_ep_pack(ids, T, top_k, n_experts, n_owners, x, d_model, wtype, rows, eids, owner_counts, inv, bad_ids,
               scratch, stream):
    """Routed rows of this device in expert order, with the rows per owner."""
    _check("ft_ep_pack",
           lib().ft_ep_pack(_ptr(ids), T, top_k, n_experts, n_owners, _ptr(x), d_model, wtype, _ptr(rows),
                            _ptr(eids), _ptr(owner_counts), _ptr(inv), _ptr(bad_ids), _ptr(scratch),
                            0 if scratch is None else scratch.numel() * scratch.element_size(), _stream(stream)))


def ft_ep_combine(y_rows, w, inv, T, top_k, d_model, wtype, y, stream):
    """Combine of the expert outputs returned by the owners (rank order)."""
    _check("ft_ep_combine",
           lib().ft_ep_combine(_ptr(y_rows), _ptr(w), _ptr(inv), T, top_k, d_model, wtype, _ptr(y), _stream(stream)))
