"""Weight formats of a slot blob, decoded from their definitions.

Test infrastructure (see oracle/__init__.py).

A slot holds every tensor one (layer, expert) pair needs ([paperlens]
"設計: 2階建てのエキスパート記憶", paper §3). The byte layout is the one
include/ft_moe.h specifies; this module implements it independently:

  fp32 / bf16: W_gate [d_ff, d], W_up [d_ff, d], W_down [d, d_ff], row-major.
  NVFP4: all 4-bit e2m1 codes (gate, up, down; two per byte, even column in
  the low nibble), then all e4m3 block scales (one per 16 consecutive
  elements along a row), times one fp32 tensor scale per matrix.

e2m1 (OCP microscaling FP4): sign bit 3, exponent bits 2..1 with bias 1,
mantissa bit 0; exponent 0 is subnormal (value = mantissa * 0.5).
e4m3 (OCP FP8 E4M3, "FN"): sign bit 7, exponent bits 6..3 with bias 7,
mantissa bits 2..0; exponent 0 is subnormal (mantissa/8 * 2^-6); exponent 15
with mantissa 7 is NaN; no infinities; max 448.

Pins: all 16 e2m1 codes against the value list of the format
(tests/golden/e2m1_values.txt); all 256 e4m3 codes against torch's
float8_e4m3fn conversion; the NVFP4 blob size against the 43 x 256 x S_e pool
size the workloads quote.
"""
from __future__ import annotations

import numpy as np

F32, BF16, NVFP4 = 0, 1, 2


def e2m1_value(code: int) -> float:
    """Value of a 4-bit e2m1 code."""
    sign = -1.0 if code & 0x8 else 1.0
    exp = (code >> 1) & 0x3
    man = code & 0x1
    if exp == 0:
        return sign * man * 0.5
    return sign * 2.0 ** (exp - 1) * (1.0 + man / 2.0)


def e4m3_value(code: int) -> float:
    """Value of an 8-bit e4m3 (FN) code; NaN for 0x7F / 0xFF."""
    sign = -1.0 if code & 0x80 else 1.0
    exp = (code >> 3) & 0xF
    man = code & 0x7
    if exp == 0xF and man == 0x7:
        return float("nan")
    if exp == 0:
        return sign * (man / 8.0) * 2.0 ** -6
    return sign * 2.0 ** (exp - 7) * (1.0 + man / 8.0)


E2M1 = np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)
E4M3 = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


def slot_bytes(d: int, d_ff: int, wtype: int) -> int:
    n = 3 * d * d_ff
    return {F32: 4 * n, BF16: 2 * n, NVFP4: n // 2 + n // 16}[wtype]


def bf16_to_f64(u16: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64 (exact: bf16 is the top half of fp32)."""
    return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _nvfp4_matrix(codes: np.ndarray, scales: np.ndarray, rows: int, K: int, tscale: float) -> np.ndarray:
    lo = codes & 0x0F
    hi = codes >> 4
    nib = np.empty(rows * K, dtype=np.uint8)
    nib[0::2] = lo
    nib[1::2] = hi
    v = E2M1[nib].reshape(rows, K)
    s = E4M3[scales].reshape(rows, K // 16)
    return v * np.repeat(s, 16, axis=1) * float(tscale)


def unpack_expert(blob: np.ndarray, d: int, d_ff: int, wtype: int, tscales=None):
    """Slot blob (uint8 array of slot_bytes) -> (W_gate, W_up, W_down) float64."""
    blob = np.ascontiguousarray(blob).view(np.uint8)
    assert blob.size == slot_bytes(d, d_ff, wtype), (blob.size, slot_bytes(d, d_ff, wtype))
    n = d * d_ff
    if wtype == F32:
        w = blob.view(np.float32).astype(np.float64)
    elif wtype == BF16:
        w = bf16_to_f64(blob.view(np.uint16))
    else:
        codes, scales = blob[: 3 * n // 2], blob[3 * n // 2:]
        ts = np.asarray(tscales, dtype=np.float32).astype(np.float64)
        cg, cu, cd = codes[: n // 2], codes[n // 2: n], codes[n: 3 * n // 2]
        sg, su, sd = scales[: n // 16], scales[n // 16: n // 8], scales[n // 8: 3 * n // 16]
        return (_nvfp4_matrix(cg, sg, d_ff, d, ts[0]),
                _nvfp4_matrix(cu, su, d_ff, d, ts[1]),
                _nvfp4_matrix(cd, sd, d, d_ff, ts[2]))
    return (w[:n].reshape(d_ff, d), w[n: 2 * n].reshape(d_ff, d), w[2 * n:].reshape(d, d_ff))
