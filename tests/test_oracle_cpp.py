"""Pins of the plain C++ oracle (oracle/moe_oracle.cpp) against the numpy
oracle and the format tables: the numpy oracle is itself pinned to a dense
brute-force evaluation, closed forms, the OCP format tables and the pages'
q* profiles, and the two share no code.

The C++ oracle rounds where the layer's plain fp32 definition rounds (each
logit, g, u, h and Y once to float, the weighted sum in float), the numpy
oracle keeps fp64 throughout; so ids and weights must agree exactly and the
outputs within a few float roundings (1e-5 of rms)."""
import numpy as np
import pytest
import torch

from conftest import read_golden
from oracle import cache as ocache
from oracle import cpp
from oracle import formats as ofmt
from oracle import moe

F32, BF16, NVFP4 = ofmt.F32, ofmt.BF16, ofmt.NVFP4


def test_e2m1_codes_against_the_format_table():
    rows = read_golden("e2m1_values.txt")
    vals = [float(r.split()[1]) for r in rows]
    assert len(vals) == 16
    for c in range(16):
        assert cpp.e2m1(c) == vals[c], c


def test_e4m3_codes_against_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        v = cpp.e4m3(c)
        assert (np.isnan(v) and np.isnan(ref[c])) or v == ref[c], c


def _blob(rng, d, d_ff, wtype):
    n = 3 * d * d_ff
    if wtype == F32:
        return rng.normal(0, 0.3, n).astype(np.float32).view(np.uint8)
    if wtype == BF16:
        return (rng.normal(0, 0.3, n).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16).view(np.uint8)
    codes = rng.integers(0, 256, n // 2, dtype=np.uint8)
    scales = rng.choice(np.array([(e << 3) | m for e in (4, 5, 6, 7, 8) for m in range(8)], np.uint8), n // 16)
    return np.concatenate([codes, scales])


@pytest.mark.parametrize("wtype", [F32, BF16, NVFP4])
def test_weight_decode_matches_the_numpy_unpacking(wtype):
    rng = np.random.default_rng(wtype)
    d, d_ff = 32, 48
    blob = _blob(rng, d, d_ff, wtype)
    ts = np.array([0.5, 0.25, 2.0], np.float32)
    W = ofmt.unpack_expert(blob, d, d_ff, wtype, ts)
    for m, (rows, cols) in enumerate(((d_ff, d), (d_ff, d), (d, d_ff))):
        for r, c in [(0, 0), (rows - 1, cols - 1), (rows // 2, 17), (3, cols - 2)]:
            assert cpp.weight(blob, wtype, d, d_ff, ts, m, r, c) == W[m][r, c], (m, r, c)


def _problem(rng, T, E, d, d_ff, wtype, per_token=False):
    x = rng.normal(0, 1, (T, d)).astype(np.float32).astype(np.float64)
    wr = rng.normal(0, 0.5, (E, d)).astype(np.float32).astype(np.float64)
    b = rng.normal(0, 0.1, (T, E) if per_token else E)
    blobs = [_blob(rng, d, d_ff, wtype) for _ in range(E)]
    ts = rng.uniform(0.05, 0.2, (E, 3)).astype(np.float32) if wtype == NVFP4 else None
    return x, wr, b, blobs, ts


@pytest.mark.parametrize("wtype,T,E,k,per_token", [(F32, 9, 8, 2, False), (BF16, 5, 6, 3, True),
                                                   (NVFP4, 4, 5, 5, False), (BF16, 3, 7, 1, False)])
def test_layer_matches_the_numpy_oracle(wtype, T, E, k, per_token):
    rng = np.random.default_rng(100 + wtype * 10 + k)
    d, d_ff = 32, 48
    x, wr, b, blobs, ts = _problem(rng, T, E, d, d_ff, wtype, per_token)
    y, ids, w = cpp.layer_forward(x, wr, b, k, blobs, wtype, d, d_ff, ts, threads=3)
    W = [ofmt.unpack_expert(bl, d, d_ff, wtype, None if ts is None else ts[e]) for e, bl in enumerate(blobs)]
    y1, ids1, w1 = moe.layer_forward(x, wr, b, k, lambda e: W[e])
    np.testing.assert_array_equal(ids, ids1)
    np.testing.assert_array_equal(w, w1)
    ids2, w2 = cpp.route(x, wr, b, k)
    np.testing.assert_array_equal(ids2, ids1)
    np.testing.assert_array_equal(w2, w1)
    rms = np.sqrt(np.mean(y1 ** 2))
    assert np.max(np.abs(y - y1)) <= 1e-5 * rms


def test_all_ties_and_duplicate_rows():
    rng = np.random.default_rng(5)
    d, d_ff, E, k, T = 16, 24, 6, 3, 4
    _, wr, _, blobs, _ = _problem(rng, T, E, d, d_ff, BF16)
    y, ids, w = cpp.layer_forward(np.zeros((T, d)), wr, np.zeros(E), k, blobs, BF16, d, d_ff)
    assert (ids == np.arange(k)).all() and (w == 1.0 / k).all() and (y == 0).all()
    wr2 = wr.copy()
    wr2[4] = wr2[1]
    x = rng.normal(0, 1, (T, d))
    _, ids2, _ = cpp.layer_forward(x, wr2, None, 5, blobs, BF16, d, d_ff)
    for t in range(T):
        pos = {int(e): j for j, e in enumerate(ids2[t])}
        if 4 in pos:
            assert 1 in pos and pos[1] < pos[4]


@pytest.mark.parametrize("L,E,C,bp,bh", [(3, 8, 5, 52700, 77300), (2, 6, 12, 11800, 47500), (4, 4, 0, 1, 1),
                                         (2, 8, 16, 77300, 77300), (3, 5, 7, 0, 100)])
def test_cache_matches_the_numpy_cache(L, E, C, bp, bh):
    """Decode and prefill calls over a random trace: the same lookup records,
    counters and slot contents as oracle/cache.ExpertCache."""
    rng = np.random.default_rng(L * 100 + E + C)
    a, b = ocache.ExpertCache(L, E, C, bp, bh), cpp.Cache(L, E, C, bp, bh)
    for step in range(40):
        layer = int(rng.integers(0, L))
        mode = ocache.PREFILL if step % 7 == 3 else ocache.DECODE
        counts = rng.integers(0, 3, E) * (rng.random(E) < 0.4)
        ra, rb = a.forward(layer, mode, counts), b.forward(layer, mode, counts)
        assert rb["lookups"] == [tuple(v) for v in ra["lookups"]]
        assert (rb["n_cur"], rb["m"], rb["qstar"], rb["qstage"]) == (ra["n_cur"], ra["m"], ra["qstar"], ra["qstage"])
    cnt = b.counters()
    for key in ("lookups", "hits", "misses", "staged", "streamed", "layer_calls"):
        assert cnt[key] == a.n[key], key
    assert b.contents() == (a.key_of, a.stamp)
    b.close()
