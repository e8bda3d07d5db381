"""Pins of oracle/formats.py: e2m1 / e4m3 decoders and the blob layout."""
import numpy as np
import pytest
import torch

import ftgen
from oracle import formats
from conftest import read_golden


def test_e2m1_all_codes_match_format_table():
    rows = [r.split() for r in read_golden("e2m1_values.txt")]
    assert len(rows) == 16
    for code, val in rows:
        got = formats.e2m1_value(int(code))
        assert got == float(val)
        assert np.signbit(got) == np.signbit(float(val)) or float(val) != 0.0


def test_e4m3_all_codes_match_torch_float8():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        got = formats.e4m3_value(c)
        if np.isnan(ref[c]):
            assert np.isnan(got), c
        else:
            assert got == ref[c], (c, got, ref[c])
    assert formats.e4m3_value(0x7E) == 448.0
    assert formats.e4m3_value(0x01) == 2.0 ** -9


def test_nvfp4_roundtrip_of_representable_values():
    # Build a blob whose decoded matrices are known exactly: pick codes and
    # scales, write them in the documented layout, decode, compare.
    d, d_ff = 32, 64
    rng = np.random.default_rng(0)
    n = d * d_ff
    mats = []
    codes_all, scales_all = [], []
    for rows, K in ((d_ff, d), (d_ff, d), (d, d_ff)):
        c = rng.integers(0, 16, size=(rows, K), dtype=np.uint8)
        s = rng.choice([0x30, 0x38, 0x40, 0x3C], size=(rows, K // 16)).astype(np.uint8)
        vals = np.array([[formats.e2m1_value(int(c[r, j])) * formats.e4m3_value(int(s[r, j // 16]))
                          for j in range(K)] for r in range(rows)])
        packed = (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8).reshape(-1)
        codes_all.append(packed)
        scales_all.append(s.reshape(-1))
        mats.append(vals)
    blob = np.concatenate(codes_all + scales_all)
    assert blob.size == formats.slot_bytes(d, d_ff, formats.NVFP4) == 3 * n // 2 + 3 * n // 16
    ts = np.array([1.0, 0.5, 2.0], dtype=np.float32)
    wg, wu, wd = formats.unpack_expert(blob, d, d_ff, formats.NVFP4, ts)
    np.testing.assert_array_equal(wg, mats[0] * 1.0)
    np.testing.assert_array_equal(wu, mats[1] * 0.5)
    np.testing.assert_array_equal(wd, mats[2] * 2.0)


def test_bf16_and_f32_unpack_layout():
    d, d_ff = 8, 16
    for wtype, dt in ((formats.F32, torch.float32), (formats.BF16, torch.bfloat16)):
        w = torch.arange(3 * d * d_ff, dtype=torch.float32).to(dt)
        blob = w.view(torch.uint8).numpy()
        wg, wu, wd = formats.unpack_expert(blob, d, d_ff, wtype)
        ref = w.to(torch.float64).numpy()
        np.testing.assert_array_equal(wg, ref[: d * d_ff].reshape(d_ff, d))
        np.testing.assert_array_equal(wu, ref[d * d_ff: 2 * d * d_ff].reshape(d_ff, d))
        np.testing.assert_array_equal(wd, ref[2 * d * d_ff:].reshape(d, d_ff))


def test_pool_size_matches_workload_shape():
    g = dict(r.split() for r in read_golden("pool_shape.txt"))
    L, E, d, dff = (int(g[k]) for k in ("layers", "experts", "d_model", "d_ff"))
    assert formats.slot_bytes(d, dff, formats.NVFP4) == int(g["nvfp4_slot_bytes"])
    assert formats.slot_bytes(d, dff, formats.BF16) == int(g["bf16_slot_bytes"])
    assert L * E * formats.slot_bytes(d, dff, formats.NVFP4) == int(g["nvfp4_pool_bytes"])
    assert ftgen.slot_bytes(d, dff, ftgen.W_NVFP4) == int(g["nvfp4_slot_bytes"])


@pytest.mark.parametrize("wtype", [ftgen.W_F32, ftgen.W_BF16, ftgen.W_NVFP4])
def test_generated_blob_decodes_to_small_weights(wtype):
    d, d_ff = 64, 128
    blob = ftgen.expert_blob(d, d_ff, wtype, seed=5).numpy()
    ts = ftgen.tensor_scales(5) if wtype == ftgen.W_NVFP4 else None
    wg, wu, wd = formats.unpack_expert(blob, d, d_ff, wtype, ts)
    for w in (wg, wu, wd):
        assert np.all(np.isfinite(w))
        assert 0.01 < np.sqrt(np.mean(w ** 2)) < 0.04
