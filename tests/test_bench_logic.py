"""Host logic of bench.py (no GPU): which roof each kernel is held against,
the dominant kernel, the shares, and the ncu traffic lookup that turns null
once a kernel's source changed."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

PEAKS = {"hbm_gbs": 6553.6, "bf16_tflops": 1672.7}


def test_roofline_classes_and_dominant_kernel():
    prof = {
        # a GEMM below the ridge (HBM time > tensor time) is held against HBM
        "gemm_tc_gateup": {"launches": 1, "ms": 1.0, "bytes": 6.0e9, "flops": 0.6e12},
        # above the ridge against the tensor peak
        "gemm_tc_down": {"launches": 1, "ms": 2.0, "bytes": 1.0e9, "flops": 2.0e12},
        "gemv_hit": {"launches": 4, "ms": 0.5, "bytes": 2.0e9, "flops": 0.0},
        "gemv_streamed": {"launches": 2, "ms": 3.0, "bytes": 0.1e9, "flops": 0.0},
        "gemv_staged": {"launches": 2, "ms": 0.2, "bytes": 0.01e9, "flops": 0.0},
        "h2d_stage_copies": {"launches": 2, "ms": 9.0, "bytes": 0.45e9, "flops": 0.0},
    }
    roof, rows = bench.roofline(prof, PEAKS, "measured", 55.0, 50.0)
    assert rows["gemm_tc_gateup"]["bound"] == "hbm" and rows["gemm_tc_gateup"]["unit"] == "GB/s"
    assert abs(rows["gemm_tc_gateup"]["achieved"] - 6000.0) < 0.01
    assert rows["gemm_tc_down"]["bound"] == "tensor" and abs(rows["gemm_tc_down"]["achieved"] - 1000.0) < 0.01
    assert rows["gemv_hit"]["bound"] == "hbm"
    # the copy engine and the staged class against the H2D copy rate, the
    # streamed class against the zero-copy read rate
    for k in ("gemv_staged", "h2d_stage_copies"):
        assert rows[k]["bound"] == "host_link" and rows[k]["peak"] == 55.0
    assert rows["gemv_streamed"]["bound"] == "host_link" and rows["gemv_streamed"]["peak"] == 50.0
    assert abs(rows["gemv_streamed"]["frac"] - round(0.1e9 / 3.0e6 / 50.0, 4)) < 1e-4
    assert abs(sum(v["share"] for v in rows.values()) - 1.0) < 1e-3
    # the copy engine's staging takes the most time: it is the dominant row
    assert roof["kernel"] == "h2d_stage_copies" and roof["bound"] == "host_link"
    assert abs(roof["frac"] - round(0.45e9 / 9.0e6 / 55.0, 4)) < 1e-4
    assert roof["algorithmic_bytes_per_launch"] == round(0.45e9 / 2)
    # without a zero-copy figure the streamed class falls back to the H2D rate
    _, rows2 = bench.roofline(prof, PEAKS, "measured", 55.0)
    assert rows2["gemv_streamed"]["peak"] == 55.0


def test_traffic_lookup_follows_the_source(tmp_path, monkeypatch):
    prof_dir = tmp_path / "profiles"
    prof_dir.mkdir()
    sha = bench._source_sha("gemv_hit")
    assert sha is not None and bench._source_sha("no_such_kernel") is None
    (prof_dir / "ncu_traffic.json").write_text(json.dumps({
        "gemv_hit": {"dram_bytes_per_launch": 123, "source_sha": sha},
        "gemv_staged": {"dram_bytes_per_launch": 456, "source_sha": "0" * 12}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # _source_sha reads the kernel sources under ROOT: give it the real ones
    os.makedirs(tmp_path / "sparse_moe_expert_topk_b200" / "csrc")
    src = os.path.join(ROOT, "sparse_moe_expert_topk_b200", "csrc", "k_gemv_mma.cu")
    (tmp_path / "sparse_moe_expert_topk_b200" / "csrc" / "k_gemv_mma.cu").write_bytes(open(src, "rb").read())
    assert bench.ncu_traffic("gemv_hit", 1) == 123
    assert bench.ncu_traffic("gemv_staged", 1) is None  # taken from an older source
    assert bench.ncu_traffic("route_decode_fused", 1) is None  # not recorded


def test_kernel_microbenchmarks_are_single_gpu(monkeypatch):
    """The kernel microbenchmark workloads run on one GPU and only for this
    implementation; other requests stop before any device is touched."""
    import pytest
    for argv in (["--workload", "hit_gemv", "--gpus", "2"], ["--workload", "stream_gemv", "--impl", "reference"],
                 ["--workload", "prefill_gemm", "--gpus", "8"]):
        monkeypatch.setattr(sys, "argv", ["bench.py", *argv])
        with pytest.raises(SystemExit) as e:
            bench.main()
        assert "one GPU" in str(e.value)


def test_unknown_workload_is_rejected(monkeypatch):
    import pytest
    monkeypatch.setattr(sys, "argv", ["bench.py", "--workload", "no_such_workload"])
    with pytest.raises((SystemExit, KeyError, ValueError)):
        bench.main()


def test_mixed_point_skips_when_the_host_cannot_hold_the_pool(monkeypatch):
    """The config-5 leg of the default line needs the 117 GB pinned pool; on a
    host without that much memory it reports why it was skipped, with and
    without the decode prefetch, and touches no device."""
    monkeypatch.setattr(bench, "host_mem_available", lambda: 64 << 30)
    for pf in (False, True):
        r = bench.mixed_point(0, 0, prefetch=pf)
        assert set(r) == {"skipped"} and "host memory" in r["skipped"]
