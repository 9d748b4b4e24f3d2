"""Measurement helpers of bench.py, on CPU: folding an ncu launch list onto the
library's profiler ids, scaling the committed DRAM traffic summary to a launch, and
the roofline object of the bench line.

The ncu CSV here is synthetic but has the layout ncu writes with --csv (one row per
launch and metric, "ID", "Kernel Name", "Metric Name", "Metric Value")."""

import argparse
import csv
import json

import pytest

import bench


def _write_csv(path, launches):
    """launches: list of (kernel name, {metric: value})."""
    with open(path, "w", newline="") as f:
        w = csv.writer(f)
        w.writerow(["ID", "Process ID", "Kernel Name", "Metric Name", "Metric Unit", "Metric Value"])
        for i, (name, metrics) in enumerate(launches):
            for mname, v in metrics.items():
                w.writerow([str(i), "1", name, mname, "", f"{v:,.3f}"])


def _args(tmp_path, log, launches):
    lp = tmp_path / "log.json"
    lp.write_text(json.dumps(log))
    cp = tmp_path / "launches.csv"
    _write_csv(cp, launches)
    return argparse.Namespace(launch_log=str(lp), traffic_csv=str(cp), traffic_out=str(tmp_path / "out.json"))


def _m(ns, rd=None, wr=None, tc=None, dt=None):
    d = {"gpu__time_duration.sum": ns}
    if rd is not None:
        d["dram__bytes_read.sum"] = rd
        d["dram__bytes_write.sum"] = wr
    if tc is not None:
        d["sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_elapsed"] = tc
    if dt is not None:
        d["dram__throughput.avg.pct_of_peak_sustained_elapsed"] = dt
    return d


LOG = {"workload": "toy", "optimizers": "muon", "source_hash": "abc",
       "launches": [{"kernel": "ns_gram", "flops": 1.0e9, "bytes": 0.0},
                    {"kernel": "muon_update", "flops": 0.0, "bytes": 4.0e6},
                    {"kernel": "ns_gram", "flops": 3.0e9, "bytes": 0.0}]}


def test_fold_aggregates_per_profiler_id(tmp_path):
    # a launch of another library first (not the library's), then the logged step
    launches = [("void at::native::elementwise_kernel<int>(int)", _m(500.0)),
                ("void mao::gemm_tc_kernel<0, 0, 1, 0>(mao::GemmParams)", _m(1000.0, 2e6, 1e6, 60.0, 10.0)),
                ("void mao::muon_update_kernel<__nv_bfloat16>(const MuonMatDev *)", _m(2000.0, 3e6, 2e6, 0.0, 80.0)),
                ("void mao::gemm_tc_kernel<0, 0, 1, 0>(mao::GemmParams)", _m(3000.0, 4e6, 1e6, 80.0, 20.0))]
    args = _args(tmp_path, LOG, launches)
    bench.fold_traffic(args)
    out = json.load(open(args.traffic_out))
    assert out["source_hash"] == "abc" and out["measured_on"] == "toy"
    g, u = out["kernels"]["ns_gram"], out["kernels"]["muon_update"]
    assert g["launches"] == 2 and u["launches"] == 1
    assert g["ncu_ms"] == pytest.approx(4000.0 / 1e6) and u["ncu_ms"] == pytest.approx(2000.0 / 1e6)
    assert g["share"] + u["share"] == pytest.approx(1.0)
    assert g["share"] == pytest.approx(4.0 / 6.0)
    # DRAM bytes per launch and per algorithmic FLOP / byte
    assert g["dram_bytes_per_launch"] == pytest.approx((3e6 + 5e6) / 2)
    assert g["dram_bytes_per_flop"] == pytest.approx(8e6 / 4e9)
    assert g["dram_bytes_per_alg_byte"] is None
    assert u["dram_bytes_per_alg_byte"] == pytest.approx(5e6 / 4e6)
    # utilisations are weighted by each launch's time
    assert g["tensor_pipe_pct"] == pytest.approx((1000 * 60.0 + 3000 * 80.0) / 4000)
    assert g["dram_pct"] == pytest.approx((1000 * 10.0 + 3000 * 20.0) / 4000)


def test_fold_rejects_a_misaligned_list(tmp_path):
    launches = [("void mao::gemm_tc_kernel<0, 0, 1, 0>(mao::GemmParams)", _m(1000.0)),
                ("void mao::gemm_tc_kernel<0, 0, 1, 0>(mao::GemmParams)", _m(2000.0)),  # the log says muon_update
                ("void mao::gemm_tc_kernel<0, 0, 1, 0>(mao::GemmParams)", _m(3000.0))]
    with pytest.raises(SystemExit, match="not aligned"):
        bench.fold_traffic(_args(tmp_path, LOG, launches))
    with pytest.raises(SystemExit, match="fewer ncu launches"):
        bench.fold_traffic(_args(tmp_path, LOG, launches[:2]))


def test_traffic_summary_scales_and_goes_stale(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "ncu_traffic.json").write_text(json.dumps({
        "source_hash": "h1", "measured_on": "toy",
        "kernels": {"pc_qr": {"dram_bytes_per_flop": 0.02, "dram_bytes_per_alg_byte": None},
                    "pc_elementwise": {"dram_bytes_per_flop": None, "dram_bytes_per_alg_byte": 0.96}}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "h1")
    t = bench.ncu_traffic("pc_qr", 1.0e12, 0.0)
    assert t["bytes"] == round(0.02 * 1.0e12) and t["by"] == "algorithmic flops" and t["scaled_from"] == "toy"
    t = bench.ncu_traffic("pc_elementwise", 0.0, 2.0e9)
    assert t["bytes"] == round(0.96 * 2.0e9) and t["by"] == "algorithmic bytes"
    assert bench.ncu_traffic("pc_chol", 1.0e9, 0.0) is None
    # changed kernel sources: the counters no longer describe them
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "h2")
    assert bench.ncu_traffic("pc_qr", 1.0e12, 0.0) is None


def test_committed_traffic_summary_matches_the_sources():
    """The committed per-kernel DRAM summary was captured on the current kernel sources
    (otherwise the bench reports no traffic)."""
    with open(bench.os.path.join(bench.ROOT, "profiles", "ncu_traffic.json")) as f:
        d = json.load(f)
    assert d["source_hash"] == bench.kernel_source_hash()


def test_roofline_of_tensor_and_hbm_kernels():
    peaks = {"bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
    # four launches of 2 ms: 1e12 useful FLOP each (0.8e12 counted by the host), 6e12 issued
    e = {"n": 4, "ms": 8.0, "flops": 4.0e12, "tc": 24.0e12, "planned": 3.2e12, "bytes": 0.0}
    r = bench.roofline_of("pc_qr", e, peaks, "fallback", {"bytes": 123, "by": "algorithmic flops",
                                                           "scaled_from": "toy"})
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["kernel"] == "pc_qr"
    assert r["achieved"] == pytest.approx(3000.0) and r["useful_tflops"] == pytest.approx(500.0)
    assert r["frac"] == pytest.approx(3000.0 / 1400.0, abs=1e-4)
    assert r["useful_tflops_host_counted"] == pytest.approx(400.0)
    assert r["traffic"] == 123 and "toy" in r["traffic_source"]
    assert r["launches"] == 4 and r["avg_launch_ms"] == pytest.approx(2.0)
    # an HBM pass: 2 launches of 1 ms moving 5 GB each
    e = {"n": 2, "ms": 2.0, "flops": 0.0, "tc": 0.0, "planned": 0.0, "bytes": 10.0e9}
    r = bench.roofline_of("pc_elementwise", e, peaks, "measured", None)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(5000.0) and r["frac"] == pytest.approx(5000.0 / 6650.0, abs=1e-4)
    assert r["traffic"] is None and "traffic_source" not in r
