"""CPU tests of the benchmark's host logic: the max-over-ranks reduction on a
world-size-2 gloo group, the reference arm (the fp64 oracle) in one process and
under torchrun with two ranks (rank 0 alone prints its one JSON line), the clock
record (median SM clock and throttle reasons of the samples inside the timed region),
the stale-profile check of the traffic figure, and the peak lookup with its fallback."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out[rank] = bench.max_over_ranks(1.5 + rank, "cpu")
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        assert dict(out) == {0: 2.5, 1: 2.5}


def test_max_over_ranks_without_process_group():
    import bench
    assert bench.max_over_ranks(3.25, "cpu") == 3.25


def _json_lines(text):
    return [json.loads(l) for l in text.splitlines() if l.startswith("{")]


def test_reference_arm_one_process():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    l = lines[0]
    assert l["impl"] == "reference" and l["unit"] == "GB/s" and l["value"] > 0
    assert l["cpu_baseline"]["kind"] == "oracle" and l["cpu_baseline"]["cores"] >= 1
    assert l["e2e"] == {"value": l["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_two_ranks_torchrun():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1 and lines[0]["impl"] == "reference" and lines[0]["n_gpus"] == 2


# ---------------------------------------------------------------------------
# clock record, stale-profile detection and peak lookup (pure host logic)
# ---------------------------------------------------------------------------
def _sampler_with(samples, max_mhz=1965):
    import bench
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.samples, s.ok, s.max_mhz = samples, True, max_mhz
    return s


def test_clock_summary_median_and_reasons_inside_the_region():
    R = __import__("bench").ClockSampler.REASONS
    samples = [(0.5, 900, R["hw_slowdown"]),                # before the region: ignored
               (1.0, 1800, R["gpu_idle"]), (1.1, 1900, R["sw_power_cap"]), (1.2, 1950, 0),
               (3.0, 700, R["sw_thermal_slowdown"])]         # after: ignored
    out = _sampler_with(samples).summary(1.0, 1.2)
    assert out["sm_mhz"] == 1900 and out["sm_max_mhz"] == 1965 and out["samples"] == 3
    assert out["reasons"] == ["sw_power_cap"]                # gpu_idle is not a throttle reason


def test_clock_summary_short_region_takes_the_nearest_samples():
    R = __import__("bench").ClockSampler.REASONS
    samples = [(0.0, 1000, 0), (1.0, 1500, R["hw_thermal_slowdown"]), (1.01, 1600, 0),
               (1.02, 1700, 0), (5.0, 500, R["hw_slowdown"])]
    out = _sampler_with(samples).summary(1.004, 1.006)       # no sample inside
    assert out["samples"] == 3 and out["sm_mhz"] == 1600
    assert out["reasons"] == ["hw_thermal_slowdown"]


def test_clock_summary_without_nvml():
    s = _sampler_with([], max_mhz=None)
    s.ok = False
    assert s.summary(0.0, 1.0) == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_profiled_traffic_scales_per_unit_and_rejects_stale_profiles(tmp_path, monkeypatch):
    import bench
    path = tmp_path / "prof.json"
    prof = {"source_hash": bench.kernel_source_hash("absorb"), "dram_bytes_per_launch": 3.0e8,
            "units_per_launch": 1.0e6, "workload": bench.WORKLOAD}
    path.write_text(json.dumps(prof))
    monkeypatch.setattr(bench, "profile_path", lambda variant, workload=bench.WORKLOAD:
                        str(path) if workload == bench.WORKLOAD else str(tmp_path / "none.json"))
    assert bench.profiled_traffic(2.0e6, "absorb") == pytest.approx(6.0e8)
    # another workload runs another kernel instantiation: no scaled guess
    assert bench.profiled_traffic(2.0e6, "absorb", "rho4-prefill") is None
    prof["source_hash"] = "0" * 16                            # taken on other kernel sources
    path.write_text(json.dumps(prof))
    assert bench.profiled_traffic(2.0e6, "absorb") is None
    path.write_text("not json")
    assert bench.profiled_traffic(2.0e6, "absorb") is None
    path.unlink()
    assert bench.profiled_traffic(2.0e6, "absorb") is None


def test_committed_traffic_summaries_are_well_formed():
    """Each committed traffic summary names the hash of the sources it was taken on; the
    bench reports traffic only while they match (otherwise null)."""
    import glob
    import bench
    paths = glob.glob(os.path.join(bench.ROOT, "profiles", "*.json"))
    assert paths
    for path in paths:
        with open(path) as f:
            prof = json.load(f)
        assert prof["units_per_launch"] > 0 and prof["dram_bytes_per_launch"] > 0
        assert len(prof["source_hash"]) == 16
        import lla_synth
        assert prof["workload"] in lla_synth.WORKLOADS
        kernel, workload = os.path.basename(path)[:-5].split(".", 1)
        assert kernel in bench.PROFILE_KERNEL.values() and workload == prof["workload"]


def test_measured_peaks_fall_back_when_the_file_is_absent(tmp_path, monkeypatch):
    import bench
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, kind = bench.measured_peaks()
    assert kind == "fallback" and peaks["hbm_gbs"] == 6650.0 and peaks["bf16_tflops"] == 1590.0
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6543.1}))
    peaks, kind = bench.measured_peaks()
    assert kind == "measured" and peaks["hbm_gbs"] == 6543.1
