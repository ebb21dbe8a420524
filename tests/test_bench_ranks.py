"""Host logic of the multi-rank benchmark, on CPU with a world-size-2 gloo group: every rank
runs its own replica, the elapsed time is the maximum over ranks, the rate counts all ranks'
tokens, and the reference arm does its work on rank 0 only."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    r, w, lr = bench.dist_env()
    ms = bench.max_over_ranks(10.0 + 5.0 * rank, w, "cpu")
    rate = bench.whole_job_rate(8192, w, ms)
    out[rank] = (r, w, lr, ms, rate)
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_timing_and_rate():
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    assert out[0][:3] == (0, 2, 0) and out[1][:3] == (1, 2, 1)
    for r in (0, 1):
        assert out[r][3] == 15.0                       # max over ranks
        assert out[r][4] == pytest.approx(2 * 8192 / 0.015)


def test_reference_arm_runs_on_rank0_only(monkeypatch, capsys):
    import argparse
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = argparse.Namespace(workload="tiny", steps=3, warmup=3)
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_line_on_rank0(monkeypatch, capsys):
    """The reference arm (the oracle on the host cores) prints one JSON line with the keys the
    benchmark contract asks for."""
    import argparse
    import json
    import bench
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    args = argparse.Namespace(workload="tiny", steps=3, warmup=3)
    assert bench.run_reference(args) == 0
    lines = [l for l in capsys.readouterr().out.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["metric"] == bench.METRIC and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"] and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == "tiny"


def test_flop_counts():
    """Algorithmic FLOPs count the recompute; model FLOPs do not (OPD workload numbers)."""
    import bench
    from synthetic import WORKLOADS
    w = WORKLOADS["opd_0p6b_4b"]
    f = bench.algorithmic_flops(w, 4916)
    sweep = 2.0 * 4916 * 151936 * (1024 + 2560)
    assert f["sweep_fwd"] == f["sweep_grad"] == sweep and f["sweep_jsd"] == 0.0
    assert f["gemm_bwd"] == 4.0 * 4916 * 151936 * 1024
    assert sum(f.values()) == pytest.approx(13.77e12, rel=1e-3)
    assert bench.model_flops(w, 4916) == pytest.approx(sum(f.values()) - sweep, rel=1e-12)
    jsd = WORKLOADS["long_jsd"]
    fj = bench.algorithmic_flops(jsd, 6144)
    assert fj["sweep_jsd"] == fj["sweep_fwd"] > 0


def test_peak_follows_the_run_clock():
    """The roofline's peak is the burst figure when the run held its clock near the burst
    measurement's, the sustained figure near the sustained measurement's clock, and the burst
    figure scaled by the clock ratio in between."""
    import bench
    peaks = {"bf16_tflops": 1630.0, "bf16_tflops_sustained": 1371.8}
    p, desc, mhz = bench.choose_peak(peaks, "measured", 1942.0, 1965.0)
    assert p == 1630.0 and "burst" in desc and mhz == 1965.0
    p, desc, mhz = bench.choose_peak(peaks, "measured", 1290.0, 1965.0)
    assert p == 1371.8 and "sustained" in desc and mhz == bench.SUSTAINED_MHZ_DEFAULT
    p, desc, mhz = bench.choose_peak(peaks, "measured", 1620.0, 1965.0)
    assert p == pytest.approx(1630.0 * 1620.0 / 1965.0) and mhz == 1620.0
    # clock fields recorded in the peaks file take precedence over the defaults
    rec = dict(peaks, clocks={"bf16_burst_sm_mhz": 1900.0, "bf16_sustained_sm_mhz_median": 1400.0})
    assert bench.peak_clocks(rec) == (1900.0, 1400.0)
    assert bench.choose_peak(rec, "measured", 1410.0, 1965.0)[0] == 1371.8
    assert bench.choose_peak(rec, "measured", 1850.0, 1965.0)[0] == 1630.0
    # no clock record: the burst figure, said so
    p, desc, _ = bench.choose_peak(peaks, "measured", None, None)
    assert p == 1630.0 and "no clock record" in desc


def test_profiled_traffic_scales_by_columns_and_checks_the_code_hash(tmp_path, monkeypatch):
    """The roofline's traffic comes from the profiling-size twin's ncu summary, scaled by the
    vocabulary columns one launch covers, and only while the summary matches the device code."""
    import bench
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "sweep_grad_opd_0p6b_4b_v24k_prof.md").write_text(
        f"kernel_source_sha: {bench.kernel_source_sha()}\n"
        "profiled_vocab_columns_per_launch: 24576\ndram_bytes_per_launch: 4.0e8\n")
    real_sha = bench.kernel_source_sha()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_sha", lambda: real_sha)
    assert bench.profiled_traffic("sweep_grad", "opd_0p6b_4b", 49152) == pytest.approx(8.0e8)
    assert bench.profiled_traffic("sweep_grad", "long_jsd", 49152) is None        # no twin
    assert bench.profiled_traffic("gemm_bwd", "opd_0p6b_4b", 49152) is None       # no summary
    monkeypatch.setattr(bench, "kernel_source_sha", lambda: "0" * 16)              # code changed
    assert bench.profiled_traffic("sweep_grad", "opd_0p6b_4b", 49152) is None
