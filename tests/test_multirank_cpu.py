"""The multi-rank bookkeeping of bench.py on CPU (two gloo ranks): every rank runs its
own replica, the job time is the max over ranks, and the throughput is the weak-scaling
sum. The path needs no data-path collective, so this is all that runs across ranks."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ms = 10.0 + 5.0 * rank                       # rank 1 is the slow one
    job_ms = bench.max_over_ranks(ms, dist, "cpu")
    tops = bench.weak_scaling_tops(8.8e12, 3, world, job_ms)
    out[rank] = (job_ms, tops)
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    port = _free_port()
    mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        job_ms, tops = out[r]
        assert job_ms == pytest.approx(15.0)
        assert tops == pytest.approx(2 * 8.8e12 * 3 / 15e-3 / 1e12)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(7.5) == 7.5
    assert bench.weak_scaling_tops(1e12, 2, 1, 1000.0) == pytest.approx(2.0)


def test_end_to_end_bound_from_the_input_copy():
    """The e2e ceiling: the step's input bytes over the measured copy time."""
    b = bench._e2e_bound(8.8e12, 1, 805306368, 14.5)
    assert b["h2d_gbs"] == pytest.approx(805306368 / 14.5e-3 / 1e9)
    assert b["h2d_bound"] == pytest.approx(8.8e12 / 14.5e-3 / 1e12)
    assert bench._e2e_bound(8.8e12, 4, 805306368, 14.5)["h2d_bound"] == pytest.approx(
        4 * 8.8e12 / 14.5e-3 / 1e12)


def test_gpus_flag_starts_its_own_ranks():
    """`--gpus 2` outside torchrun: the script re-executes itself under torchrun with two
    ranks, and rank 0 reports the max over ranks (rank 1 is the slow one)."""
    import json
    import subprocess
    import sys
    probe = os.path.join(os.path.dirname(os.path.abspath(__file__)), "replica_probe.py")
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    r = subprocess.run([sys.executable, probe, "--gpus", "2"], capture_output=True, text=True,
                       timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    out = json.loads(lines[0])
    assert out["world"] == 2
    assert out["job_ms"] == pytest.approx(15.0)
    assert out["tops"] == pytest.approx(2 * 8.8e12 * 3 / 15e-3 / 1e12)


def test_gpus_flag_must_match_torchrun_world(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "4")
    with pytest.raises(SystemExit):
        bench.maybe_relaunch(2, "bench.py", [])
    bench.maybe_relaunch(4, "bench.py", [])      # consistent: nothing to do
    bench.maybe_relaunch(None, "bench.py", [])


def test_peaks_and_quant_bytes():
    peaks = {"bf16_tflops": 1660.9, "bf16_tflops_sustained": 1399.1, "hbm_gbs": 6541.8}
    mixed, int8, bf16, which = bench.tensor_peaks(peaks, False, 140.0)
    assert which == "burst" and bf16 == 1660.9
    assert mixed == pytest.approx(1 / (0.5 / 3321.8 + 0.5 / 1660.9))
    mixed8, _, _, _ = bench.tensor_peaks(peaks, True, 140.0)
    assert mixed8 == pytest.approx(3321.8)
    assert bench.tensor_peaks(peaks, False, 5000.0)[3] == "sustained"
    b = bench.quant_bytes(2, 32, 16384, 16384, 128, False, False)
    n = 2 * 32 * 16384 * 128
    assert b["algorithmic"] == 6 * n + 4 * 2 * 32 * 128 + 4 * 2 * 32 * (128 + 256)
    assert b["moved"] == b["algorithmic"] + 2 * n


def test_clock_summary_keeps_the_timed_region_only():
    # samples as the NVML poller records them: (time, SM MHz, max SM MHz, active reasons)
    c = bench.ClockSampler(0)
    c.source = "nvml"
    c.samples = [(0.90, 1965.0, 1965.0, {"hw_slowdown"}),      # before the timed region
                 (1.00, 1965.0, 1965.0, set()),
                 (1.05, 1800.0, 1965.0, {"sw_power_cap"}),
                 (1.10, 1850.0, 1965.0, set()),
                 (1.50, 210.0, 1965.0, set())]                  # after it
    c.t0, c.t1 = 1.0, 1.1
    s = c.summary()
    assert s["samples"] == 3 and s["sm_mhz"] == 1850.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["source"] == "nvml"
    c.t0, c.t1 = 2.0, 2.1                                       # no sample inside
    assert c.summary()["samples"] == 0 and c.summary()["sm_mhz"] is None
