"""bench.py on the CPU: the N > 1 path, where two gloo ranks run the same
aggregation the GPU ranks run over NCCL (one independent replica per rank,
no data exchange; the job's time is the slowest rank's), the peak
choice, and the reference arm's contract line."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, q):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        local_ms = [12.0, 15.0][rank]  # rank 1 is the slower replica
        worst = bench.max_over_ranks(local_ms, torch.device("cpu"))
        value = bench.whole_job_tflops(world, 2.0e12, 10, worst)
        q.put((rank, worst, value))
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, worst, value in got:
        assert worst == 15.0
        # 2 replicas x 10 steps x 2 TFLOP over 15 ms
        assert value == pytest.approx(2 * 2.0e12 * 10 / 15e-3 / 1e12)


def test_single_rank_is_its_own_maximum():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5
    assert bench.whole_job_tflops(1, 1.0e12, 4, 2.0) == pytest.approx(1.0e12 * 4 / 2e-3 / 1e12)


def test_peak_choice_follows_the_timed_region(tmp_path, monkeypatch):
    """A kernel timed inside a long (power-capped) region is rated against
    the sustained bf16 figure, a short burst against the burst figure."""
    import json

    import bench
    peaks = {"bf16_tflops": 1615.5, "bf16_tflops_sustained": 1402.0, "hbm_gbs": 6559.0}
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(peaks))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peak, burst, kind = bench.tensor_peak(1360.0)
    assert (peak, burst) == (1402.0, 1615.5) and "sustained" in kind
    peak, burst, kind = bench.tensor_peak(22.0)
    assert (peak, burst) == (1615.5, 1615.5) and "burst" in kind
    monkeypatch.setattr(bench, "ROOT", str(tmp_path / "absent"))
    assert bench.tensor_peak(22.0)[0] == 1590.0 and bench.tensor_peak(2000.0)[0] == 1400.0


def _bench(args, env_extra=None):
    import subprocess
    env = dict(os.environ, **(env_extra or {}))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, capture_output=True, text=True,
                          env=env, timeout=600)


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` (the CPU oracle, the one other place the
    benchmark runs it) prints one JSON line with the contract's keys, the
    GPU arm's metric and unit, and an e2e object with no host copies."""
    import json

    sys.path.insert(0, ROOT)
    import bench
    r = _bench(["--impl", "reference", "--config", "tiny", "--steps", "1", "--warmup", "3"])
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "TFLOP/s"
    assert d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 3 and d["higher_is_better"] is True
    assert d["value"] > 0 and d["config"]["workload"] == bench.CONFIGS["tiny"].name
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_without_work():
    r = _bench(["--impl", "reference", "--config", "tiny", "--steps", "1", "--warmup", "3"],
               {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_bench_rejects_fewer_than_three_warmup_steps():
    r = _bench(["--impl", "reference", "--config", "tiny", "--steps", "1", "--warmup", "2"])
    assert r.returncode != 0 and "warmup" in r.stderr
