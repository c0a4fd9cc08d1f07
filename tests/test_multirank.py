"""The N > 1 path of bench.py on the CPU: two gloo ranks run the same
aggregation the GPU ranks run over NCCL (one independent replica per rank,
no data exchange; the job's time is the slowest rank's)."""
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
