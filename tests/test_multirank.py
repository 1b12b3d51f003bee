"""The multi-rank (replica) path of bench.py, on CPU with the gloo backend:
ranks agree on the slowest rank's time, whole-job throughput counts every
rank's tokens, and the reference arm runs on rank 0 only."""

import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        t = bench.reduce_max(10.0 + 5.0 * rank)  # rank 1 is the slow one
        v = bench.job_throughput(1000, 4, world, t)
        q.put((rank, t, v))
    finally:
        dist.destroy_process_group()


def test_ranks_agree_on_max_time_and_job_throughput():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [r[1] for r in res] == [15.0, 15.0]
    # 2 ranks x 1000 tokens x 4 steps over the slowest rank's 15 ms
    assert res[0][2] == pytest.approx(2 * 1000 * 4 / 0.015)


def test_single_process_reduce_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.5) == 3.5


def test_reference_arm_skips_non_zero_ranks(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    import synth
    monkeypatch.setenv("RANK", "1")

    class Args:
        steps, warmup, gpus = 1, 0, 2

    bench.run_reference(Args(), synth.preset("tiny"))
    assert capsys.readouterr().out == ""


def test_reference_arm_line_carries_the_contract_keys(monkeypatch, capsys):
    """Rank 0 prints one JSON line: the metric keys, the oracle as its own CPU
    baseline, and an e2e block with no host copies."""
    import json
    sys.path.insert(0, ROOT)
    import bench
    import synth
    monkeypatch.setenv("RANK", "0")

    class Args:
        steps, warmup, gpus = 2, 1, 1

    bench.run_reference(Args(), bench.resolve_schedule(synth.preset("tiny"), use_oracle=True))
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in rec, key
    assert rec["impl"] == "reference" and rec["steps"] == 2 and rec["warmup"] == 1 and rec["value"] > 0
    assert rec["unit"] == bench.UNIT and rec["metric"] == bench.METRIC and rec["higher_is_better"] is True
    assert "workload" in rec["config"]
    cb = rec["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == rec["value"] and cb["cores"] >= 1 and cb["sample"]
    assert rec["e2e"] == {"value": rec["value"], "unit": rec["unit"], "h2d_bytes_per_step": 0,
                          "d2h_bytes_per_step": 0}
