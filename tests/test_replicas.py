"""The N > 1 path of the bench on CPU: two `gloo` ranks stand in for two
replicas (the layer has no exchange step, so the GPUs run independent
replicas and only the timing is reduced across ranks)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        w, r, _ = bench._dist()
        bench._barrier(w)
        ms = 100.0 + 50.0 * r                 # the second replica is slower
        mx = bench._maxreduce(ms, w)
        out.put((r, w, mx, bench._job_rate(w, 16384, 10, mx)))
        bench._barrier(w)
    finally:
        dist.destroy_process_group()


def test_two_replicas_time_is_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, w, mx, rate in res:
        assert w == 2 and mx == 150.0
        # both replicas' tokens over the slowest replica's time
        assert rate == pytest.approx(2 * 16384 * 10 / 0.150)


def test_reference_arm_runs_on_rank_0_only(monkeypatch):
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("LOCAL_RANK", "1")

    class A:
        config = "tiny"; tokens = 0; experts = 0; steps = 1; warmup = 0; gpus = 2
    assert bench.run_reference(A()) is None     # returns at once, no oracle work
