"""Host logic of the multi-GPU bench path, on CPU with the gloo backend.

The step does not shard: N GPUs run N independent replicas, and the only
cross-rank operations are a barrier and the maximum of the per-rank times.
These tests run that logic in two processes, and check that the reference arm
does work on rank 0 alone.
"""
import datetime
import os
import socket

import pytest

import bench


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, queue):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = 5.0 + 2.5 * rank                       # rank 1 is the slow one
        slowest = bench.max_over_ranks(ms, world, "cpu")
        dist.barrier()
        queue.put((rank, slowest, bench.replicas_value(world, 1, 256, slowest)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_value_with_two_gloo_ranks():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    got = sorted(queue.get(timeout=10) for _ in range(2))
    for rank, slowest, value in got:
        assert slowest == pytest.approx(7.5)       # both ranks see the slowest time
        assert value == pytest.approx(2 * 256 / 7.5e-3)  # all ranks' tokens over that time


def test_single_rank_is_a_no_op_and_value_counts_every_replica():
    assert bench.max_over_ranks(3.25, 1, "cpu") == 3.25
    assert bench.replicas_value(1, 1, 256, 10.0) == pytest.approx(25600.0)
    assert bench.replicas_value(8, 1, 256, 10.0) == pytest.approx(8 * 25600.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    """Ranks other than 0 return at once, without building the oracle or
    printing anything."""
    import synth_inputs as si

    monkeypatch.setenv("RANK", "1")
    args = type("Args", (), {"gpus": 2, "steps": 1, "warmup": 0})()
    assert bench.run_reference(args, si.workload("a4b_p2k")) is None
    assert capsys.readouterr().out == ""
