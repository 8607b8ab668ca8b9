"""The multi-GPU host logic of bench.py (data-parallel replicas) with two gloo ranks
on the CPU: the LoRA weight gradients are summed over the ranks, timings reduce to
their maximum, rank 0 alone prints the JSON line, and the reference arm does no
work on ranks other than 0."""
import contextlib
import io
import json
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import bench
    rep = bench.Replicas("gloo", None, timeout_s=60)
    grads = [torch.full((4,), float(rank + 1)), torch.arange(3, dtype=torch.float32) * (rank + 1)]
    rep.allreduce_grads(grads)
    ms = rep.max_over_ranks(10.0 + rank)
    rep.barrier()
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        rep.emit({"rank": rank, "ms": ms})
    q.put((rank, [g.tolist() for g in grads], ms, out.getvalue()))
    rep.close()


def test_two_gloo_replicas():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        rank, grads, ms, printed = q.get(timeout=120)
        res[rank] = (grads, ms, printed)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in range(world):
        grads, ms, printed = res[rank]
        assert grads[0] == [3.0] * 4                   # 1 + 2
        assert grads[1] == [0.0, 3.0, 6.0]             # arange * (1 + 2)
        assert ms == 11.0                              # max over ranks
    assert json.loads(res[0][2]) == {"rank": 0, "ms": 11.0}
    assert res[1][2] == ""


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr("sys.argv", ["bench.py", "--impl", "reference", "--gpus", "2"])
    bench.reference_arm(bench.parse())
    assert capsys.readouterr().out == ""
