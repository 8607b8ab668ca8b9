"""The multi-GPU host logic of bench.py (data-parallel replicas) with two gloo ranks
on the CPU: the LoRA weight gradients, one flat FP32 buffer, are summed over the
ranks in one collective and rounded to BF16 once afterwards; timings reduce to their
maximum, rank 0 alone prints the JSON line, and the reference arm does no work on
ranks other than 0."""
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
    calls = []
    real = rep.dist.all_reduce
    rep.dist.all_reduce = lambda t, *a, **k: (calls.append(t.dtype), real(t, *a, **k))[1]
    # one flat FP32 bucket: the two ranks' values sum exactly in FP32 and only then round
    bucket = torch.tensor([1.0, 2.0 ** -9, 3.0, 1.0 + 2.0 ** -8], dtype=torch.float32) * (rank + 1)
    rep.allreduce_bucket(bucket)
    with pytest.raises(TypeError):
        rep.allreduce_bucket(bucket.to(torch.bfloat16))
    ms = rep.max_over_ranks(10.0 + rank)
    rep.barrier()
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        rep.emit({"rank": rank, "ms": ms})
    n_bucket_calls = sum(1 for d in calls if d == torch.float32)
    q.put((rank, bucket.tolist(), bucket.to(torch.bfloat16).float().tolist(), n_bucket_calls, ms, out.getvalue()))
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
        rank, summed, rounded, n_calls, ms, printed = q.get(timeout=120)
        res[rank] = (summed, rounded, n_calls, ms, printed)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in range(world):
        summed, rounded, n_calls, ms, printed = res[rank]
        assert summed == [3.0, 3 * 2.0 ** -9, 9.0, 3.0 + 3 * 2.0 ** -8]      # the sum, exact in FP32
        # rounded once from the FP32 sum: 3 + 3/256 = 3.01171875 lies between the BF16
        # values 3.0 and 3.015625 and rounds to the nearer 3.015625; rounding each rank's
        # value first (1 + 2^-8 -> 1.0 by RNE, 2 + 2^-7 -> 2.0) would give 3.0
        assert rounded == [3.0, 3 * 2.0 ** -9, 9.0, 3.015625]
        assert n_calls == 1                                                 # one collective for the bucket
        assert ms == 11.0                                                   # max over ranks
    assert json.loads(res[0][4]) == {"rank": 0, "ms": 11.0}
    assert res[1][4] == ""


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr("sys.argv", ["bench.py", "--impl", "reference", "--gpus", "2"])
    bench.reference_arm(bench.parse())
    assert capsys.readouterr().out == ""
