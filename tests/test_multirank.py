"""Data-parallel host logic of bench.py on two gloo ranks, on the CPU.

Each rank draws its own tokens against the same weights, the job's time is
the slowest rank's (all-reduce MAX), the whole-job value counts every rank's
tokens, and only rank 0 prints its JSON line.  The GPU work between these
steps is covered by the GPU tests; here no CUDA device is touched."""
import contextlib
import datetime
import io
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from mixture_experts_layer_sqrt_b200 import synth
        p = synth.PROBLEMS["tiny_f32"]
        a = bench.rank_arrays(p, rank, synth)
        # fingerprints of this rank's tokens and weights, gathered on every rank
        fp = torch.tensor([float(np.abs(a["x"]).sum()), float(np.abs(a["w_gate"]).sum()),
                           float(np.abs(a["w_router"]).sum())], dtype=torch.float64)
        allfp = [torch.zeros_like(fp) for _ in range(world)]
        dist.all_gather(allfp, fp)
        slowest = bench.max_over_ranks(10.0 + rank, dist, "cpu")
        value = bench.whole_job_value(world, p.T, slowest)
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            bench.emit({"metric": "m", "value": value, "n_gpus": world}, rank)
        q.put((rank, [t.tolist() for t in allfp], slowest, value, buf.getvalue()))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_ranks_shard_tokens_and_take_the_slowest_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    got = {}
    for _ in range(world):
        rank, fps, slowest, value, printed = q.get(timeout=120)
        got[rank] = (fps, slowest, value, printed)
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    fps = got[0][0]
    assert got[1][0] == fps                       # both ranks saw the same gathered fingerprints
    assert fps[0][0] != fps[1][0]                 # different tokens per rank
    assert fps[0][1:] == fps[1][1:]               # identical weights
    for r in range(world):
        assert got[r][1] == 11.0                  # max over ranks of 10 + rank
        assert got[r][2] == pytest.approx(world * 64 / 11.0e-3)
    assert '"n_gpus": 2' in got[0][3] and got[1][3] == ""


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3"])
    monkeypatch.setattr(bench, "run_reference", lambda *a: pytest.fail("rank 1 ran the reference arm"))
    bench.main()
    assert capsys.readouterr().out == ""
