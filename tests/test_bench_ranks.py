"""The multi-rank plumbing of bench.py on CPU: two gloo ranks (no GPU, no kernels).

Checks what --gpus N relies on: the process group comes up from the torchrun
environment, max-over-ranks gives every rank the slowest figure, each rank
draws its own independent batch, and the reference arm runs on rank 0 only."""
import argparse
import io
import multiprocessing as mp
import os
import socket
import sys
from contextlib import redirect_stdout

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE="2", LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    from speculative_decoding_tree_va_b200 import synth
    r, local, dist = bench.dist_setup(2, backend="gloo")
    slowest = bench.max_over_ranks(10.0 + 3.0 * r, dist, device="cpu")
    wl = synth.WORKLOADS["fp32-tiny"]
    inp = synth.make_inputs(wl, seed=bench.rank_seed(wl, r), with_tensors=False)
    dist.barrier()
    dist.destroy_process_group()
    q.put((r, local, slowest, float(inp.lp.sum()), int(inp.tok.sum())))


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r for r, *_ in res] == [0, 1] and [l for _, l, *_ in res] == [0, 1]
    assert all(s == 13.0 for _, _, s, _, _ in res)          # the max over both ranks
    assert res[0][3:] != res[1][3:]                          # independent batches


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    args = argparse.Namespace(workload="fp32-tiny", gpus=2, steps=1, warmup=0, cpu_seconds=1.0)
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(args)
    assert buf.getvalue() == ""
