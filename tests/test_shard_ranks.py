"""Sharding one long prefix across ranks, on CPU: two gloo ranks, the oracle in
place of the kernels.

Each rank computes its share of the S-way split partition with the oracle's
attention over each split's key range, merges its share locally with the
oracle's merge, the shares are gathered through the process group, and rank
0 merges them.  The result must equal the unsplit oracle at fp64 rounding
(1e-12): the split assignment covers every split once and the gather keeps
every rank's partial in rank order."""
import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from speculative_decoding_tree_va_b200.shard import split_share  # noqa: E402


@pytest.mark.parametrize("S,world", [(s, w) for s in (1, 2, 3, 7, 16, 64) for w in (1, 2, 3, 8)])
def test_split_share_covers_every_split_once(S, world):
    shares = [split_share(S, world, r) for r in range(world)]
    covered = [s for f, c in shares for s in range(f, f + c)]
    assert covered == list(range(S))                       # contiguous, in rank order, once each
    counts = [c for _, c in shares]
    assert max(counts) - min(counts) <= 1


@pytest.mark.parametrize("S", [1, 2, 3, 5, 16, 64])
def test_split_bounds_partition(S):
    from speculative_decoding_tree_va_b200 import synth
    kv = np.array([1, 33, 255, 256, 257, 2081, 4096, 8225, 65 * 64 * 20, 131071], np.int32)
    b = synth.split_bounds(kv, S)
    assert b.shape == (kv.size, S, 2)
    for r in range(kv.size):
        lo, hi = b[r, :, 0].astype(np.int64), b[r, :, 1].astype(np.int64)
        assert lo[0] == 0 and hi[-1] == kv[r]
        assert np.all(hi[:-1] == lo[1:]) and np.all(hi >= lo)   # contiguous, ordered
        assert np.all((lo % 256 == 0) | (lo == kv[r]))            # every edge but kv_len aligned
        exact = np.arange(S) * kv[r] / S                          # nearest multiple of 256
        assert np.all(np.abs(lo[1:] - exact[1:]) <= 128)
        assert np.all(np.abs((hi - lo) - kv[r] / S) < 256)


def test_split_share_rejects_bad_arguments():
    for bad in ((0, 2, 0), (4, 0, 0), (4, 2, 2), (4, 2, -1)):
        with pytest.raises(ValueError):
            split_share(*bad)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    from speculative_decoding_tree_va_b200 import synth
    # two long requests of the long-prefix shape, scaled so the oracle runs every row
    return synth.make_inputs(synth.WORKLOADS["bf16-long-prefix"], B=2, H=4, P=(1800, 2600),
                             budget=12)


def _rank_main(rank, world, S, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    from speculative_decoding_tree_va_b200 import shard, synth
    from _harness import oracle_mask

    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    inp = _inputs()
    parents = oracle.build_trees(inp.lp, inp.tok, inp.wl.budget)["parent"]
    mask = oracle_mask(parents)
    bounds = synth.split_bounds(inp.kv_len, S)
    rows = inp.wl.B * inp.T * inp.wl.H

    def attention(lo=None, hi=None):
        return oracle.attention_rows(inp.q_nope, inp.q_pe, inp.c_kv, inp.k_pe, inp.page_table,
                                     inp.kv_len, mask, scale=synth.SCALE, dtype=inp.wl.dtype,
                                     key_lo=lo, key_hi=hi)

    def compute(first, count):
        parts = [attention(bounds[:, s, 0], bounds[:, s, 1]) for s in range(first, first + count)]
        return (torch.from_numpy(np.stack([o for o, _ in parts])),
                torch.from_numpy(np.stack([l for _, l in parts])))

    def merge(o, lse):
        out, l = oracle.merge(o.numpy(), lse.numpy())
        return torch.from_numpy(out), torch.from_numpy(l)

    def empty():
        return (torch.zeros(rows, 512, dtype=torch.float64),
                torch.full((rows,), float("-inf"), dtype=torch.float64))

    res = shard.sharded_verify(S, rank, world, dist, compute, merge, merge, empty)
    if rank == 0:
        ref_out, ref_lse = attention()
        out, lse = res[0].numpy(), res[1].numpy()
        fin = np.isfinite(ref_lse)
        q.put((rank, float(np.abs(out - ref_out).max()),
               float(np.abs(lse[fin] - ref_lse[fin]).max()),
               bool(np.array_equal(np.isfinite(lse), fin))))
    else:
        q.put((rank, res is None, 0.0, True))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("S,world", [(8, 2), (3, 2), (1, 2)])
def test_two_gloo_ranks_shard_one_long_prefix(S, world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, S, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(world))
    rank0 = res[0]
    assert rank0[0] == 0
    assert rank0[3], "empty-row pattern differs"
    assert rank0[1] <= 1e-12 and rank0[2] <= 1e-12, rank0
    assert all(r[1] is True for r in res[1:])               # only rank 0 holds the result
