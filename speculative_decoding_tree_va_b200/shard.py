"""One long prefix sharded across GPUs: split-KV partials per rank, one gather, one merge.

The pages name a flash-decode split with an LSE merge for long prefixes as a
production step ("The Milestone Commit: Cementing Phase 1 of a Custom CUDA
Speculative Decoding Engine", section "How Decisions Were Made", production
notes: flash+merge for long prefixes).  Across GPUs the same partition is
shared out: the key range of every request is cut into S splits exactly as
``va_verify_attn`` cuts it, rank r computes the contiguous block of splits
``split_share(S, world, r)`` with ``va_verify_attn_partials``, merges them
locally into one partial (``va_merge`` with an fp32 output), and the ranks'
single partials are gathered so that one rank merges them into the final
output.  The merge is an exact re-association of the softmax sums, so the
result equals the one-GPU result up to rounding.

Traffic of the exchange: one fp32 partial per rank, rows x (512 + 1) x 4
bytes (rows = B * T * H), instead of every split's partials.  Remote partials
land in this rank's own memory through the collective before any kernel reads
them.

The steps are plain functions of callables so that the rank plumbing runs on
CPU ranks (``gloo``) in the tests; ``ShardedStep`` binds them to the CUDA
library and NCCL.

Problems a split meets (a bad kv_len or page index, an expired wait) are
reported by each rank's partials call in that rank's ``req_status``; the
final merge does not see them, so a request flagged on any rank is to be
treated as failed (its merged rows are not emptied across ranks, unlike a
one-GPU split call, whose merge empties them).
"""
from __future__ import annotations

from typing import Callable, Tuple


def split_share(S: int, world: int, rank: int) -> Tuple[int, int]:
    """(first, count): the contiguous block of the S splits that `rank` computes.

    Blocks differ in size by at most one; the first S % world ranks take the
    larger ones.  A rank beyond S gets count 0 (an empty share)."""
    if S < 1 or world < 1 or not 0 <= rank < world:
        raise ValueError(f"bad split share: S={S}, world={world}, rank={rank}")
    base, extra = divmod(S, world)
    count = base + (1 if rank < extra else 0)
    first = rank * base + min(rank, extra)
    return first, count


def local_partial(first: int, count: int, compute: Callable, merge_local: Callable,
                  empty: Callable):
    """This rank's single partial (o [rows, 512], lse [rows]).

    compute(first, count) -> (o [count, rows, 512], lse [count, rows]);
    merge_local(o, lse) -> their LSE merge; empty() -> zeros and -inf (a rank
    with no split contributes weight 0)."""
    if count == 0:
        return empty()
    o, lse = compute(first, count)
    if count == 1:
        return o[0], lse[0]
    return merge_local(o, lse)


def gather_partials(o, lse, dist, group=None):
    """Every rank's (o, lse) stacked along a new first axis, on every rank."""
    world = dist.get_world_size(group)
    # the output is the ranks' tensors concatenated along the first axis (the
    # form every backend accepts), then viewed with a rank axis
    o_all = o.new_empty((world * o.shape[0],) + tuple(o.shape[1:]))
    l_all = lse.new_empty((world * lse.shape[0],) + tuple(lse.shape[1:]))
    dist.all_gather_into_tensor(o_all, o.contiguous(), group=group)
    dist.all_gather_into_tensor(l_all, lse.contiguous(), group=group)
    return o_all.view((world,) + tuple(o.shape)), l_all.view((world,) + tuple(lse.shape))


def sharded_verify(S: int, rank: int, world: int, dist, compute: Callable, merge_local: Callable,
                   merge_final: Callable, empty: Callable, group=None, root: int = 0):
    """One sharded verify step; returns the merged (out, lse) on `root`, None elsewhere."""
    first, count = split_share(S, world, rank)
    o, lse = local_partial(first, count, compute, merge_local, empty)
    o_all, l_all = gather_partials(o, lse, dist, group)
    if rank != root:
        return None
    return merge_final(o_all, l_all)


class ShardedStep:
    """The sharded step on GPUs through the CUDA library, with buffers made once.

    `args` are the va_verify_attn arguments of the whole batch (every rank
    holds the batch; out / lse are written on `root` only) with an explicit
    split count S = args.num_splits."""

    def __init__(self, va, args, rank: int, world: int, dist, device, group=None, root: int = 0):
        import torch
        self.va, self.args, self.rank, self.world = va, args, rank, world
        self.dist, self.group, self.root = dist, group, root
        self.S = args.num_splits
        if self.S < 1:
            raise ValueError("a sharded step needs an explicit split count")
        self.first, self.count = split_share(self.S, world, rank)
        rows = args.B * args.T * args.H
        f32 = dict(device=device, dtype=torch.float32)
        c = max(self.count, 1)
        self.o_part = torch.empty(c, rows, 512, **f32)
        self.l_part = torch.empty(c, rows, **f32)
        # the partial this rank contributes: its one split in place, the local
        # merge of several, or zeros and -inf for an empty share
        self.o_local = self.o_part[0] if self.count == 1 else torch.zeros(rows, 512, **f32)
        self.l_local = (self.l_part[0] if self.count == 1 else
                        torch.full((rows,), float("-inf"), **f32))
        self.o_all = torch.empty(world * rows, 512, **f32)   # ranks along the first axis
        self.l_all = torch.empty(world * rows, **f32)
        need = va.partials_workspace_bytes(args)
        self.ws = torch.empty(max(need, 256), device=device, dtype=torch.uint8)
        self.pargs = va.VaAttnArgs.from_buffer_copy(args)
        self.pargs.workspace, self.pargs.workspace_bytes = self.ws.data_ptr(), self.ws.numel()
        self.lib = va.load_library()

    def _merge(self, o, lse, S, out_ptr, lse_ptr, dtype, stream):
        a = self.args
        r = self.lib.va_merge(o.data_ptr(), lse.data_ptr(), S, a.B, a.T, a.H, dtype, out_ptr,
                              lse_ptr, stream)
        if r:
            raise RuntimeError(f"va_merge failed ({r})")

    def __call__(self):
        import ctypes
        va, stream = self.va, self.va._stream()
        if self.count > 0:
            r = self.lib.va_verify_attn_partials(ctypes.byref(self.pargs), self.first, self.count,
                                                 ctypes.c_void_p(self.o_part.data_ptr()),
                                                 ctypes.c_void_p(self.l_part.data_ptr()), stream)
            if r:
                raise RuntimeError(f"va_verify_attn_partials failed ({r})")
            if self.count > 1:
                self._merge(self.o_part, self.l_part, self.count, self.o_local.data_ptr(),
                            self.l_local.data_ptr(), va.VA_F32, stream)
        self.dist.all_gather_into_tensor(self.o_all, self.o_local, group=self.group)
        self.dist.all_gather_into_tensor(self.l_all, self.l_local, group=self.group)
        if self.rank == self.root:
            self._merge(self.o_all, self.l_all, self.world, self.args.out, self.args.lse,
                        self.args.dtype, stream)
