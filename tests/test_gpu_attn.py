"""GPU parity of va_verify_attn / va_merge against the fp64 oracle.

Paths: "f32" (CUDA-core FFMA kernel), "tc" (bf16 tcgen05 kernel, the default
for bf16) and "cc" (bf16 on the CUDA-core kernel, VA_FLAG_BF16_CUDA_CORES).
Bars: fp32 max_abs <= 1e-5; bf16 out max_abs <= 1e-2 and lse <= 1e-3.
"""
import dataclasses

import numpy as np
import pytest

import oracle
from speculative_decoding_tree_va_b200 import synth
from _harness import check_gpu_mask, compare, oracle_rows, to_device, trees_for

pytestmark = pytest.mark.gpu

BF16_PATHS = ["tc", "cc"]


@pytest.fixture(scope="module")
def va():
    import torch
    assert torch.cuda.is_available()
    import speculative_decoding_tree_va_b200 as m
    m.load_library()
    return m


def run_gpu(va, inp, parents, path, num_splits=1, rows=None):
    """Mask + attention on the GPU; returns numpy (out, lse) rows and the GPU's mask.

    The mask is returned for a bit-exact check against the oracle's; the oracle
    never computes with it."""
    import torch
    d = to_device(inp, parents)
    mask, status = va.build_tree_mask(d["parents"])
    flags = va.VA_FLAG_BF16_CUDA_CORES if path == "cc" else 0
    req_status = torch.zeros(inp.wl.B, dtype=torch.int32, device="cuda")
    out, lse = va.verify_attn(d["q_nope"], d["q_pe"], d["c_kv"], d["k_pe"], d["page_table"],
                              d["kv_len"], mask, scale=synth.SCALE, num_splits=num_splits,
                              flags=flags, req_status=req_status, kv_scale=inp.wl.kv_scale)
    torch.cuda.synchronize()
    assert (req_status.cpu().numpy() == 0).all()
    out = out.float().reshape(-1, synth.D_LATENT)
    lse = lse.reshape(-1)
    if rows is not None:
        idx = torch.from_numpy(rows.astype(np.int64)).cuda()
        out, lse = out[idx], lse[idx]
    return out.cpu().numpy(), lse.cpu().numpy(), mask.cpu().numpy().view(np.uint64)


def check_full(va, inp, path, num_splits=1, parents=None, what=""):
    if parents is None:
        parents = trees_for(inp)["parent"]
    out, lse, mask = run_gpu(va, inp, parents, path, num_splits)
    check_gpu_mask(mask, parents, what or inp.wl.name)
    ref_out, ref_lse = oracle_rows(inp, parents=parents)
    return compare(out, lse, ref_out, ref_lse, inp.wl.dtype, what or inp.wl.name)


def paths_for(dtype):
    return ["f32"] if dtype == "f32" else BF16_PATHS


# --- the two fp32 workloads in full -------------------------------------------

@pytest.mark.parametrize("name", ["fp32-tiny", "fp32-page-test"])
def test_fp32_workloads_full(va, name):
    inp = synth.make_inputs(synth.WORKLOADS[name])
    check_full(va, inp, "f32")


# --- bf16 workloads, scaled so the oracle runs every row ---------------------

SMALL = [
    ("bf16-deep", dict(B=2, P=700)),
    ("bf16-b64-ragged", dict(B=5, P=(130, 1400))),
    ("bf16-long-prefix", dict(B=1, P=3000, H=16)),
]


@pytest.mark.parametrize("path", BF16_PATHS)
@pytest.mark.parametrize("name,kw", SMALL)
def test_bf16_workloads_scaled(va, path, name, kw):
    inp = synth.make_inputs(synth.WORKLOADS[name], **kw)
    check_full(va, inp, path)


@pytest.mark.parametrize("path", ["f32"] + BF16_PATHS)
@pytest.mark.parametrize("S", [2, 3, 16])
def test_split_kv_matches_unsplit_oracle(va, path, S):
    name = "fp32-page-test" if path == "f32" else "bf16-long-prefix"
    inp = synth.make_inputs(synth.WORKLOADS[name], B=2, H=8, P=(1500, 4000))
    check_full(va, inp, path, num_splits=S)


@pytest.mark.parametrize("path", ["f32"] + BF16_PATHS)
def test_planner_chosen_splits_match_the_oracle(va, path):
    """num_splits = 0: the library picks the split count (and the caller's workspace size)."""
    import torch
    name = "fp32-page-test" if path == "f32" else "bf16-long-prefix"
    inp = synth.make_inputs(synth.WORKLOADS[name], B=1, H=16, P=6000)
    parents = trees_for(inp)["parent"]
    d = to_device(inp, parents)
    mask, _ = va.build_tree_mask(d["parents"])
    flags = va.VA_FLAG_BF16_CUDA_CORES if path == "cc" else 0
    out = torch.empty(*d["q_nope"].shape, dtype=d["q_nope"].dtype, device="cuda")
    lse = torch.empty(*d["q_nope"].shape[:3], dtype=torch.float32, device="cuda")
    args = va.make_args(d["q_nope"], d["q_pe"], d["c_kv"], d["k_pe"], d["page_table"], d["kv_len"],
                        mask, out, lse, scale=synth.SCALE, num_splits=0, flags=flags)
    S = va.num_splits(args)
    assert S > 1  # one request of 6000 keys leaves most SMs idle without a split
    out, lse = va.verify_attn(d["q_nope"], d["q_pe"], d["c_kv"], d["k_pe"], d["page_table"],
                              d["kv_len"], mask, scale=synth.SCALE, num_splits=0, flags=flags)
    torch.cuda.synchronize()
    check_gpu_mask(mask.cpu().numpy(), parents)
    ref_out, ref_lse = oracle_rows(inp, parents=parents)
    compare(out.float().cpu().numpy().reshape(-1, 512), lse.cpu().numpy().reshape(-1),
            ref_out, ref_lse, inp.wl.dtype, f"{path}, {S} planned splits")


# --- edge cases ----------------------------------------------------------------

def edge_inputs(dtype, B=2, H=8, P=0, budget=8, topk=8, max_depth=15, seed=5):
    wl = synth.WORKLOADS["fp32-tiny" if dtype == "f32" else "bf16-deep"]
    wl = dataclasses.replace(wl, paged=True)
    return synth.make_inputs(wl, B=B, H=H, P=P, budget=budget, topk=topk,
                             max_depth=max_depth, seed=seed)


@pytest.mark.parametrize("dtype,path", [("f32", "f32"), ("bf16", "tc"), ("bf16", "cc")])
@pytest.mark.parametrize("case", [
    dict(P=0, budget=0),                 # T = 1, no prefix: the root sees itself
    dict(P=0, budget=8),                 # tree tail only
    dict(P=1, budget=64, H=16),          # maxbudget, T = 65 (two mask words)
    dict(P=63, budget=64, topk=1),       # deep chain, depth 15, underfull tree (padding)
    dict(P=64, budget=32, H=16),
    dict(P=(5, 600), budget=20, topk=3, B=4),
    dict(P=257, budget=64, topk=2, H=64, B=1),
    dict(P=100, budget=10, H=1),
    dict(P=(60, 70), budget=33, H=3, B=3),
    dict(P=(1, 300), budget=0, H=1, B=1100, max_depth=1),  # more requests than the kernel ranks
])
def test_edge_cases(va, dtype, path, case):
    inp = edge_inputs(dtype, **case)
    check_full(va, inp, path, what=f"{case}")


# CUDA-core calls with fewer (request, 32-row tile) segments than SMs and an
# automatic split count take the balanced plan: contiguous ranges of 32-key
# tiles over one CTA per SM, a segment's partials in up to `slots` slots.
BALANCED = [
    dict(P=(5, 900), budget=20, topk=3, B=3, H=5),   # ragged lengths, partial row tiles
    dict(P=4000, budget=0, H=1, B=1),                  # one 1-row segment over ~30 CTAs
    dict(P=(1, 3000), budget=64, topk=2, H=2, B=2),   # T = 65, two mask words
    dict(P=(300, 330), budget=8, H=32, B=4),          # kv_len below the page capacity
]


@pytest.mark.parametrize("dtype,path", [("f32", "f32"), ("bf16", "cc")])
@pytest.mark.parametrize("case", BALANCED)
def test_balanced_plan_matches_the_oracle(va, dtype, path, case):
    import torch
    inp = edge_inputs(dtype, **case)
    if case.get("P") == (300, 330):
        inp.kv_len[:] = np.minimum(inp.kv_len, inp.kv_len.min())  # empty tiles at every tail
    d = to_device(inp, trees_for(inp)["parent"])
    mask, _ = va.build_tree_mask(d["parents"])
    out = torch.empty(*d["q_nope"].shape, dtype=d["q_nope"].dtype, device="cuda")
    lse = torch.empty(*d["q_nope"].shape[:3], dtype=torch.float32, device="cuda")
    flags = va.VA_FLAG_BF16_CUDA_CORES if path == "cc" else 0
    args = va.make_args(d["q_nope"], d["q_pe"], d["c_kv"], d["k_pe"], d["page_table"], d["kv_len"],
                        mask, out, lse, scale=synth.SCALE, num_splits=0, flags=flags)
    assert va.num_splits(args) > 1
    check_full(va, inp, path, num_splits=0, what=f"balanced {case}")


@pytest.mark.parametrize("dtype,path", [("f32", "f32"), ("bf16", "tc"), ("bf16", "cc")])
@pytest.mark.parametrize("shape", ["chain", "star"])
def test_chain_and_star_trees(va, dtype, path, shape):
    inp = edge_inputs(dtype, B=2, H=8, P=(90, 300), budget=40)
    T = inp.T
    p = np.array([-1] + (list(range(T - 1)) if shape == "chain" else [0] * (T - 1)), np.int32)
    check_full(va, inp, path, parents=np.stack([p, p]))


@pytest.mark.parametrize("dtype,path", [("f32", "f32"), ("bf16", "tc"), ("bf16", "cc")])
def test_values_beyond_kv_len_do_not_leak(va, dtype, path):
    inp = edge_inputs(dtype, B=3, H=8, P=(70, 200), budget=16)
    big = 3.0e4
    for b in range(inp.wl.B):
        n = int(inp.kv_len[b])
        last = inp.page_table[b, (n - 1) // 64]
        for arr in (inp.c_kv, inp.k_pe):
            v = np.full(arr.shape[2], big, np.float32)
            arr[last, n % 64 or 64:] = synth.bf16_round(v) if dtype == "bf16" else v
    check_full(va, inp, path)


@pytest.mark.parametrize("dtype,path", [("f32", "f32"), ("bf16", "tc"), ("bf16", "cc")])
def test_poisoned_request_stays_contained(va, dtype, path):
    """NaN in one request's queries and +inf in its keys reach no other request."""
    inp = edge_inputs(dtype, B=3, H=8, P=(70, 400), budget=12)
    nan_, inf_ = (np.uint16(0x7FC0), np.uint16(0x7F80)) if dtype == "bf16" else (np.nan, np.inf)
    inp.q_nope[0, 1, 2, 5] = nan_
    inp.c_kv[inp.page_table[0, 0], 3, 7] = inf_
    inp.k_pe[inp.page_table[0, 1], 9, 2] = inf_
    parents = trees_for(inp)["parent"]
    out, lse, mask = run_gpu(va, inp, parents, path)
    check_gpu_mask(mask, parents)
    R = inp.T * inp.wl.H
    rows = np.arange(R, 3 * R, dtype=np.int32)
    ref_out, ref_lse = oracle_rows(inp, parents=parents, rows=rows)
    compare(out[R:], lse[R:], ref_out, ref_lse, dtype, "requests 1-2")
    assert not np.isfinite(out[:R]).all()   # the poisoned request does see its own inputs


@pytest.mark.parametrize("dtype,path", [("f32", "f32"), ("bf16", "tc"), ("bf16", "cc")])
@pytest.mark.parametrize("num_splits", [1, 3, 0])  # one pass, a split, the planner's choice
def test_bad_kv_len_and_page_are_flagged(va, dtype, path, num_splits):
    """A flagged request comes out empty even when only one of its splits
    meets the bad page."""
    import torch
    inp = edge_inputs(dtype, B=3, H=8, P=(300, 600), budget=8)
    parents = trees_for(inp)["parent"]
    d = to_device(inp, parents)
    mask, _ = va.build_tree_mask(d["parents"])
    kv = d["kv_len"].clone()
    kv[1] = 3                                   # shorter than T
    pt = d["page_table"].clone()
    pt[2, 0] = inp.num_pages + 5                # page out of range
    st = torch.zeros(3, dtype=torch.int32, device="cuda")
    flags = va.VA_FLAG_BF16_CUDA_CORES if path == "cc" else 0
    out, lse = va.verify_attn(d["q_nope"], d["q_pe"], d["c_kv"], d["k_pe"], pt, kv, mask,
                              scale=synth.SCALE, num_splits=num_splits, req_status=st,
                              flags=flags)
    torch.cuda.synchronize()
    assert st.cpu().tolist() == [0, va.VA_ERR_INVALID_ARG, va.VA_ERR_INVALID_ARG]
    assert torch.isneginf(lse[1:]).all() and not out[1:].float().abs().sum()
    check_gpu_mask(mask.cpu().numpy(), parents)
    ref_out, ref_lse = oracle_rows(inp, parents=parents,
                                   rows=np.arange(inp.T * inp.wl.H, dtype=np.int32))
    compare(out[0].float().cpu().numpy().reshape(-1, 512), lse[0].cpu().numpy().reshape(-1),
            ref_out, ref_lse, dtype)


# --- partials of split subsets (the per-GPU step of a sharded long prefix) ----

@pytest.mark.parametrize("path", ["f32"] + BF16_PATHS)
def test_partials_of_split_subsets_match_the_oracle(va, path):
    """Splits computed in three disjoint groups: each partial equals the oracle's
    attention over that split's key range, and va_merge over all of them equals
    the unsplit oracle."""
    import torch
    name = "fp32-page-test" if path == "f32" else "bf16-long-prefix"
    inp = synth.make_inputs(synth.WORKLOADS[name], B=2, H=8, P=(2500, 4000))
    parents = trees_for(inp)["parent"]
    d = to_device(inp, parents)
    mask, _ = va.build_tree_mask(d["parents"])
    check_gpu_mask(mask.cpu().numpy(), parents)
    S = 8
    B, T, H = inp.wl.B, inp.T, inp.wl.H
    flags = va.VA_FLAG_BF16_CUDA_CORES if path == "cc" else 0
    args = va.make_args(d["q_nope"], d["q_pe"], d["c_kv"], d["k_pe"], d["page_table"],
                        d["kv_len"], mask, torch.empty(0, device="cuda"),
                        torch.empty(0, device="cuda"), scale=synth.SCALE, num_splits=S,
                        flags=flags)
    args.out = args.lse = None                       # not used by a partials-only call
    need = va.partials_workspace_bytes(args)
    ws = torch.empty(max(need, 256), device="cuda", dtype=torch.uint8)
    args.workspace, args.workspace_bytes = ws.data_ptr(), ws.numel()
    o_all = torch.full((S, B, T, H, 512), float("nan"), device="cuda")
    l_all = torch.full((S, B, T, H), float("nan"), device="cuda")
    for first, count in ((0, 3), (3, 1), (4, 4)):
        va.verify_attn_partials(args, first, count, o_all[first:first + count],
                                l_all[first:first + count])
    torch.cuda.synchronize()
    bounds = synth.split_bounds(inp.kv_len, S)
    dt = inp.wl.dtype
    for s in range(S):
        ref_o, ref_l = oracle_rows(inp, parents=parents, key_lo=bounds[:, s, 0],
                                   key_hi=bounds[:, s, 1])
        # partials are fp32 on every path: the bar is the query dtype's
        compare(o_all[s].cpu().numpy().reshape(-1, 512), l_all[s].cpu().numpy().reshape(-1),
                ref_o, ref_l, dt, f"{path} partial {s} of {S}")
    out, lse = va.merge(o_all, l_all, d["dtype"])
    torch.cuda.synchronize()
    ref_out, ref_lse = oracle_rows(inp, parents=parents)
    compare(out.float().cpu().numpy().reshape(-1, 512), lse.cpu().numpy().reshape(-1),
            ref_out, ref_lse, dt, f"{path} merged partials")


# --- merge ---------------------------------------------------------------------

@pytest.mark.parametrize("out_dtype", ["f32", "bf16"])
@pytest.mark.parametrize("S", [1, 2, 7, 33, 64])
def test_merge_against_oracle(va, out_dtype, S):
    import torch
    rng = np.random.default_rng(S)
    B, T, H = 2, 5, 3
    o = rng.standard_normal((S, B, T, H, 512)).astype(np.float32)
    l = (rng.standard_normal((S, B, T, H)) * 3).astype(np.float32)
    l[rng.random(l.shape) < 0.3] = -np.inf      # empty chunks
    l[:, 0, 0, 0] = -np.inf                     # a row with every chunk empty
    tdt = torch.float32 if out_dtype == "f32" else torch.bfloat16
    out, lse = va.merge(torch.from_numpy(o).cuda(), torch.from_numpy(l).cuda(), tdt)
    torch.cuda.synchronize()
    ref_out, ref_lse = oracle.merge(o.reshape(S, -1, 512), l.reshape(S, -1))
    compare(out.float().cpu().numpy().reshape(-1, 512), lse.cpu().numpy().reshape(-1),
            ref_out, ref_lse, out_dtype)


# --- full-size workloads on sampled rows ---------------------------------------

FULL = [("bf16-deep", 1), ("bf16-b64-ragged", 1), ("bf16-long-prefix", 16)]
# the long-prefix workload splits its prefix into 16 to 64 chunks; the wider
# splits run on the tensor-core path (the CUDA-core path shares the split code)
FULL_TC_ONLY = [("bf16-long-prefix", 32), ("bf16-long-prefix", 64)]


@pytest.mark.parametrize("path,name,S",
                         [(p, n, s) for p in BF16_PATHS for n, s in FULL] +
                         [("tc", n, s) for n, s in FULL_TC_ONLY])
def test_full_size_sampled_rows(va, path, name, S):
    inp = synth.make_inputs(synth.WORKLOADS[name])
    B, T, H = inp.wl.B, inp.T, inp.wl.H
    n_rand = 96 if name == "bf16-long-prefix" else 256
    rows = synth.sample_rows(7, B, T, H, n_rand,
                             full_request=None if name == "bf16-long-prefix" else 0)
    parents = trees_for(inp)["parent"]
    out, lse, mask = run_gpu(va, inp, parents, path, num_splits=S, rows=rows)
    check_gpu_mask(mask, parents, name)
    ref_out, ref_lse = oracle_rows(inp, parents=parents, rows=rows)
    compare(out, lse, ref_out, ref_lse, "bf16", f"{name}, {path}, S={S}")
