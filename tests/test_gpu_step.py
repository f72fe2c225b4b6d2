"""GPU tests of the greedy accept walk and of the whole on-device verify step
(tree build -> mask -> verify attention -> accept) captured in one CUDA graph."""
import ctypes
import json
import os

import numpy as np
import pytest

import oracle
from speculative_decoding_tree_va_b200 import synth
from _harness import compare, oracle_rows, to_device

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def va():
    import torch
    assert torch.cuda.is_available()
    import speculative_decoding_tree_va_b200 as m
    m.load_library()
    return m


def synthetic_target(rng, par, tok, p_match=0.75):
    """Target greedy tokens that follow some child with probability p_match."""
    B, T = par.shape
    target = rng.integers(0, 1 << 20, size=(B, T)).astype(np.int32)
    for b in range(B):
        for t in range(T):
            kids = [i for i in range(t + 1, T) if par[b, i] == t]
            if kids and rng.random() < p_match:
                target[b, t] = tok[b, kids[int(rng.integers(0, len(kids)))]]
    return target


def gpu_accept(va, par, tok, tgt):
    import torch
    path, alen, nxt = va.tree_accept(*(torch.from_numpy(np.ascontiguousarray(a, np.int32)).cuda()
                                       for a in (par, tok, tgt)))
    torch.cuda.synchronize()
    return path.cpu().numpy(), alen.cpu().numpy(), nxt.cpu().numpy()


def test_accept_golden(va):
    g = json.load(open(os.path.join(GOLDEN, "tree_accept.json")))
    par = np.array([g["parents"]], np.int32)
    tok = np.array([g["tokens"]], np.int32)
    for case in g["cases"]:
        path, alen, nxt = gpu_accept(va, par, tok, np.array([case["target_next"]], np.int32))
        n = case["accept_len"]
        assert alen[0] == n and nxt[0] == case["next_token"]
        assert path[0, :n].tolist() == case["path"] and (path[0, n:] == -1).all()


@pytest.mark.parametrize("name,p_match", [("bf16-b64-ragged", 0.75), ("bf16-deep", 0.9),
                                          ("fp32-tiny", 0.5), ("bf16-deep", 1.0)])
def test_accept_bit_exact(va, name, p_match):
    wl = synth.WORKLOADS[name]
    inp = synth.make_inputs(wl, with_tensors=False)
    trees = oracle.build_trees(inp.lp, inp.tok, wl.budget)
    par, tok = trees["parent"], trees["token"]
    tgt = synthetic_target(np.random.default_rng(3), par, tok, p_match)
    ref = oracle.tree_accept(par, tok, tgt)
    got = gpu_accept(va, par, tok, tgt)
    for r, g in zip(ref, got):
        assert np.array_equal(r, g)
    if p_match == 1.0:  # always follows a child: accepts down to a leaf
        assert (ref[1] >= 2).all()


def test_accept_malformed_links_are_ignored(va):
    rng = np.random.default_rng(7)
    B, T = 33, 20
    par = np.array([[-1] + [int(rng.integers(-1, i)) for i in range(1, T)] for _ in range(B)],
                   np.int32)
    par[::3, 5] = 9      # parent after the child: ignored by both sides
    par[1::4, 7] = -7
    tok = rng.integers(0, 4, size=(B, T)).astype(np.int32)  # many equal sibling tokens
    tgt = rng.integers(0, 4, size=(B, T)).astype(np.int32)
    ref = oracle.tree_accept(par, tok, tgt)
    got = gpu_accept(va, par, tok, tgt)
    for r, g in zip(ref, got):
        assert np.array_equal(r, g)


def test_greedy_step_in_one_cuda_graph(va):
    """Build -> mask -> verify -> accept chained on the device, captured once and
    replayed twice; every stage checked against the oracle."""
    import torch
    wl = synth.WORKLOADS["bf16-b64-ragged"]
    inp = synth.make_inputs(wl, B=6, H=16, P=(200, 1500))
    B, L, K = inp.lp.shape
    T, H = inp.T, inp.q_nope.shape[2]
    lib = va.load_library()
    d = to_device(inp, np.zeros((B, T), np.int32))
    lp = torch.from_numpy(inp.lp).cuda()
    tk = torch.from_numpy(inp.tok).cuda()
    i32 = dict(device="cuda", dtype=torch.int32)
    parents, tokens, depth = (torch.empty(B, T, **i32) for _ in range(3))
    n_nodes = torch.empty(B, **i32)
    mask = torch.empty(B, T, (T + 63) // 64, device="cuda", dtype=torch.int64)
    tstat = torch.empty(B, **i32)
    out = torch.empty(B, T, H, 512, device="cuda", dtype=torch.bfloat16)
    lse = torch.empty(B, T, H, device="cuda", dtype=torch.float32)
    ref_tree = oracle.build_trees(inp.lp, inp.tok, wl.budget)
    tgt_h = synthetic_target(np.random.default_rng(11), ref_tree["parent"], ref_tree["token"])
    tgt = torch.from_numpy(tgt_h).cuda()
    path, alen, nxt = torch.empty(B, T, **i32), torch.empty(B, **i32), torch.empty(B, **i32)
    args = va.make_args(d["q_nope"], d["q_pe"], d["c_kv"], d["k_pe"], d["page_table"],
                        d["kv_len"], mask, out, lse, scale=synth.SCALE, num_splits=1)
    ws = torch.empty(max(va.workspace_bytes(args), 256), device="cuda", dtype=torch.uint8)
    args.workspace, args.workspace_bytes = ws.data_ptr(), ws.numel()
    P = lambda t: ctypes.c_void_p(t.data_ptr())

    def step(stream):
        s = ctypes.c_void_p(stream.cuda_stream)
        assert lib.va_build_tree(P(lp), P(tk), B, L, K, wl.budget, P(parents), P(tokens),
                                 P(depth), P(n_nodes), s) == 0
        assert lib.va_build_tree_mask(P(parents), B, T, P(mask), P(tstat), s) == 0
        assert lib.va_verify_attn(ctypes.byref(args), s) == 0
        assert lib.va_tree_accept(P(parents), P(tokens), P(tgt), B, T, P(path), P(alen),
                                  P(nxt), s) == 0

    side = torch.cuda.Stream()
    with torch.cuda.stream(side):  # warm up (module loads, attribute setup) before capture
        step(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        step(side)
    ref_mask, _ = oracle.ancestor_mask(ref_tree["parent"])
    ref_out, ref_lse = oracle_rows(inp, parents=ref_tree["parent"])
    ref_acc = oracle.tree_accept(ref_tree["parent"], ref_tree["token"], tgt_h)
    for _ in range(2):
        out.zero_()
        path.fill_(-5)
        g.replay()
        torch.cuda.synchronize()
        assert np.array_equal(parents.cpu().numpy(), ref_tree["parent"])
        assert np.array_equal(tokens.cpu().numpy(), ref_tree["token"])
        assert np.array_equal(mask.cpu().numpy().view(np.uint64), ref_mask)
        compare(out.float().cpu().numpy().reshape(-1, 512), lse.cpu().numpy().reshape(-1),
                ref_out, ref_lse, "bf16", "graph step")
        for r, got in zip(ref_acc, (path, alen, nxt)):
            assert np.array_equal(r, got.cpu().numpy())
