"""Pins of the fp64 oracle against facts fixed outside the oracle itself.

Each check is chosen so that a plausible slip in the oracle (a dropped rope
term, a wrong scale, an off-by-one in the tail position, a transposed page
index, a wrong tie-break, a missing self bit) fails at least one of them:

* hand-worked 3-node trees (tests/golden/three_node_trees.json),
* hand-worked forced-tie best-first expansion (tests/golden/tree_ties.json),
* brute force: dense masked softmax via numpy matmul + scipy logsumexp,
  with visibility from an independent recursive ancestor definition,
* invariants: chain tree == causal attention, popcount == depth + 1,
  root and self bits, page-table permutation invariance, split + merge ==
  unsplit, special cases (identical keys, P = 0 and T = 1, q = 0),
* best-first builder == brute-force top-B enumeration of all paths, and
  == an independent heapq expansion with tuple keys.
"""
import heapq
import itertools
import json
import math
import os

import numpy as np
import pytest
from scipy.special import logsumexp

import oracle
from speculative_decoding_tree_va_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
DC, DR = synth.D_LATENT, synth.D_ROPE


# ---------------------------------------------------------------------------
# independent helpers (written from the definitions, not from oracle.cpp)
# ---------------------------------------------------------------------------

def ancestors(parents, t):
    """Set of nodes on the root path of t (t included), by recursion."""
    if parents[t] == -1:
        return {t}
    return {t} | ancestors(parents, parents[t])


def logical_kv(c_kv, k_pe, page_table, b, n, page=64):
    """Gather the first n keys of request b in logical order."""
    idx = [page_table[b][j // page] * page + j % page for j in range(n)]
    ck = c_kv.reshape(-1, c_kv.shape[-1])[idx]
    kp = k_pe.reshape(-1, k_pe.shape[-1])[idx]
    return ck.astype(np.float64), kp.astype(np.float64)


def dense_reference(q_nope, q_pe, c_kv, k_pe, page_table, kv_len, parents, scale):
    """Dense masked softmax with library primitives (matmul, logsumexp)."""
    B, T, H, _ = q_nope.shape
    out = np.zeros((B, T, H, DC))
    lse = np.full((B, T, H), -np.inf)
    for b in range(B):
        n = int(kv_len[b])
        P = n - T
        ck, kp = logical_kv(c_kv, k_pe, page_table, b, n)
        for t in range(T):
            if t > 0 and parents[b][t] == -1:
                continue
            vis = np.zeros(n, bool)
            vis[:P] = True
            for i in ancestors(list(parents[b]), t):
                vis[P + i] = True
            q = q_nope[b, t].astype(np.float64)
            qp = q_pe[b, t].astype(np.float64)
            s = scale * (q @ ck.T + qp @ kp.T)          # [H, n]
            s = np.where(vis[None, :], s, -np.inf)
            l = logsumexp(s, axis=1)
            w = np.exp(s - l[:, None])
            out[b, t] = w @ ck
            lse[b, t] = l
    return out, lse


def small_inputs(seed, B=2, T=5, H=3, P=(0, 9), parents=None):
    rng = np.random.default_rng(seed)
    if parents is None:
        parents = []
        for _ in range(B):
            p = [-1] + [int(rng.integers(0, i)) for i in range(1, T)]
            parents.append(p)
    parents = np.array(parents, np.int32)
    if isinstance(P, tuple):
        prefix = rng.integers(P[0], P[1] + 1, size=B)
    else:
        prefix = np.full(B, P)
    kv_len = (prefix + T).astype(np.int32)
    pages = (kv_len + 63) // 64
    num_pages = int(pages.sum())
    perm = rng.permutation(num_pages)
    pt = np.full((B, int(pages.max())), -1, np.int32)
    o = 0
    for b in range(B):
        pt[b, :pages[b]] = perm[o:o + pages[b]]
        o += pages[b]
    q_nope = rng.standard_normal((B, T, H, DC)).astype(np.float32)
    q_pe = rng.standard_normal((B, T, H, DR)).astype(np.float32)
    c_kv = rng.standard_normal((num_pages, 64, DC)).astype(np.float32)
    k_pe = rng.standard_normal((num_pages, 64, DR)).astype(np.float32)
    return dict(q_nope=q_nope, q_pe=q_pe, c_kv=c_kv, k_pe=k_pe, page_table=pt,
                kv_len=kv_len, parents=parents)


def run_oracle(d, scale, rows=None, key_lo=None, key_hi=None):
    mask, status = oracle.ancestor_mask(d["parents"])
    out, lse = oracle.attention_rows(d["q_nope"], d["q_pe"], d["c_kv"], d["k_pe"],
                                     d["page_table"], d["kv_len"], mask, scale=scale,
                                     dtype="f32", rows=rows, key_lo=key_lo, key_hi=key_hi)
    return out, lse, mask, status


# ---------------------------------------------------------------------------
# hand-worked attention cases
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("scale,alpha", [(math.log(2.0), 1.0), (0.5 * math.log(2.0), 2.0)])
def test_hand_worked_three_node_trees(scale, alpha):
    g = json.load(open(os.path.join(GOLDEN, "three_node_trees.json")))
    P, a, bvals = g["P"], g["a"], g["b"]
    T = 3
    n = P + T
    for case in g["cases"]:
        q_nope = np.zeros((1, T, 1, DC), np.float32)
        q_pe = np.zeros((1, T, 1, DR), np.float32)
        q_nope[..., 0] = alpha
        q_pe[..., 0] = alpha
        c_kv = np.zeros((1, 64, DC), np.float32)
        k_pe = np.zeros((1, 64, DR), np.float32)
        for j in range(n):
            c_kv[0, j, 0] = a[j]
            k_pe[0, j, 0] = bvals[j]
            c_kv[0, j, 1 + j] = 1.0
        mask, status = oracle.ancestor_mask(np.array([case["parents"]], np.int32))
        assert status[0] == 0
        out, lse = oracle.attention_rows(q_nope, q_pe, c_kv, k_pe, np.zeros((1, 1), np.int32),
                                         np.array([n], np.int32), mask, scale=scale, dtype="f32")
        for row in case["rows"]:
            t = row["node"]
            o, l = out[t], lse[t]
            if row["den"] == 0:
                assert l == -np.inf and not o.any()
                continue
            w = np.array(row["weights_num"], np.float64) / row["den"]
            exp = np.zeros(DC)
            exp[0] = float(np.dot(w, a))
            exp[1:1 + n] = w
            np.testing.assert_allclose(o, exp, rtol=0, atol=1e-14)
            assert abs(l - math.log(row["den"])) < 1e-13


# ---------------------------------------------------------------------------
# brute force + invariants
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("seed", [1, 2, 3])
def test_oracle_matches_dense_bruteforce(seed):
    d = small_inputs(seed, B=2, T=6, H=3, P=(0, 70))
    scale = synth.SCALE
    out, lse, _, status = run_oracle(d, scale)
    assert (status == 0).all()
    ref_out, ref_lse = dense_reference(d["q_nope"], d["q_pe"], d["c_kv"], d["k_pe"],
                                       d["page_table"], d["kv_len"], d["parents"], scale)
    np.testing.assert_allclose(out, ref_out.reshape(out.shape), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse.reshape(-1), rtol=0, atol=1e-12)


def test_chain_tree_equals_causal_attention():
    T, H, P = 7, 2, 20
    d = small_inputs(11, B=1, T=T, H=H, P=P, parents=[[-1] + list(range(T - 1))])
    out, lse, _, _ = run_oracle(d, synth.SCALE)
    out = out.reshape(1, T, H, DC)
    lse = lse.reshape(1, T, H)
    n = P + T
    ck, kp = logical_kv(d["c_kv"], d["k_pe"], d["page_table"], 0, n)
    for t in range(T):
        for h in range(H):
            pos = P + t  # the query token's own position
            s = np.array([synth.SCALE * (np.dot(d["q_nope"][0, t, h].astype(np.float64), ck[j])
                                         + np.dot(d["q_pe"][0, t, h].astype(np.float64), kp[j]))
                          for j in range(pos + 1)])
            m = s.max()
            e = np.exp(s - m)
            ref = (e[:, None] * ck[:pos + 1]).sum(0) / e.sum()
            np.testing.assert_allclose(out[0, t, h], ref, atol=1e-12, rtol=0)
            assert abs(lse[0, t, h] - (m + math.log(e.sum()))) < 1e-12


def test_mask_invariants_on_builder_trees():
    inp = synth.make_inputs(synth.WORKLOADS["bf16-b64-ragged"], B=8, with_tensors=False)
    trees = oracle.build_trees(inp.lp, inp.tok, inp.wl.budget)
    mask, status = oracle.ancestor_mask(trees["parent"])
    assert (status == 0).all()
    B, T = trees["parent"].shape
    for b in range(B):
        for t in range(T):
            bits = [i for i in range(T) if (int(mask[b, t, i // 64]) >> (i % 64)) & 1]
            assert bits[0] == 0 and t in bits
            assert len(bits) == trees["depth"][b, t] + 1
            assert set(bits) == ancestors(list(trees["parent"][b]), t)
            assert max(bits) == t


@pytest.mark.parametrize("bad", [[0, 0, 1], [-1, 1, 0], [-1, 0, 3], [-1, -2, 0], [-1, -1, 1]])
def test_mask_rejects_malformed_parents(bad):
    mask, status = oracle.ancestor_mask(np.array([bad, [-1, 0, 0]], np.int32))
    assert status[0] == 1 and status[1] == 0
    assert not mask[0].any()


def test_mask_two_words_at_max_qlen():
    T = synth.MAX_QLEN
    parents = np.array([[-1] + list(range(T - 1))], np.int32)
    mask, status = oracle.ancestor_mask(parents)
    assert mask.shape == (1, T, 2) and status[0] == 0
    assert int(mask[0, T - 1, 0]) == 0xFFFFFFFFFFFFFFFF and int(mask[0, T - 1, 1]) == 1
    assert int(mask[0, 63, 1]) == 0 and int(mask[0, 64, 1]) == 1


def test_page_permutation_invariance():
    d = small_inputs(5, B=2, T=5, H=2, P=(100, 200))
    out1, lse1, _, _ = run_oracle(d, synth.SCALE)
    # move every page to a new physical slot, same logical contents
    num_pages = d["c_kv"].shape[0]
    perm = np.random.default_rng(9).permutation(num_pages)
    c2 = np.empty_like(d["c_kv"])
    k2 = np.empty_like(d["k_pe"])
    c2[perm] = d["c_kv"]
    k2[perm] = d["k_pe"]
    pt2 = np.where(d["page_table"] >= 0, perm[np.maximum(d["page_table"], 0)], -1).astype(np.int32)
    d2 = dict(d, c_kv=c2, k_pe=k2, page_table=pt2)
    out2, lse2, _, _ = run_oracle(d2, synth.SCALE)
    assert np.array_equal(out1, out2) and np.array_equal(lse1, lse2)


def test_split_merge_equals_unsplit():
    d = small_inputs(7, B=2, T=6, H=2, P=(300, 700))
    full_out, full_lse, _, _ = run_oracle(d, synth.SCALE)
    for S in (2, 3, 5):
        bounds = synth.split_bounds(d["kv_len"], S, align=64)
        parts = [run_oracle(d, synth.SCALE, key_lo=bounds[:, s, 0], key_hi=bounds[:, s, 1])
                 for s in range(S)]
        o_part = np.stack([p[0] for p in parts])
        l_part = np.stack([p[1] for p in parts])
        out, lse = oracle.merge(o_part, l_part)
        np.testing.assert_allclose(out, full_out, atol=1e-12, rtol=0)
        np.testing.assert_allclose(lse, full_lse, atol=1e-12, rtol=0)


def test_merge_special_cases():
    rng = np.random.default_rng(3)
    o = rng.standard_normal((1, 4, 8))
    l = rng.standard_normal((1, 4))
    out, lse = oracle.merge(o, l)
    assert np.array_equal(out, o[0]) and np.array_equal(lse, l[0])
    o2 = np.concatenate([o, rng.standard_normal((1, 4, 8))])
    l2 = np.concatenate([l, np.full((1, 4), -np.inf)])
    out, lse = oracle.merge(o2, l2)
    np.testing.assert_allclose(out, o[0], atol=1e-15)
    np.testing.assert_allclose(lse, l[0], atol=1e-15)
    out, lse = oracle.merge(np.zeros((3, 2, 8)), np.full((3, 2), -np.inf))
    assert not out.any() and (lse == -np.inf).all()
    # two equal chunks: lse + ln 2, same output
    out, lse = oracle.merge(np.concatenate([o, o]), np.concatenate([l, l]))
    np.testing.assert_allclose(out, o[0], atol=1e-14)
    np.testing.assert_allclose(lse, l[0] + math.log(2.0), atol=1e-14)


def test_special_cases():
    rng = np.random.default_rng(4)
    # identical keys: out = mean of visible c_kv, lse = s + ln |V|
    T, H, P = 4, 2, 5
    d = small_inputs(12, B=1, T=T, H=H, P=P, parents=[[-1, 0, 1, 1]])
    ck = rng.standard_normal(DC).astype(np.float32)
    kp = rng.standard_normal(DR).astype(np.float32)
    d["c_kv"][:] = ck
    d["k_pe"][:] = kp
    out, lse, _, _ = run_oracle(d, synth.SCALE)
    out = out.reshape(T, H, DC)
    lse = lse.reshape(T, H)
    vis = [P + len(ancestors([-1, 0, 1, 1], t)) for t in range(T)]
    for t in range(T):
        for h in range(H):
            s = synth.SCALE * (np.dot(d["q_nope"][0, t, h].astype(np.float64), ck.astype(np.float64))
                               + np.dot(d["q_pe"][0, t, h].astype(np.float64), kp.astype(np.float64)))
            np.testing.assert_allclose(out[t, h], ck.astype(np.float64), atol=1e-13)
            assert abs(lse[t, h] - (s + math.log(vis[t]))) < 1e-12
    # P = 0, T = 1: the root sees only itself
    d = small_inputs(13, B=1, T=1, H=3, P=0, parents=[[-1]])
    out, lse, _, _ = run_oracle(d, synth.SCALE)
    kr = d["page_table"][0, 0] * 64
    ckr = d["c_kv"].reshape(-1, DC)[kr].astype(np.float64)
    kpr = d["k_pe"].reshape(-1, DR)[kr].astype(np.float64)
    for h in range(3):
        np.testing.assert_allclose(out[h], ckr, atol=0, rtol=0)
        s = synth.SCALE * (np.dot(d["q_nope"][0, 0, h].astype(np.float64), ckr)
                           + np.dot(d["q_pe"][0, 0, h].astype(np.float64), kpr))
        assert abs(lse[h] - s) < 1e-12
    # q = 0: uniform average over the visible keys, lse = ln |V|
    d = small_inputs(14, B=1, T=3, H=1, P=9, parents=[[-1, 0, 0]])
    d["q_nope"][:] = 0
    d["q_pe"][:] = 0
    out, lse, _, _ = run_oracle(d, 0.7)
    ck, _ = logical_kv(d["c_kv"], d["k_pe"], d["page_table"], 0, 12)
    for t, keys in enumerate([list(range(9)) + [9], list(range(9)) + [9, 10],
                              list(range(9)) + [9, 11]]):
        np.testing.assert_allclose(out[t], ck[keys].mean(0), atol=1e-13)
        assert abs(lse[t] - math.log(len(keys))) < 1e-13


def test_padding_rows_are_empty():
    d = small_inputs(15, B=1, T=4, H=2, P=10, parents=[[-1, 0, -1, -1]])
    out, lse, mask, status = run_oracle(d, synth.SCALE)
    assert status[0] == 0
    out = out.reshape(4, 2, DC)
    lse = lse.reshape(4, 2)
    assert not out[2:].any() and (lse[2:] == -np.inf).all()
    assert np.isfinite(lse[:2]).all()


# ---------------------------------------------------------------------------
# best-first builder
# ---------------------------------------------------------------------------

def test_builder_hand_worked_ties():
    g = json.load(open(os.path.join(GOLDEN, "tree_ties.json")))
    lp = np.array(g["lp"], np.float64)
    tok = np.array(g["tok"], np.int32)
    for case in g["cases"]:
        t = oracle.build_tree(lp, tok, case["budget"])
        assert t["n"] == case["n"]
        assert t["parent"].tolist() == case["parent"]
        assert t["depth"].tolist() == case["depth"]
        assert t["token"].tolist() == case["token"]


def enumerate_paths(lp, L, K):
    """Every path (tuple of ranks) of length 1..L with its score (fsum)."""
    out = []
    for d in range(1, L + 1):
        for ranks in itertools.product(range(K), repeat=d):
            out.append((math.fsum(lp[i][r] for i, r in enumerate(ranks)), ranks))
    return out


def node_paths(tree):
    paths = {0: ()}
    for i in range(1, tree["n"]):
        paths[i] = paths[int(tree["parent"][i])] + (int(tree["rank"][i]),)
    return paths


@pytest.mark.parametrize("K,L,budget,seed", [(2, 3, 6, 0), (3, 3, 12, 1), (3, 4, 20, 2),
                                              (2, 4, 30, 3), (1, 4, 9, 4)])
def test_builder_equals_bruteforce_topB(K, L, budget, seed):
    rng = np.random.default_rng(seed)
    lp = -np.sort(rng.exponential(1.0, size=(L, K)), axis=1)   # descending, tie-free
    tok = rng.integers(0, 4096, size=(L, K)).astype(np.int32)
    tree = oracle.build_tree(lp, tok, budget)
    allp = sorted(enumerate_paths(lp, L, K), key=lambda x: -x[0])
    n_expect = min(budget, len(allp)) + 1
    assert tree["n"] == n_expect
    paths = node_paths(tree)
    assert set(paths[i] for i in range(1, tree["n"])) == set(p for _, p in allp[:n_expect - 1])
    # node order is best-first: scores non-increasing, each equal to its path sum
    sc = tree["score"][:tree["n"]]
    assert (np.diff(sc[1:]) <= 0).all()
    for i in range(1, tree["n"]):
        p = paths[i]
        assert abs(sc[i] - math.fsum(lp[k][r] for k, r in enumerate(p))) < 1e-12
        assert tree["token"][i] == tok[len(p) - 1][p[-1]]
        assert tree["depth"][i] == len(p)
    # padding entries
    assert (tree["parent"][tree["n"]:] == -1).all()


def heapq_builder(lp, K, L, budget):
    """Independent expansion with Python heapq and tuple keys (-score, parent, rank)."""
    parent, depth, score = [-1], [0], [0.0]
    heap = [(-(0.0 + lp[0][0]), 0, 0, 1)]
    while len(parent) < budget + 1 and heap:
        neg, p, r, d = heapq.heappop(heap)
        node = len(parent)
        parent.append(p)
        depth.append(d)
        score.append(-neg)
        if r + 1 < K:
            heapq.heappush(heap, (-(score[p] + lp[d - 1][r + 1]), p, r + 1, d))
        if d + 1 <= L:
            heapq.heappush(heap, (-(score[node] + lp[d][0]), node, 0, d + 1))
    return parent, depth


@pytest.mark.parametrize("name", ["fp32-tiny", "bf16-deep", "bf16-b64-ragged"])
def test_builder_equals_heapq_on_workload_trees(name):
    wl = synth.WORKLOADS[name]
    inp = synth.make_inputs(wl, B=min(wl.B, 8), with_tensors=False)
    for b in range(inp.lp.shape[0]):
        t = oracle.build_tree(inp.lp[b], inp.tok[b], wl.budget)
        par, dep = heapq_builder(inp.lp[b], wl.topk, wl.max_depth, wl.budget)
        assert t["parent"][:t["n"]].tolist() == par
        assert t["depth"][:t["n"]].tolist() == dep
        assert t["n"] == wl.T  # these workloads always fill the budget
        assert t["depth"].max() <= wl.max_depth


# ---------------------------------------------------------------------------
# greedy tree accept
# ---------------------------------------------------------------------------

def test_tree_accept_hand_worked():
    g = json.load(open(os.path.join(GOLDEN, "tree_accept.json")))
    par = np.array([g["parents"]], np.int32)
    tok = np.array([g["tokens"]], np.int32)
    for case in g["cases"]:
        path, alen, nxt = oracle.tree_accept(par, tok, np.array([case["target_next"]], np.int32))
        n = case["accept_len"]
        assert alen[0] == n and nxt[0] == case["next_token"], case["name"]
        assert path[0, :n].tolist() == case["path"] and (path[0, n:] == -1).all(), case["name"]


def accept_bruteforce(parents, tokens, target):
    """Deepest node whose whole root path follows the target's greedy tokens."""
    T = len(parents)
    best = [0]
    for node in range(1, T):
        if parents[node] == -1:
            continue
        chain = [node]
        while parents[chain[-1]] != -1:
            chain.append(parents[chain[-1]])
        chain = chain[::-1]  # root first
        if chain[0] != 0:
            continue
        if all(tokens[c] == target[p] for p, c in zip(chain, chain[1:])) and len(chain) > len(best):
            best = chain
    return best, target[best[-1]]


@pytest.mark.parametrize("seed", range(6))
def test_tree_accept_bruteforce(seed):
    rng = np.random.default_rng(seed)
    inp = synth.make_inputs(synth.WORKLOADS["bf16-b64-ragged"], B=16, topk=3,
                            seed=1000 + seed, with_tensors=False)
    trees = oracle.build_trees(inp.lp, inp.tok, inp.wl.budget)
    par, tok = trees["parent"], trees["token"]
    B, T = par.shape
    # target agrees with the first child's token with probability 0.7
    target = rng.integers(0, 4096, size=(B, T)).astype(np.int32)
    for b in range(B):
        for t in range(T):
            kids = [i for i in range(T) if par[b, i] == t]
            if kids and rng.random() < 0.7:
                target[b, t] = tok[b, kids[int(rng.integers(0, len(kids)))]]
    path, alen, nxt = oracle.tree_accept(par, tok, target)
    for b in range(B):
        chain, nt = accept_bruteforce(list(par[b]), list(tok[b]), list(target[b]))
        assert path[b, :alen[b]].tolist() == chain and nxt[b] == nt
        assert alen[b] == len(chain) and (path[b, alen[b]:] == -1).all()


# ---------------------------------------------------------------------------
# FP8 E4M3 latent cache
# ---------------------------------------------------------------------------

def test_e4m3_decoder_closed_forms():
    g = json.load(open(os.path.join(GOLDEN, "e4m3_codes.json")))
    codes = np.array([int(c["code"], 16) for c in g["codes"]], np.uint8)
    got = oracle.decode_e4m3(codes)
    for c, v in zip(g["codes"], got):
        want = math.ldexp(c["num"], c["exp2"])
        assert v == want and math.copysign(1.0, v) == math.copysign(1.0, want), c
    nans = oracle.decode_e4m3(np.array([int(c, 16) for c in g["nan_codes"]], np.uint8))
    assert np.isnan(nans).all()


def test_e4m3_decoder_matches_torch_on_all_codes():
    import torch
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.decode_e4m3(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.array_equal(np.signbit(got[ok]), np.signbit(ref[ok]))


def fp8_case(seed, B=2, T=6, H=3, P=(0, 70)):
    """small_inputs with the cache replaced by E4M3 codes (all finite codes used)."""
    d = small_inputs(seed, B=B, T=T, H=H, P=P)
    rng = np.random.default_rng(seed + 100)
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    d["c_kv"] = rng.choice(finite, size=d["c_kv"].shape).astype(np.uint8)
    d["k_pe"] = rng.choice(finite, size=d["k_pe"].shape).astype(np.uint8)
    return d


@pytest.mark.parametrize("seed,kv_scale", [(4, 0.4375), (5, 1.0 / 448.0), (6, 3.0)])
def test_fp8_cache_matches_dense_bruteforce(seed, kv_scale):
    """The oracle on codes == the numpy brute force on torch-decoded, scaled values."""
    import torch
    d = fp8_case(seed)
    dec = lambda a: torch.from_numpy(a).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mask, status = oracle.ancestor_mask(d["parents"])
    out, lse = oracle.attention_rows(d["q_nope"], d["q_pe"], d["c_kv"], d["k_pe"],
                                     d["page_table"], d["kv_len"], mask, scale=synth.SCALE,
                                     dtype="f32", kv_dtype="fp8_e4m3", kv_scale=kv_scale)
    ref_out, ref_lse = dense_reference(d["q_nope"], d["q_pe"], kv_scale * dec(d["c_kv"]),
                                       kv_scale * dec(d["k_pe"]), d["page_table"], d["kv_len"],
                                       d["parents"], synth.SCALE)
    live = np.isfinite(ref_lse.reshape(-1))
    assert live.any()
    np.testing.assert_allclose(out, ref_out.reshape(out.shape), rtol=1e-12,
                               atol=1e-12 * max(1.0, 448 * kv_scale))
    np.testing.assert_allclose(lse[live], ref_lse.reshape(-1)[live], rtol=1e-12, atol=1e-9)


def test_fp8_cache_identical_keys_closed_form():
    """Every visible key the same code c: out = kv_scale * value(c), lse = s + ln(count)."""
    T, H, P, kv_scale = 4, 2, 10, 0.4375
    d = small_inputs(21, B=1, T=T, H=H, P=P, parents=[[-1, 0, 1, 1]])
    d["c_kv"] = np.full(d["c_kv"].shape, 0x3F, np.uint8)     # 1.875
    d["k_pe"] = np.full(d["k_pe"].shape, 0xC0, np.uint8)     # -2
    mask, _ = oracle.ancestor_mask(d["parents"])
    out, lse = oracle.attention_rows(d["q_nope"], d["q_pe"], d["c_kv"], d["k_pe"],
                                     d["page_table"], d["kv_len"], mask, scale=synth.SCALE,
                                     dtype="f32", kv_dtype="fp8_e4m3", kv_scale=kv_scale)
    depth = [0, 1, 2, 2]
    for t in range(T):
        for h in range(H):
            r = t * H + h
            q = d["q_nope"][0, t, h].astype(np.float64)
            qp = d["q_pe"][0, t, h].astype(np.float64)
            s = synth.SCALE * kv_scale * (1.875 * q.sum() - 2.0 * qp.sum())
            np.testing.assert_allclose(out[r], np.full(DC, kv_scale * 1.875), rtol=1e-14)
            assert abs(lse[r] - (s + math.log(P + depth[t] + 1))) < 1e-10
