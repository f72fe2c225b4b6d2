"""GPU parity of the tree kernels (bit-exact against the oracle)."""
import json
import os

import numpy as np
import pytest

import oracle
from speculative_decoding_tree_va_b200 import synth

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def va():
    import torch
    assert torch.cuda.is_available()
    import speculative_decoding_tree_va_b200 as m
    m.load_library()
    return m


def gpu_trees(va, lp, tok, budget):
    import torch
    p, t, d, n = va.build_tree(torch.from_numpy(lp).cuda(), torch.from_numpy(tok).cuda(), budget)
    torch.cuda.synchronize()
    return p.cpu().numpy(), t.cpu().numpy(), d.cpu().numpy(), n.cpu().numpy()


@pytest.mark.parametrize("name", synth.WORKLOAD_ORDER)
def test_builder_bit_exact_on_workloads(va, name):
    inp = synth.make_inputs(synth.WORKLOADS[name], with_tensors=False)
    ref = oracle.build_trees(inp.lp, inp.tok, inp.wl.budget)
    p, t, d, n = gpu_trees(va, inp.lp, inp.tok, inp.wl.budget)
    assert np.array_equal(p, ref["parent"])
    assert np.array_equal(t, ref["token"])
    assert np.array_equal(d, ref["depth"])
    assert np.array_equal(n, ref["n"])


def test_builder_ties_and_underfull(va):
    g = json.load(open(os.path.join(GOLDEN, "tree_ties.json")))
    lp = np.array(g["lp"], np.float64)[None]
    tok = np.array(g["tok"], np.int32)[None]
    for case in g["cases"]:
        p, t, d, n = gpu_trees(va, lp, tok, case["budget"])
        assert p[0].tolist() == case["parent"]
        assert d[0].tolist() == case["depth"]
        assert t[0].tolist() == case["token"]
        assert n[0] == case["n"]


@pytest.mark.parametrize("K,L,budget", [(1, 15, 64), (2, 15, 64), (8, 15, 64), (16, 3, 64),
                                        (3, 2, 64), (5, 1, 0), (8, 15, 1)])
def test_builder_random_with_forced_ties(va, K, L, budget):
    rng = np.random.default_rng(K * 100 + L)
    B = 37
    # quantised log-probs force many exact ties between paths
    lp = -np.sort(rng.integers(0, 4, size=(B, L, K)).astype(np.float64) * 0.5, axis=2)
    tok = rng.integers(0, 50000, size=(B, L, K)).astype(np.int32)
    ref = oracle.build_trees(lp, tok, budget)
    p, t, d, n = gpu_trees(va, lp, tok, budget)
    assert np.array_equal(p, ref["parent"]) and np.array_equal(t, ref["token"])
    assert np.array_equal(d, ref["depth"]) and np.array_equal(n, ref["n"])


def gpu_mask(va, parents):
    import torch
    m, s = va.build_tree_mask(torch.from_numpy(np.ascontiguousarray(parents, np.int32)).cuda())
    torch.cuda.synchronize()
    return m.cpu().numpy().view(np.uint64), s.cpu().numpy()


@pytest.mark.parametrize("name", synth.WORKLOAD_ORDER)
def test_mask_bit_exact_on_workload_trees(va, name):
    inp = synth.make_inputs(synth.WORKLOADS[name], with_tensors=False)
    parents = oracle.build_trees(inp.lp, inp.tok, inp.wl.budget)["parent"]
    ref_m, ref_s = oracle.ancestor_mask(parents)
    m, s = gpu_mask(va, parents)
    assert np.array_equal(m, ref_m) and np.array_equal(s, ref_s)


def test_mask_shapes_and_malformed(va):
    rng = np.random.default_rng(0)
    cases = []
    for T in (1, 2, 3, 33, 63, 64, 65):
        cases.append(np.array([-1] + list(range(T - 1)), np.int32))               # chain
        cases.append(np.array([-1] + [0] * (T - 1), np.int32))                    # star
        cases.append(np.array([-1] + [int(rng.integers(0, i)) for i in range(1, T)], np.int32))
        if T > 3:                                                                  # underfull
            c = np.array([-1] + [int(rng.integers(0, i)) for i in range(1, T)], np.int32)
            c[T // 2:] = -1
            cases.append(c)
            bad = c.copy(); bad[T - 1] = T // 2          # parent is absent
            cases.append(bad)
            bad2 = c.copy(); bad2[2] = 2                 # self parent
            cases.append(bad2)
            bad3 = c.copy(); bad3[0] = 0                 # root with a parent
            cases.append(bad3)
            bad4 = c.copy(); bad4[1] = -5
            cases.append(bad4)
    for c in cases:
        T = c.shape[0]
        batch = np.stack([c, np.array([-1] + [0] * (T - 1), np.int32), c])
        ref_m, ref_s = oracle.ancestor_mask(batch)
        m, s = gpu_mask(va, batch)
        assert np.array_equal(m, ref_m), c
        assert np.array_equal(s, np.where(ref_s == 0, 0, va.VA_ERR_INVALID_TREE))
