"""GPU parity of va_verify_attn with an FP8 E4M3 latent cache
(VA_FLAG_KV_FP8_E4M3) against the fp64 oracle, which decodes the codes itself.

Paths: "f32" (fp32 queries, CUDA-core kernel widening codes as it stages
them), "tc" (bf16 queries: the pages are widened into bf16 scratch pages, then
the tensor-core kernel runs with the cache scale folded in) and "cc" (bf16
queries on the CUDA-core kernel, VA_FLAG_BF16_CUDA_CORES).  Widening is exact
on every path and the oracle decodes the codes itself, so the bars are those
of the query dtype: fp32 max_abs <= 1e-5; bf16 out <= 1e-2, lse <= 1e-3.
"""
import dataclasses

import numpy as np
import pytest

from speculative_decoding_tree_va_b200 import synth
from _harness import check_gpu_mask, compare, oracle_rows, to_device, trees_for
from test_gpu_attn import check_full, run_gpu

pytestmark = pytest.mark.gpu

NAMES = {"f32": "fp32-fp8kv", "bf16": "bf16-fp8kv-deep"}
PATHS = [("f32", "f32"), ("bf16", "tc"), ("bf16", "cc")]


@pytest.fixture(scope="module")
def va():
    import torch
    assert torch.cuda.is_available()
    import speculative_decoding_tree_va_b200 as m
    m.load_library()
    return m


def fp8_inputs(dtype, kv_scale=None, **kw):
    wl = synth.WORKLOADS[NAMES[dtype]]
    if kv_scale is not None:
        wl = dataclasses.replace(wl, kv_scale=kv_scale)
    return synth.make_inputs(wl, **kw)


def test_fp32_fp8kv_workload_full(va):
    inp = synth.make_inputs(synth.WORKLOADS["fp32-fp8kv"])
    check_full(va, inp, "f32", num_splits=inp.wl.splits)


@pytest.mark.parametrize("path", ["tc", "cc"])
def test_bf16_fp8kv_scaled_full(va, path):
    inp = fp8_inputs("bf16", B=2, P=700)
    check_full(va, inp, path)


@pytest.mark.parametrize("dtype,path", PATHS)
@pytest.mark.parametrize("S", [1, 3, 16])
def test_fp8kv_split_kv(va, dtype, path, S):
    inp = fp8_inputs(dtype, B=2, H=8, P=1500, budget=20)
    check_full(va, inp, path, num_splits=S, what=f"S={S}")


@pytest.mark.parametrize("dtype,path", PATHS)
@pytest.mark.parametrize("case", [
    dict(P=0, budget=0, B=2, H=8),               # T = 1, no prefix
    dict(P=1, budget=64, H=16, B=2),             # T = 65 (two mask words)
    dict(P=63, budget=64, topk=1, B=2, H=8),     # deep chain, underfull tree
    dict(P=(5, 600), budget=20, topk=3, B=4, H=8),
    dict(P=(1, 300), budget=0, H=1, B=1100, max_depth=1),
])
def test_fp8kv_edge_shapes(va, dtype, path, case):
    inp = fp8_inputs(dtype, **case)
    check_full(va, inp, path, what=f"{case}")


@pytest.mark.parametrize("dtype,path", PATHS)
def test_every_finite_code(va, dtype, path):
    """All 254 finite codes (both zeros, subnormals, +-448) in the cache; the
    scale (the float32 nearest 1/448) keeps every cached value within about [-1, 1]."""
    inp = fp8_inputs(dtype, kv_scale=float(np.float32(1.0 / 448.0)), B=2, H=8, P=(200, 500),
                     budget=16)
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    for arr in (inp.c_kv, inp.k_pe):
        flat = arr.reshape(-1)
        flat[:] = np.resize(finite, flat.size)
    check_full(va, inp, path)


@pytest.mark.parametrize("dtype,path", PATHS)
def test_nan_codes_beyond_kv_len_do_not_leak(va, dtype, path):
    inp = fp8_inputs(dtype, B=3, H=8, P=(70, 200), budget=16)
    for b in range(inp.wl.B):
        n = int(inp.kv_len[b])
        last = inp.page_table[b, (n - 1) // 64]
        if n % 64:
            inp.c_kv[last, n % 64:] = 0x7F
            inp.k_pe[last, n % 64:] = 0xFF
    check_full(va, inp, path)


@pytest.mark.parametrize("dtype,path", PATHS)
def test_fp8kv_bad_page_is_flagged(va, dtype, path):
    import torch
    inp = fp8_inputs(dtype, B=2, H=8, P=(70, 200), budget=8)
    parents = trees_for(inp)["parent"]
    d = to_device(inp, parents)
    mask, _ = va.build_tree_mask(d["parents"])
    pt = d["page_table"].clone()
    pt[1, 0] = -3
    st = torch.zeros(2, dtype=torch.int32, device="cuda")
    flags = va.VA_FLAG_BF16_CUDA_CORES if path == "cc" else 0
    out, lse = va.verify_attn(d["q_nope"], d["q_pe"], d["c_kv"], d["k_pe"], pt, d["kv_len"], mask,
                              scale=synth.SCALE, num_splits=1, req_status=st, flags=flags,
                              kv_scale=inp.wl.kv_scale)
    torch.cuda.synchronize()
    assert st.cpu().tolist() == [0, va.VA_ERR_INVALID_ARG]
    assert torch.isneginf(lse[1]).all() and not out[1].float().abs().sum()
    check_gpu_mask(mask.cpu().numpy(), parents)
    ref_out, ref_lse = oracle_rows(inp, parents=parents,
                                   rows=np.arange(inp.T * inp.wl.H, dtype=np.int32))
    compare(out[0].float().cpu().numpy().reshape(-1, 512), lse[0].cpu().numpy().reshape(-1),
            ref_out, ref_lse, dtype)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_uint8_cache_noalloc_and_flag_agree(va, dtype):
    """A uint8 cache, a float8_e4m3fn cache and va_verify_attn_noalloc (whose
    fixed array then also holds the widened pages for bf16) give the same bits."""
    import torch
    inp = fp8_inputs(dtype, B=2, H=8, P=900, budget=12)
    parents = trees_for(inp)["parent"]
    d = to_device(inp, parents)
    mask, _ = va.build_tree_mask(d["parents"])
    common = dict(scale=synth.SCALE, num_splits=3, kv_scale=inp.wl.kv_scale)
    out_a, lse_a = va.verify_attn(d["q_nope"], d["q_pe"], d["c_kv"], d["k_pe"], d["page_table"],
                                  d["kv_len"], mask, **common)
    out_b, lse_b = va.verify_attn(d["q_nope"], d["q_pe"], d["c_kv"].view(torch.uint8),
                                  d["k_pe"].view(torch.uint8), d["page_table"], d["kv_len"], mask,
                                  **common)
    out_c, lse_c = torch.empty_like(out_a), torch.empty_like(lse_a)
    args = va.make_args(d["q_nope"], d["q_pe"], d["c_kv"], d["k_pe"], d["page_table"],
                        d["kv_len"], mask, out_c, lse_c, **common)
    assert args.flags & va.VA_FLAG_KV_FP8_E4M3
    va.verify_attn_noalloc(args)
    torch.cuda.synchronize()
    for o, l in ((out_b, lse_b), (out_c, lse_c)):
        assert torch.equal(o, out_a) and torch.equal(l, lse_a)


def test_full_size_bf16_fp8kv_sampled_rows(va):
    inp = synth.make_inputs(synth.WORKLOADS["bf16-fp8kv-deep"])
    B, T, H = inp.wl.B, inp.T, inp.wl.H
    rows = synth.sample_rows(7, B, T, H, 256, full_request=None)
    parents = trees_for(inp)["parent"]
    out, lse, mask = run_gpu(va, inp, parents, "tc", num_splits=inp.wl.splits, rows=rows)
    check_gpu_mask(mask, parents)
    ref_out, ref_lse = oracle_rows(inp, parents=parents, rows=rows)
    compare(out, lse, ref_out, ref_lse, "bf16", "bf16-fp8kv-deep")
