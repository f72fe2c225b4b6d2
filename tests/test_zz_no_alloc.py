"""va_verify_attn_noalloc against va_verify_attn (GPU).

The no-allocation entry point serves callers that cannot allocate device
memory when they run the verify step (memory planned once at start-up, or a
path where an allocation's possible device synchronisation is not
acceptable).  It runs the same kernels as the workspace-based call with the
workspace in the library's fixed array, so its results must be the same bits;
the first call of each case is also compared with the fp64 oracle.  This
file is collected last on purpose; it also passes alone in a fresh process.
"""
import ctypes

import pytest

from speculative_decoding_tree_va_b200 import synth
from _harness import compare, oracle_rows, to_device, trees_for

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def va():
    import torch
    assert torch.cuda.is_available()
    import speculative_decoding_tree_va_b200 as m
    m.load_library()
    return m


def _setup(va, name, path, **kw):
    import torch
    inp = synth.make_inputs(synth.WORKLOADS[name], **kw)
    parents = trees_for(inp)["parent"]
    d = to_device(inp, parents)
    if inp.wl.kv == "fp8_e4m3":
        d["c_kv"], d["k_pe"] = d["c_kv"].view(torch.uint8), d["k_pe"].view(torch.uint8)
    mask, _ = va.build_tree_mask(d["parents"])
    flags = va.VA_FLAG_BF16_CUDA_CORES if path == "cc" else 0
    B, T, H = inp.wl.B, inp.T, inp.wl.H

    def outputs():
        return (torch.full((B, T, H, 512), float("nan"), device="cuda", dtype=d["dtype"]),
                torch.full((B, T, H), float("nan"), device="cuda", dtype=torch.float32))
    return inp, parents, d, mask, flags, outputs


@pytest.mark.parametrize("name,path,S", [("bf16-long-prefix", "tc", 4),
                                         ("bf16-b64-ragged", "tc", 3),
                                         ("bf16-b64-ragged", "tc", 1),
                                         ("bf16-long-prefix", "cc", 5),
                                         ("fp32-page-test", "f32", 6),
                                         ("bf16-fp8kv-deep", "tc", 1),
                                         ("bf16-fp8kv-deep", "tc", 3)])
def test_noalloc_matches_workspace_call_twice(va, name, path, S):
    import torch
    inp, parents, d, mask, flags, outputs = _setup(va, name, path, B=2, H=8, P=(1500, 3000))
    ref_out, ref_lse = outputs()
    va.verify_attn(d["q_nope"], d["q_pe"], d["c_kv"], d["k_pe"], d["page_table"], d["kv_len"],
                   mask, scale=synth.SCALE, num_splits=S, flags=flags, out=ref_out, lse=ref_lse,
                   kv_scale=inp.wl.kv_scale)
    for call in range(2):  # the fixed array keeps the previous call's contents
        out, lse = outputs()
        args = va.make_args(d["q_nope"], d["q_pe"], d["c_kv"], d["k_pe"], d["page_table"],
                            d["kv_len"], mask, out, lse, scale=synth.SCALE, num_splits=S,
                            flags=flags, kv_scale=inp.wl.kv_scale)
        assert va.num_splits(args) == S
        assert bool(args.flags & va.VA_FLAG_KV_FP8_E4M3) == (inp.wl.kv == "fp8_e4m3")
        va.verify_attn_noalloc(args)
        torch.cuda.synchronize()
        assert torch.equal(out, ref_out), f"call {call}: output differs from the workspace call"
        assert torch.equal(lse, ref_lse), f"call {call}: lse differs from the workspace call"
        if call == 0:
            ref_o, ref_l = oracle_rows(inp, parents=parents)
            compare(out.float().cpu().numpy().reshape(-1, 512), lse.cpu().numpy().reshape(-1),
                    ref_o, ref_l, inp.wl.dtype, f"noalloc {name} {path} S={S}")


def test_noalloc_rejects_partials_beyond_the_array(va):
    inp, parents, d, mask, flags, outputs = _setup(va, "bf16-long-prefix", "tc", B=2, H=64,
                                                   P=4000)
    out, lse = outputs()
    # 64 splits x 2 x 65 x 64 rows x 2052 bytes is far above the fixed array
    args = va.make_args(d["q_nope"], d["q_pe"], d["c_kv"], d["k_pe"], d["page_table"],
                        d["kv_len"], mask, out, lse, scale=synth.SCALE, num_splits=64)
    rows = 64 * 2 * 65 * 64
    assert rows * 2052 > va.NOALLOC_SCRATCH_BYTES
    st = va.load_library().va_verify_attn_noalloc(ctypes.byref(args), va._stream())
    assert st == va.VA_ERR_UNSUPPORTED
