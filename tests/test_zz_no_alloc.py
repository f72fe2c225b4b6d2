"""va_verify_attn_noalloc against va_verify_attn (GPU).

The no-allocation entry point serves callers that cannot allocate device
memory when they run the verify step (memory planned once at start-up, or a
path where an allocation's possible device synchronisation is not
acceptable).  It must give the same results as the workspace-based call.
This file is collected last on purpose; it also passes alone in a fresh
process.
"""
import ctypes

import numpy as np
import pytest

from speculative_decoding_tree_va_b200 import synth
from _harness import TOL, to_device, trees_for

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
    d = to_device(inp, trees_for(inp)["parent"])
    mask, _ = va.build_tree_mask(d["parents"])
    flags = va.VA_FLAG_BF16_CUDA_CORES if path == "cc" else 0
    B, T, H = inp.wl.B, inp.T, inp.wl.H

    def outputs():
        return (torch.full((B, T, H, 512), float("nan"), device="cuda", dtype=d["dtype"]),
                torch.full((B, T, H), float("nan"), device="cuda", dtype=torch.float32))
    return inp, d, mask, flags, outputs


@pytest.mark.parametrize("name,path,S", [("bf16-long-prefix", "tc", 4),
                                         ("bf16-b64-ragged", "tc", 3),
                                         ("bf16-long-prefix", "cc", 5),
                                         ("fp32-page-test", "f32", 6)])
def test_noalloc_matches_workspace_call_twice(va, name, path, S):
    import torch
    inp, d, mask, flags, outputs = _setup(va, name, path, B=2, H=8, P=(1500, 3000))
    ref_out, ref_lse = outputs()
    va.verify_attn(d["q_nope"], d["q_pe"], d["c_kv"], d["k_pe"], d["page_table"], d["kv_len"],
                   mask, scale=synth.SCALE, num_splits=S, flags=flags, out=ref_out, lse=ref_lse)
    tol = TOL[inp.wl.dtype]
    for call in range(2):  # the fixed array keeps the previous call's contents
        out, lse = outputs()
        args = va.make_args(d["q_nope"], d["q_pe"], d["c_kv"], d["k_pe"], d["page_table"],
                            d["kv_len"], mask, out, lse, scale=synth.SCALE, num_splits=S,
                            flags=flags)
        assert va.num_splits(args) == S
        va.verify_attn_noalloc(args)
        torch.cuda.synchronize()
        o = out.float().cpu().numpy()
        r = ref_out.float().cpu().numpy()
        assert np.isfinite(o).all(), f"call {call}: output not fully written"
        assert float(np.abs(o - r).max()) <= tol["out"], f"call {call}"
        l, rl = lse.cpu().numpy(), ref_lse.cpu().numpy()
        fin = np.isfinite(rl)
        assert np.array_equal(np.isfinite(l), fin)
        assert float(np.abs(l[fin] - rl[fin]).max()) <= tol["lse"], f"call {call}"


def test_noalloc_rejects_partials_beyond_the_array(va):
    inp, d, mask, flags, outputs = _setup(va, "bf16-long-prefix", "tc", B=2, H=64, P=4000)
    out, lse = outputs()
    # 64 splits x 2 x 65 x 64 rows x 2052 bytes is far above the fixed array
    args = va.make_args(d["q_nope"], d["q_pe"], d["c_kv"], d["k_pe"], d["page_table"],
                        d["kv_len"], mask, out, lse, scale=synth.SCALE, num_splits=64)
    rows = 64 * 2 * 65 * 64
    assert rows * 2052 > va.NOALLOC_SCRATCH_BYTES
    st = va.load_library().va_verify_attn_noalloc(ctypes.byref(args), va._stream())
    assert st == va.VA_ERR_UNSUPPORTED
