"""Failure detection on the GPU without a fault: the attention kernels'
barrier waits are bounded, and an expired wait comes back as a status.

VA_FLAG_TEST_STALL_MMA makes the tensor-core kernel issue no tensor-core
work, so every wait on tensor-core completion runs into its 1 s bound (a flag
that nothing sets); VA_FLAG_TEST_STALL_COPIES makes the CUDA-core kernel arm
its staging barrier without issuing the copies.  The tests check the
per-request status, the output of flagged rows, the timeout counter, and that
the same context then runs a normal call."""
import numpy as np
import pytest

from speculative_decoding_tree_va_b200 import synth
from _harness import check_gpu_mask, compare, oracle_rows, to_device, trees_for

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def va():
    import torch
    assert torch.cuda.is_available()
    import speculative_decoding_tree_va_b200 as m
    m.load_library()
    return m


def test_expired_waits_flag_requests_and_leave_the_context_usable(va):
    import torch
    inp = synth.make_inputs(synth.WORKLOADS["bf16-deep"], B=2, H=16, P=(100, 300), budget=8)
    parents = trees_for(inp)["parent"]
    d = to_device(inp, parents)
    mask, _ = va.build_tree_mask(d["parents"])
    call = dict(scale=synth.SCALE, num_splits=1)
    before = va.device_timeouts()
    st = torch.zeros(inp.wl.B, dtype=torch.int32, device="cuda")
    out, lse = va.verify_attn(d["q_nope"], d["q_pe"], d["c_kv"], d["k_pe"], d["page_table"],
                              d["kv_len"], mask, req_status=st, flags=va.VA_FLAG_TEST_STALL_MMA,
                              **call)
    torch.cuda.synchronize()
    assert st.cpu().tolist() == [va.VA_ERR_CUDA] * inp.wl.B
    assert torch.isneginf(lse).all() and not out.float().abs().sum()
    assert va.device_timeouts() > before

    st.zero_()
    out, lse = va.verify_attn(d["q_nope"], d["q_pe"], d["c_kv"], d["k_pe"], d["page_table"],
                              d["kv_len"], mask, req_status=st, **call)
    torch.cuda.synchronize()
    assert st.cpu().tolist() == [0] * inp.wl.B
    check_gpu_mask(mask.cpu().numpy(), parents)
    ref_out, ref_lse = oracle_rows(inp, parents=parents)
    compare(out.float().cpu().numpy().reshape(-1, 512), lse.cpu().numpy().reshape(-1),
            ref_out, ref_lse, "bf16", "after the stalled call")


@pytest.mark.parametrize("num_splits", [1, 0])  # one CTA per row tile; the balanced plan
def test_expired_staging_waits_of_the_cuda_core_kernel(va, num_splits):
    """VA_FLAG_TEST_STALL_COPIES arms the fp32 kernel's staging barrier without
    issuing the bulk copies, so its bounded wait expires (no copy in flight)."""
    import torch
    inp = synth.make_inputs(synth.WORKLOADS["fp32-page-test"], B=2, H=16, P=(900, 1800))
    parents = trees_for(inp)["parent"]
    d = to_device(inp, parents)
    mask, _ = va.build_tree_mask(d["parents"])
    call = dict(scale=synth.SCALE, num_splits=num_splits)
    before = va.device_timeouts()
    st = torch.zeros(inp.wl.B, dtype=torch.int32, device="cuda")
    out, lse = va.verify_attn(d["q_nope"], d["q_pe"], d["c_kv"], d["k_pe"], d["page_table"],
                              d["kv_len"], mask, req_status=st,
                              flags=va.VA_FLAG_TEST_STALL_COPIES, **call)
    torch.cuda.synchronize()
    assert st.cpu().tolist() == [va.VA_ERR_CUDA] * inp.wl.B
    assert torch.isneginf(lse).all() and not out.abs().sum()
    assert va.device_timeouts() > before

    st.zero_()
    out, lse = va.verify_attn(d["q_nope"], d["q_pe"], d["c_kv"], d["k_pe"], d["page_table"],
                              d["kv_len"], mask, req_status=st, **call)
    torch.cuda.synchronize()
    assert st.cpu().tolist() == [0] * inp.wl.B
    ref_out, ref_lse = oracle_rows(inp, parents=parents)
    compare(out.cpu().numpy().reshape(-1, 512), lse.cpu().numpy().reshape(-1),
            ref_out, ref_lse, "f32", "after the stalled call")
