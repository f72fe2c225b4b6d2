"""Shared test plumbing: synthetic inputs -> (oracle, CUDA library) -> comparison.

Inputs come from ``speculative_decoding_tree_va_b200.synth``; trees for both
sides come from the oracle's builder (an oracle input, never a CUDA output).
"""
from __future__ import annotations

import numpy as np

import oracle
from speculative_decoding_tree_va_b200 import synth

TOL = {  # max_abs bars: fp32 configs 1e-5; bf16 configs out 1e-2, lse 1e-3
    "f32": dict(out=1e-5, lse=1e-5),
    "bf16": dict(out=1e-2, lse=1e-3),
}


def trees_for(inp: synth.Inputs):
    return oracle.build_trees(inp.lp, inp.tok, inp.wl.budget)


def to_device(inp: synth.Inputs, parents: np.ndarray, device="cuda"):
    """Torch tensors of one workload (values as float32 or bfloat16)."""
    import torch
    dt = torch.float32 if inp.wl.dtype == "f32" else torch.bfloat16

    def vals(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        if inp.wl.dtype == "bf16":
            t = t.view(torch.int16).view(torch.bfloat16)
        return t.to(device)

    def cache(a):
        if inp.wl.kv == "fp8_e4m3":
            return torch.from_numpy(np.ascontiguousarray(a)).view(torch.float8_e4m3fn).to(device)
        return vals(a)

    return dict(
        q_nope=vals(inp.q_nope), q_pe=vals(inp.q_pe), c_kv=cache(inp.c_kv), k_pe=cache(inp.k_pe),
        page_table=torch.from_numpy(inp.page_table).to(device),
        kv_len=torch.from_numpy(inp.kv_len).to(device),
        parents=torch.from_numpy(np.ascontiguousarray(parents, np.int32)).to(device),
        dtype=dt)


def oracle_rows(inp: synth.Inputs, mask: np.ndarray, rows=None, key_lo=None, key_hi=None):
    return oracle.attention_rows(inp.q_nope, inp.q_pe, inp.c_kv, inp.k_pe, inp.page_table,
                                 inp.kv_len, mask, scale=synth.SCALE, dtype=inp.wl.dtype,
                                 rows=rows, key_lo=key_lo, key_hi=key_hi, **kv_kwargs(inp))


def kv_kwargs(inp: synth.Inputs) -> dict:
    """Cache storage arguments of the oracle for this workload."""
    if inp.wl.kv == "fp8_e4m3":
        return dict(kv_dtype="fp8_e4m3", kv_scale=inp.wl.kv_scale)
    return {}


def compare(out_gpu, lse_gpu, out_ref, lse_ref, dtype: str, what: str = ""):
    """Element-wise check of (out, lse) rows against the oracle at the dtype's bar.

    -inf lse (absent rows) must match exactly, with an all-zero output."""
    out_gpu = np.asarray(out_gpu, np.float64).reshape(out_ref.shape)
    lse_gpu = np.asarray(lse_gpu, np.float64).reshape(lse_ref.shape)
    tol = TOL[dtype]
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), empty), f"{what}: empty-row pattern differs"
    assert not out_gpu[empty].any(), f"{what}: absent rows not zero"
    assert np.isfinite(out_gpu).all() and np.isfinite(lse_gpu[~empty]).all(), f"{what}: non-finite"
    err = np.abs(out_gpu - out_ref)
    d_out = float(err.max()) if out_ref.size else 0.0
    d_lse = float(np.abs(lse_gpu[~empty] - lse_ref[~empty]).max()) if (~empty).any() else 0.0
    if dtype == "bf16":
        # bf16 outputs: the bar is 1e-2, except where storing the exact value
        # in bf16 alone costs more (half an ulp = 2^-8 |x| reaches 1e-2 at
        # |x| >= 2.56); there the storage rounding plus 2e-3 is allowed.
        bar = np.maximum(tol["out"], np.abs(out_ref) * 2.0 ** -8 + 2e-3)
        worst = float((err - bar).max()) if out_ref.size else -1.0
        assert worst <= 0, f"{what}: out max_abs {d_out:.3e} over the bf16 bar"
    else:
        assert d_out <= tol["out"], f"{what}: out max_abs {d_out:.3e} > {tol['out']}"
    assert d_lse <= tol["lse"], f"{what}: lse max_abs {d_lse:.3e} > {tol['lse']}"
    return d_out, d_lse
