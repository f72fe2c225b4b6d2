"""Shared test plumbing: synthetic inputs -> (oracle, CUDA library) -> comparison.

Inputs come from ``speculative_decoding_tree_va_b200.synth``; trees for both
sides come from the oracle's builder (an oracle input, never a CUDA output),
and the oracle derives its visibility mask from those parent pointers itself
(``oracle_rows``): no value the CUDA library computes ever enters the oracle.
"""
from __future__ import annotations

import json
import os

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


def oracle_mask(parents: np.ndarray) -> np.ndarray:
    """The oracle's own ancestor mask of [B, T] parent pointers (uint64 [B, T, W])."""
    mask, _ = oracle.ancestor_mask(np.asarray(parents, np.int32))
    return mask


def check_gpu_mask(gpu_mask, parents: np.ndarray, what: str = ""):
    """The library's mask must equal the oracle's bit for bit."""
    got = np.ascontiguousarray(np.asarray(gpu_mask)).view(np.uint64)
    ref = oracle_mask(parents)
    assert got.shape == ref.shape and np.array_equal(got, ref), f"{what}: tree mask differs"


def oracle_rows(inp: synth.Inputs, *, parents: np.ndarray, rows=None, key_lo=None, key_hi=None):
    """fp64 oracle rows of one workload; the mask comes from ``parents`` through the
    oracle's own ancestor walk."""
    return oracle.attention_rows(inp.q_nope, inp.q_pe, inp.c_kv, inp.k_pe, inp.page_table,
                                 inp.kv_len, oracle_mask(parents), scale=synth.SCALE,
                                 dtype=inp.wl.dtype, rows=rows, key_lo=key_lo, key_hi=key_hi,
                                 **kv_kwargs(inp))


def kv_kwargs(inp: synth.Inputs) -> dict:
    """Cache storage arguments of the oracle for this workload."""
    if inp.wl.kv == "fp8_e4m3":
        return dict(kv_dtype="fp8_e4m3", kv_scale=inp.wl.kv_scale)
    return {}


def _log(rec: dict):
    """Print one parity record; with VA_PARITY_LOG set, also append it as a JSON line."""
    print("[parity] " + json.dumps(rec))
    path = os.environ.get("VA_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(rec) + "\n")


def compare(out_gpu, lse_gpu, out_ref, lse_ref, dtype: str, what: str = ""):
    """Element-wise check of (out, lse) rows against the oracle at the dtype's bar.

    -inf lse (absent rows) must match exactly, with an all-zero output.  Returns
    (out max_abs, lse max_abs, elements that needed the bf16 storage allowance)
    and logs them (``_log``)."""
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
        relaxed = int((err > tol["out"]).sum())
        worst = float((err - bar).max()) if out_ref.size else -1.0
    else:
        relaxed, worst = 0, d_out - tol["out"]
    _log({"what": what, "dtype": dtype, "elements": int(out_ref.size), "out_max_abs": d_out,
          "lse_max_abs": d_lse, "out_over_plain_bar": relaxed})
    if dtype == "bf16":
        assert worst <= 0, f"{what}: out max_abs {d_out:.3e} over the bf16 bar"
    else:
        assert worst <= 0, f"{what}: out max_abs {d_out:.3e} > {tol['out']}"
    assert d_lse <= tol["lse"], f"{what}: lse max_abs {d_lse:.3e} > {tol['lse']}"
    return d_out, d_lse, relaxed
