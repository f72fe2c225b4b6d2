"""The whole greedy verify step from a plain C program (tests/c/va_step.c): cudaMalloc'd
buffers, va_build_tree_mask, va_verify_attn with the library's split planning,
va_tree_accept -- no Python in the calling process.  Its outputs are compared with the
oracle here."""
import os
import subprocess

import numpy as np
import pytest

import oracle
from speculative_decoding_tree_va_b200 import synth
from _harness import compare, oracle_rows, trees_for

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def test_c_program_runs_the_step(tmp_path):
    inp = synth.make_inputs(synth.WORKLOADS["bf16-b64-ragged"], B=3, H=16, P=(300, 5000))
    trees = trees_for(inp)
    par, tok = trees["parent"], trees["token"]
    rng = np.random.default_rng(21)
    tgt = rng.integers(0, 1 << 20, size=par.shape).astype(np.int32)
    for b in range(par.shape[0]):            # follow the lowest-index child
        for i in range(par.shape[1] - 1, 0, -1):
            if par[b, i] >= 0:
                tgt[b, par[b, i]] = tok[b, i]
    B, T, H = inp.q_nope.shape[:3]
    files = dict(q_nope=inp.q_nope, q_pe=inp.q_pe, c_kv=inp.c_kv, k_pe=inp.k_pe,
                 page_table=inp.page_table, kv_len=inp.kv_len, parents=par, tokens=tok, target=tgt)
    for name, arr in files.items():
        np.ascontiguousarray(arr).tofile(tmp_path / f"{name}.bin")
    (tmp_path / "dims.txt").write_text(f"{B} {T} {H} {inp.num_pages} {inp.page_table.shape[1]}\n")

    pkg = os.path.join(ROOT, "speculative_decoding_tree_va_b200")
    exe = str(tmp_path / "va_step")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(CUDA, "include"), os.path.join(ROOT, "tests", "c", "va_step.c"),
                    "-L", pkg, "-lverifyattn", "-Wl,-rpath," + pkg,
                    "-L", os.path.join(CUDA, "lib64"), "-lcudart", "-Wl,-rpath," + os.path.join(CUDA, "lib64"),
                    "-o", exe], check=True)
    r = subprocess.run([exe, str(tmp_path)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "step ok" in r.stdout

    out = np.fromfile(tmp_path / "out.bin", np.uint16).astype(np.uint32) << 16
    out = out.view(np.float32).reshape(-1, synth.D_LATENT)
    lse = np.fromfile(tmp_path / "lse.bin", np.float32)
    ref_out, ref_lse = oracle_rows(inp, parents=par)
    compare(out, lse, ref_out, ref_lse, "bf16", "C program")
    path, alen, nxt = oracle.tree_accept(par, tok, tgt)
    assert np.array_equal(np.fromfile(tmp_path / "path.bin", np.int32).reshape(B, T), path)
    assert np.array_equal(np.fromfile(tmp_path / "accept_len.bin", np.int32), alen)
    assert np.array_equal(np.fromfile(tmp_path / "next_token.bin", np.int32), nxt)
