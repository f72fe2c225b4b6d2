"""bench.py's algorithmic work count: flops per visible (row, key) and bytes per key
for each cache storage type (CPU only)."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from speculative_decoding_tree_va_b200 import synth  # noqa: E402


def _work(name, **kw):
    inp = synth.make_inputs(synth.WORKLOADS[name], with_tensors=False, **kw)
    depth = np.full((inp.wl.B, inp.T), -1, np.int32)
    depth[:, 0] = 0                                   # root only: P + 1 visible keys per row
    return inp, bench.work(inp, depth)


def test_flops_count_visible_keys_only():
    inp, (flops, _) = _work("bf16-deep", B=2, P=100)
    H = inp.wl.H
    assert flops == 2 * (100 + 1) * H * (2 * 576 + 2 * 512)


def test_bytes_per_key_follow_the_cache_type():
    sizes = {}
    for name in ("bf16-deep", "bf16-fp8kv-deep"):
        inp, (_, nbytes) = _work(name, B=2, P=100)
        rows = inp.wl.B * inp.T * inp.wl.H
        q_out = rows * (576 * 2 + 512 * 2 + 4)
        sizes[name] = (nbytes - q_out) / float(inp.kv_len.astype(np.int64).sum())
    assert sizes == {"bf16-deep": 1152.0, "bf16-fp8kv-deep": 576.0}
