"""The input generator's FP8 E4M3 rounding (used only to fill synthetic
caches) agrees with torch's float -> float8_e4m3fn conversion."""
import numpy as np

from speculative_decoding_tree_va_b200 import synth


def test_e4m3_codes_match_torch_rounding():
    import torch
    rng = np.random.default_rng(1)
    x = rng.standard_normal(100000) * np.exp(rng.uniform(-12.0, 7.0, 100000))
    ties = np.array([2.0 ** -10, 1.5 * 2.0 ** -9, 2.5 * 2.0 ** -9, 1.0625, 1.1875, -1.0625,
                     0.0, -0.0, 448.0, 464.0, 1e6, -1e6])
    x = np.concatenate([x, ties]).astype(np.float32)
    ours = synth.e4m3_codes(x)
    ref = torch.from_numpy(np.clip(x, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_fp8_workload_cache_statistics():
    """Unit-variance latents at a 5-sigma scale: no NaN codes, rms ~ 1, |value| <= 5."""
    inp = synth.make_inputs(synth.WORKLOADS["fp32-fp8kv"])
    for codes in (inp.c_kv, inp.k_pe):
        assert codes.dtype == np.uint8
        assert not np.isin(codes, [0x7F, 0xFF]).any()
    assert synth.KV_SCALE_5SIGMA == float(np.float32(synth.KV_SCALE_5SIGMA))
