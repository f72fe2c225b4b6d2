"""Seeded synthetic inputs for tree-verify MLA attention.

This module only draws random numbers and lays them out; it holds none of
the method's arithmetic (no tree building, no masks, no attention).  Both
sides of every parity check take their inputs from here: the CUDA library
through its Python binding, and the fp64 oracle through its test wrapper.

Shapes follow the DDTree verify step described on "The Milestone Commit:
Cementing Phase 1 of a Custom CUDA Speculative Decoding Engine" (section
"The Context": masked softmax over the concatenated prefix and tree tail, in
the absorbed MLA latent space) with d_latent = 512, d_rope = 64 and
scale = 1/sqrt(192).  The drafter output that feeds the tree builder is the
per-depth top-k of a log-softmax over N(0, 2^2) logits ("Strategic Pivots in
CUDA Kernel Engineering...", section "Why This Message Was Written": the
builder takes the drafter's top-k log probabilities and token ids).

Draw order for one workload (one numpy PCG64 stream, seed 0xDD7EE000 + i):
  1. per request, per depth 1..L: VOCAB logits -> log-softmax -> top-k,
  2. ragged prefix lengths,
  3. the page permutation,
  4. q_nope, q_pe, c_kv, k_pe (N(0,1); rounded to bf16 by
     round-to-nearest-even for bf16 workloads).  Workloads whose latent cache
     is kept as FP8 E4M3 codes store c_kv / kv_scale and k_pe / kv_scale
     rounded to the nearest code (``e4m3_codes``), the way such a cache is
     filled from the model's latents with one calibrated scale; the cache
     then stands for kv_scale times the coded values.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Tuple, Union

import numpy as np

D_LATENT = 512
D_ROPE = 64
PAGE_SIZE = 64
VOCAB = 4096
MAX_QLEN = 65
MAX_DEPTH = 15
SCALE = 1.0 / math.sqrt(192.0)


KV_SCALE_5SIGMA = float(np.float32(5.0 / 448.0))


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic verify-step workload (sizes of the tree-verify step)."""

    name: str
    dtype: str                    # "f32" or "bf16"
    B: int                        # requests
    H: int                        # heads
    P: Union[int, Tuple[int, int]]  # prefix length, or inclusive uniform range
    budget: int                   # draft nodes excluding the root; T = budget + 1
    topk: int                     # drafter top-k per depth
    max_depth: int = MAX_DEPTH
    paged: bool = True            # shuffled 64-token pages (else identity table)
    splits: int = 1               # split-KV chunks for the flash-decode path (0: the library plans)
    seed_index: int = 0
    kv: str = "same"              # latent cache storage: "same" as dtype, or "fp8_e4m3" codes
    kv_scale: float = 1.0         # value of one cache unit (FP8 cache only)

    @property
    def T(self) -> int:
        return self.budget + 1

    @property
    def seed(self) -> int:
        return 0xDD7EE000 + self.seed_index


WORKLOADS = {
    "fp32-tiny": Workload("fp32-tiny", "f32", B=1, H=8, P=128, budget=8, topk=8,
                          paged=False, seed_index=0),
    "fp32-page-test": Workload("fp32-page-test", "f32", B=1, H=64, P=2048, budget=32,
                               topk=8, paged=False, splits=0, seed_index=1),
    "bf16-deep": Workload("bf16-deep", "bf16", B=16, H=64, P=4096, budget=64, topk=2,
                          paged=True, seed_index=2),
    "bf16-b64-ragged": Workload("bf16-b64-ragged", "bf16", B=64, H=64, P=(512, 8192),
                                budget=32, topk=8, paged=True, seed_index=3),
    "bf16-long-prefix": Workload("bf16-long-prefix", "bf16", B=4, H=64, P=131072,
                                 budget=64, topk=8, paged=True, splits=16, seed_index=4),
    # FP8 latent cache (one scale per tensor) under the fp32 and bf16 query
    # shapes above.  The scale maps 5 standard deviations of the unit-variance
    # latents to the largest code (448); it is the float32 nearest 5/448, so
    # both sides of a parity check use exactly the same number.
    "fp32-fp8kv": Workload("fp32-fp8kv", "f32", B=1, H=64, P=2048, budget=32, topk=8,
                           paged=True, splits=0, seed_index=5, kv="fp8_e4m3",
                           kv_scale=KV_SCALE_5SIGMA),
    "bf16-fp8kv-deep": Workload("bf16-fp8kv-deep", "bf16", B=16, H=64, P=4096, budget=64,
                                topk=2, paged=True, seed_index=6, kv="fp8_e4m3",
                                kv_scale=KV_SCALE_5SIGMA),
}
WORKLOAD_ORDER = ["fp32-tiny", "fp32-page-test", "bf16-deep", "bf16-b64-ragged",
                  "bf16-long-prefix"]


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns uint16 bit patterns.

    Inputs are finite draws, so the 32-bit sum cannot wrap (only NaN bit
    patterns lie within 0x8000 of 2^32) and no NaN handling is needed.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((u + (0x7FFF + ((u >> 16) & 1))) >> 16).astype(np.uint16)


def bf16_to_f32(u: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 (exact)."""
    return (u.astype(np.uint32) << 16).view(np.float32)


def e4m3_codes(x: np.ndarray) -> np.ndarray:
    """Nearest FP8 E4M3 codes (uint8) of x: ties go to the even mantissa,
    magnitudes beyond 448 saturate to +-448, and the sign bit follows x.
    Magnitudes below 2^-6 land on the subnormal grid (steps of 2^-9)."""
    x = np.asarray(x, np.float64)
    a = np.minimum(np.abs(x), 448.0)
    _, E = np.frexp(a)                       # a = f * 2^E with f in [0.5, 1)
    step = np.ldexp(1.0, np.maximum(E - 1, -6) - 3)
    r = np.rint(a / step) * step             # round half to even on the step count
    _, E2 = np.frexp(r)
    normal = r >= 2.0 ** -6
    field = np.where(normal, E2 - 1 + 7, 0)
    man = np.where(normal, np.ldexp(r, -(E2 - 1)) * 8 - 8, r * 2.0 ** 9)
    sign = np.signbit(x).astype(np.int64) << 7
    return (sign | (field.astype(np.int64) << 3) | man.astype(np.int64)).astype(np.uint8)


def drafter_topk(rng: np.random.Generator, L: int, K: int, vocab: int = VOCAB,
                 sigma: float = 2.0) -> Tuple[np.ndarray, np.ndarray]:
    """Synthetic drafter output: per-depth top-K log-probs (descending) and token ids.

    Row d (0-based) belongs to tree depth d + 1.  Equal log-probs keep token-id
    order (stable sort), so the table is a deterministic function of the draw.
    """
    logits = rng.normal(0.0, sigma, size=(L, vocab))
    mx = logits.max(axis=1, keepdims=True)
    lse = mx + np.log(np.exp(logits - mx).sum(axis=1, keepdims=True))
    logp = logits - lse
    order = np.argsort(-logp, axis=1, kind="stable")[:, :K]
    lp = np.take_along_axis(logp, order, axis=1)
    return np.ascontiguousarray(lp, dtype=np.float64), np.ascontiguousarray(order, dtype=np.int32)


@dataclasses.dataclass
class Inputs:
    """Host arrays of one workload.  Values of bf16 workloads are uint16 bit patterns;
    an FP8 cache holds uint8 E4M3 codes."""

    wl: Workload
    lp: np.ndarray          # [B, L, K] float64 drafter log-probs
    tok: np.ndarray         # [B, L, K] int32 drafter token ids
    prefix: np.ndarray      # [B] int32 prefix lengths P_b
    kv_len: np.ndarray      # [B] int32 = P_b + T
    page_table: np.ndarray  # [B, max_pages] int32 (unused entries = -1)
    num_pages: int
    q_nope: np.ndarray      # [B, T, H, 512]
    q_pe: np.ndarray        # [B, T, H, 64]
    c_kv: np.ndarray        # [num_pages, 64, 512]
    k_pe: np.ndarray        # [num_pages, 64, 64]

    @property
    def T(self) -> int:
        return self.wl.T

    @property
    def max_pages(self) -> int:
        return self.page_table.shape[1]


def make_inputs(wl: Workload, *, B: Optional[int] = None, H: Optional[int] = None,
                P=None, budget: Optional[int] = None, topk: Optional[int] = None,
                max_depth: Optional[int] = None, seed: Optional[int] = None,
                with_tensors: bool = True) -> Inputs:
    """Draw one workload (optionally with overridden sizes, e.g. a scaled-down case)."""
    if any(v is not None for v in (B, H, P, budget, topk, max_depth)):
        wl = dataclasses.replace(
            wl,
            B=wl.B if B is None else B, H=wl.H if H is None else H,
            P=wl.P if P is None else P, budget=wl.budget if budget is None else budget,
            topk=wl.topk if topk is None else topk,
            max_depth=wl.max_depth if max_depth is None else max_depth)
    rng = np.random.default_rng(wl.seed if seed is None else seed)
    Bn, T, Hn = wl.B, wl.T, wl.H
    L, K = wl.max_depth, wl.topk

    lp = np.empty((Bn, L, K), np.float64)
    tok = np.empty((Bn, L, K), np.int32)
    for b in range(Bn):
        lp[b], tok[b] = drafter_topk(rng, L, K)

    if isinstance(wl.P, tuple):
        lo, hi = wl.P
        prefix = rng.integers(lo, hi + 1, size=Bn).astype(np.int32)
    else:
        prefix = np.full(Bn, wl.P, np.int32)
    kv_len = (prefix + T).astype(np.int32)

    pages_per = (kv_len + PAGE_SIZE - 1) // PAGE_SIZE
    num_pages = int(pages_per.sum())
    max_pages = int(pages_per.max())
    if wl.paged:
        phys = rng.permutation(num_pages).astype(np.int32)
    else:
        phys = np.arange(num_pages, dtype=np.int32)
    page_table = np.full((Bn, max_pages), -1, np.int32)
    off = 0
    for b in range(Bn):
        n = int(pages_per[b])
        page_table[b, :n] = phys[off:off + n]
        off += n

    def draw(shape):
        x = rng.standard_normal(size=shape, dtype=np.float32)
        return bf16_round(x) if wl.dtype == "bf16" else x

    if with_tensors:
        q_nope = draw((Bn, T, Hn, D_LATENT))
        q_pe = draw((Bn, T, Hn, D_ROPE))
        if wl.kv == "fp8_e4m3":
            c_kv = e4m3_codes(rng.standard_normal(size=(num_pages, PAGE_SIZE, D_LATENT),
                                                  dtype=np.float32) / wl.kv_scale)
            k_pe = e4m3_codes(rng.standard_normal(size=(num_pages, PAGE_SIZE, D_ROPE),
                                                  dtype=np.float32) / wl.kv_scale)
        else:
            c_kv = draw((num_pages, PAGE_SIZE, D_LATENT))
            k_pe = draw((num_pages, PAGE_SIZE, D_ROPE))
    else:
        q_nope = q_pe = c_kv = k_pe = None
    return Inputs(wl, lp, tok, prefix, kv_len, page_table, num_pages,
                  q_nope, q_pe, c_kv, k_pe)


def sample_rows(rng_seed: int, B: int, T: int, H: int, n: int,
                full_request: Optional[int] = 0) -> np.ndarray:
    """Flat row ids (b*T + t)*H + h for sampled parity checks: every row of one
    request (if given) plus n seeded random rows, sorted and unique."""
    rng = np.random.default_rng(rng_seed)
    rows = [rng.integers(0, B * T * H, size=n)]
    if full_request is not None:
        rows.append(np.arange(full_request * T * H, (full_request + 1) * T * H))
    return np.unique(np.concatenate(rows)).astype(np.int32)


def split_bounds(kv_len: np.ndarray, splits: int, align: int = 256) -> np.ndarray:
    """Key ranges [lo, hi) of the flash-decode split, as the library's header
    fixes them: the edge between split s - 1 and split s is s * kv_len / S
    rounded to the nearest multiple of align (ties up), at most kv_len; the
    first split starts at 0 and the last ends at kv_len."""
    kv = kv_len.astype(np.int64)
    edges = [np.zeros_like(kv)]
    for s in range(1, splits):
        e = (2 * s * kv + splits * align) // (2 * splits * align) * align
        edges.append(np.minimum(e, kv))
    edges.append(kv)
    out = np.zeros((kv.shape[0], splits, 2), np.int32)
    for s in range(splits):
        out[:, s, 0] = edges[s]
        out[:, s, 1] = edges[s + 1]
    return out
