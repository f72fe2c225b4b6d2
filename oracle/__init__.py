"""fp64 oracle for DDTree tree-verify MLA attention -- TEST INFRASTRUCTURE ONLY.

Thin ctypes wrapper around ``oracle.cpp`` (plain single-threaded C++ in
fp64).  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` may import this package.  The CUDA library neither imports
nor links it, and it shares no code with the library.

Every function cites the page section it restates inside ``oracle.cpp``.
All functions here pin to the pages or to mathematics through the CPU tests
in ``tests/test_oracle_pins.py``; none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.cpp with g++ (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-o", _LIB + ".tmp", _SRC]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.or_build_tree.argtypes = [P, P, i32, i32, i32, P, P, P, P, P]
        lib.or_build_tree.restype = i32
        lib.or_ancestor_mask.argtypes = [P, i32, i32, P, P]
        lib.or_ancestor_mask.restype = None
        lib.or_attention_rows.argtypes = [i32, i32, i32, i32, i32, f64, i32, i32, f64,
                                          P, P, P, P, i32, P, i32, P, P, P, P,
                                          i32, P, P, P]
        lib.or_attention_rows.restype = None
        lib.or_merge.argtypes = [P, P, i32, i64, i32, P, P]
        lib.or_merge.restype = None
        lib.or_tree_accept.argtypes = [P, P, P, i32, i32, P, P, P]
        lib.or_tree_accept.restype = None
        lib.or_decode_e4m3.argtypes = [P, i64, P]
        lib.or_decode_e4m3.restype = None
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def build_tree(lp: np.ndarray, tok: np.ndarray, budget: int) -> dict:
    """Best-first tree of one request from its [L, K] drafter table."""
    lib = _load()
    lp = np.ascontiguousarray(lp, np.float64)
    tok = np.ascontiguousarray(tok, np.int32)
    L, K = lp.shape
    T = budget + 1
    parent = np.empty(T, np.int32)
    token = np.empty(T, np.int32)
    depth = np.empty(T, np.int32)
    rank = np.empty(T, np.int32)
    score = np.empty(T, np.float64)
    n = lib.or_build_tree(_ptr(lp), _ptr(tok), L, K, budget, _ptr(parent), _ptr(token),
                          _ptr(depth), _ptr(rank), _ptr(score))
    return dict(n=int(n), parent=parent, token=token, depth=depth, rank=rank, score=score)


def build_trees(lp: np.ndarray, tok: np.ndarray, budget: int) -> dict:
    """Trees of a batch: lp/tok [B, L, K] -> stacked [B, T] arrays."""
    trees = [build_tree(lp[b], tok[b], budget) for b in range(lp.shape[0])]
    out = {k: np.stack([t[k] for t in trees]) for k in ("parent", "token", "depth", "rank", "score")}
    out["n"] = np.array([t["n"] for t in trees], np.int32)
    return out


def ancestor_mask(parents: np.ndarray):
    """[B, T] parent pointers -> ([B, T, W] uint64 mask, [B] int32 status)."""
    lib = _load()
    parents = np.ascontiguousarray(parents, np.int32)
    B, T = parents.shape
    W = (T + 63) // 64
    mask = np.zeros((B, T, W), np.uint64)
    status = np.zeros(B, np.int32)
    lib.or_ancestor_mask(_ptr(parents), B, T, _ptr(mask), _ptr(status))
    return mask, status


def decode_e4m3(codes: np.ndarray) -> np.ndarray:
    """FP8 E4M3 codes (uint8) -> float64 values (NaN for the two NaN codes)."""
    lib = _load()
    codes = np.ascontiguousarray(codes, np.uint8)
    out = np.empty(codes.shape, np.float64)
    lib.or_decode_e4m3(_ptr(codes), codes.size, _ptr(out))
    return out


_DTYPES = {"f32": (0, np.float32), "bf16": (1, np.uint16), "fp8_e4m3": (2, np.uint8)}


def attention_rows(q_nope, q_pe, c_kv, k_pe, page_table, kv_len, mask, *, scale: float,
                   dtype: str, rows: Optional[np.ndarray] = None, key_lo=None, key_hi=None,
                   page_size: int = 64, kv_dtype: Optional[str] = None, kv_scale: float = 1.0):
    """Masked attention for flat rows (b*T + t)*H + h (all rows if ``rows`` is None).

    q_nope [B,T,H,Dc], q_pe [B,T,H,Dr] as float32 arrays (dtype "f32") or uint16
    bf16 bit patterns (dtype "bf16"); c_kv [pages,page,Dc], k_pe [pages,page,Dr]
    in kv_dtype (default: dtype; "fp8_e4m3" = uint8 FP8 E4M3 codes), each cached
    element standing for kv_scale times its stored value.
    Returns (out [n, Dc] float64, lse [n] float64).
    """
    lib = _load()
    B, T, H, Dc = q_nope.shape
    Dr = q_pe.shape[-1]
    dt, want = _DTYPES[dtype]
    if dt == 2:
        raise ValueError("queries are f32 or bf16")
    kdt, kwant = _DTYPES[kv_dtype or dtype]
    arrs = [np.ascontiguousarray(a, want) for a in (q_nope, q_pe)]
    arrs += [np.ascontiguousarray(a, kwant) for a in (c_kv, k_pe)]
    page_table = np.ascontiguousarray(page_table, np.int32)
    kv_len = np.ascontiguousarray(kv_len, np.int32)
    mask = np.ascontiguousarray(mask, np.uint64)
    if rows is not None:
        rows = np.ascontiguousarray(rows, np.int32)
        n = rows.shape[0]
    else:
        n = B * T * H
    lo = None if key_lo is None else np.ascontiguousarray(key_lo, np.int32)
    hi = None if key_hi is None else np.ascontiguousarray(key_hi, np.int32)
    out = np.zeros((n, Dc), np.float64)
    lse = np.zeros(n, np.float64)
    lib.or_attention_rows(B, T, H, Dc, Dr, float(scale), dt, kdt, float(kv_scale),
                          *[_ptr(a) for a in arrs],
                          page_size, _ptr(page_table), page_table.shape[1], _ptr(kv_len),
                          _ptr(mask), _ptr(lo), _ptr(hi), n, _ptr(rows), _ptr(out), _ptr(lse))
    return out, lse


def merge(o_part: np.ndarray, lse_part: np.ndarray):
    """Merge split partials: o_part [S, rows, D], lse_part [S, rows] -> (out, lse)."""
    lib = _load()
    o_part = np.ascontiguousarray(o_part, np.float64)
    lse_part = np.ascontiguousarray(lse_part, np.float64)
    S, R, D = o_part.shape
    out = np.zeros((R, D), np.float64)
    lse = np.zeros(R, np.float64)
    lib.or_merge(_ptr(o_part), _ptr(lse_part), S, R, D, _ptr(out), _ptr(lse))
    return out, lse


def tree_accept(parents: np.ndarray, tokens: np.ndarray, target_next: np.ndarray):
    """Greedy accept walk: [B, T] parents/tokens/target_next -> (path [B,T], accept_len [B],
    next_token [B])."""
    lib = _load()
    parents = np.ascontiguousarray(parents, np.int32)
    tokens = np.ascontiguousarray(tokens, np.int32)
    target_next = np.ascontiguousarray(target_next, np.int32)
    B, T = parents.shape
    path = np.empty((B, T), np.int32)
    alen = np.empty(B, np.int32)
    nxt = np.empty(B, np.int32)
    lib.or_tree_accept(_ptr(parents), _ptr(tokens), _ptr(target_next), B, T, _ptr(path),
                       _ptr(alen), _ptr(nxt))
    return path, alen, nxt
