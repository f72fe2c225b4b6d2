"""CPU checks of the C ABI: the library loads, exports what the header declares,
and rejects bad arguments on the host before launching anything."""
import ctypes
import glob
import os
import re

import pytest

import speculative_decoding_tree_va_b200 as va
from speculative_decoding_tree_va_b200 import build as va_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    va_build.build()
    return va.load_library()


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(va_\w+)\s*\(", text, flags=re.M))
    return names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert {"va_verify_attn", "va_build_tree_mask", "va_merge", "va_build_tree"} <= names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    assert set(va.EXPORTS) <= names


def test_max_qlen_and_status_strings(lib):
    assert lib.va_max_qlen() == 65
    assert lib.va_status_string(0) == b"VA_OK"
    assert lib.va_status_string(4) == b"VA_ERR_INVALID_TREE"
    assert lib.va_status_string(99) == b"VA_ERR_UNKNOWN"


def args(**kw):
    a = va.VaAttnArgs()
    a.dtype, a.B, a.H, a.T, a.scale = va.VA_BF16, 2, 64, 33, 0.07
    fake = 1 << 20  # aligned, never dereferenced: every case below fails host checks
    for f in ("q_nope", "q_pe", "c_kv", "k_pe", "page_table", "kv_len", "tree_mask", "out", "lse"):
        setattr(a, f, fake)
    a.num_pages, a.page_size, a.max_pages = 100, 64, 50
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("bad,status", [
    (dict(T=66), va.VA_ERR_INVALID_ARG), (dict(T=0), va.VA_ERR_INVALID_ARG),
    (dict(H=0), va.VA_ERR_INVALID_ARG), (dict(dtype=7), va.VA_ERR_INVALID_ARG),
    (dict(page_size=32), va.VA_ERR_UNSUPPORTED), (dict(num_splits=65), va.VA_ERR_INVALID_ARG),
    (dict(q_nope=None), va.VA_ERR_INVALID_ARG), (dict(c_kv=(1 << 20) + 8), va.VA_ERR_INVALID_ARG),
    (dict(flags=16), va.VA_ERR_INVALID_ARG), (dict(num_pages=0), va.VA_ERR_INVALID_ARG),
    (dict(num_splits=4), va.VA_ERR_INVALID_ARG),  # split without a workspace
    (dict(scale=float("nan")), va.VA_ERR_INVALID_ARG),
    (dict(B=65536), va.VA_ERR_UNSUPPORTED),     # beyond the launches' request axis
    # the bounded-wait test hook exists only on the tensor-core path
    (dict(flags=va.VA_FLAG_TEST_STALL_MMA, dtype=va.VA_F32), va.VA_ERR_INVALID_ARG),
    (dict(flags=va.VA_FLAG_TEST_STALL_MMA | va.VA_FLAG_BF16_CUDA_CORES), va.VA_ERR_INVALID_ARG),
    # FP8 cache: the scale must be finite and positive; no tensor-core test hook
    (dict(flags=va.VA_FLAG_KV_FP8_E4M3), va.VA_ERR_INVALID_ARG),  # kv_scale left at 0
    (dict(flags=va.VA_FLAG_KV_FP8_E4M3, kv_scale=-0.5), va.VA_ERR_INVALID_ARG),
    (dict(flags=va.VA_FLAG_KV_FP8_E4M3, kv_scale=float("nan")), va.VA_ERR_INVALID_ARG),
    (dict(flags=va.VA_FLAG_KV_FP8_E4M3, kv_scale=float("inf")), va.VA_ERR_INVALID_ARG),
    (dict(flags=va.VA_FLAG_KV_FP8_E4M3 | va.VA_FLAG_TEST_STALL_MMA, kv_scale=0.5),
     va.VA_ERR_INVALID_ARG),
    # the staging-wait hook exists only for fp32 queries on an fp32 cache
    (dict(flags=va.VA_FLAG_TEST_STALL_COPIES), va.VA_ERR_INVALID_ARG),
    (dict(flags=va.VA_FLAG_TEST_STALL_COPIES | va.VA_FLAG_BF16_CUDA_CORES), va.VA_ERR_INVALID_ARG),
    (dict(flags=va.VA_FLAG_TEST_STALL_COPIES | va.VA_FLAG_KV_FP8_E4M3, kv_scale=0.5,
          dtype=va.VA_F32), va.VA_ERR_INVALID_ARG),
    (dict(flags=va.VA_FLAG_TEST_STALL_COPIES | va.VA_FLAG_TEST_STALL_MMA, dtype=va.VA_F32),
     va.VA_ERR_INVALID_ARG),
])
def test_verify_attn_host_checks(lib, bad, status):
    a = args(**bad)
    assert lib.va_verify_attn(ctypes.byref(a), None) == status


def test_zero_batch_is_a_noop(lib):
    a = args(B=0)
    assert lib.va_verify_attn(ctypes.byref(a), None) == va.VA_OK
    assert lib.va_build_tree_mask(None, 0, 5, None, None, None) == va.VA_OK
    assert lib.va_merge(None, None, 2, 0, 5, 8, 0, None, None, None) == va.VA_OK


def test_other_host_checks(lib):
    assert lib.va_build_tree_mask(None, 1, 66, None, None, None) == va.VA_ERR_INVALID_ARG
    assert lib.va_build_tree_mask(None, 1, 5, None, None, None) == va.VA_ERR_INVALID_ARG
    assert lib.va_build_tree(None, None, 1, 16, 8, 32, None, None, None, None, None) == \
        va.VA_ERR_INVALID_ARG  # depth > 15
    assert lib.va_build_tree(None, None, 1, 15, 8, 65, None, None, None, None, None) == \
        va.VA_ERR_INVALID_ARG  # T = 66
    assert lib.va_merge(None, None, 65, 1, 5, 8, 0, None, None, None) == va.VA_ERR_INVALID_ARG
    assert lib.va_merge(None, None, 2, 1, 5, 8, 3, None, None, None) == va.VA_ERR_INVALID_ARG


def test_split_planning_and_workspace(lib):
    # tensor cores: the request order (int32 [B]) first; explicit split count:
    # partials [S,B,T,H,512] f32 + [S,B,T,H] f32 + the splits' status int32
    # [B]; every part 256-byte aligned
    a = args(num_splits=16)
    rows = 2 * 33 * 64
    order = 256
    o = (16 * rows * 512 * 4 + 255) // 256 * 256
    l = (16 * rows * 4 + 255) // 256 * 256 + 256
    assert lib.va_num_splits(ctypes.byref(a)) == 16
    assert lib.va_workspace_bytes(ctypes.byref(a)) == order + o + l
    assert lib.va_workspace_bytes(ctypes.byref(args(num_splits=1))) == order
    assert lib.va_workspace_bytes(ctypes.byref(args(num_splits=1, B=300))) == 5 * 256
    # the CUDA-core kernel needs no order; single pass: no workspace at all
    assert lib.va_workspace_bytes(ctypes.byref(args(num_splits=1, dtype=va.VA_F32))) == 0
    assert lib.va_workspace_bytes(ctypes.byref(args(num_splits=1, flags=va.VA_FLAG_BF16_CUDA_CORES))) == 0
    assert lib.va_workspace_bytes(ctypes.byref(args(num_splits=16, dtype=va.VA_F32))) == o + l
    # auto: a big batch needs no split; a long, small batch splits
    assert lib.va_num_splits(ctypes.byref(args(B=64, max_pages=129))) == 1
    s = lib.va_num_splits(ctypes.byref(args(B=4, T=65, max_pages=2050)))
    assert s > 1 and (4 * 33 * s) % 74 >= 0
    assert lib.va_num_splits(ctypes.byref(args(T=66))) == -va.VA_ERR_INVALID_ARG


def _balanced_slots_brute_force(B, T, H, max_pages, sms=148):
    """Partials per row of the balanced CUDA-core plan, by listing every CTA's
    tile range: segments = B * ceil(T H / 32), 2 max_pages virtual tiles each,
    G = min(sms, tiles / 4) CTAs (fewer while a segment would need more than
    64 partials); None where the plan does not apply."""
    q = B * (-(-T * H // 32))
    if q >= sms:
        return None
    vt = 2 * max_pages
    U = q * vt
    G = min(sms, U // 4)
    while G > q:
        owners = [set() for _ in range(q)]
        for c in range(G):
            for u in range(c * U // G, (c + 1) * U // G):
                owners[u // vt].add(c)
        assert sum(len(o) for o in owners) >= q
        slots = max(len(o) for o in owners)
        if slots <= 64:
            return slots if slots >= 2 else None
        G -= 1
    return None


@pytest.mark.parametrize("B,T,H,max_pages", [
    (1, 33, 64, 33),    # the fp32 page-test shape
    (3, 21, 5, 15),     # partial row tiles
    (1, 1, 1, 63),      # one 1-row segment
    (2, 65, 2, 48),
    (4, 9, 32, 2),      # too few tiles per CTA: the plain planner
    (1, 65, 64, 2050),  # a long prefix with 131 segments
])
def test_balanced_cuda_core_plan(lib, B, T, H, max_pages):
    """Without a device the planner takes 148 SMs, like a B200."""
    want = _balanced_slots_brute_force(B, T, H, max_pages)
    for kw in (dict(dtype=va.VA_F32), dict(flags=va.VA_FLAG_BF16_CUDA_CORES)):
        got = lib.va_num_splits(ctypes.byref(args(B=B, T=T, H=H, max_pages=max_pages, **kw)))
        if want is None:
            assert got >= 1 and (got & (got - 1)) == 0  # the power-of-two planner
        else:
            assert got == want, (B, T, H, max_pages, kw)
    # the tensor-core kernel never takes the balanced plan
    tc = lib.va_num_splits(ctypes.byref(args(B=B, T=T, H=H, max_pages=max_pages)))
    assert tc >= 1 and (tc & (tc - 1)) == 0  # the power-of-two planner


def test_balanced_cta_of_is_the_inverse_of_the_ranges():
    """The balanced plan's kernel finds a segment's first and last CTA (its
    partial slots, and who marks the unused ones) with
    cta_of(u) = floor((u G + G - 1) / U), the CTA whose range
    [c U / G, (c + 1) U / G) holds virtual tile u.  Checked against the ranges
    themselves: every tile has exactly one owner, a segment's owners are
    consecutive CTAs from cta_of(first tile) to cta_of(last tile), and so slot
    c - cta_of(first) is unique per segment and below the plan's slot count."""
    import random
    rng = random.Random(7)
    cta_of = lambda u, U, G: (u * G + G - 1) // U
    for _ in range(300):
        q = rng.randint(1, 40)
        vt = rng.randint(1, 300)
        U = q * vt
        G = rng.randint(q + 1, max(q + 1, min(148, U // 4 if U >= 4 * (q + 1) else q + 1)))
        owner = [None] * U
        for c in range(G):
            for u in range(c * U // G, (c + 1) * U // G):
                assert owner[u] is None
                owner[u] = c
        assert None not in owner
        for u in range(U):
            assert cta_of(u, U, G) == owner[u], (u, U, G)
        for seg in range(q):
            owners = sorted({owner[u] for u in range(seg * vt, (seg + 1) * vt)})
            assert owners == list(range(owners[0], owners[-1] + 1))
            assert owners[0] == cta_of(seg * vt, U, G)
            assert owners[-1] == cta_of((seg + 1) * vt - 1, U, G)


def test_fp8_cache_split_planning_and_workspace(lib):
    """An FP8 cache keeps the query type's kernel (bf16: tensor cores, fp32: CUDA
    cores), so the auto split count is that kernel's; bf16 on the tensor cores
    adds the widened pages to the workspace."""
    fp8 = dict(flags=va.VA_FLAG_KV_FP8_E4M3, kv_scale=0.4375)
    for dt in (va.VA_BF16, va.VA_F32):
        for B, T, mp in ((1, 33, 33), (4, 65, 2050), (16, 65, 66), (64, 33, 129)):
            a = args(dtype=dt, B=B, T=T, max_pages=mp, **fp8)
            plain = args(dtype=dt, B=B, T=T, max_pages=mp)
            assert lib.va_num_splits(ctypes.byref(a)) == lib.va_num_splits(ctypes.byref(plain))
    # the two planners differ here, so the routing is visible
    tc = args(B=4, T=65, max_pages=2050, **fp8)
    cc = args(B=4, T=65, max_pages=2050, flags=fp8["flags"] | va.VA_FLAG_BF16_CUDA_CORES,
              kv_scale=0.4375)
    assert lib.va_num_splits(ctypes.byref(tc)) != lib.va_num_splits(ctypes.byref(cc))
    # single pass: the request order, then the widened cache (B * max_pages
    # pages) and its page table
    a = args(num_splits=1, **fp8)                     # B = 2, max_pages = 50
    pages = 2 * 50
    up = lambda x: (x + 255) // 256 * 256
    want = up(pages * 64 * 512 * 2) + up(pages * 64 * 64 * 2) + up(pages * 4)
    assert lib.va_workspace_bytes(ctypes.byref(a)) == 256 + want
    assert lib.va_workspace_bytes(ctypes.byref(args(num_splits=1, dtype=va.VA_F32, **fp8))) == 0
    # with splits the partials and the splits' status come between the order
    # and the widened cache
    a = args(num_splits=4, **fp8)
    rows = 2 * 33 * 64
    parts = up(4 * rows * 512 * 4) + up(4 * rows * 4) + up(2 * 4)
    assert lib.va_workspace_bytes(ctypes.byref(a)) == 256 + parts + want
    # the no-allocation entry point refuses, before any launch, what its fixed array cannot hold
    big = args(B=64, max_pages=129, num_splits=1, **fp8)
    assert lib.va_verify_attn_noalloc(ctypes.byref(big), None) == va.VA_ERR_UNSUPPORTED


def test_partials_host_checks(lib):
    """va_verify_attn_partials: explicit partition, split range inside it, its own
    output arrays; out and lse may be NULL; no launch on any failed check."""
    f = ctypes.c_void_p(1 << 20)
    ws = dict(workspace=1 << 24, workspace_bytes=1 << 20)
    call = lambda a, first, count, o=f, l=f: lib.va_verify_attn_partials(ctypes.byref(a), first,
                                                                         count, o, l, None)
    assert call(args(num_splits=0, **ws), 0, 1) == va.VA_ERR_INVALID_ARG     # planned: refused
    assert call(args(num_splits=8, **ws), -1, 2) == va.VA_ERR_INVALID_ARG
    assert call(args(num_splits=8, **ws), 7, 2) == va.VA_ERR_INVALID_ARG     # past the last split
    assert call(args(num_splits=8, **ws), 3, 0) == va.VA_ERR_INVALID_ARG
    assert call(args(num_splits=8, **ws), 0, 2, o=None) == va.VA_ERR_INVALID_ARG
    assert call(args(num_splits=8, **ws), 0, 2, o=ctypes.c_void_p((1 << 20) + 4)) == \
        va.VA_ERR_INVALID_ARG                                                # o_part misaligned
    assert call(args(num_splits=8), 0, 2) == va.VA_ERR_INVALID_ARG           # no workspace (order)
    assert call(args(num_splits=8, T=66, **ws), 0, 2) == va.VA_ERR_INVALID_ARG
    assert call(args(num_splits=8, B=0, out=None, lse=None), 0, 2) == va.VA_OK
    # its workspace is that of a single-split call: no partials in it
    a = args(num_splits=8)
    assert va.partials_workspace_bytes(a) == 256
    assert va.partials_workspace_bytes(args(num_splits=8, dtype=va.VA_F32)) == 0


def test_c99_program_uses_the_host_api(tmp_path):
    """The header is plain C99 and the library links into a C program with no Python."""
    import subprocess
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pkg = os.path.join(root, "speculative_decoding_tree_va_b200")
    exe = str(tmp_path / "va_host_checks")
    subprocess.run(["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror",
                    "-I", os.path.join(root, "include"), os.path.join(root, "tests", "c", "va_host_checks.c"),
                    "-L", pkg, "-lverifyattn", "-Wl,-rpath," + pkg, "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "host checks ok" in r.stdout
    # the binding's copy of the fixed no-allocation array size is the header's
    m = re.search(r"VA_NOALLOC_SCRATCH_BYTES=(\d+)", r.stdout)
    assert m and int(m.group(1)) == va.NOALLOC_SCRATCH_BYTES
