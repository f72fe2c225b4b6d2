"""Python binding of libverifyattn (tree-verify MLA attention for DDTree, sm_100a).

Argument marshalling only: every step runs in the CUDA library's kernels.
Torch tensors cross the C ABI as raw device pointers plus the current CUDA
stream, the bridge shape the pages describe (page "The Capstone Commit:
Validating a Native CUDA DDTree Inference Engine", section "The Message
Itself": ctypes bindings accepting torch CUDA tensors via data_ptr and the
current stream).  The library must be built in-tree
(``python -m speculative_decoding_tree_va_b200.build``); importing the calls
without it raises -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("VA_LIB", os.path.join(HERE, "libverifyattn.so"))

VA_OK, VA_ERR_INVALID_ARG, VA_ERR_UNSUPPORTED, VA_ERR_CUDA, VA_ERR_INVALID_TREE = range(5)
VA_F32, VA_BF16 = 0, 1
VA_FLAG_BF16_CUDA_CORES = 1
VA_FLAG_TEST_STALL_MMA = 2  # test hook: the tensor-core kernel's bounded waits expire
VA_FLAG_TEST_STALL_COPIES = 8  # test hook: the CUDA-core kernel's staging waits expire
VA_FLAG_KV_FP8_E4M3 = 4     # latent cache as FP8 E4M3 codes times kv_scale
D_LATENT, D_ROPE, PAGE_SIZE, MAX_QLEN = 512, 64, 64, 65

EXPORTS = ("va_max_qlen", "va_status_string", "va_build_tree", "va_build_tree_mask",
           "va_workspace_bytes", "va_num_splits", "va_verify_attn", "va_merge",
           "va_device_timeouts", "va_verify_attn_noalloc", "va_tree_accept",
           "va_verify_attn_partials")
NOALLOC_SCRATCH_BYTES = 32 << 20


class VaAttnArgs(ctypes.Structure):
    """Mirror of ``va_attn_args`` in include/verifyattn.h."""

    _fields_ = [
        ("dtype", ctypes.c_int), ("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int),
        ("scale", ctypes.c_float),
        ("q_nope", ctypes.c_void_p), ("q_pe", ctypes.c_void_p),
        ("c_kv", ctypes.c_void_p), ("k_pe", ctypes.c_void_p),
        ("num_pages", ctypes.c_int), ("page_size", ctypes.c_int),
        ("page_table", ctypes.c_void_p), ("max_pages", ctypes.c_int),
        ("kv_len", ctypes.c_void_p), ("tree_mask", ctypes.c_void_p),
        ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p), ("req_status", ctypes.c_void_p),
        ("num_splits", ctypes.c_int), ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t), ("flags", ctypes.c_int),
        ("kv_scale", ctypes.c_float),
    ]


class VerifyAttnError(RuntimeError):
    pass


_lib = None


def load_library(path: Optional[str] = None):
    """Load libverifyattn.so (raises if it has not been built)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise VerifyAttnError(f"libverifyattn not built: {p} missing "
                              "(run python -m speculative_decoding_tree_va_b200.build)")
    lib = ctypes.CDLL(p)
    V, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.va_max_qlen.argtypes, lib.va_max_qlen.restype = [], I
    lib.va_status_string.argtypes, lib.va_status_string.restype = [I], ctypes.c_char_p
    lib.va_build_tree.argtypes = [V, V, I, I, I, I, V, V, V, V, V]
    lib.va_build_tree.restype = I
    lib.va_build_tree_mask.argtypes = [V, I, I, V, V, V]
    lib.va_build_tree_mask.restype = I
    lib.va_workspace_bytes.argtypes, lib.va_workspace_bytes.restype = [ctypes.POINTER(VaAttnArgs)], Z
    lib.va_num_splits.argtypes, lib.va_num_splits.restype = [ctypes.POINTER(VaAttnArgs)], I
    lib.va_verify_attn.argtypes = [ctypes.POINTER(VaAttnArgs), V]
    lib.va_verify_attn.restype = I
    lib.va_merge.argtypes = [V, V, I, I, I, I, I, V, V, V]
    lib.va_merge.restype = I
    lib.va_device_timeouts.argtypes, lib.va_device_timeouts.restype = [], ctypes.c_uint
    lib.va_tree_accept.argtypes = [V, V, V, I, I, V, V, V, V]
    lib.va_tree_accept.restype = I
    lib.va_verify_attn_noalloc.argtypes = [ctypes.POINTER(VaAttnArgs), V]
    lib.va_verify_attn_noalloc.restype = I
    lib.va_verify_attn_partials.argtypes = [ctypes.POINTER(VaAttnArgs), I, I, V, V, V]
    lib.va_verify_attn_partials.restype = I
    if path is None:
        _lib = lib
    return lib


def _check(status: int, what: str):
    if status != VA_OK:
        name = load_library().va_status_string(status).decode()
        raise VerifyAttnError(f"{what} failed: {name}")


def _stream(stream=None):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def max_qlen() -> int:
    return load_library().va_max_qlen()


def device_timeouts() -> int:
    """Expired bounded waits in the tensor-core kernel since load (synchronises)."""
    return int(load_library().va_device_timeouts())


def build_tree(lp, tok, budget: int, stream=None):
    """GPU best-first draft trees.  lp float64 [B, L, K], tok int32 [B, L, K] (cuda).

    Returns (parents, tokens, depth) int32 [B, budget + 1] and n_nodes int32 [B]."""
    import torch
    B, L, K = lp.shape
    T = budget + 1
    kw = dict(device=lp.device, dtype=torch.int32)
    parents, tokens, depth = (torch.empty(B, T, **kw) for _ in range(3))
    n_nodes = torch.empty(B, **kw)
    _check(load_library().va_build_tree(_ptr(lp.contiguous()), _ptr(tok.contiguous()), B, L, K,
                                        budget, _ptr(parents), _ptr(tokens), _ptr(depth),
                                        _ptr(n_nodes), _stream(stream)), "va_build_tree")
    return parents, tokens, depth, n_nodes


def tree_accept(parents, tokens, target_next, stream=None):
    """Greedy accept walk.  int32 [B, T] cuda tensors -> (path [B, T], accept_len [B],
    next_token [B])."""
    import torch
    B, T = parents.shape
    kw = dict(device=parents.device, dtype=torch.int32)
    path = torch.empty(B, T, **kw)
    alen = torch.empty(B, **kw)
    nxt = torch.empty(B, **kw)
    _check(load_library().va_tree_accept(_ptr(parents.contiguous()), _ptr(tokens.contiguous()),
                                         _ptr(target_next.contiguous()), B, T, _ptr(path),
                                         _ptr(alen), _ptr(nxt), _stream(stream)), "va_tree_accept")
    return path, alen, nxt


def build_tree_mask(parents, stream=None):
    """parents int32 [B, T] (cuda) -> (mask int64 [B, T, W] holding uint64 bits, status int32 [B])."""
    import torch
    B, T = parents.shape
    W = (T + 63) // 64
    mask = torch.empty(B, T, W, device=parents.device, dtype=torch.int64)
    status = torch.empty(B, device=parents.device, dtype=torch.int32)
    _check(load_library().va_build_tree_mask(_ptr(parents.contiguous()), B, T, _ptr(mask),
                                             _ptr(status), _stream(stream)), "va_build_tree_mask")
    return mask, status


def _fp8_cache(c_kv) -> bool:
    import torch
    return c_kv.dtype in (torch.uint8, torch.float8_e4m3fn)


def make_args(q_nope, q_pe, c_kv, k_pe, page_table, kv_len, tree_mask, out, lse, *, scale: float,
              num_splits: int = 0, workspace=None, req_status=None, flags: int = 0,
              kv_scale: float = 1.0) -> VaAttnArgs:
    """Fill a VaAttnArgs from torch tensors (no checks beyond what the library does).

    A uint8 or float8_e4m3fn cache (c_kv, k_pe) sets VA_FLAG_KV_FP8_E4M3 with
    kv_scale, the value of one cache unit."""
    import torch
    B, T, H, _ = q_nope.shape
    dt = {torch.float32: VA_F32, torch.bfloat16: VA_BF16}[q_nope.dtype]
    a = VaAttnArgs()
    a.dtype, a.B, a.H, a.T, a.scale = dt, B, H, T, float(scale)
    a.q_nope, a.q_pe, a.c_kv, a.k_pe = (t.data_ptr() for t in (q_nope, q_pe, c_kv, k_pe))
    a.num_pages, a.page_size = c_kv.shape[0], c_kv.shape[1]
    a.page_table, a.max_pages = page_table.data_ptr(), page_table.shape[1]
    a.kv_len, a.tree_mask = kv_len.data_ptr(), tree_mask.data_ptr()
    a.out, a.lse = out.data_ptr(), lse.data_ptr()
    a.req_status = None if req_status is None else req_status.data_ptr()
    a.num_splits = num_splits
    a.workspace = None if workspace is None else workspace.data_ptr()
    a.workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    a.flags = flags
    if _fp8_cache(c_kv):
        a.flags |= VA_FLAG_KV_FP8_E4M3
        a.kv_scale = float(kv_scale)
    return a


def workspace_bytes(args: VaAttnArgs) -> int:
    return int(load_library().va_workspace_bytes(ctypes.byref(args)))


def num_splits(args: VaAttnArgs) -> int:
    """The split count va_verify_attn uses for these arguments (for the balanced
    CUDA-core plan, the number of partials per row it merges)."""
    return int(load_library().va_num_splits(ctypes.byref(args)))


def verify_attn_args(args: VaAttnArgs, stream=None):
    _check(load_library().va_verify_attn(ctypes.byref(args), _stream(stream)), "va_verify_attn")


def verify_attn(q_nope, q_pe, c_kv, k_pe, page_table, kv_len, tree_mask, *, scale: float,
                num_splits: int = 0, out=None, lse=None, workspace=None, req_status=None,
                flags: int = 0, kv_scale: float = 1.0, stream=None):
    """Tree-verify MLA-absorb attention.  Allocates out/lse/workspace when not given.

    q_nope [B,T,H,512], q_pe [B,T,H,64] (float32 or bfloat16, cuda); c_kv
    [pages,64,512], k_pe [pages,64,64] in the query dtype, or FP8 E4M3 codes
    (uint8 / float8_e4m3fn) standing for kv_scale times their values;
    page_table int32 [B, max_pages], kv_len int32 [B], tree_mask int64 [B,T,W]
    from build_tree_mask.  Returns (out, lse) in the query dtype."""
    import torch
    B, T, H, _ = q_nope.shape
    if out is None:
        out = torch.empty(B, T, H, D_LATENT, device=q_nope.device, dtype=q_nope.dtype)
    if lse is None:
        lse = torch.empty(B, T, H, device=q_nope.device, dtype=torch.float32)
    args = make_args(q_nope, q_pe, c_kv, k_pe, page_table, kv_len, tree_mask, out, lse,
                     scale=scale, num_splits=num_splits, workspace=workspace,
                     req_status=req_status, flags=flags, kv_scale=kv_scale)
    need = workspace_bytes(args)
    if need and workspace is None:
        workspace = torch.empty(need, device=q_nope.device, dtype=torch.uint8)
        args.workspace, args.workspace_bytes = workspace.data_ptr(), need
    verify_attn_args(args, stream)
    return out, lse


def verify_attn_noalloc(args: VaAttnArgs, stream=None):
    """va_verify_attn_noalloc: split-KV partials in the library's fixed device
    array instead of a workspace (for callers that cannot allocate)."""
    _check(load_library().va_verify_attn_noalloc(ctypes.byref(args), _stream(stream)),
           "va_verify_attn_noalloc")


def partials_workspace_bytes(args: VaAttnArgs) -> int:
    """Workspace of va_verify_attn_partials: that of the same call with one split."""
    one = VaAttnArgs.from_buffer_copy(args)
    one.num_splits = 1
    return workspace_bytes(one)


def verify_attn_partials(args: VaAttnArgs, split_first: int, split_count: int, o_part, lse_part,
                         stream=None):
    """va_verify_attn_partials: splits [split_first, split_first + split_count) of the
    args.num_splits-way partition into o_part float [count, B, T, H, 512] and
    lse_part float [count, B, T, H] (cuda tensors), no merge."""
    _check(load_library().va_verify_attn_partials(ctypes.byref(args), split_first, split_count,
                                                  _ptr(o_part), _ptr(lse_part), _stream(stream)),
           "va_verify_attn_partials")


def merge(o_part, lse_part, out_dtype, stream=None):
    """o_part float [S,B,T,H,512], lse_part float [S,B,T,H] -> (out, lse)."""
    import torch
    S, B, T, H, _ = o_part.shape
    dt = {torch.float32: VA_F32, torch.bfloat16: VA_BF16}[out_dtype]
    out = torch.empty(B, T, H, D_LATENT, device=o_part.device, dtype=out_dtype)
    lse = torch.empty(B, T, H, device=o_part.device, dtype=torch.float32)
    _check(load_library().va_merge(_ptr(o_part.contiguous()), _ptr(lse_part.contiguous()), S, B, T,
                                   H, dt, _ptr(out), _ptr(lse), _stream(stream)), "va_merge")
    return out, lse
