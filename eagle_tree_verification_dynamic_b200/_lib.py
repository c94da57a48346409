"""ctypes binding of libeagle_tree.so (argument marshalling only).

Every function here checks shapes, allocates outputs / workspaces with torch
on the tensors' device and calls the C entry point of the same name on the
current CUDA stream.  All arithmetic happens in the library's kernels.  There
is no fallback: if the shared library is missing or a call fails, an
exception is raised.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libeagle_tree.so")

F32, BF16 = 0, 1
MAX_NODES, MAX_TOPK, MAX_DEPTH, MAX_POOL = 128, 32, 16, 4096

_c_p = ctypes.c_void_p
_c_i = ctypes.c_int
_c_ll = ctypes.c_longlong
_c_sz = ctypes.c_size_t
_c_f = ctypes.c_float


class EagleError(RuntimeError):
    pass


class TreeStruct(ctypes.Structure):
    _fields_ = [("tokens", _c_p), ("parents", _c_p), ("depth", _c_p), ("logV", _c_p),
                ("gid", _c_p), ("draft_row", _c_p), ("row_lse", _c_p)]


class StepIn(ctypes.Structure):
    _fields_ = [("draft_logits", _c_p), ("target_logits", _c_p), ("logits_dtype", _c_i),
                ("B", _c_i), ("V", _c_i), ("depth", _c_i), ("k", _c_i), ("m", _c_i),
                ("q", _c_p), ("k_cache", _c_p), ("v_cache", _c_p), ("prefix_len", _c_p), ("Lmax", _c_i),
                ("k_tree", _c_p), ("v_tree", _c_p), ("Hq", _c_i), ("Hkv", _c_i), ("D", _c_i), ("window", _c_i),
                ("scale", _c_f), ("uniforms", _c_p), ("sampling_rule", _c_i),
                ("block_table", _c_p), ("page_size", _c_i), ("pages_per_seq", _c_i), ("num_pages", _c_i)]


class CostTableStruct(ctypes.Structure):
    _fields_ = [("nB", _c_i), ("nL", _c_i), ("nN", _c_i), ("B", _c_p), ("L", _c_p), ("N", _c_p), ("us", _c_p)]


class StepOut(ctypes.Structure):
    _fields_ = [("tree", TreeStruct), ("mask", _c_p), ("pos", _c_p), ("attn_out", _c_p),
                ("accepted_len", _c_p), ("path", _c_p), ("bonus", _c_p)]


_SIGS = {
    "eagle_status_string": (ctypes.c_char_p, [_c_i]),
    "eagle_last_cuda_error": (ctypes.c_char_p, []),
    "eagle_version": (_c_i, []),
    "eagle_row_stats_workspace_bytes": (_c_sz, [_c_ll, _c_i, _c_i, _c_i]),
    "eagle_row_stats": (_c_i, [_c_p, _c_i, _c_ll, _c_i, _c_i, _c_p, _c_p, _c_p, _c_p, _c_sz, _c_p]),
    "eagle_tree_build_workspace_bytes": (_c_sz, [_c_i, _c_i, _c_i, _c_i, _c_i]),
    "eagle_tree_build": (_c_i, [_c_p, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i,
                                ctypes.POINTER(TreeStruct), ctypes.POINTER(_c_i), _c_p, _c_sz, _c_p]),
    "eagle_tree_mask": (_c_i, [_c_p, _c_p, _c_p, _c_i, _c_i, _c_p, _c_p, _c_p]),
    "eagle_tree_attention_workspace_bytes": (_c_sz, [_c_i, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i]),
    "eagle_tree_attention": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_i, _c_p, _c_p, _c_p, _c_p, _c_i, _c_i,
                                    _c_i, _c_i, _c_i, _c_i, _c_f, _c_p, _c_p, _c_sz, _c_p]),
    "eagle_debug_attention_wait_probe": (None, [ctypes.c_ulonglong]),
    "eagle_tree_build_noalloc": (_c_i, [_c_p, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i,
                                        ctypes.POINTER(TreeStruct), ctypes.POINTER(_c_i), _c_p]),
    "eagle_verify_step_workspace_bytes": (_c_sz, [ctypes.POINTER(StepIn)]),
    "eagle_verify_step_attention_status_offset": (_c_sz, [ctypes.POINTER(StepIn)]),
    "eagle_verify_step": (_c_i, [ctypes.POINTER(StepIn), ctypes.POINTER(StepOut), ctypes.POINTER(_c_i), _c_p,
                                 _c_sz, _c_p]),
    "eagle_tree_grow_state_bytes": (_c_sz, [_c_i, _c_i, _c_i, _c_i, _c_i]),
    "eagle_tree_grow_begin": (_c_i, [_c_p, _c_i, _c_i, _c_i, _c_i, _c_i, _c_p, _c_sz, _c_p, _c_p, _c_p]),
    "eagle_tree_grow_level": (_c_i, [_c_p, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i, _c_p, _c_sz, _c_p, _c_p, _c_p]),
    "eagle_tree_grow_gains": (_c_i, [_c_i, _c_i, _c_i, _c_i, _c_i, _c_p, _c_sz, _c_p, _c_p]),
    "eagle_tree_grow_level_width": (_c_i, [_c_p, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i, _c_p, _c_sz, _c_p,
                                           _c_p, _c_p]),
    "eagle_tree_grow_frontier_logv": (_c_i, [_c_i, _c_i, _c_i, _c_i, _c_i, _c_p, _c_sz, _c_p, _c_p]),
    "eagle_tree_grow_finish_widths": (_c_i, [_c_i, _c_i, _c_i, _c_i, _c_i, _c_i, _c_p, _c_p, _c_sz,
                                             ctypes.POINTER(TreeStruct), ctypes.POINTER(_c_i), _c_p]),
    "eagle_size_level_width": (_c_i, [ctypes.POINTER(CostTableStruct), ctypes.c_double, ctypes.c_double, _c_i, _c_p,
                                      _c_i, _c_i, ctypes.c_double, ctypes.POINTER(_c_i), _c_p]),
    "eagle_tree_grow_finish": (_c_i, [_c_i, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i, _c_p, _c_sz,
                                      ctypes.POINTER(TreeStruct), ctypes.POINTER(_c_i), _c_p]),
    "eagle_static_tree_rows": (_c_i, [_c_p, _c_p, _c_i]),
    "eagle_static_tree_workspace_bytes": (_c_sz, [_c_i, _c_i, _c_i, _c_p, _c_p, _c_i]),
    "eagle_static_tree_build": (_c_i, [_c_p, _c_i, _c_i, _c_i, _c_i, _c_p, _c_p, _c_i, ctypes.POINTER(TreeStruct),
                                       _c_p, _c_sz, _c_p]),
    "eagle_cost_at": (ctypes.c_double, [ctypes.POINTER(CostTableStruct), ctypes.c_double, ctypes.c_double,
                                        ctypes.c_double]),
    "eagle_size_keep_level": (_c_i, [ctypes.POINTER(CostTableStruct), ctypes.c_double, ctypes.c_double, _c_i, _c_i,
                                     _c_p, _c_i, ctypes.c_double, ctypes.POINTER(_c_i),
                                     ctypes.POINTER(ctypes.c_double)]),
    "eagle_tree_attention_paged": (_c_i, [_c_p, _c_p, _c_p, _c_i, _c_i, _c_p, _c_i, _c_p, _c_p, _c_p, _c_p, _c_p,
                                          _c_i, _c_i, _c_i, _c_i, _c_i, _c_i, _c_f, _c_p, _c_p, _c_sz, _c_p]),
    "eagle_kv_compact_paged": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_p, _c_i, _c_p, _c_i,
                                      _c_i, _c_i, _c_i, _c_i, _c_p]),
    "eagle_kv_compact": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i,
                                _c_p]),
    "eagle_accept_workspace_bytes": (_c_sz, [_c_i, _c_i, _c_i, _c_i]),
    "eagle_accept_with_rule": (_c_i, [_c_p, _c_i, _c_p, _c_i, _c_p, _c_i, _c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i,
                                      _c_i, _c_i, _c_p, _c_p, _c_p, _c_p, _c_sz, _c_p]),
    "eagle_accept": (_c_i, [_c_p, _c_i, _c_p, _c_i, _c_p, _c_i, _c_p, _c_p, _c_p, _c_p, _c_i, _c_i,
                            _c_i, _c_i, _c_p, _c_p, _c_p, _c_p, _c_sz, _c_p]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load the shared library (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise EagleError(f"{LIB_PATH} is missing: build it with eagle_tree_verification_dynamic_b200.build")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def exported_names():
    return list(_SIGS)


def _check(status: int, what: str):
    if status != 0:
        msg = lib().eagle_status_string(status).decode()
        cuda = lib().eagle_last_cuda_error().decode()
        raise EagleError(f"{what}: {msg}" + (f" ({cuda})" if cuda and status == 7 else ""))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise EagleError(f"unsupported logits dtype {t.dtype}")


def _need_cuda(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise EagleError("tensors must be on a CUDA device")
            if not t.is_contiguous():
                raise EagleError("tensors must be contiguous")


def _workspace(nbytes: int, device) -> torch.Tensor:
    # torch's caching allocator returns blocks aligned to at least 512 bytes
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


# ---------------------------------------------------------------- row stats
def row_stats_workspace_bytes(rows: int, V: int, dtype_code: int, k: int) -> int:
    return lib().eagle_row_stats_workspace_bytes(rows, V, dtype_code, k)


def row_stats_into(logits: torch.Tensor, k: int, tok: torch.Tensor, val: torch.Tensor, lse, ws: torch.Tensor):
    """The vocabulary sweep into preallocated outputs (tok [rows][k] int32, val [rows][k] f32, lse [rows] f64
    or None) and workspace."""
    rows, V = logits.reshape(-1, logits.shape[-1]).shape
    dt = _dtype_code(logits)
    _check(lib().eagle_row_stats(_ptr(logits), dt, rows, V, k, _ptr(tok), _ptr(val), _ptr(lse), _ptr(ws),
                                 ws.numel(), _stream(logits.device)), "eagle_row_stats")


def row_stats(logits: torch.Tensor, k: int, want_lse: bool = True):
    """logits [rows][V] -> (topk_token [rows][k] int32, topk_logit [rows][k] f32, lse [rows] f64)."""
    _need_cuda(logits)
    rows, V = logits.reshape(-1, logits.shape[-1]).shape
    dev = logits.device
    tok = torch.empty(rows, k, dtype=torch.int32, device=dev)
    val = torch.empty(rows, k, dtype=torch.float32, device=dev)
    lse = torch.empty(rows, dtype=torch.float64, device=dev) if want_lse else None
    dt = _dtype_code(logits)
    nb = lib().eagle_row_stats_workspace_bytes(rows, V, dt, k)
    ws = _workspace(nb, dev)
    _check(lib().eagle_row_stats(_ptr(logits), dt, rows, V, k, _ptr(tok), _ptr(val), _ptr(lse),
                                 _ptr(ws), nb, _stream(dev)), "eagle_row_stats")
    return tok, val, lse


# --------------------------------------------------------------- tree build
@dataclass
class Tree:
    tokens: torch.Tensor     # [B][n] int32
    parents: torch.Tensor    # [B][n] int32
    depth: torch.Tensor      # [B][n] int32
    logV: torch.Tensor       # [B][n] float32
    gid: torch.Tensor        # [B][n] int32
    draft_row: torch.Tensor  # [B][n+1] int32
    row_lse: torch.Tensor    # [B][R] float64
    n: int

    def struct(self) -> TreeStruct:
        return TreeStruct(*[ctypes.c_void_p(t.data_ptr()) for t in
                            (self.tokens, self.parents, self.depth, self.logV, self.gid,
                             self.draft_row, self.row_lse)])


def pool_size(depth: int, k: int) -> int:
    return k + (depth - 1) * k * k


def alloc_tree(B: int, R: int, depth: int, k: int, m: int, device) -> Tree:
    n = min(m, pool_size(depth, k))
    i32 = dict(dtype=torch.int32, device=device)
    return Tree(tokens=torch.empty(B, n, **i32), parents=torch.empty(B, n, **i32),
                depth=torch.empty(B, n, **i32), logV=torch.empty(B, n, dtype=torch.float32, device=device),
                gid=torch.empty(B, n, **i32), draft_row=torch.empty(B, n + 1, **i32),
                row_lse=torch.empty(B, R, dtype=torch.float64, device=device), n=n)


def tree_build_workspace_bytes(B, R, V, dtype_code, k) -> int:
    return lib().eagle_tree_build_workspace_bytes(B, R, V, dtype_code, k)


def tree_build_into(draft_logits: torch.Tensor, depth: int, k: int, m: int, tree: Tree,
                    ws: torch.Tensor) -> int:
    B, R, V = draft_logits.shape
    dt = _dtype_code(draft_logits)
    st = tree.struct()
    n_out = _c_i(0)
    _check(lib().eagle_tree_build(_ptr(draft_logits), dt, B, R, V, depth, k, m, ctypes.byref(st),
                                  ctypes.byref(n_out), _ptr(ws), ws.numel(), _stream(draft_logits.device)),
           "eagle_tree_build")
    return n_out.value


def tree_build(draft_logits: torch.Tensor, depth: int, k: int, m: int) -> Tree:
    """draft_logits [B][R][V] (f32 or bf16) -> Tree."""
    _need_cuda(draft_logits)
    B, R, V = draft_logits.shape
    tree = alloc_tree(B, R, depth, k, m, draft_logits.device)
    nb = tree_build_workspace_bytes(B, R, V, _dtype_code(draft_logits), k)
    tree_build_into(draft_logits, depth, k, m, tree, _workspace(nb, draft_logits.device))
    return tree


# ---------------------------------------------------------------- tree mask
def tree_mask_into(parents, depth, prefix_len, mask, pos):
    B, n = parents.shape
    _check(lib().eagle_tree_mask(_ptr(parents), _ptr(depth), _ptr(prefix_len), B, n, _ptr(mask), _ptr(pos),
                                 _stream(parents.device)), "eagle_tree_mask")


def tree_mask(parents: torch.Tensor, depth: Optional[torch.Tensor] = None,
              prefix_len: Optional[torch.Tensor] = None):
    """parents [B][n] -> (mask [B][n][2] uint64 as int64, pos [B][n] int32 or None)."""
    _need_cuda(parents, depth, prefix_len)
    B, n = parents.shape
    mask = torch.empty(B, n, 2, dtype=torch.int64, device=parents.device)
    pos = torch.empty(B, n, dtype=torch.int32, device=parents.device) if depth is not None else None
    tree_mask_into(parents, depth, prefix_len, mask, pos)
    return mask, pos


# ----------------------------------------------------------- tree attention
def attention_workspace_bytes(B, n, Hq, Hkv, D, Lmax, window=0) -> int:
    return lib().eagle_tree_attention_workspace_bytes(B, n, Hq, Hkv, D, Lmax, window)


def tree_attention_into(q, k_cache, v_cache, prefix_len, k_tree, v_tree, mask, pos, out, ws,
                        window: int = 0, scale: float = 0.0):
    B, n, Hq, D = q.shape
    Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
    _check(lib().eagle_tree_attention(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(prefix_len), Lmax,
                                      _ptr(k_tree), _ptr(v_tree), _ptr(mask), _ptr(pos), B, n, Hq, Hkv, D,
                                      window, scale, _ptr(out), _ptr(ws), ws.numel(), _stream(q.device)),
           "eagle_tree_attention")


def tree_attention(q, k_cache, v_cache, prefix_len, k_tree, v_tree, mask, pos=None, window: int = 0,
                   scale: float = 0.0, check: bool = True) -> torch.Tensor:
    """q [B][n][Hq][D] bf16, caches [B][Hkv][Lmax][D] bf16, tree K/V [B][n][Hkv][D] bf16 -> out bf16."""
    _need_cuda(q, k_cache, v_cache, prefix_len, k_tree, v_tree, mask, pos)
    for t in (q, k_cache, v_cache, k_tree, v_tree):
        if t.dtype != torch.bfloat16:
            raise EagleError("attention tensors must be bf16")
    B, n, Hq, D = q.shape
    Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
    out = torch.empty_like(q)
    ws = _workspace(attention_workspace_bytes(B, n, Hq, Hkv, D, Lmax, window), q.device)
    tree_attention_into(q, k_cache, v_cache, prefix_len, k_tree, v_tree, mask, pos, out, ws, window, scale)
    if check:
        check_attention_status(ws)
    return out


def attention_wait_probe(limit_ns: int):
    """Diagnostics: make every following attention launch take its abort path
    after a bounded wait of limit_ns that nothing completes (0 turns it off)."""
    lib().eagle_debug_attention_wait_probe(int(limit_ns))


def check_attention_status(ws: torch.Tensor):
    """Read the device status word the attention kernel keeps in its workspace
    header (synchronises the stream).  1: a bounded wait inside the kernel gave
    up; 3: a paged cache named a page outside its pool for a key in use."""
    code = int(ws[:4].view(torch.int32).item())
    if code != 0:
        raise EagleError(f"eagle_tree_attention: device status {code}")


# ------------------------------------------------------- paged prefix cache
def tree_attention_paged_into(q, k_pages, v_pages, block_table, prefix_len, k_tree, v_tree, mask, pos, out, ws,
                              window: int = 0, scale: float = 0.0):
    """k_pages / v_pages [num_pages][Hkv][page_size][D] bf16, block_table [B][pages_per_seq] int32."""
    B, n, Hq, D = q.shape
    num_pages, Hkv, ps = k_pages.shape[0], k_pages.shape[1], k_pages.shape[2]
    _check(lib().eagle_tree_attention_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), num_pages, ps, _ptr(block_table),
                                            block_table.shape[1], _ptr(prefix_len), _ptr(k_tree), _ptr(v_tree),
                                            _ptr(mask), _ptr(pos), B, n, Hq, Hkv, D, window, scale, _ptr(out),
                                            _ptr(ws), ws.numel(), _stream(q.device)), "eagle_tree_attention_paged")


def tree_attention_paged(q, k_pages, v_pages, block_table, prefix_len, k_tree, v_tree, mask, pos=None,
                         window: int = 0, scale: float = 0.0, check: bool = True) -> torch.Tensor:
    """Tree attention over a paged prefix cache -> out [B][n][Hq][D] bf16 (raises on a device status when
    check, e.g. a page id outside the pool for a key in use)."""
    _need_cuda(q, k_pages, v_pages, block_table, prefix_len, k_tree, v_tree, mask, pos)
    B, n, Hq, D = q.shape
    Hkv, ps = k_pages.shape[1], k_pages.shape[2]
    out = torch.empty_like(q)
    ws = _workspace(attention_workspace_bytes(B, n, Hq, Hkv, D, block_table.shape[1] * ps, window), q.device)
    tree_attention_paged_into(q, k_pages, v_pages, block_table, prefix_len, k_tree, v_tree, mask, pos, out, ws,
                              window, scale)
    if check:
        check_attention_status(ws)
    return out


def kv_compact_paged_into(k_tree, v_tree, path, accepted_len, prefix_len, k_pages, v_pages, block_table,
                          new_prefix_len):
    """kv_compact into a paged cache (pools updated in place); new lengths into new_prefix_len."""
    B, n, Hkv, D = k_tree.shape
    _check(lib().eagle_kv_compact_paged(_ptr(k_tree), _ptr(v_tree), _ptr(path), _ptr(accepted_len), _ptr(prefix_len),
                                        _ptr(k_pages), _ptr(v_pages), k_pages.shape[0], k_pages.shape[2],
                                        _ptr(block_table), block_table.shape[1], _ptr(new_prefix_len), B, n, Hkv, D,
                                        path.shape[1], _stream(k_tree.device)), "eagle_kv_compact_paged")


def kv_compact_paged(k_tree, v_tree, path, accepted_len, prefix_len, k_pages, v_pages, block_table) -> torch.Tensor:
    """kv_compact into a paged cache (pools updated in place) -> new prefix lengths [B] int32."""
    _need_cuda(k_tree, v_tree, path, accepted_len, prefix_len, k_pages, v_pages, block_table)
    new_len = torch.empty_like(prefix_len)
    kv_compact_paged_into(k_tree, v_tree, path, accepted_len, prefix_len, k_pages, v_pages, block_table, new_len)
    return new_len


# -------------------------------------------------------------------- accept
def accept_workspace_bytes(B, n, V, dtype_code) -> int:
    return lib().eagle_accept_workspace_bytes(B, n, V, dtype_code)


SAMPLE_WITH_REPLACEMENT, SAMPLE_WITHOUT_REPLACEMENT = 0, 1


def accept_into(target_logits, tokens, parents, draft_row, depth, uniforms, draft_logits, draft_lse,
                accepted_len, path, bonus, ws, without_replacement: bool = False):
    B, n1, V = target_logits.shape
    n = n1 - 1
    R = draft_logits.shape[1] if draft_logits is not None else 0
    ddt = _dtype_code(draft_logits) if draft_logits is not None else 0
    rule = SAMPLE_WITHOUT_REPLACEMENT if without_replacement else SAMPLE_WITH_REPLACEMENT
    _check(lib().eagle_accept_with_rule(_ptr(target_logits), _dtype_code(target_logits), _ptr(draft_logits), ddt,
                                        _ptr(draft_lse), R, _ptr(tokens), _ptr(parents), _ptr(draft_row),
                                        _ptr(uniforms), rule, B, n, V, depth, _ptr(accepted_len), _ptr(path),
                                        _ptr(bonus), _ptr(ws), ws.numel(), _stream(target_logits.device)),
           "eagle_accept_with_rule")


def accept(target_logits, tokens, parents, draft_row, depth: int, uniforms=None, draft_logits=None,
           draft_lse=None, without_replacement: bool = False):
    """-> (accepted_len [B] int32, path [B][depth] int32, bonus [B] int32).  without_replacement: after a
    sampled child is rejected its token leaves the draft distribution (q renormalised)."""
    _need_cuda(target_logits, tokens, parents, draft_row, uniforms, draft_logits, draft_lse)
    B, n1, V = target_logits.shape
    dev = target_logits.device
    acc = torch.empty(B, dtype=torch.int32, device=dev)
    path = torch.empty(B, depth, dtype=torch.int32, device=dev)
    bonus = torch.empty(B, dtype=torch.int32, device=dev)
    ws = _workspace(accept_workspace_bytes(B, n1 - 1, V, _dtype_code(target_logits)), dev)
    accept_into(target_logits, tokens, parents, draft_row, depth, uniforms, draft_logits, draft_lse,
                acc, path, bonus, ws, without_replacement)
    return acc, path, bonus


# ---------------------------------------------------------------- one step
def step_in(draft_logits, target_logits, depth, k, m, q, k_cache, v_cache, prefix_len, k_tree, v_tree,
            uniforms=None, window: int = 0, scale: float = 0.0, without_replacement: bool = False,
            block_table=None) -> StepIn:
    """The C step's inputs: draft_logits [B][R][V] and target_logits [B][n+1][V] (f32 or bf16),
    q [B][n][Hq][D], caches [B][Hkv][Lmax][D], tree K/V [B][n][Hkv][D] (bf16), prefix_len [B] int32,
    uniforms [B][2][n+1] f32 or None (greedy)."""
    B, R, V = draft_logits.shape
    Hq, D = q.shape[2], q.shape[3]
    Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
    paged = (_ptr(block_table), k_cache.shape[2], block_table.shape[1], k_cache.shape[0]) if block_table is not None \
        else (None, 0, 0, 0)
    return StepIn(_ptr(draft_logits), _ptr(target_logits), _dtype_code(draft_logits), B, V, depth, k, m,
                  _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(prefix_len), 0 if block_table is not None else Lmax,
                  _ptr(k_tree), _ptr(v_tree), Hq, Hkv, D, window, scale, _ptr(uniforms),
                  SAMPLE_WITHOUT_REPLACEMENT if without_replacement else SAMPLE_WITH_REPLACEMENT, *paged)


def step_workspace_bytes(si: StepIn) -> int:
    return lib().eagle_verify_step_workspace_bytes(ctypes.byref(si))


def step_into(si: StepIn, tree: Tree, mask, pos, attn_out, accepted_len, path, bonus, ws: torch.Tensor,
              device) -> int:
    """Enqueue one whole step (build + fused mask, attention, acceptance) on the current stream."""
    so = StepOut(tree.struct(), _ptr(mask), _ptr(pos), _ptr(attn_out), _ptr(accepted_len), _ptr(path), _ptr(bonus))
    n_out = _c_i(0)
    _check(lib().eagle_verify_step(ctypes.byref(si), ctypes.byref(so), ctypes.byref(n_out), _ptr(ws), ws.numel(),
                                   _stream(device)), "eagle_verify_step")
    return n_out.value


def step_attention_status(si: StepIn, ws: torch.Tensor):
    """Read the attention's device status word from a step workspace (synchronises)."""
    off = lib().eagle_verify_step_attention_status_offset(ctypes.byref(si))
    check_attention_status(ws[off:])


# ------------------------------------------------------- KV-cache compaction
def kv_compact_into(k_tree, v_tree, path, accepted_len, prefix_len, k_cache, v_cache, new_prefix_len):
    """Append the accepted path's tree keys/values to the caches (in place); new lengths into new_prefix_len."""
    B, n, Hkv, D = k_tree.shape
    Lmax, depth = k_cache.shape[2], path.shape[1]
    _check(lib().eagle_kv_compact(_ptr(k_tree), _ptr(v_tree), _ptr(path), _ptr(accepted_len), _ptr(prefix_len),
                                  _ptr(k_cache), _ptr(v_cache), _ptr(new_prefix_len), B, n, Hkv, D, Lmax, depth,
                                  _stream(k_tree.device)), "eagle_kv_compact")


def kv_compact(k_tree, v_tree, path, accepted_len, prefix_len, k_cache, v_cache) -> torch.Tensor:
    """k_tree / v_tree [B][n][Hkv][D] bf16, path [B][depth], accepted_len [B], prefix_len [B] int32,
    caches [B][Hkv][Lmax][D] bf16 (updated in place) -> new prefix lengths [B] int32."""
    _need_cuda(k_tree, v_tree, path, accepted_len, prefix_len, k_cache, v_cache)
    new_len = torch.empty_like(prefix_len)
    kv_compact_into(k_tree, v_tree, path, accepted_len, prefix_len, k_cache, v_cache, new_len)
    return new_len


# ---------------------------------------------------- tree grown per level
class TreeGrower:
    """The build one level at a time: begin(root rows [B][V]) and level(rows [B][k][V], level) each return the
    new frontier (tokens [B][k], parent slots [B][k]); gains() the last level's per-sequence gain [B] (device,
    float64); finish(m, levels) returns the Tree over the first `levels` levels (equal to tree_build of that
    depth on the same rows)."""

    def __init__(self, B: int, V: int, depth: int, k: int, dtype: torch.dtype, device):
        self.B, self.V, self.depth, self.k = B, V, depth, k
        self.dt = F32 if dtype == torch.float32 else BF16
        self.device = torch.device(device)
        nb = lib().eagle_tree_grow_state_bytes(B, V, self.dt, depth, k)
        self.state = _workspace(nb, self.device)
        self.ftok = torch.empty(B, k, dtype=torch.int32, device=self.device)
        self.fpar = torch.empty(B, k, dtype=torch.int32, device=self.device)
        self.gain = torch.empty(B, dtype=torch.float64, device=self.device)
        self.flogv = torch.empty(B, k, dtype=torch.float64, device=self.device)

    def begin(self, root_logits: torch.Tensor):
        _check(lib().eagle_tree_grow_begin(_ptr(root_logits), self.dt, self.B, self.V, self.depth, self.k,
                                           _ptr(self.state), self.state.numel(), _ptr(self.ftok), _ptr(self.fpar),
                                           _stream(self.device)), "eagle_tree_grow_begin")
        return self.ftok, self.fpar

    def level(self, level_logits: torch.Tensor, level: int):
        _check(lib().eagle_tree_grow_level(_ptr(level_logits), self.dt, self.B, self.V, self.depth, self.k, level,
                                           _ptr(self.state), self.state.numel(), _ptr(self.ftok), _ptr(self.fpar),
                                           _stream(self.device)), "eagle_tree_grow_level")
        return self.ftok, self.fpar

    def level_width(self, level_logits: torch.Tensor, level: int, width: int):
        """A level drafted from the first `width` frontier slots only: level_logits [B][width][V]."""
        _check(lib().eagle_tree_grow_level_width(_ptr(level_logits), self.dt, self.B, self.V, self.depth, self.k,
                                                 level, width, _ptr(self.state), self.state.numel(), _ptr(self.ftok),
                                                 _ptr(self.fpar), _stream(self.device)), "eagle_tree_grow_level_width")
        return self.ftok, self.fpar

    def frontier_logv(self) -> torch.Tensor:
        """The last level's k best candidates per sequence, log V in rank order [B][k] (device, float64)."""
        _check(lib().eagle_tree_grow_frontier_logv(self.dt, self.B, self.V, self.depth, self.k, _ptr(self.state),
                                                   self.state.numel(), _ptr(self.flogv), _stream(self.device)),
               "eagle_tree_grow_frontier_logv")
        return self.flogv

    def finish_widths(self, widths) -> Tree:
        """The tree keeping the widths[l-1] best candidates of each level l drafted."""
        levels = len(widths)
        w = (ctypes.c_int * levels)(*[int(x) for x in widths])
        R = 1 + (self.depth - 1) * self.k
        tree = alloc_tree(self.B, R, levels, self.k, max(1, sum(int(x) for x in widths)), self.device)
        st = tree.struct()
        n_out = _c_i(0)
        _check(lib().eagle_tree_grow_finish_widths(self.dt, self.B, self.V, self.depth, self.k, levels, w,
                                                   _ptr(self.state), self.state.numel(), ctypes.byref(st),
                                                   ctypes.byref(n_out), _stream(self.device)),
               "eagle_tree_grow_finish_widths")
        return tree

    def gains(self) -> torch.Tensor:
        _check(lib().eagle_tree_grow_gains(self.dt, self.B, self.V, self.depth, self.k, _ptr(self.state),
                                           self.state.numel(), _ptr(self.gain), _stream(self.device)),
               "eagle_tree_grow_gains")
        return self.gain

    def finish(self, m: int, levels: Optional[int] = None) -> Tree:
        levels = self.depth if levels is None else levels
        R = 1 + (self.depth - 1) * self.k
        tree = alloc_tree(self.B, R, levels, self.k, m, self.device)
        st = tree.struct()
        n_out = _c_i(0)
        _check(lib().eagle_tree_grow_finish(self.dt, self.B, self.V, self.depth, self.k, levels, m,
                                            _ptr(self.state), self.state.numel(), ctypes.byref(st),
                                            ctypes.byref(n_out), _stream(self.device)), "eagle_tree_grow_finish")
        return tree


# --------------------------------------------------------------- static tree
def _template(parents, ranks):
    p = (ctypes.c_int32 * len(parents))(*[int(v) for v in parents])
    r = (ctypes.c_int32 * len(ranks))(*[int(v) for v in ranks])
    if len(parents) != len(ranks):
        raise EagleError("static tree: parents and ranks differ in length")
    return p, r


def static_template_from_paths(paths):
    """A static tree written as rank paths -> (parents, ranks) in template order.

    Each path lists sibling ranks from the root: (0,) is the root's likeliest child, (0, 1) that child's
    second likeliest, and so on.  Every prefix of a path must itself be a path.  Nodes are numbered by
    (depth, path), so a parent precedes its children and siblings follow their rank."""
    keyed = sorted({tuple(int(r) for r in p) for p in paths}, key=lambda p: (len(p), p))
    if not keyed or any(len(p) == 0 for p in keyed):
        raise EagleError("static tree: empty path")
    node_of = {p: i + 1 for i, p in enumerate(keyed)}
    parents, ranks = [], []
    for p in keyed:
        if len(p) > 1 and p[:-1] not in node_of:
            raise EagleError(f"static tree: path {p} has no parent path {p[:-1]}")
        parents.append(0 if len(p) == 1 else node_of[p[:-1]])
        ranks.append(p[-1])
    return parents, ranks


def static_tree_rows(parents, ranks) -> int:
    """Number of draft rows R the template needs (row 0 = root, then each node with a child)."""
    p, r = _template(parents, ranks)
    R = lib().eagle_static_tree_rows(p, r, len(parents))
    if R < 0:
        raise EagleError("static tree: invalid template")
    return R


def static_tree_build(draft_logits: torch.Tensor, parents, ranks) -> Tree:
    """EAGLE-1 fixed tree: draft_logits [B][R][V] (R = static_tree_rows), template parents/ranks
    (host sequences, node i+1 at index i) -> Tree with n = len(parents) nodes in template order."""
    _need_cuda(draft_logits)
    B, R, V = draft_logits.shape
    n = len(parents)
    p, r = _template(parents, ranks)
    dev = draft_logits.device
    dt = _dtype_code(draft_logits)
    i32 = dict(dtype=torch.int32, device=dev)
    tree = Tree(tokens=torch.empty(B, n, **i32), parents=torch.empty(B, n, **i32), depth=torch.empty(B, n, **i32),
                logV=torch.empty(B, n, dtype=torch.float32, device=dev), gid=torch.empty(B, n, **i32),
                draft_row=torch.empty(B, n + 1, **i32), row_lse=torch.empty(B, R, dtype=torch.float64, device=dev),
                n=n)
    nb = lib().eagle_static_tree_workspace_bytes(B, V, dt, p, r, n)
    ws = _workspace(max(nb, 256), dev)
    st = tree.struct()
    _check(lib().eagle_static_tree_build(_ptr(draft_logits), dt, B, R, V, p, r, n, ctypes.byref(st), _ptr(ws),
                                         ws.numel(), _stream(dev)), "eagle_static_tree_build")
    return tree
