"""Thin ctypes binding of ``libhs2.so`` (include/hs2.h) over torch tensors.

Argument marshalling only: torch provides device memory and the current
stream; every step of the Hybrid-Block path runs in the library's CUDA
kernels.  If the library is missing or fails to load, every call raises --
there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhs2.so")

HS2_F32, HS2_BF16, HS2_E4M3 = 0, 1, 2
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT = range(6)

_DTYPE = {torch.float32: HS2_F32, torch.bfloat16: HS2_BF16, torch.uint8: HS2_E4M3,
          torch.float8_e4m3fn: HS2_E4M3}


class Cache(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("dtype", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("num_slots", ctypes.c_int64)]


class Heads(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("batch", ctypes.c_int32),
                ("num_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32)]


class HS2Error(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"hs2 error {code}: {msg}")
        self.code = code


_lib = None
EXPORTS = ["hs2_full_attn_select_workspace", "hs2_full_attn_select", "hs2_full_attn_select_marked",
           "hs2_full_attn_select_blocks", "hs2_full_attn_select_fused",
           "hs2_full_attn_select_static", "hs2_full_attn_select_static_status", "hs2_selftest_bounded_wait_static",
           "hs2_sparse_attn",
           "hs2_workspace_status", "hs2_selftest_bounded_wait", "hs2_selftest_grid_barrier",
           "hs2_kv_bridge_workspace", "hs2_kv_bridge_append",
           "hs2_copy_peak", "hs2_last_error", "hs2_version"]


def lib():
    """The loaded library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m long_context_decode_full_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        L.hs2_full_attn_select_workspace.argtypes = [I32, I32, I32, I32, I64]
        L.hs2_full_attn_select_workspace.restype = SZ
        L.hs2_full_attn_select.argtypes = [ctypes.POINTER(Heads), ctypes.POINTER(Cache), ctypes.POINTER(Cache),
                                           P, P, I32, I32, I32, ctypes.POINTER(Heads), P, P, SZ, P]
        L.hs2_full_attn_select.restype = ctypes.c_int
        L.hs2_full_attn_select_marked.argtypes = L.hs2_full_attn_select.argtypes + [P]
        L.hs2_full_attn_select_marked.restype = ctypes.c_int
        L.hs2_full_attn_select_fused.argtypes = L.hs2_full_attn_select.argtypes
        L.hs2_full_attn_select_fused.restype = ctypes.c_int
        L.hs2_full_attn_select_blocks.argtypes = [ctypes.POINTER(Heads), ctypes.POINTER(Cache), ctypes.POINTER(Cache),
                                                  P, P, I32, I32, I32, I32, ctypes.POINTER(Heads), P, P, SZ, P]
        L.hs2_full_attn_select_blocks.restype = ctypes.c_int
        L.hs2_full_attn_select_static.argtypes = [ctypes.POINTER(Heads), ctypes.POINTER(Cache),
                                                  ctypes.POINTER(Cache), P, P, I32, I32, I32,
                                                  ctypes.POINTER(Heads), P, P]
        L.hs2_full_attn_select_static.restype = ctypes.c_int
        L.hs2_full_attn_select_static_status.argtypes = [P]
        L.hs2_full_attn_select_static_status.restype = ctypes.c_int
        L.hs2_selftest_bounded_wait_static.argtypes = [P]
        L.hs2_selftest_bounded_wait_static.restype = ctypes.c_int
        L.hs2_sparse_attn.argtypes = [ctypes.POINTER(Heads), ctypes.POINTER(Cache), ctypes.POINTER(Cache), P, I32,
                                      ctypes.POINTER(Heads), P]
        L.hs2_sparse_attn.restype = ctypes.c_int
        L.hs2_workspace_status.argtypes = [P, SZ, P]
        L.hs2_workspace_status.restype = ctypes.c_int
        L.hs2_kv_bridge_workspace.argtypes = [I32, I32, I32, I32]
        L.hs2_kv_bridge_workspace.restype = SZ
        L.hs2_kv_bridge_append.argtypes = [P, I32, I32, P, P, P, P, I32, ctypes.POINTER(Cache),
                                           ctypes.POINTER(Cache), P, SZ, P]
        L.hs2_kv_bridge_append.restype = ctypes.c_int
        L.hs2_selftest_bounded_wait.argtypes = [P, SZ, P]
        L.hs2_selftest_bounded_wait.restype = ctypes.c_int
        L.hs2_selftest_grid_barrier.argtypes = [P, SZ, P]
        L.hs2_selftest_grid_barrier.restype = ctypes.c_int
        L.hs2_copy_peak.argtypes = [P, P, SZ, P]
        L.hs2_copy_peak.restype = ctypes.c_int
        L.hs2_last_error.argtypes = []
        L.hs2_last_error.restype = ctypes.c_char_p
        L.hs2_version.argtypes = []
        L.hs2_version.restype = ctypes.c_int
        _lib = L
    return _lib


def _check(rc: int):
    if rc != OK:
        raise HS2Error(rc, lib().hs2_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(name, t, dtypes, dim=None, shape=None):
    """The C ABI takes bare pointers: check what they cannot carry (element
    type, rank, shape, contiguity, a CUDA device) before the call."""
    if t is None:
        return
    dtypes = dtypes if isinstance(dtypes, tuple) else (dtypes,)
    if t.dtype not in dtypes:
        raise HS2Error(ERR_INVALID_ARG, f"{name}: dtype {t.dtype}, expected {' or '.join(map(str, dtypes))}")
    if dim is not None and t.dim() != dim:
        raise HS2Error(ERR_INVALID_ARG, f"{name}: {t.dim()} dimensions, expected {dim}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise HS2Error(ERR_INVALID_ARG, f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise HS2Error(ERR_INVALID_ARG, f"{name}: not contiguous")


def _need_cuda(**tensors):
    """Checked after every element type and shape, so a type error is
    reported as such whatever the device."""
    for name, t in tensors.items():
        if t is not None and not t.is_cuda:
            raise HS2Error(ERR_INVALID_ARG, f"{name}: not on a CUDA device")


def _need_lens(seq_lens, page_table, B):
    _need("seq_lens", seq_lens, torch.int32, shape=(B,))
    if page_table is not None:
        _need("page_table", page_table, torch.int32, dim=2)
        if page_table.shape[0] != B:
            raise HS2Error(ERR_INVALID_ARG, f"page_table: {page_table.shape[0]} rows for batch {B}")


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def cache_desc(kv: torch.Tensor, scale: Optional[torch.Tensor], page_size: int) -> Cache:
    assert kv.dim() == 3 and kv.is_contiguous(), "cache must be a contiguous [num_slots, Hkv, d] tensor"
    return Cache(kv.data_ptr(), None if scale is None else scale.data_ptr(), _DTYPE[kv.dtype], kv.shape[1],
                 kv.shape[2], page_size, kv.shape[0])


def heads_desc(x: torch.Tensor) -> Heads:
    assert x.dim() == 3 and x.is_contiguous(), "q/out must be a contiguous [B, H, d] tensor"
    return Heads(x.data_ptr(), _DTYPE[x.dtype], x.shape[0], x.shape[1], x.shape[2])


def full_workspace_bytes(batch: int, num_kv_heads: int, group: int, head_dim: int, t_cap: int) -> int:
    return int(lib().hs2_full_attn_select_workspace(batch, num_kv_heads, group, head_dim, t_cap))


def alloc_workspace(batch, num_kv_heads, group, head_dim, t_cap, device="cuda") -> torch.Tensor:
    n = full_workspace_bytes(batch, num_kv_heads, group, head_dim, t_cap)
    if n == 0:
        raise HS2Error(ERR_INVALID_ARG, "invalid workspace shape")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def full_attn_select(q, k, v, seq_lens, page_table=None, page_size=None, window=128, k_global=1024,
                     k_scale=None, v_scale=None, out=None, idx_out=None, workspace=None, stream=None,
                     mark_event=None, fused=False):
    """Full-attention layer + token selection.  Returns (out, idx) where idx
    holds selected slots [B, Hkv, window + k_global], ascending, -1 padded.
    ``mark_event`` (a recorded-once torch.cuda.Event) is recorded between the
    attention kernel and the selection kernels.  ``fused`` runs the attention
    and the selection's score pass in one cooperative persistent kernel
    (hs2_full_attn_select_fused; no mark event)."""
    B, Hq, d = q.shape
    Hkv = k.shape[1]
    _need_lens(seq_lens, page_table, B)
    _need("idx_out", idx_out, torch.int32, shape=(B, Hkv, window + k_global))
    _need_cuda(q=q, k=k, v=v, seq_lens=seq_lens, page_table=page_table, idx_out=idx_out)
    if page_size is None:
        assert page_table is None, "page_size is required with a page table"
        page_size = k.shape[0] // B
    max_pages = 1 if page_table is None else page_table.shape[1]
    t_cap = page_size * max_pages
    if out is None:
        out = torch.empty_like(q)
    if idx_out is None:
        idx_out = torch.empty(B, Hkv, window + k_global, dtype=torch.int32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(B, Hkv, Hq // Hkv, d, t_cap, q.device)
    kc, vc = cache_desc(k, k_scale, page_size), cache_desc(v, v_scale, page_size)
    qd, od = heads_desc(q), heads_desc(out)
    if fused:
        assert mark_event is None, "the fused call records no mark event"
        _check(lib().hs2_full_attn_select_fused(ctypes.byref(qd), ctypes.byref(kc), ctypes.byref(vc),
                                                _ptr(seq_lens), _ptr(page_table), max_pages, window, k_global,
                                                ctypes.byref(od), _ptr(idx_out), _ptr(workspace), workspace.numel(),
                                                _stream(stream)))
        return out, idx_out
    ev = None if mark_event is None else ctypes.c_void_p(mark_event.cuda_event)
    _check(lib().hs2_full_attn_select_marked(ctypes.byref(qd), ctypes.byref(kc), ctypes.byref(vc),
                                             _ptr(seq_lens), _ptr(page_table), max_pages, window, k_global,
                                             ctypes.byref(od), _ptr(idx_out), _ptr(workspace), workspace.numel(),
                                             _stream(stream), ev))
    return out, idx_out


def full_attn_select_blocks(q, k, v, seq_lens, page_table=None, page_size=None, window=128, k_global=1024,
                            block=16, k_scale=None, v_scale=None, out=None, idx_out=None, workspace=None,
                            stream=None):
    """Full-attention layer + BLOCK-level selection (the first-generation
    comparator): the same attention output, and idx [B, Hkv, window + k_global]
    with the slots of the k_global / block best blocks' positions and the
    window, ascending, -1 padded."""
    B, Hq, d = q.shape
    Hkv = k.shape[1]
    _need_lens(seq_lens, page_table, B)
    _need("idx_out", idx_out, torch.int32, shape=(B, Hkv, window + k_global))
    _need_cuda(q=q, k=k, v=v, seq_lens=seq_lens, page_table=page_table, idx_out=idx_out)
    if page_size is None:
        assert page_table is None, "page_size is required with a page table"
        page_size = k.shape[0] // B
    max_pages = 1 if page_table is None else page_table.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if idx_out is None:
        idx_out = torch.empty(B, Hkv, window + k_global, dtype=torch.int32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(B, Hkv, Hq // Hkv, d, page_size * max_pages, q.device)
    kc, vc = cache_desc(k, k_scale, page_size), cache_desc(v, v_scale, page_size)
    qd, od = heads_desc(q), heads_desc(out)
    _check(lib().hs2_full_attn_select_blocks(ctypes.byref(qd), ctypes.byref(kc), ctypes.byref(vc), _ptr(seq_lens),
                                             _ptr(page_table), max_pages, window, k_global, block, ctypes.byref(od),
                                             _ptr(idx_out), _ptr(workspace), workspace.numel(), _stream(stream)))
    return out, idx_out


def full_attn_select_static(q, k, v, seq_lens, page_table=None, page_size=None, window=128, k_global=1024,
                            k_scale=None, v_scale=None, out=None, idx_out=None, stream=None):
    """full_attn_select() without a workspace: the library's own fixed 32 MiB
    device scratch is used (for callers that may not allocate).  Calls that
    overlap on the GPU race on that scratch; static_status() reports an
    expired device wait of these calls."""
    B, Hq, d = q.shape
    Hkv = k.shape[1]
    _need_lens(seq_lens, page_table, B)
    _need("idx_out", idx_out, torch.int32, shape=(B, Hkv, window + k_global))
    _need_cuda(q=q, k=k, v=v, seq_lens=seq_lens, page_table=page_table, idx_out=idx_out)
    if page_size is None:
        assert page_table is None, "page_size is required with a page table"
        page_size = k.shape[0] // B
    max_pages = 1 if page_table is None else page_table.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if idx_out is None:
        idx_out = torch.empty(B, Hkv, window + k_global, dtype=torch.int32, device=q.device)
    kc, vc = cache_desc(k, k_scale, page_size), cache_desc(v, v_scale, page_size)
    qd, od = heads_desc(q), heads_desc(out)
    _check(lib().hs2_full_attn_select_static(ctypes.byref(qd), ctypes.byref(kc), ctypes.byref(vc),
                                             _ptr(seq_lens), _ptr(page_table), max_pages, window, k_global,
                                             ctypes.byref(od), _ptr(idx_out), _stream(stream)))
    return out, idx_out


def static_status(stream=None) -> int:
    """Synchronises the stream, returns and clears the sticky device error flag
    of full_attn_select_static() calls in the current CUDA context."""
    return int(lib().hs2_full_attn_select_static_status(_stream(stream)))


def sparse_attn(q_l, k, v, idx, k_scale=None, v_scale=None, page_size=1, out=None, stream=None):
    """Sparse-attention layer over the rows listed in ``idx`` (slots)."""
    _need("idx", idx, torch.int32, dim=3)
    _need_cuda(q=q_l, k=k, v=v, idx=idx)
    if out is None:
        out = torch.empty_like(q_l)
    kc, vc = cache_desc(k, k_scale, page_size), cache_desc(v, v_scale, page_size)
    qd, od = heads_desc(q_l), heads_desc(out)
    _check(lib().hs2_sparse_attn(ctypes.byref(qd), ctypes.byref(kc), ctypes.byref(vc), _ptr(idx), idx.shape[-1],
                                 ctypes.byref(od), _stream(stream)))
    return out


def hybrid_block_step(q_full, q_sparse: Sequence[torch.Tensor], k, v, seq_lens, page_table=None, page_size=None,
                      window=128, k_global=1024, k_scale=None, v_scale=None, outs=None, idx_out=None,
                      workspace=None, stream=None, fused=False):
    """One decode step of a Hybrid Block: the full layer (attention + token
    selection) then every sparse layer with its own query, all reusing the
    same cache and the same index list.  Returns (outs, idx).  ``fused``
    selects the fused full-layer call (see full_attn_select)."""
    outs = outs if outs is not None else [None] * (1 + len(q_sparse))
    o0, idx = full_attn_select(q_full, k, v, seq_lens, page_table, page_size, window, k_global, k_scale, v_scale,
                               outs[0], idx_out, workspace, stream, fused=fused)
    ps = page_size if page_size is not None else k.shape[0] // q_full.shape[0]
    res = [o0]
    for i, q in enumerate(q_sparse):
        res.append(sparse_attn(q, k, v, idx, k_scale, v_scale, ps, outs[1 + i], stream))
    return res, idx


def workspace_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronises the stream, returns and clears the sticky device error flag."""
    return int(lib().hs2_workspace_status(_ptr(workspace), workspace.numel(), _stream(stream)))


def kv_bridge_workspace_bytes(batch: int, d_model: int, num_kv_heads: int, head_dim: int) -> int:
    return int(lib().hs2_kv_bridge_workspace(batch, d_model, num_kv_heads, head_dim))


def kv_bridge_append(hidden, w_k, w_v, k, v, seq_lens, page_table=None, page_size=None, k_scale=None, v_scale=None,
                     workspace=None, stream=None):
    """KV Bridging append: writes the new token's K/V rows (hidden [B, d_model]
    bf16 times w_k / w_v [d_model, Hkv * d] bf16) at position seq_lens[b] - 1
    of the caches k / v (and the E4M3 scales).  A workspace passed in must
    have been zero-filled once (see kv_bridge_workspace_bytes)."""
    _need("hidden", hidden, torch.bfloat16, dim=2)
    B, dm = hidden.shape
    if k.dim() != 3:
        raise HS2Error(ERR_INVALID_ARG, "k: expected a [num_slots, Hkv, d] cache")
    N = k.shape[1] * k.shape[2]
    _need("w_k", w_k, torch.bfloat16, shape=(dm, N))
    _need("w_v", w_v, torch.bfloat16, shape=(dm, N))
    _need_lens(seq_lens, page_table, B)
    _need("k_scale", k_scale, torch.float32, shape=k.shape[:2])
    _need("v_scale", v_scale, torch.float32, shape=v.shape[:2])
    _need_cuda(hidden=hidden, w_k=w_k, w_v=w_v, k=k, v=v, seq_lens=seq_lens, page_table=page_table,
               k_scale=k_scale, v_scale=v_scale)
    if page_size is None:
        assert page_table is None, "page_size is required with a page table"
        page_size = k.shape[0] // B
    max_pages = 1 if page_table is None else page_table.shape[1]
    if workspace is None:
        n = kv_bridge_workspace_bytes(B, dm, k.shape[1], k.shape[2])
        if n == 0:
            raise HS2Error(ERR_INVALID_ARG, "invalid KV bridge shape")
        workspace = torch.zeros(n, dtype=torch.uint8, device=hidden.device)
    kc, vc = cache_desc(k, k_scale, page_size), cache_desc(v, v_scale, page_size)
    _check(lib().hs2_kv_bridge_append(_ptr(hidden), B, dm, _ptr(w_k), _ptr(w_v), _ptr(seq_lens), _ptr(page_table),
                                      max_pages, ctypes.byref(kc), ctypes.byref(vc), _ptr(workspace),
                                      workspace.numel(), _stream(stream)))


def selftest_bounded_wait(workspace: torch.Tensor, stream=None):
    """Makes one bounded device wait expire on purpose (it sets the sticky flag)."""
    _check(lib().hs2_selftest_bounded_wait(_ptr(workspace), workspace.numel(), _stream(stream)))


def selftest_grid_barrier(workspace: torch.Tensor, stream=None):
    """Makes the fused call's grid barrier expire on purpose (two CTAs wait for
    a third that never comes; it sets the sticky flag)."""
    _check(lib().hs2_selftest_grid_barrier(_ptr(workspace), workspace.numel(), _stream(stream)))


def copy_peak(dst: torch.Tensor, src: torch.Tensor, stream=None):
    _check(lib().hs2_copy_peak(_ptr(dst), _ptr(src), src.numel() * src.element_size(), _stream(stream)))


def version() -> int:
    return int(lib().hs2_version())


def last_error() -> str:
    return lib().hs2_last_error().decode()
