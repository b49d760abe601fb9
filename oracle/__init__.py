"""ctypes binding of the fp64 CPU oracle (``hs2_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg import this package; the product library never does.
The oracle is built with gcc (``build()``), independent of nvcc and of the
CUDA sources.

Inputs are raw stored bytes (numpy arrays of float32, uint16 bf16 bit
patterns, or uint8 E4M3 codes plus float32 scales), so the oracle sees exactly
the bytes the CUDA library sees.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hs2_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libhs2_oracle.so")

F32, BF16, E4M3 = 0, 1, 2
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc into ``oracle/libhs2_oracle.so``."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P, I, I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        lib.orc_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.orc_e4m3_value.restype = ctypes.c_double
        lib.orc_full_attn_select.argtypes = [P, I, I, I, P, P, P, P, I, I, I, P, P, I, I, I, I, I64,
                                             P, P, P, P, P]
        lib.orc_full_attn_select.restype = I
        lib.orc_sparse_attn.argtypes = [P, I, I, I, P, P, P, P, I, I, I, P, I, P]
        lib.orc_sparse_attn.restype = I
        lib.orc_e4m3_encode.argtypes = [ctypes.c_double]
        lib.orc_e4m3_encode.restype = ctypes.c_uint8
        lib.orc_bf16_encode.argtypes = [ctypes.c_double]
        lib.orc_bf16_encode.restype = ctypes.c_uint16
        lib.orc_e4m3_row.argtypes = [P, I, P, P]
        lib.orc_e4m3_row.restype = None
        lib.orc_kv_bridge.argtypes = [P, I, I, P, P, I, P, P]
        lib.orc_kv_bridge.restype = I
        lib.orc_select_blocks.argtypes = [P, I64, I, I, I, P, I, I, I, P]
        lib.orc_select_blocks.restype = I
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


_STORE = {F32: np.float32, BF16: np.uint16, E4M3: np.uint8}


def e4m3_value(code: int) -> float:
    """Exact value of one E4M3 code (NaN for the two NaN codes)."""
    return _load().orc_e4m3_value(code)


def full_attn_select(q, q_dtype, k, v, kv_dtype, seq_lens, page_table=None, page_size=None,
                     window=128, k_global=1024, k_scale=None, v_scale=None):
    """Full-attention layer + token selection for a batch.

    q: [B, Hq, d] stored elements; k, v: [num_slots, Hkv, d] stored elements;
    seq_lens: [B]; page_table: [B, max_pages] or None (contiguous, each sequence
    owns ``page_size`` consecutive slots).  Returns a dict with ``out``
    [B,Hq,d] f64, ``lse`` [B,Hq], ``score`` [B,Hkv,t_cap] (NaN beyond T_b),
    ``idx`` [B,Hkv,window+k_global] int32 slots (-1 pad) and ``n_sel`` [B,Hkv].
    """
    lib = _load()
    q = _c(q, _STORE[q_dtype])
    k = _c(k, _STORE[kv_dtype])
    v = _c(v, _STORE[kv_dtype])
    B, Hq, d = q.shape
    Hkv = k.shape[1]
    assert k.shape[2] == d and Hq % Hkv == 0
    seq_lens = _c(seq_lens, np.int32)
    if page_table is not None:
        page_table = _c(page_table, np.int32)
        max_pages = page_table.shape[1]
    else:
        max_pages = 1
    if page_size is None:
        assert page_table is None
        page_size = k.shape[0] // B
    t_cap = int(seq_lens.max()) if len(seq_lens) else 0
    if kv_dtype == E4M3:
        k_scale = _c(k_scale, np.float32)
        v_scale = _c(v_scale, np.float32)
    out = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    score = np.full((B, Hkv, max(t_cap, 1)), np.nan)
    L = window + k_global
    idx = np.full((B, Hkv, L), -1, np.int32)
    n_sel = np.zeros((B, Hkv), np.int32)
    rc = lib.orc_full_attn_select(_ptr(q), q_dtype, B, Hq, _ptr(k), _ptr(k_scale), _ptr(v),
                                  _ptr(v_scale), kv_dtype, Hkv, d, _ptr(seq_lens),
                                  _ptr(page_table), max_pages, page_size, window, k_global,
                                  max(t_cap, 1), _ptr(out), _ptr(lse), _ptr(score), _ptr(idx),
                                  _ptr(n_sel))
    if rc != 0:
        raise MemoryError("oracle allocation failed")
    return {"out": out, "lse": lse, "score": score, "idx": idx, "n_sel": n_sel}


def sparse_attn(q, q_dtype, k, v, kv_dtype, idx, k_scale=None, v_scale=None):
    """Sparse layer for a batch: softmax over the slots listed in ``idx``
    [B, Hkv, L] (-1 entries ignored).  Returns out [B, Hq, d] float64."""
    lib = _load()
    q = _c(q, _STORE[q_dtype])
    k = _c(k, _STORE[kv_dtype])
    v = _c(v, _STORE[kv_dtype])
    idx = _c(idx, np.int32)
    B, Hq, d = q.shape
    Hkv = k.shape[1]
    if kv_dtype == E4M3:
        k_scale = _c(k_scale, np.float32)
        v_scale = _c(v_scale, np.float32)
    out = np.zeros((B, Hq, d))
    rc = lib.orc_sparse_attn(_ptr(q), q_dtype, B, Hq, _ptr(k), _ptr(k_scale), _ptr(v),
                             _ptr(v_scale), kv_dtype, Hkv, d, _ptr(idx), idx.shape[2], _ptr(out))
    if rc != 0:
        raise MemoryError("oracle allocation failed")
    return out


def e4m3_encode(x: float) -> int:
    """The E4M3 code nearest to x (ties to even), saturated at +-448."""
    return int(_load().orc_e4m3_encode(float(x)))


def bf16_encode(x: float) -> int:
    """The bf16 bit pattern nearest to x (ties to even)."""
    return int(_load().orc_bf16_encode(float(x)))


def e4m3_row(x):
    """One row of values -> (uint8 E4M3 codes, fp32 scale = max|x| / 448)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    codes = np.zeros(x.shape[-1], np.uint8)
    scale = np.zeros(1, np.float32)
    _load().orc_e4m3_row(_ptr(x), x.shape[-1], _ptr(codes), _ptr(scale))
    return codes, float(scale[0])


def kv_bridge(h, wk, wv):
    """KV Bridging projections of one decode step: h [B, d_model] and
    wk / wv [d_model, n] as bf16 bit patterns -> (k, v) float64 [B, n]."""
    h = _c(h, np.uint16)
    wk, wv = _c(wk, np.uint16), _c(wv, np.uint16)
    B, dm = h.shape
    n = wk.shape[1]
    assert wk.shape == (dm, n) and wv.shape == (dm, n)
    k = np.zeros((B, n), np.float64)
    v = np.zeros((B, n), np.float64)
    rc = _load().orc_kv_bridge(_ptr(h), B, dm, _ptr(wk), _ptr(wv), n, _ptr(k), _ptr(v))
    assert rc == 0
    return k, v


def select_blocks(score, T, window, k_global, block):
    """Block-level selection (first-generation HySparse) over one score row:
    the taken positions, ascending (window included)."""
    score = np.ascontiguousarray(np.asarray(score, np.float64)[:T])
    idx = np.full(window + k_global, -1, np.int32)
    n = _load().orc_select_blocks(_ptr(score), int(T), window, k_global, block, None, 1, max(int(T), 1), 0,
                                  _ptr(idx))
    if n < 0:
        raise ValueError("block size must divide k_global")
    return idx[:n].copy()


def full_attn_select_blocks(q, q_dtype, k, v, kv_dtype, seq_lens, page_table=None, page_size=None,
                            window=128, k_global=1024, block=64, k_scale=None, v_scale=None):
    """The full layer with block-level instead of token-level selection: the
    same attention output and group scores, and ``idx`` [B, Hkv, window +
    k_global] slots of the taken blocks' positions plus the window."""
    r = full_attn_select(q, q_dtype, k, v, kv_dtype, seq_lens, page_table, page_size, window, k_global,
                         k_scale, v_scale)
    seq_lens = _c(seq_lens, np.int32)
    B, Hkv = r["idx"].shape[:2]
    if page_table is not None:
        page_table = _c(page_table, np.int32)
        max_pages = page_table.shape[1]
    else:
        max_pages = 1
        page_size = k.shape[0] // B if page_size is None else page_size
    idx = np.full((B, Hkv, window + k_global), -1, np.int32)
    n_sel = np.zeros((B, Hkv), np.int32)
    for b in range(B):
        T = int(seq_lens[b])
        for h in range(Hkv):
            row = np.ascontiguousarray(r["score"][b, h, :max(T, 1)])
            out = idx[b, h]
            n = _load().orc_select_blocks(_ptr(row), T, window, k_global, block, _ptr(page_table), max_pages,
                                          page_size, b, out.ctypes.data_as(ctypes.c_void_p))
            if n < 0:
                raise ValueError("block size must divide k_global")
            n_sel[b, h] = n
    r["idx"], r["n_sel"] = idx, n_sel
    return r
