"""ctypes front end of the fp64 oracle (test infrastructure only)."""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import numpy as np

from .build import LIB, build

_lib = None

F16, BF16 = 0, 1


def library_path() -> str:
    return LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_decode.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, I,
                                      ctypes.c_double, I, P, P]
        lib.oracle_decode.restype = I
        lib.oracle_combine.argtypes = [P, P, I, ctypes.c_long, I, P, P]
        lib.oracle_combine.restype = I
        lib.oracle_f16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_f16_to_double.restype = ctypes.c_double
        lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_double.restype = ctypes.c_double
        _lib = lib
    return _lib


def _bits(x) -> np.ndarray:
    """16-bit storage of a torch fp16/bf16 tensor or a numpy uint16 array."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch
    assert x.dtype in (torch.float16, torch.bfloat16)
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def decode(q, k_cache, v_cache, block_table, cache_seqlens, *, Hkv: int,
           page_size: int, dtype: str, scale: float, causal: bool,
           max_pages_per_seq: Optional[int] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Exact attention in fp64.

    q [B, q_len, Hq, D]; k_cache/v_cache [num_pages, page_size, Hkv, D]
    (or [B, page_size, Hkv, D] when block_table is None); block_table
    [B, max_pages_per_seq] int32 or None; cache_seqlens [B] int32.
    Returns (out [B, q_len, Hq, D] float64, lse [B, Hq, q_len] float64).
    """
    lib = _load()
    qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
    B, q_len, Hq, D = qb.shape
    L = np.ascontiguousarray(np.asarray(cache_seqlens, dtype=np.int32))
    bt = None
    mpps = 1
    if block_table is not None:
        bt = np.ascontiguousarray(np.asarray(block_table, dtype=np.int32))
        mpps = bt.shape[1] if max_pages_per_seq is None else max_pages_per_seq
    out = np.empty((B, q_len, Hq, D), dtype=np.float64)
    lse = np.empty((B, Hq, q_len), dtype=np.float64)
    rc = lib.oracle_decode(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(bt), _ptr(L), B, q_len, Hq,
                           Hkv, D, page_size, mpps, BF16 if dtype == "bf16" else F16,
                           float(scale), int(bool(causal)), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_decode: bad shape arguments")
    return out, lse


def decode_varlen(q, cu_seqlens_q, k_cache, v_cache, block_table, cache_seqlens, *, Hkv: int,
                  page_size: int, dtype: str, scale: float, causal: bool) -> Tuple[np.ndarray, np.ndarray]:
    """Exact attention for rows with their own number of queries, in fp64.

    The packed-query layout of a varlen call: row b's queries are
    q[cu_seqlens_q[b] : cu_seqlens_q[b + 1]] ("MXFlashAttn 1.4.0",
    flash_attn_varlen_func; "MixedQuantSparseFlashMlaMetadata 算子解析",
    参数说明: cu_seqlens of B + 1 entries, starting at 0, non-decreasing).  Each
    row is the plain decode of decode() with its own q_len_b; with causal
    the row's queries are its last q_len_b cache entries (query t sees the
    first L_b - q_len_b + t + 1 keys).

    q [total_q, Hq, D]; caches and block_table as for decode().
    Returns (out [total_q, Hq, D] float64, lse [Hq, total_q] float64).
    """
    qb = _bits(q)
    total_q, Hq, D = qb.shape
    cu = np.asarray(cu_seqlens_q, dtype=np.int64)
    L = np.asarray(cache_seqlens, dtype=np.int32)
    if cu.ndim != 1 or cu[0] != 0 or cu[-1] != total_q or (np.diff(cu) < 0).any():
        raise ValueError("cu_seqlens_q: B + 1 non-decreasing offsets from 0 to total_q")
    out = np.zeros((total_q, Hq, D), dtype=np.float64)
    lse = np.zeros((Hq, total_q), dtype=np.float64)
    bt = None if block_table is None else np.asarray(block_table, dtype=np.int32)
    for b in range(cu.size - 1):
        q0, q1 = int(cu[b]), int(cu[b + 1])
        if q1 == q0:
            continue
        row_bt = None if bt is None else bt[b:b + 1]
        if bt is None:  # contiguous cache: row b only
            kc, vc = _bits(k_cache)[b:b + 1], _bits(v_cache)[b:b + 1]
        else:
            kc, vc = _bits(k_cache), _bits(v_cache)
        o, l = decode(qb[None, q0:q1], kc, vc, row_bt, L[b:b + 1], Hkv=Hkv, page_size=page_size,
                      dtype=dtype, scale=scale, causal=causal)
        out[q0:q1] = o[0]
        lse[:, q0:q1] = l[0]
    return out, lse


def append_kv(k_cache, v_cache, k_new, v_new, block_table, cache_seqlens, *, page_size: int):
    """Write each row's new tokens into copies of the caches; return the copies.

    The new keys and values that a decode call appends before attending
    ("Flash-Attention GQA 性能调优: pack_gqa 与 num_splits", the k / v arguments
    of flash_attn_with_kvcache next to cache_seqlens; "MXFlashAttn 1.4.0",
    能力矩阵: paged KV append).  Row b's new token t goes to logical position
    L_b + t of the row (L_b = cache_seqlens[b]): page
    block_table[b, (L_b + t) // page_size], slot (L_b + t) % page_size, or
    row b, slot L_b + t of a contiguous cache (block_table None).  The
    values are copied bit for bit.

    k_cache/v_cache as for decode(); k_new/v_new [B, q_len, Hkv, D].
    """
    kb, vb = _bits(k_cache).copy(), _bits(v_cache).copy()
    knb, vnb = _bits(k_new), _bits(v_new)
    B, q_len = knb.shape[0], knb.shape[1]
    L = np.asarray(cache_seqlens, dtype=np.int64)
    bt = None if block_table is None else np.asarray(block_table, dtype=np.int64)
    for b in range(B):
        for t in range(q_len):
            pos = int(L[b]) + t
            if bt is None:
                page, slot = b, pos
            else:
                page, slot = int(bt[b, pos // page_size]), pos % page_size
            kb[page, slot] = knb[b, t]
            vb[page, slot] = vnb[b, t]
    return kb, vb


def combine(o_part: np.ndarray, lse_part: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Exact LSE merge.  o_part [S, rows, D], lse_part [S, rows] (float64)."""
    lib = _load()
    o_part = np.ascontiguousarray(o_part, dtype=np.float64)
    lse_part = np.ascontiguousarray(lse_part, dtype=np.float64)
    S, rows, D = o_part.shape
    out = np.empty((rows, D), dtype=np.float64)
    lse = np.empty((rows,), dtype=np.float64)
    rc = lib.oracle_combine(_ptr(o_part), _ptr(lse_part), S, rows, D, _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_combine: bad shape arguments")
    return out, lse


def f16_to_double(bits: int) -> float:
    return _load().oracle_f16_to_double(bits)


def bf16_to_double(bits: int) -> float:
    return _load().oracle_bf16_to_double(bits)
