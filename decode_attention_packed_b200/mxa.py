"""Python binding of libmxa.so (the C ABI in include/mxa.h).

Argument marshalling only: every step of the decode path runs in the CUDA
kernels of libmxa.so.  Torch tensors supply device memory and the current
stream.  There is no fallback: if the library is missing this module raises
on import.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIBRARY = os.path.join(_HERE, "libmxa.so")

if not os.path.exists(LIBRARY):
    raise ImportError(f"libmxa.so is not built ({LIBRARY}); run "
                      "`python -m decode_attention_packed_b200.build`")

_lib = ctypes.CDLL(LIBRARY)

MXA_OK, MXA_ERR_INVALID_ARG, MXA_ERR_UNSUPPORTED, MXA_ERR_WORKSPACE, MXA_ERR_CUDA, MXA_ERR_TIMEOUT = range(6)
MXA_F16, MXA_BF16 = 0, 1
MXA_SCHED_UNIFORM, MXA_SCHED_BALANCED = 0, 1

EXPORTED = ("mxa_status_string", "mxa_should_pack_gqa", "mxa_num_splits_heuristic", "mxa_plan",
            "mxa_plan_balanced",
            "mxa_decode_fwd", "mxa_decode_fwd_with_plan", "mxa_combine", "mxa_device_error",
            "mxa_decode_fwd_noalloc", "mxa_decode_fwd_append", "mxa_decode_fwd_varlen",
            "mxa_decode_fwd_f32out", "mxa_decode_workspace_size")

SIZE_MAX = ctypes.c_size_t(-1).value


class mxa_decode_params_t(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("q_len", ctypes.c_int), ("Hq", ctypes.c_int),
                ("Hkv", ctypes.c_int), ("D", ctypes.c_int), ("num_pages", ctypes.c_int),
                ("page_size", ctypes.c_int), ("max_pages_per_seq", ctypes.c_int),
                ("max_seqlen_k", ctypes.c_int), ("dtype", ctypes.c_int)]


class mxa_plan_t(ctypes.Structure):
    _fields_ = [("num_splits", ctypes.c_int), ("schedule", ctypes.c_int), ("grid", ctypes.c_int),
                ("units", ctypes.c_int), ("rows_per_tile", ctypes.c_int),
                ("block_tokens", ctypes.c_int), ("ctas_per_sm", ctypes.c_int),
                ("sm_count", ctypes.c_int), ("needs_combine", ctypes.c_int),
                ("unit_cost", ctypes.c_int), ("workspace_bytes", ctypes.c_size_t)]

    def as_dict(self) -> dict:
        return {name: getattr(self, name) for name, _ in self._fields_}


_P = ctypes.c_void_p
_I = ctypes.c_int
_lib.mxa_status_string.argtypes = [_I]
_lib.mxa_status_string.restype = ctypes.c_char_p
_lib.mxa_should_pack_gqa.argtypes = [_I, _I, _I, _I]
_lib.mxa_should_pack_gqa.restype = _I
_lib.mxa_num_splits_heuristic.argtypes = [_I, _I, _I, _I, _I, _I, _I, ctypes.c_double]
_lib.mxa_num_splits_heuristic.restype = _I
_lib.mxa_plan.argtypes = [ctypes.POINTER(mxa_decode_params_t), _I, _I, ctypes.POINTER(mxa_plan_t)]
_lib.mxa_plan.restype = _I
_lib.mxa_plan_balanced.argtypes = [ctypes.POINTER(mxa_decode_params_t), _I, _I, ctypes.POINTER(mxa_plan_t)]
_lib.mxa_plan_balanced.restype = _I
_lib.mxa_decode_fwd.argtypes = [_P, _P, _P, _P, _P, ctypes.POINTER(mxa_decode_params_t),
                                ctypes.c_float, _I, _I, _P, ctypes.c_size_t, _P, _P, _P]
_lib.mxa_decode_fwd.restype = _I
_lib.mxa_decode_fwd_with_plan.argtypes = [_P, _P, _P, _P, _P, ctypes.POINTER(mxa_decode_params_t),
                                          ctypes.c_float, _I, ctypes.POINTER(mxa_plan_t), _P,
                                          ctypes.c_size_t, _P, _P, _P]
_lib.mxa_decode_fwd_with_plan.restype = _I
_lib.mxa_decode_fwd_f32out.argtypes = _lib.mxa_decode_fwd_with_plan.argtypes
_lib.mxa_decode_fwd_f32out.restype = _I
_lib.mxa_decode_workspace_size.argtypes = [ctypes.POINTER(mxa_decode_params_t), _I]
_lib.mxa_decode_workspace_size.restype = ctypes.c_size_t
_lib.mxa_decode_fwd_append.argtypes = [_P, _P, _P, _P, _P, _P, _P, ctypes.POINTER(mxa_decode_params_t),
                                       ctypes.c_float, _I, ctypes.POINTER(mxa_plan_t), _P, ctypes.c_size_t,
                                       _P, _P, _P]
_lib.mxa_decode_fwd_append.restype = _I
_lib.mxa_decode_fwd_varlen.argtypes = [_P, _P, _I, _P, _P, _P, _P, ctypes.POINTER(mxa_decode_params_t),
                                       ctypes.c_float, _I, ctypes.POINTER(mxa_plan_t), _P, ctypes.c_size_t,
                                       _P, _P, _P]
_lib.mxa_decode_fwd_varlen.restype = _I
_lib.mxa_decode_fwd_noalloc.argtypes = [_P, _P, _P, _P, _P, ctypes.POINTER(mxa_decode_params_t),
                                        ctypes.c_float, _I, _I, _P, _P, _P]
_lib.mxa_decode_fwd_noalloc.restype = _I
_lib.mxa_combine.argtypes = [_P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P]
_lib.mxa_combine.restype = _I
_lib.mxa_device_error.argtypes = [_I]
_lib.mxa_device_error.restype = _I


class MxaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {mxa_status_string(code)}")


def _check(code: int, where: str) -> None:
    if code != MXA_OK:
        raise MxaError(code, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


# --------------------------------------------------------------------------
# the C calls, same names
# --------------------------------------------------------------------------

def mxa_status_string(code: int) -> str:
    return _lib.mxa_status_string(code).decode()


def mxa_should_pack_gqa(varlen_q: int, seqlen_q: int, qhead_per_khead: int, block_m: int) -> int:
    return _lib.mxa_should_pack_gqa(varlen_q, seqlen_q, qhead_per_khead, block_m)


def mxa_num_splits_heuristic(tiles, sm_count, slots, num_n_blocks, max_splits, causal,
                             num_m_blocks, kv_head_bytes) -> int:
    return _lib.mxa_num_splits_heuristic(tiles, sm_count, slots, num_n_blocks, max_splits,
                                         int(causal), num_m_blocks, float(kv_head_bytes))


def mxa_plan(params: mxa_decode_params_t, num_splits: int = 0, sm_count: int = 0) -> mxa_plan_t:
    plan = mxa_plan_t()
    _check(_lib.mxa_plan(ctypes.byref(params), num_splits, sm_count, ctypes.byref(plan)), "mxa_plan")
    return plan


def mxa_plan_balanced(params: mxa_decode_params_t, grid: int, sm_count: int = 0) -> mxa_plan_t:
    plan = mxa_plan_t()
    _check(_lib.mxa_plan_balanced(ctypes.byref(params), grid, sm_count, ctypes.byref(plan)),
           "mxa_plan_balanced")
    return plan


def mxa_decode_fwd(q, k_cache, v_cache, block_table, cache_seqlens, params, scale, causal,
                   num_splits, workspace, out, lse, stream=None) -> None:
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.mxa_decode_fwd(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                               _ptr(cache_seqlens), ctypes.byref(params), float(scale), int(causal),
                               int(num_splits), _ptr(workspace), ws_bytes, _ptr(out), _ptr(lse),
                               _stream(stream)), "mxa_decode_fwd")


def mxa_decode_fwd_with_plan(q, k_cache, v_cache, block_table, cache_seqlens, params, scale, causal,
                             plan, workspace, out, lse, stream=None) -> None:
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.mxa_decode_fwd_with_plan(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                         _ptr(cache_seqlens), ctypes.byref(params), float(scale),
                                         int(causal), ctypes.byref(plan), _ptr(workspace), ws_bytes,
                                         _ptr(out), _ptr(lse), _stream(stream)),
           "mxa_decode_fwd_with_plan")


def mxa_decode_fwd_f32out(q, k_cache, v_cache, block_table, cache_seqlens, params, scale, causal,
                          plan, workspace, out, lse, stream=None) -> None:
    """As mxa_decode_fwd_with_plan with a float32 `out`: O before its rounding
    to the input type."""
    if out.dtype != torch.float32:
        raise TypeError("mxa_decode_fwd_f32out writes a float32 out")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.mxa_decode_fwd_f32out(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                      _ptr(cache_seqlens), ctypes.byref(params), float(scale),
                                      int(causal), ctypes.byref(plan), _ptr(workspace), ws_bytes,
                                      _ptr(out), _ptr(lse), _stream(stream)),
           "mxa_decode_fwd_f32out")


def mxa_decode_workspace_size(params: mxa_decode_params_t, num_splits: int = 0) -> int:
    """Workspace bytes of mxa_plan(params, num_splits); SIZE_MAX when refused."""
    return int(_lib.mxa_decode_workspace_size(ctypes.byref(params), int(num_splits)))


def mxa_decode_fwd_append(q, k_cache, v_cache, k_new, v_new, block_table, cache_seqlens, params, scale,
                          causal, plan, workspace, out, lse, stream=None) -> None:
    """Write k_new / v_new [B, q_len, Hkv, D] at positions cache_seqlens[b] + t of
    the cache, then decode over cache_seqlens[b] + q_len keys (see mxa.h)."""
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.mxa_decode_fwd_append(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_new), _ptr(v_new),
                                      _ptr(block_table), _ptr(cache_seqlens), ctypes.byref(params),
                                      float(scale), int(causal), ctypes.byref(plan), _ptr(workspace), ws_bytes,
                                      _ptr(out), _ptr(lse), _stream(stream)), "mxa_decode_fwd_append")


def mxa_decode_fwd_varlen(q, cu_seqlens_q, k_cache, v_cache, block_table, cache_seqlens, params, scale,
                          causal, plan, workspace, out, lse, stream=None) -> None:
    """Decode rows with their own query counts: q [total_q, Hq, D], row b's
    queries at cu_seqlens_q[b] .. cu_seqlens_q[b + 1] - 1; params.q_len bounds
    every count.  out [total_q, Hq, D], lse [Hq, total_q] (see mxa.h)."""
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.mxa_decode_fwd_varlen(_ptr(q), _ptr(cu_seqlens_q), int(q.shape[0]), _ptr(k_cache),
                                      _ptr(v_cache), _ptr(block_table), _ptr(cache_seqlens), ctypes.byref(params),
                                      float(scale), int(causal), ctypes.byref(plan), _ptr(workspace), ws_bytes,
                                      _ptr(out), _ptr(lse), _stream(stream)), "mxa_decode_fwd_varlen")


def mxa_decode_fwd_noalloc(q, k_cache, v_cache, block_table, cache_seqlens, params, scale, causal,
                           num_splits, out, lse, stream=None) -> None:
    """Decode with the library's fixed 16 MiB scratch array instead of a
    workspace, for callers that cannot allocate device memory (see
    include/mxa.h: first call per device before any stream capture; calls
    that overlap on the GPU race on the shared array)."""
    _check(_lib.mxa_decode_fwd_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                       _ptr(cache_seqlens), ctypes.byref(params), float(scale),
                                       int(causal), int(num_splits), _ptr(out), _ptr(lse),
                                       _stream(stream)), "mxa_decode_fwd_noalloc")


def mxa_combine(o_part, lse_part, out, lse=None, stream=None) -> None:
    """o_part [S, B, q_len, Hq, D] fp32, lse_part [S, B, Hq, q_len] fp32 -> out [B, q_len, Hq, D]."""
    S, B, q_len, Hq, D = o_part.shape
    dtype = MXA_BF16 if out.dtype == torch.bfloat16 else MXA_F16
    _check(_lib.mxa_combine(_ptr(o_part), _ptr(lse_part), S, B, q_len, Hq, D, dtype, _ptr(out),
                            _ptr(lse), _stream(stream)), "mxa_combine")


def mxa_device_error(reset: bool = False) -> int:
    return _lib.mxa_device_error(int(reset))


# --------------------------------------------------------------------------
# convenience: shapes from tensors
# --------------------------------------------------------------------------

def params_for(q: torch.Tensor, k_cache: torch.Tensor, block_table: Optional[torch.Tensor],
               max_seqlen_k: Optional[int] = None) -> mxa_decode_params_t:
    """Problem shape from the tensors.  Without `max_seqlen_k` the bound is
    the cache capacity of a row (no device read)."""
    B, q_len, Hq, D = q.shape
    num_pages, page_size, Hkv, Dk = k_cache.shape
    assert Dk == D
    if block_table is None:
        mpps = 1
        cap = page_size
    else:
        mpps = block_table.shape[1]
        cap = mpps * page_size
    if max_seqlen_k is None:
        max_seqlen_k = cap
    if q.dtype == torch.bfloat16:
        dt = MXA_BF16
    elif q.dtype == torch.float16:
        dt = MXA_F16
    else:
        raise TypeError("q must be float16 or bfloat16")
    return mxa_decode_params_t(B, q_len, Hq, Hkv, D, num_pages, page_size, mpps, int(max_seqlen_k), dt)


@dataclass
class Prepared:
    """A planned call with its workspace: the two-phase use of the library."""
    params: mxa_decode_params_t
    plan: mxa_plan_t
    workspace: Optional[torch.Tensor]


def prepare(q, k_cache, block_table, *, max_seqlen_k=None, num_splits=0, plan=None,
            device=None) -> Prepared:
    params = params_for(q, k_cache, block_table, max_seqlen_k)
    if plan is None:
        plan = mxa_plan(params, num_splits)
    ws = None
    if plan.workspace_bytes:
        ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=device or q.device)
    return Prepared(params, plan, ws)


def decode(q, k_cache, v_cache, block_table, cache_seqlens, *, scale=None, causal=False,
           num_splits=0, max_seqlen_k=None, out=None, lse=None, prepared: Optional[Prepared] = None,
           return_lse=True, stream=None, k_new=None, v_new=None, out_dtype=None):
    """out [B, q_len, Hq, D] (and lse [B, Hq, q_len] fp32) for one decode step.

    With k_new / v_new [B, q_len, Hkv, D] the step first writes them into the
    cache at positions cache_seqlens[b] + t and attends to cache_seqlens[b] +
    q_len keys; max_seqlen_k must then bound those lengths.  out_dtype =
    torch.float32 returns O before its rounding to q's type
    (mxa_decode_fwd_f32out)."""
    if scale is None:
        scale = q.shape[-1] ** -0.5
    if prepared is None:
        prepared = prepare(q, k_cache, block_table, max_seqlen_k=max_seqlen_k, num_splits=num_splits)
    f32 = out_dtype == torch.float32 or (out is not None and out.dtype == torch.float32)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device) if f32 else torch.empty_like(q)
    if lse is None and return_lse:
        B, q_len, Hq, _ = q.shape
        lse = torch.empty((B, Hq, q_len), dtype=torch.float32, device=q.device)
    if (k_new is None) != (v_new is None):
        raise ValueError("k_new and v_new go together")
    if f32:
        if k_new is not None:
            raise ValueError("a float32 output is not offered with k_new / v_new")
        mxa_decode_fwd_f32out(q, k_cache, v_cache, block_table, cache_seqlens, prepared.params, scale, causal,
                              prepared.plan, prepared.workspace, out, lse, stream)
    elif k_new is None:
        mxa_decode_fwd_with_plan(q, k_cache, v_cache, block_table, cache_seqlens, prepared.params, scale,
                                 causal, prepared.plan, prepared.workspace, out, lse, stream)
    else:
        mxa_decode_fwd_append(q, k_cache, v_cache, k_new, v_new, block_table, cache_seqlens, prepared.params,
                              scale, causal, prepared.plan, prepared.workspace, out, lse, stream)
    return out, lse


def decode_varlen(q, cu_seqlens_q, k_cache, v_cache, block_table, cache_seqlens, *, max_seqlen_q,
                  scale=None, causal=False, num_splits=0, max_seqlen_k=None, out=None, lse=None,
                  prepared: Optional[Prepared] = None, return_lse=True, stream=None):
    """out [total_q, Hq, D] (and lse [Hq, total_q] fp32) for rows with their
    own query counts: q [total_q, Hq, D], cu_seqlens_q [B + 1] int32 on the
    device, max_seqlen_q >= every row's count (it sizes the plan)."""
    total_q, Hq, D = q.shape
    B = cu_seqlens_q.shape[0] - 1
    if scale is None:
        scale = D ** -0.5
    if prepared is None:
        # planned as B rows of max_seqlen_q queries (a shape-only tensor)
        shape = torch.empty((B, int(max_seqlen_q), Hq, D), dtype=q.dtype, device="meta")
        params = params_for(shape, k_cache, block_table, max_seqlen_k)
        plan = mxa_plan(params, num_splits)
        ws = None
        if plan.workspace_bytes:
            ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=q.device)
        prepared = Prepared(params, plan, ws)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((Hq, total_q), dtype=torch.float32, device=q.device)
    mxa_decode_fwd_varlen(q, cu_seqlens_q, k_cache, v_cache, block_table, cache_seqlens, prepared.params,
                          scale, causal, prepared.plan, prepared.workspace, out, lse, stream)
    return out, lse
