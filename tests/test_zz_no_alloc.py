"""mxa_decode_fwd_noalloc: decode for callers that cannot allocate device
memory (a serving loop whose memory is fixed at start-up, a plugin under
another framework's allocator, a loop where an allocation could synchronise
the device).  It keeps split results in the library's fixed 16 MiB array
instead of a caller workspace.

Called through the C ABI on two calls in a row.  Each call is compared with
mxa_decode_fwd (caller workspace) and with the fp64 oracle, within the
parity tolerance of the other GPU tests, and the second call must leave the
device's free memory and torch's allocated bytes exactly where the first
left them: the entry point allocates nothing.  (The first call on a device
may load the library's device code, and with it the array, under CUDA's
lazy module loading; that is why the memory is compared from the first call
on.)  This file is collected last so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from decode_attention_packed_b200.workloads import WORKLOADS, make_inputs
from tests.tolerance import assert_lse_close, assert_out_close

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from decode_attention_packed_b200 import mxa


@pytest.fixture(scope="module", autouse=True)
def _needs_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("i", [1, 2, 4])
def test_noalloc_matches_workspace_entry_point(i):
    inp = make_inputs(WORKLOADS[i])
    w = inp.w
    d = "cuda"
    q, k, v = inp.q.to(d), inp.k_cache.to(d), inp.v_cache.to(d)
    bt, sl = inp.block_table.to(d), inp.cache_seqlens.to(d)
    params = mxa.params_for(q, k, bt, inp.max_seqlen_k)
    plan = mxa.mxa_plan(params, 0)
    assert plan.workspace_bytes > 0          # this plan does use scratch memory

    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=d)
    ref_out = torch.empty_like(q)
    ref_lse = torch.empty((w.B, w.Hq, w.q_len), dtype=torch.float32, device=d)
    rc = mxa._lib.mxa_decode_fwd(_p(q), _p(k), _p(v), _p(bt), _p(sl), ctypes.byref(params), w.scale,
                                 int(w.causal), 0, _p(ws), plan.workspace_bytes, _p(ref_out),
                                 _p(ref_lse), _stream())
    assert rc == mxa.MXA_OK
    torch.cuda.synchronize()
    ref_o = ref_out.float().cpu().double().numpy()
    ref_l = ref_lse.cpu().double().numpy()
    oro, orl = oracle.decode(inp.q, inp.k_cache, inp.v_cache, inp.block_table, inp.cache_seqlens, Hkv=w.Hkv,
                             page_size=inp.page_size, dtype=w.dtype, scale=w.scale, causal=w.causal)

    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.q_len), dtype=torch.float32, device=d)
    torch.cuda.synchronize()
    mem = None
    for call in range(2):
        out.fill_(float("nan"))
        lse.fill_(float("nan"))
        rc = mxa._lib.mxa_decode_fwd_noalloc(_p(q), _p(k), _p(v), _p(bt), _p(sl), ctypes.byref(params),
                                             w.scale, int(w.causal), 0, _p(out), _p(lse), _stream())
        assert rc == mxa.MXA_OK, mxa.mxa_status_string(rc)
        torch.cuda.synchronize()
        assert mxa.mxa_device_error(True) == mxa.MXA_OK
        now = (torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated())
        if mem is not None:
            assert now == mem, f"device memory changed across calls: {mem} -> {now}"
        mem = now
        # the same result as the entry point with a caller workspace ...
        assert_out_close(out.cpu(), ref_o, w.dtype, what=f"noalloc call {call}")
        assert_lse_close(lse.cpu(), ref_l, what=f"noalloc lse call {call}")
        # ... and as the oracle
        assert_out_close(out.cpu(), oro, w.dtype, what=f"noalloc call {call} vs oracle")
        assert_lse_close(lse.cpu(), orl, what=f"noalloc lse call {call} vs oracle")


def test_noalloc_refuses_plans_beyond_its_array():
    # 2048 units cut into 8 uniform splits: 16384 CTAs, ~268 MB of split scratch
    params = mxa.mxa_decode_params_t(256, 1, 64, 8, 128, 65536, 16, 256, 4096, mxa.MXA_BF16)
    plan = mxa.mxa_plan(params, 8)
    assert plan.workspace_bytes > 16 << 20
    rc = mxa._lib.mxa_decode_fwd_noalloc(None, None, None, None, None, ctypes.byref(params), 0.088, 0,
                                         8, None, None, _stream())
    assert rc == mxa.MXA_ERR_WORKSPACE
