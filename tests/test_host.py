"""Host-side checks of libmxa.so that need no GPU: the library loads and
exports every symbol include/mxa.h declares, the planner and the packing and
split rules follow the pages' worked cases, and bad arguments are refused
with status codes before anything is launched."""
import ctypes
import os
import re

import pytest
import torch

from decode_attention_packed_b200 import mxa
from decode_attention_packed_b200.mxa import (MXA_ERR_INVALID_ARG, MXA_ERR_UNSUPPORTED,
                                              MXA_ERR_WORKSPACE, MXA_OK, MXA_SCHED_BALANCED,
                                              MXA_SCHED_UNIFORM, mxa_decode_params_t, mxa_plan_t)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden", "heuristics_pack_gqa_num_splits.txt")


def header_symbols():
    text = open(os.path.join(ROOT, "include", "mxa.h")).read()
    return sorted(set(re.findall(r"MXA_API\s+[\w\s\*]*?\b(mxa_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = header_symbols()
    assert len(names) >= 8, names
    lib = ctypes.CDLL(mxa.LIBRARY)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/mxa.h but not exported"
    assert sorted(mxa.EXPORTED) == names


@pytest.mark.parametrize("splits", [1, 2, 3, 8, 16, 64])
def test_workspace_size_is_the_uniform_plans(splits):
    # the first phase of the two-phase call: the size mxa_plan puts in the
    # plan, from the shape alone (no device for a uniform plan)
    for p in (params(), params(B=5, q_len=4, Hq=32, Hkv=8, D=128, max_seqlen_k=8192, max_pages_per_seq=128),
              params(B=3, q_len=1, Hq=16, Hkv=8, D=64, max_seqlen_k=300, max_pages_per_seq=19)):
        plan = mxa.mxa_plan(p, splits, sm_count=148)
        assert mxa.mxa_decode_workspace_size(p, splits) == plan.workspace_bytes
        assert (plan.workspace_bytes > 0) == (splits > 1)


def test_workspace_size_refusals():
    assert mxa.mxa_decode_workspace_size(params(), -1) == mxa.SIZE_MAX
    assert mxa.mxa_decode_workspace_size(params(D=96), 2) == mxa.SIZE_MAX
    assert mxa.mxa_decode_workspace_size(params(Hq=30, Hkv=8), 2) == mxa.SIZE_MAX
    assert mxa._lib.mxa_decode_workspace_size(None, 2) == mxa.SIZE_MAX


def test_status_strings():
    for code in range(6):
        assert mxa.mxa_status_string(code).startswith("MXA_")
    assert "UNKNOWN" in mxa.mxa_status_string(99)


def golden_rows(kind):
    for line in open(GOLDEN):
        line = line.split("#")[0].split()
        if line and line[0] == kind:
            yield [int(x) for x in line[1:]]


def test_pack_gqa_rule_worked_cases():
    rows = list(golden_rows("pack"))
    assert rows
    for varlen, seqlen_q, qpk, block_m, expect in rows:
        assert mxa.mxa_should_pack_gqa(varlen, seqlen_q, qpk, block_m) == expect


@pytest.mark.parametrize("q_len,G", [(1, 2), (1, 4), (1, 8), (4, 8), (8, 2), (2, 16)])
def test_pack_gqa_holds_for_every_decode_shape(q_len, G):
    """The kernels always pack; the rule agrees for small q_len (block_m 16)."""
    assert mxa.mxa_should_pack_gqa(0, q_len, G, 16) == 1


def test_num_splits_rule_worked_cases():
    rows = list(golden_rows("splits"))
    assert rows
    for batch, hkv, m_rows, seqlen_k, block_m, block_n, sms, max_splits, expect in rows:
        tiles = batch * hkv * ((m_rows + block_m - 1) // block_m)
        n_blocks = (seqlen_k + block_n - 1) // block_n
        got = mxa.mxa_num_splits_heuristic(tiles, sms, sms, n_blocks, max_splits, 0, 1,
                                           seqlen_k * 128 * 4.0)
        assert got == expect, (batch, got, expect)


def test_num_splits_wave_efficiency():
    # 16 tiles on 148 slots: eff(s) = 16s/148 / ceil(16s/148); best 1.0 (s = 37);
    # smallest s with eff >= 0.85 is 8 (128/148 = 0.865; 7 gives 0.757)
    assert mxa.mxa_num_splits_heuristic(16, 148, 148, 128, 128, 0, 1, 1e6) == 8
    # the same on 296 slots (two CTAs per SM): 16 (256/296 = 0.865)
    assert mxa.mxa_num_splits_heuristic(16, 148, 296, 128, 128, 0, 1, 1e6) == 16
    # enough tiles: one split
    assert mxa.mxa_num_splits_heuristic(256, 148, 296, 64, 64, 0, 1, 1e6) == 1
    # the large-KV-head exception: non-causal, several query tiles
    big = 200 * 1024 * 1024
    assert mxa.mxa_num_splits_heuristic(256, 148, 296, 4096, 128, 0, 4, big) == 4
    assert mxa.mxa_num_splits_heuristic(256, 148, 296, 4096, 128, 1, 4, big) == 1
    assert mxa.mxa_num_splits_heuristic(0, 148, 296, 4096, 128, 0, 1, 1.0) == 0


def params(**kw):
    base = dict(B=2, q_len=1, Hq=64, Hkv=8, D=128, num_pages=512, page_size=64,
                max_pages_per_seq=256, max_seqlen_k=16384, dtype=mxa.MXA_BF16)
    base.update(kw)
    return mxa_decode_params_t(*[base[f] for f, _ in mxa_decode_params_t._fields_])


def test_plan_long_context_split():
    plan = mxa.mxa_plan(params(), 0, sm_count=148)
    assert plan.schedule == MXA_SCHED_BALANCED
    # one full wave of two CTAs per SM over 16 units of 256 blocks
    assert plan.units == 16 and plan.grid == 296 and plan.num_splits == 19
    assert plan.ctas_per_sm == 2 and plan.block_tokens == 64
    assert plan.needs_combine == 1 and plan.workspace_bytes > 0
    # each unit is charged a fixed cost besides its KV blocks, in quarter
    # blocks: one block per two packed query rows (8 rows here), one block for
    # one or two rows, a block and a half for three or four, at most six
    assert plan.unit_cost == 16
    assert mxa.mxa_plan_balanced(params(), 100, sm_count=148).unit_cost == 16
    assert mxa.mxa_plan(params(), 3, sm_count=148).unit_cost == 0
    costs = {(q, hq): mxa.mxa_plan(params(q_len=q, Hq=hq), 0, sm_count=148).unit_cost
             for q, hq in [(1, 8), (1, 16), (1, 32), (4, 32), (8, 64)]}
    assert costs == {(1, 8): 4, (1, 16): 4, (1, 32): 6, (4, 32): 24, (8, 64): 24}
    # a D = 256 block carries twice the bytes, so the same work is half the blocks
    costs = {(q, hq): mxa.mxa_plan(params(q_len=q, Hq=hq, D=256), 0, sm_count=148).unit_cost
             for q, hq in [(1, 16), (1, 32), (2, 32), (4, 32)]}
    assert costs == {(1, 16): 4, (1, 32): 4, (2, 32): 8, (4, 32): 12}


def test_plan_does_not_split_tiny_problems():
    # one unit of 4 blocks: pieces would be under 4 blocks, so one CTA
    p = params(B=1, Hq=4, Hkv=1, D=64, max_seqlen_k=512, max_pages_per_seq=8, num_pages=8)
    plan = mxa.mxa_plan(p, 0, sm_count=148)
    assert plan.grid == 1 and plan.needs_combine == 0 and plan.workspace_bytes == 0
    # 1024 units of up to 256 blocks: capped by the wave
    p = params(B=128, Hq=16, Hkv=8, D=64, max_seqlen_k=16384, max_pages_per_seq=1024, num_pages=20000)
    assert mxa.mxa_plan(p, 0, sm_count=148).grid == 296


def test_plan_uniform_and_row_tiles():
    plan = mxa.mxa_plan(params(B=16, q_len=4, Hq=32), 4, sm_count=148)
    assert plan.schedule == MXA_SCHED_UNIFORM and plan.grid == 16 * 8 * 4
    p1 = mxa.mxa_plan(params(B=16, q_len=4, Hq=32), 1, sm_count=148)
    assert p1.needs_combine == 0 and p1.workspace_bytes == 0
    # 8 query heads per KV head x 4 tokens = 32 packed rows = 2 row tiles
    p2 = mxa.mxa_plan(params(B=3, q_len=4, Hq=64), 1, sm_count=148)
    assert p2.units == 3 * 8 * 2
    # D = 64 stages carry 128 keys
    assert mxa.mxa_plan(params(D=64), 1, sm_count=148).block_tokens == 128


def test_plan_switches_to_uniform_past_the_balanced_row_limit():
    # the balanced prologue scans at most 12288 rows in shared memory; past
    # that the automatic plan uses the page's num_splits rule (uniform)
    at = mxa.mxa_plan(params(B=12288, max_seqlen_k=256, max_pages_per_seq=4, num_pages=50000), 0,
                      sm_count=148)
    past = mxa.mxa_plan(params(B=12289, max_seqlen_k=256, max_pages_per_seq=4, num_pages=50000), 0,
                        sm_count=148)
    assert at.schedule == MXA_SCHED_BALANCED
    assert past.schedule == MXA_SCHED_UNIFORM and past.num_splits == 1  # 98k units fill the GPU
    p = mxa_plan_t()
    pp = params(B=12289, max_seqlen_k=256, max_pages_per_seq=4, num_pages=50000)
    assert mxa._lib.mxa_plan_balanced(ctypes.byref(pp), 296, 148, ctypes.byref(p)) == MXA_ERR_UNSUPPORTED


@pytest.mark.parametrize("kw,code", [
    (dict(D=96), MXA_ERR_UNSUPPORTED),
    (dict(D=512), MXA_ERR_UNSUPPORTED),
    (dict(D=192), MXA_ERR_UNSUPPORTED),
    (dict(Hq=12, Hkv=8), MXA_ERR_INVALID_ARG),
    (dict(q_len=0), MXA_ERR_INVALID_ARG),
    (dict(B=-1), MXA_ERR_INVALID_ARG),
    (dict(page_size=0), MXA_ERR_INVALID_ARG),
    (dict(dtype=7), MXA_ERR_INVALID_ARG),
])
def test_plan_refuses_bad_shapes(kw, code):
    plan = mxa_plan_t()
    p = params(**kw)
    assert mxa._lib.mxa_plan(ctypes.byref(p), 0, 148, ctypes.byref(plan)) == code


def test_plan_head_dim_256_holds_one_cta_per_sm():
    # 64-key stages of 64 KiB, three in the ring: one CTA per SM, so the
    # automatic plan's full wave is one CTA per SM
    p = params(D=256, B=32, Hq=16, Hkv=4, max_seqlen_k=4096, max_pages_per_seq=256, num_pages=8192, page_size=16)
    plan = mxa.mxa_plan(p, 0, sm_count=148)
    assert plan.ctas_per_sm == 1 and plan.block_tokens == 64
    assert plan.schedule == MXA_SCHED_BALANCED and plan.grid == 148
    for D, cps, T in ((64, 2, 128), (128, 2, 64)):
        q = mxa.mxa_plan(params(D=D), 0, sm_count=148)
        assert (q.ctas_per_sm, q.block_tokens) == (cps, T)
    # a 16-row piece of head dim 256 is 16 KiB in float32: the workspace holds
    # two such slots per CTA after the counters
    u = mxa.mxa_plan(p, 3, sm_count=148)
    assert u.workspace_bytes >= u.grid * 2 * 16 * 256 * 4


def _run_with_plan(p, plan, *, q=1, k=1, v=1, bt=1, sl=1, out=1, ws=None, ws_bytes=0, lse=None,
                   scale=0.125, causal=0):
    f = lambda x: None if x is None else ctypes.c_void_p(x * 4096)
    return mxa._lib.mxa_decode_fwd_with_plan(f(q), f(k), f(v), f(bt), f(sl), ctypes.byref(p),
                                             scale, causal, ctypes.byref(plan), f(ws), ws_bytes,
                                             f(out), f(lse), None)


def test_run_refuses_bad_arguments_before_launch():
    p = params()
    plan = mxa.mxa_plan(p, 0, sm_count=148)
    assert _run_with_plan(p, plan, q=None) == MXA_ERR_INVALID_ARG
    assert _run_with_plan(p, plan, out=None) == MXA_ERR_INVALID_ARG
    assert _run_with_plan(p, plan, sl=None) == MXA_ERR_INVALID_ARG
    assert _run_with_plan(p, plan, ws=None) == MXA_ERR_WORKSPACE
    assert _run_with_plan(p, plan, ws=1, ws_bytes=plan.workspace_bytes - 1) == MXA_ERR_WORKSPACE
    assert _run_with_plan(p, plan, scale=float("nan")) == MXA_ERR_INVALID_ARG
    assert _run_with_plan(p, plan, causal=2) == MXA_ERR_INVALID_ARG
    # misaligned pointer
    f = lambda x: ctypes.c_void_p(x)
    assert mxa._lib.mxa_decode_fwd_with_plan(f(4096 + 2), f(4096), f(4096), f(4096), f(4096),
                                             ctypes.byref(p), 0.1, 0, ctypes.byref(plan), f(4096),
                                             plan.workspace_bytes, f(4096), None, None) == MXA_ERR_INVALID_ARG
    # a page size the gather does not tile (paged) ...
    p12 = params(page_size=12, max_pages_per_seq=2048)
    assert _run_with_plan(p12, mxa.mxa_plan(p12, 1, sm_count=148)) == MXA_ERR_UNSUPPORTED
    # ... block table too narrow for max_seqlen_k
    pn = params(max_pages_per_seq=8)
    assert _run_with_plan(pn, mxa.mxa_plan(pn, 1, sm_count=148)) == MXA_ERR_INVALID_ARG
    # a uniform plan whose grid does not match units x splits
    bad = mxa.mxa_plan(p, 2, sm_count=148)
    bad.grid += 1
    assert _run_with_plan(p, bad, ws=1, ws_bytes=1 << 30) == MXA_ERR_INVALID_ARG
    # a balanced plan's fixed unit cost must lie in 0..256 quarter blocks
    for cost in (-1, 257):
        bad = mxa.mxa_plan(p, 0, sm_count=148)
        bad.unit_cost = cost
        assert _run_with_plan(p, bad, ws=1, ws_bytes=1 << 30) == MXA_ERR_INVALID_ARG
    # nothing to do for B = 0
    p0 = params(B=0)
    assert _run_with_plan(p0, mxa.mxa_plan(p0, 1, sm_count=148)) == MXA_OK


def test_append_refuses_bad_arguments_before_launch():
    # the append entry point checks like the plain run, and needs both new-token arrays
    p = params()
    plan = mxa.mxa_plan(p, 0, sm_count=148)
    f = lambda x: None if x is None else ctypes.c_void_p(x * 4096)
    call = lambda **kw: mxa._lib.mxa_decode_fwd_append(
        f(kw.get("q", 1)), f(1), f(1), f(kw.get("k_new", 1)), f(kw.get("v_new", 1)), f(1), f(1),
        ctypes.byref(p), 0.125, 0, ctypes.byref(plan), f(1), 1 << 30, f(1), None, None)
    assert call(k_new=None) == MXA_ERR_INVALID_ARG
    assert call(v_new=None) == MXA_ERR_INVALID_ARG
    assert call(q=None) == MXA_ERR_INVALID_ARG
    misaligned = mxa._lib.mxa_decode_fwd_append(f(1), f(1), f(1), ctypes.c_void_p(4096 + 8), f(1), f(1), f(1),
                                                ctypes.byref(p), 0.125, 0, ctypes.byref(plan), f(1), 1 << 30,
                                                f(1), None, None)
    assert misaligned == MXA_ERR_INVALID_ARG
    p0 = params(B=0)
    assert mxa._lib.mxa_decode_fwd_append(None, None, None, None, None, f(1), None, ctypes.byref(p0), 0.125, 0,
                                          ctypes.byref(mxa.mxa_plan(p0, 1, sm_count=148)), None, 0, None, None,
                                          None) == MXA_OK  # nothing to do for B = 0 (paged layout)


def test_shapes_whose_position_sums_overflow_are_refused():
    # B rows x max KV blocks fits 32 bits, but not once every row's unit cost
    # (up to 64 blocks) is added: the balanced prologue's sums would overflow
    ok = params(B=1000, Hq=1, Hkv=1, page_size=64, num_pages=16, max_pages_per_seq=2147000,
                max_seqlen_k=2147000 * 64)
    assert mxa.mxa_plan(ok, 0, sm_count=148).schedule in (MXA_SCHED_BALANCED, mxa.MXA_SCHED_UNIFORM)
    big = params(B=1000, Hq=1, Hkv=1, page_size=64, num_pages=16, max_pages_per_seq=2147483,
                 max_seqlen_k=2147483 * 64)
    with pytest.raises(mxa.MxaError) as e:
        mxa.mxa_plan(big, 0, sm_count=148)
    assert e.value.code == mxa.MXA_ERR_UNSUPPORTED


def test_varlen_refuses_bad_arguments_before_launch():
    p = params()
    plan = mxa.mxa_plan(p, 0, sm_count=148)
    f = lambda x: None if x is None else ctypes.c_void_p(x * 4096)
    call = lambda **kw: mxa._lib.mxa_decode_fwd_varlen(
        f(kw.get("q", 1)), kw.get("cu", f(1)), kw.get("total_q", 8), f(1), f(1), f(1), f(1),
        ctypes.byref(kw.get("p", p)), 0.125, 0, ctypes.byref(kw.get("plan", plan)), f(1), 1 << 30, f(1), None,
        None)
    assert call(cu=None) == MXA_ERR_INVALID_ARG
    assert call(cu=ctypes.c_void_p(4096 + 2)) == MXA_ERR_INVALID_ARG  # offsets are int32
    assert call(total_q=-1) == MXA_ERR_INVALID_ARG
    assert call(q=None) == MXA_ERR_INVALID_ARG
    assert call(total_q=0) == MXA_OK  # no query: nothing to write, nothing launched
    # a balanced plan whose per-row sums fit 32 bits for one row tile per
    # head, but not for the two tiles (q_len 2 x 16 heads) a varlen row may use
    big = params(B=1000, q_len=2, Hq=16, Hkv=1, D=128, page_size=64, num_pages=16,
                 max_pages_per_seq=1073700, max_seqlen_k=1073700 * 64)
    bplan = mxa.mxa_plan_balanced(big, 296, sm_count=148)
    bplan.unit_cost = 256
    assert call(p=big, plan=bplan) == mxa.MXA_ERR_UNSUPPORTED


def test_combine_refuses_bad_arguments():
    f = lambda x: None if x is None else ctypes.c_void_p(x * 4096)
    c = mxa._lib.mxa_combine
    assert c(f(1), f(1), 0, 2, 1, 4, 64, 0, f(1), None, None) == MXA_ERR_INVALID_ARG
    assert c(f(1), f(1), 2, 2, 1, 4, 66, 0, f(1), None, None) == MXA_ERR_INVALID_ARG
    assert c(None, f(1), 2, 2, 1, 4, 64, 0, f(1), None, None) == MXA_ERR_INVALID_ARG
    assert c(f(1), f(1), 2, 0, 1, 4, 64, 0, f(1), None, None) == MXA_OK


def test_params_from_tensors():
    q = torch.empty(3, 2, 8, 64, dtype=torch.float16)
    k = torch.empty(40, 16, 2, 64, dtype=torch.float16)
    bt = torch.zeros(3, 7, dtype=torch.int32)
    p = mxa.params_for(q, k, bt)
    assert (p.B, p.q_len, p.Hq, p.Hkv, p.D, p.num_pages, p.page_size, p.max_pages_per_seq,
            p.max_seqlen_k, p.dtype) == (3, 2, 8, 2, 64, 40, 16, 7, 112, mxa.MXA_F16)
