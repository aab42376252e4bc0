"""GPU parity: the CUDA path of libmxa.so against the fp64 oracle, element
by element, on the same seeded inputs.

Covers the five decode workloads at their full sizes in the launch
configuration the benchmark times, the split sweeps, both schedules with
many grid sizes, ragged and edge lengths, every supported page size and the
contiguous layout, grouped-query ratios and query lengths (causal and not),
rows that see no key, garbage (NaN) in unused cache slots, the public
combine, determinism and the device failure record.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from decode_attention_packed_b200.workloads import WORKLOADS, Workload, make_inputs, workload
from tests.tolerance import assert_lse_close, assert_out_close

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from decode_attention_packed_b200 import mxa


@pytest.fixture(scope="module", autouse=True)
def _needs_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def run_oracle(inp):
    w = inp.w
    return oracle.decode(inp.q, inp.k_cache, inp.v_cache, inp.block_table, inp.cache_seqlens,
                         Hkv=w.Hkv, page_size=inp.page_size, dtype=w.dtype, scale=w.scale,
                         causal=w.causal)


def to_dev(inp):
    d = "cuda"
    bt = None if inp.block_table is None else inp.block_table.to(d)
    return inp.q.to(d), inp.k_cache.to(d), inp.v_cache.to(d), bt, inp.cache_seqlens.to(d)


def run_gpu(inp, num_splits=0, plan=None, dev=None, return_lse=True):
    q, k, v, bt, sl = dev if dev is not None else to_dev(inp)
    prep = mxa.prepare(q, k, bt, max_seqlen_k=inp.max_seqlen_k, num_splits=num_splits, plan=plan)
    out, lse = mxa.decode(q, k, v, bt, sl, scale=inp.w.scale, causal=inp.w.causal, prepared=prep,
                          return_lse=return_lse)
    torch.cuda.synchronize()
    assert mxa.mxa_device_error(True) == mxa.MXA_OK
    return out.cpu(), (None if lse is None else lse.cpu()), prep.plan


def check(inp, out, lse, ref=None):
    ro, rl = run_oracle(inp) if ref is None else ref
    err = assert_out_close(out, ro, inp.w.dtype)
    if lse is not None:
        assert_lse_close(lse, rl)
    return err


_cache = {}


def full(i):
    if i not in _cache:
        inp = make_inputs(WORKLOADS[i])
        _cache[i] = (inp, run_oracle(inp), to_dev(inp))
    return _cache[i]


# --------------------------------------------------------------------------
# the five workloads at full size
# --------------------------------------------------------------------------

@pytest.mark.parametrize("i", range(len(WORKLOADS)))
def test_workload_full_size(i):
    inp, ref, dev = full(i)
    out, lse, plan = run_gpu(inp, num_splits=inp.w.num_splits, dev=dev)
    err = check(inp, out, lse, ref)
    print(f"{inp.w.name}: plan={plan.as_dict()} max|err|={err:.3e}")


@pytest.mark.parametrize("s", [1, 2, 4, 8, 16])
def test_long_context_split_sweep(s):
    inp, ref, dev = full(3)
    out, lse, plan = run_gpu(inp, num_splits=s, dev=dev)
    assert plan.schedule == mxa.MXA_SCHED_UNIFORM and plan.grid == 16 * s
    check(inp, out, lse, ref)


@pytest.mark.parametrize("s", [1, 3, 8])
def test_ragged_uniform_splits(s):
    inp, ref, dev = full(1)
    out, lse, _ = run_gpu(inp, num_splits=s, dev=dev)
    check(inp, out, lse, ref)


@pytest.mark.parametrize("grid", [1, 2, 7, 148, 296, 1000, 5000])
def test_ragged_balanced_grids(grid):
    inp, ref, dev = full(4)
    q, k, v, bt, sl = dev
    plan = mxa.mxa_plan_balanced(mxa.params_for(q, k, bt, inp.max_seqlen_k), grid)
    assert plan.grid == grid and plan.schedule == mxa.MXA_SCHED_BALANCED
    out, lse, _ = run_gpu(inp, plan=plan, dev=dev)
    check(inp, out, lse, ref)


@pytest.mark.parametrize("unit_cost", [0, 1, 2, 5, 64, 256])
@pytest.mark.parametrize("grid", [3, 296, 1500])
def test_balanced_unit_costs(grid, unit_cost):
    # the fixed cost per unit (quarter blocks, shared out over the rows in
    # whole blocks) moves every range boundary; every block must still be
    # read exactly once and every split unit merged
    inp, ref, dev = full(4)
    q, k, v, bt, sl = dev
    plan = mxa.mxa_plan_balanced(mxa.params_for(q, k, bt, inp.max_seqlen_k), grid)
    plan.unit_cost = unit_cost
    out, lse, _ = run_gpu(inp, plan=plan, dev=dev)
    check(inp, out, lse, ref)


@pytest.mark.parametrize("unit_cost", [0, 3, 6, 64, 256])
def test_balanced_unit_costs_edge_lengths(unit_cost):
    # rows of every length class, including L = 0 rows that hold no unit
    inp = make_inputs(wl())
    dev = to_dev(inp)
    q, k, v, bt, sl = dev
    plan = mxa.mxa_plan_balanced(mxa.params_for(q, k, bt, inp.max_seqlen_k), 37)
    plan.unit_cost = unit_cost
    out, lse, _ = run_gpu(inp, plan=plan, dev=dev)
    check(inp, out, lse)


@pytest.mark.parametrize("D,dtype,G", [(128, "bf16", 16), (64, "f16", 1), (128, "f16", 3)])
@pytest.mark.parametrize("grid", [40, 130])
def test_one_unit_in_many_pieces(D, dtype, G, grid):
    # a single long row cut into more pieces than one landing's LSE slots
    # hold: the merge lands its pieces in several batches and takes the row
    # statistics from global memory
    w = Workload(name="many", B=1, q_len=1, Hq=G, Hkv=1, D=D, dtype=dtype, page_size=64, causal=False,
                 lengths="const:16000", seed=77)
    inp = make_inputs(w)
    dev = to_dev(inp)
    q, k, v, bt, sl = dev
    plan = mxa.mxa_plan_balanced(mxa.params_for(q, k, bt, inp.max_seqlen_k), grid)
    assert plan.needs_combine == 1
    out, lse, _ = run_gpu(inp, plan=plan, dev=dev)
    check(inp, out, lse)


@pytest.mark.parametrize("grid", [5, 6, 12, 13, 100, 300])
def test_rows_of_one_length(grid):
    # Rows all of one length: the balanced ranges then fall at the same
    # offsets in every unit, or straddle two units, depending on the grid
    # (6 units of 47 blocks here, over 5 to 300 CTAs).
    w = Workload(name="even", B=3, q_len=1, Hq=8, Hkv=2, D=128, dtype="bf16", page_size=16, causal=False,
                 lengths="const:3000", seed=93)
    inp = make_inputs(w)
    dev = to_dev(inp)
    q, k, v, bt, sl = dev
    plan = mxa.mxa_plan_balanced(mxa.params_for(q, k, bt, inp.max_seqlen_k), grid)
    out, lse, _ = run_gpu(inp, plan=plan, dev=dev)
    check(inp, out, lse)


@pytest.mark.parametrize("B", [12288, 12289])
def test_row_limit_of_the_balanced_schedule(B):
    # the largest batch the balanced prologue scans, and one row more (the
    # automatic plan then uses the uniform schedule)
    w = Workload(name="rows", B=B, q_len=1, Hq=2, Hkv=1, D=64, dtype="f16", page_size=16, causal=False,
                 lengths="uniform:0:64", seed=90)
    inp = make_inputs(w)
    out, lse, plan = run_gpu(inp)
    assert plan.schedule == (mxa.MXA_SCHED_BALANCED if B <= 12288 else mxa.MXA_SCHED_UNIFORM)
    check(inp, out, lse)


# --------------------------------------------------------------------------
# shapes and edges at sizes the oracle finishes in seconds
# --------------------------------------------------------------------------

EDGE_LENGTHS = [0, 1, 2, 15, 16, 17, 63, 64, 65, 127, 128, 129, 255, 257, 1023, 1025, 1500, 3000, 4096]


def wl(**kw):
    base = dict(name="case", B=len(EDGE_LENGTHS), q_len=1, Hq=8, Hkv=2, D=128, dtype="bf16",
                page_size=16, causal=False, lengths="list:" + ",".join(map(str, EDGE_LENGTHS)), seed=11)
    base.update(kw)
    return Workload(**base)


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("num_splits", [0, 1, 3])
def test_edge_lengths(D, dtype, num_splits):
    inp = make_inputs(wl(D=D, dtype=dtype))
    out, lse, _ = run_gpu(inp, num_splits=num_splits)
    check(inp, out, lse)
    assert (out[0] == 0).all() and torch.isneginf(lse[0]).all()   # the L = 0 row


@pytest.mark.parametrize("page", [0, 8, 16, 32, 64, 128, 256, 192])
@pytest.mark.parametrize("D", [64, 128, 256])
def test_page_sizes(page, D):
    if page == 192 and D == 64:
        pytest.skip("192 neither divides nor is a multiple of the 128-key stage of D = 64")
    inp = make_inputs(wl(page_size=page, D=D, lengths="list:1,100,700,1030,2049", B=5, seed=page + D))
    for s in (0, 2):
        out, lse, _ = run_gpu(inp, num_splits=s)
        check(inp, out, lse)


def test_page_size_not_tiling_is_refused():
    inp = make_inputs(wl(page_size=24, lengths="list:50", B=1))
    with pytest.raises(mxa.MxaError) as e:
        run_gpu(inp)
    assert e.value.code == mxa.MXA_ERR_UNSUPPORTED


@pytest.mark.parametrize("G", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("q_len", [1, 2, 4, 8])
@pytest.mark.parametrize("causal", [False, True])
def test_groups_and_query_lengths(G, q_len, causal):
    inp = make_inputs(wl(Hq=2 * G, Hkv=2, q_len=q_len, causal=causal, D=64 if G % 2 else 128,
                         lengths="list:3,9,130,1025", B=4, page_size=32, seed=G * 10 + q_len))
    for s in (0, 1):
        out, lse, plan = run_gpu(inp, num_splits=s)
        assert plan.units == 4 * 2 * math.ceil(q_len * G / 16)
        check(inp, out, lse)


def test_causal_rows_with_no_key():
    inp = make_inputs(wl(q_len=8, causal=True, Hq=16, Hkv=4, lengths="list:1,3,7,8,9", B=5, seed=5))
    out, lse, _ = run_gpu(inp)
    check(inp, out, lse)
    assert torch.isneginf(lse[0, :, :7]).all() and (out[0, :7] == 0).all()


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_nan_in_unused_cache_slots(dtype):
    """Slots past L_b in a row's last page and pages no row uses hold NaN:
    the result is the same as with clean memory."""
    w = wl(dtype=dtype, lengths="list:5,33,70,0", B=4, page_size=32, seed=21)
    inp = make_inputs(w)
    ref = run_oracle(inp)
    extra = torch.full((3,) + tuple(inp.k_cache.shape[1:]), float("nan"), dtype=inp.k_cache.dtype)
    inp.k_cache = torch.cat([inp.k_cache, extra])
    inp.v_cache = torch.cat([inp.v_cache, extra.clone()])
    for b, L in enumerate(inp.cache_seqlens.tolist()):
        if L % 32:
            pg = int(inp.block_table[b, L // 32])
            inp.k_cache[pg, L % 32:] = float("nan")
            inp.v_cache[pg, L % 32:] = float("nan")
    for s in (0, 1, 2):
        out, lse, _ = run_gpu(inp, num_splits=s)
        check(inp, out, lse, ref)


def test_contiguous_with_spare_capacity():
    inp = make_inputs(wl(page_size=0, lengths="list:1,77,300,0,513", B=5, seed=3), max_seqlen_k=600)
    inp.v_cache[:, 513:] = float("nan")   # capacity past every row's length
    for s in (0, 1, 4):
        out, lse, _ = run_gpu(inp, num_splits=s)
        check(inp, out, lse)


def test_lse_is_optional_and_runs_are_deterministic():
    inp, ref, dev = full(1)
    o1, _, _ = run_gpu(inp, dev=dev, return_lse=False)
    o2, l2, _ = run_gpu(inp, dev=dev)
    assert torch.equal(o1, o2)
    check(inp, o2, l2, ref)


# --------------------------------------------------------------------------
# public combine
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_combine_matches_exact_merge(dtype):
    rng = np.random.default_rng(9)
    S, B, q_len, Hq, D = 5, 3, 2, 4, 64
    o = rng.standard_normal((S, B, q_len, Hq, D)).astype(np.float32)
    lse = (rng.standard_normal((S, B, Hq, q_len)) * 4).astype(np.float32)
    lse[1, 0] = -np.inf                 # an empty split
    lse[:, 2, 1, 0] = -np.inf           # a row with no key in any split
    rows_o = o.transpose(0, 1, 2, 3, 4).reshape(S, -1, D)
    rows_l = lse.transpose(0, 1, 3, 2).reshape(S, -1)    # [S, B*q_len*Hq] in (b, t, h) order
    ro, rl = oracle.combine(rows_o.astype(np.float64), rows_l.astype(np.float64))
    out = torch.empty((B, q_len, Hq, D), dtype=torch.bfloat16 if dtype == "bf16" else torch.float16,
                      device="cuda")
    lse_out = torch.empty((B, Hq, q_len), dtype=torch.float32, device="cuda")
    mxa.mxa_combine(torch.from_numpy(o).cuda(), torch.from_numpy(lse).cuda(), out, lse_out)
    torch.cuda.synchronize()
    assert_out_close(out.cpu(), ro.reshape(B, q_len, Hq, D), dtype)
    assert_lse_close(lse_out.cpu(), rl.reshape(B, q_len, Hq).transpose(0, 2, 1))


# --------------------------------------------------------------------------
# CUDA graphs: a decode step captured once and replayed
# --------------------------------------------------------------------------

def test_decode_replays_in_a_cuda_graph():
    inp, ref, dev = full(1)
    q, k, v, bt, sl = dev
    w = inp.w
    prep = mxa.prepare(q, k, bt, max_seqlen_k=inp.max_seqlen_k)
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.q_len), dtype=torch.float32, device=q.device)
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):  # first call outside the capture (kernel attributes, maps)
        mxa.decode(q, k, v, bt, sl, scale=w.scale, causal=w.causal, prepared=prep, out=out, lse=lse)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        mxa.decode(q, k, v, bt, sl, scale=w.scale, causal=w.causal, prepared=prep, out=out, lse=lse)
    out.zero_()
    lse.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert mxa.mxa_device_error(True) == mxa.MXA_OK
    check(inp, out.cpu(), lse.cpu(), ref)


@pytest.mark.parametrize("bad_page", [10**6, -5])
def test_a_page_id_outside_the_pool_reads_as_zeros_and_is_reported(bad_page):
    # row 1 (70 keys, pages of 16) has its logical page 2 pointing outside the
    # pool: the call must attend to zeros there (as if that page held zero
    # keys and values), leave the other rows alone, and report the entry
    w = Workload(name="badpage", B=3, q_len=1, Hq=8, Hkv=2, D=128, dtype="bf16", page_size=16, causal=False,
                 lengths="list:40,70,33", seed=545)
    inp = make_inputs(w)
    bt_bad = inp.block_table.clone()
    bt_bad[1, 2] = bad_page
    d = "cuda"
    assert mxa.mxa_device_error(True) == mxa.MXA_OK
    out, lse = mxa.decode(inp.q.to(d), inp.k_cache.to(d), inp.v_cache.to(d), bt_bad.to(d),
                          inp.cache_seqlens.to(d), scale=w.scale, causal=False, max_seqlen_k=inp.max_seqlen_k)
    torch.cuda.synchronize()
    assert mxa.mxa_device_error(True) == mxa.MXA_ERR_INVALID_ARG
    # the oracle on a pool with one more page, all zeros, in that entry's place
    zero = torch.zeros((1,) + tuple(inp.k_cache.shape[1:]), dtype=inp.k_cache.dtype)
    k_ref, v_ref = torch.cat([inp.k_cache, zero]), torch.cat([inp.v_cache, zero])
    bt_ref = inp.block_table.clone()
    bt_ref[1, 2] = inp.k_cache.shape[0]
    ro, rl = oracle.decode(inp.q, k_ref, v_ref, bt_ref, inp.cache_seqlens, Hkv=w.Hkv, page_size=16, dtype=w.dtype,
                           scale=w.scale, causal=False)
    assert_out_close(out.cpu(), ro, w.dtype)
    assert_lse_close(lse.cpu(), rl)


@pytest.mark.parametrize("bad_len", [70, -3, 2**31 - 1, -2**31])
def test_a_length_outside_the_bound_is_clamped_and_reported(bad_len):
    # row 1's length lies outside [0, max_seqlen_k = 64]: the call must stay
    # inside its buffers, attend to the clamped length (64 keys, or none),
    # leave the other rows alone, and report the breach
    w = Workload(name="badlen", B=3, q_len=1, Hq=8, Hkv=2, D=128, dtype="bf16", page_size=16, causal=False,
                 lengths="list:40,70,33", seed=546)
    inp = make_inputs(w)  # a block table wide enough for 70 keys
    d = "cuda"
    sl = inp.cache_seqlens.clone()
    sl[1] = bad_len
    pad = 64
    out_buf = torch.full((3 + 2 * pad, 1, 8, 128), 7.0, dtype=torch.bfloat16, device=d)
    out = out_buf[pad:pad + 3]
    for num_splits in (0, 3):
        assert mxa.mxa_device_error(True) == mxa.MXA_OK
        _, lse = mxa.decode(inp.q.to(d), inp.k_cache.to(d), inp.v_cache.to(d), inp.block_table.to(d), sl.to(d),
                            scale=w.scale, causal=False, max_seqlen_k=64, num_splits=num_splits, out=out)
        torch.cuda.synchronize()
        assert mxa.mxa_device_error(True) == mxa.MXA_ERR_INVALID_ARG
        assert (out_buf[:pad] == 7).all() and (out_buf[pad + 3:] == 7).all()
        ref_len = torch.tensor([40, min(max(bad_len, 0), 64), 33], dtype=torch.int32)
        ro, rl = oracle.decode(inp.q, inp.k_cache, inp.v_cache, inp.block_table, ref_len, Hkv=2, page_size=16,
                               dtype="bf16", scale=w.scale, causal=False)
        assert_out_close(out.cpu(), ro, "bf16")
        assert_lse_close(lse.cpu(), rl)


def test_lengths_at_the_bounds_are_not_reported():
    # 0 and max_seqlen_k themselves are valid lengths
    w = Workload(name="edgelen", B=3, q_len=1, Hq=8, Hkv=2, D=128, dtype="bf16", page_size=16, causal=False,
                 lengths="list:0,64,33", seed=547)
    inp = make_inputs(w)
    assert mxa.mxa_device_error(True) == mxa.MXA_OK
    out, lse, _ = run_gpu(inp)
    check(inp, out, lse)



# --------------------------------------------------------------------------
# head dim 256: 64-key stages of 64 KiB, one CTA per SM
# --------------------------------------------------------------------------

def test_head_dim_256_full_size():
    inp = make_inputs(workload("gqa_decode_hd256"))
    ref = run_oracle(inp)
    for s in (0, 1, 4):
        out, lse, plan = run_gpu(inp, num_splits=s)
        assert plan.ctas_per_sm == 1 and plan.block_tokens == 64
        err = check(inp, out, lse, ref)
        print(f"gqa_decode_hd256 splits={s}: grid {plan.grid} max|err|={err:.3e}")


@pytest.mark.parametrize("G,q_len,causal", [(1, 1, False), (2, 4, True), (4, 4, True), (8, 2, False),
                                            (16, 1, False), (4, 8, True)])
def test_head_dim_256_groups_and_query_lengths(G, q_len, causal):
    inp = make_inputs(wl(Hq=2 * G, Hkv=2, q_len=q_len, causal=causal, D=256, lengths="list:1,9,130,1025,3000",
                         B=5, page_size=32, seed=600 + G * 10 + q_len))
    for s in (0, 2):
        out, lse, _ = run_gpu(inp, num_splits=s)
        check(inp, out, lse)


@pytest.mark.parametrize("grid", [1, 7, 148, 1000])
def test_head_dim_256_balanced_grids(grid):
    inp = make_inputs(wl(D=256, lengths="uniform:0:3000", B=24, Hq=16, Hkv=4, page_size=64, seed=640))
    q, k, v, bt, sl = to_dev(inp)
    plan = mxa.mxa_plan_balanced(mxa.params_for(q, k, bt, inp.max_seqlen_k), grid)
    out, lse, _ = run_gpu(inp, plan=plan, dev=(q, k, v, bt, sl))
    check(inp, out, lse)


# --------------------------------------------------------------------------
# repeated calls on a garbage workspace
# --------------------------------------------------------------------------

@pytest.mark.parametrize("name,grid", [("ragged_varlen", 296), ("gqa_decode", 296), ("spec_mtp_small_q", 296),
                                       ("long_context_split_kv", 296), ("gqa_decode_hd256", 148)])
def test_repeated_calls_on_a_garbage_workspace(name, grid):
    # 200 calls in a row, each on a workspace whose every byte is 0xFF (NaN
    # partial results, all-ones arrival counters): every call must match the
    # oracle.  A read of a partial result before it is written shows up as
    # NaN; a read of a shared-memory tile while it is being refilled for the
    # next segment shows up as a wrong row in a few calls out of a hundred.
    w = workload(name)
    inp = make_inputs(w)
    ro, _ = run_oracle(inp)
    q, k, v, bt, sl = to_dev(inp)
    params = mxa.params_for(q, k, bt, inp.max_seqlen_k)
    plan = mxa.mxa_plan_balanced(params, grid)
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    lse = torch.empty((w.B, w.Hq, w.q_len), dtype=torch.float32, device="cuda")
    ref = torch.from_numpy(ro).cuda()
    worst = torch.zeros((), dtype=torch.float64, device="cuda")
    for _ in range(200):
        ws.fill_(255)
        out.fill_(float("nan"))
        mxa.mxa_decode_fwd_f32out(q, k, v, bt, sl, params, w.scale, w.causal, plan, ws, out, lse)
        err = torch.nan_to_num((out.double() - ref).abs(), nan=1e9).max()
        worst = torch.maximum(worst, err)
    torch.cuda.synchronize()
    assert mxa.mxa_device_error(True) == mxa.MXA_OK
    assert worst.item() <= 2e-3, f"worst |err| over 200 calls: {worst.item():.3e}"


@pytest.mark.parametrize("name,grid", [("ragged_varlen", 296), ("long_context_split_kv", 296), ("gqa_decode", 1000),
                                       ("spec_mtp_small_q", 296)])
def test_results_do_not_depend_on_which_piece_merges(name, grid):
    # A split unit is merged by whichever of its pieces arrives last, or by a
    # piece that finds all the others already there and merges at once,
    # without storing its own rows.  Which piece that is, and where the
    # pieces land (the staging buffer, a ring stage, the whole ring), changes
    # from call to call.  The arithmetic is the same in every case and in the
    # same order, so every call returns the same output and LSE, bit for bit.
    w = workload(name)
    inp = make_inputs(w)
    q, k, v, bt, sl = to_dev(inp)
    params = mxa.params_for(q, k, bt, inp.max_seqlen_k)
    plan = mxa.mxa_plan_balanced(params, grid)
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    lse = torch.empty((w.B, w.Hq, w.q_len), dtype=torch.float32, device="cuda")
    mxa.mxa_decode_fwd_f32out(q, k, v, bt, sl, params, w.scale, w.causal, plan, ws, out, lse)
    out0, lse0 = out.clone(), lse.clone()
    differ = torch.zeros((), dtype=torch.int64, device="cuda")
    for _ in range(100):
        mxa.mxa_decode_fwd_f32out(q, k, v, bt, sl, params, w.scale, w.causal, plan, ws, out, lse)
        differ += (out.view(torch.int32) != out0.view(torch.int32)).sum()
        differ += (lse.view(torch.int32) != lse0.view(torch.int32)).sum()
    torch.cuda.synchronize()
    assert mxa.mxa_device_error(True) == mxa.MXA_OK
    assert differ.item() == 0, f"{differ.item()} values differ from the first call's over 100 calls"
