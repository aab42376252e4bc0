"""GPU parity of the computation itself: mxa_decode_fwd_f32out writes O in
float32, the value the kernels hold before their one rounding to the input
type ("SmallQ FlashAttention (Vector)" README, 精度策略: fp32 dot products
and accumulation, output acc * (1 / rowSum) rounded once at the end).

Against the fp64 oracle these outputs are held to the raw 2e-3 of the
parity bar, with no allowance for a 16-bit output's rounding, and LSE to
1e-4.  The 16-bit output of the ordinary entry point must be exactly this
float32 output rounded to nearest even: the same kernels run, in the same
order, and only the final store differs.

Each test prints the raw max |err| it saw; `python -m tests.report_errors`
prints the per-workload table.
"""
import numpy as np
import pytest
import torch

import oracle
from decode_attention_packed_b200.workloads import WORKLOADS, Workload, make_inputs
from tests.tolerance import assert_lse_close, assert_out_raw

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from decode_attention_packed_b200 import mxa


@pytest.fixture(scope="module", autouse=True)
def _needs_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def oracle_of(inp):
    w = inp.w
    return oracle.decode(inp.q, inp.k_cache, inp.v_cache, inp.block_table, inp.cache_seqlens, Hkv=w.Hkv,
                         page_size=inp.page_size, dtype=w.dtype, scale=w.scale, causal=w.causal)


def both_outputs(inp, num_splits=0, plan=None):
    """The float32 and the 16-bit output of one plan on the same device inputs."""
    d = "cuda"
    q, k, v = inp.q.to(d), inp.k_cache.to(d), inp.v_cache.to(d)
    bt = None if inp.block_table is None else inp.block_table.to(d)
    sl = inp.cache_seqlens.to(d)
    prep = mxa.prepare(q, k, bt, max_seqlen_k=inp.max_seqlen_k, num_splits=num_splits, plan=plan)
    o32, l32 = mxa.decode(q, k, v, bt, sl, scale=inp.w.scale, causal=inp.w.causal, prepared=prep,
                          out_dtype=torch.float32)
    o16, l16 = mxa.decode(q, k, v, bt, sl, scale=inp.w.scale, causal=inp.w.causal, prepared=prep)
    torch.cuda.synchronize()
    assert mxa.mxa_device_error(True) == mxa.MXA_OK
    assert o32.dtype == torch.float32 and o16.dtype == q.dtype
    return o32.cpu(), l32.cpu(), o16.cpu(), l16.cpu(), prep.plan


def check(inp, num_splits=0, plan=None, ref=None):
    ro, rl = oracle_of(inp) if ref is None else ref
    o32, l32, o16, l16, plan = both_outputs(inp, num_splits, plan)
    err = assert_out_raw(o32, ro)
    assert_lse_close(l32, rl)
    # the 16-bit call is the float32 result rounded once, to nearest even
    assert torch.equal(o32.to(o16.dtype).view(torch.int16), o16.view(torch.int16))
    assert torch.equal(l32, l16)
    return err, plan


_full = {}


def full(i):
    if i not in _full:
        inp = make_inputs(WORKLOADS[i])
        _full[i] = (inp, oracle_of(inp))
    return _full[i]


@pytest.mark.parametrize("i", range(len(WORKLOADS)))
def test_workload_full_size_raw(i):
    inp, ref = full(i)
    err, plan = check(inp, num_splits=inp.w.num_splits, ref=ref)
    print(f"{inp.w.name}: raw max|err| (float32 O) = {err:.3e}, plan grid {plan.grid}")


@pytest.mark.parametrize("s", [1, 2, 4, 8, 16])
def test_long_context_split_sweep_raw(s):
    inp, ref = full(3)
    check(inp, num_splits=s, ref=ref)


@pytest.mark.parametrize("grid", [1, 7, 148, 1000])
def test_ragged_balanced_grids_raw(grid):
    inp, ref = full(4)
    d = "cuda"
    bt = inp.block_table.to(d)
    plan = mxa.mxa_plan_balanced(mxa.params_for(inp.q, inp.k_cache, bt, inp.max_seqlen_k), grid)
    check(inp, plan=plan, ref=ref)


EDGE = [0, 1, 2, 15, 16, 17, 63, 64, 65, 127, 128, 129, 255, 257, 1023, 1025, 1500, 3000, 4096]


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("f16", 64), ("bf16", 64), ("f16", 128), ("bf16", 256),
                                     ("f16", 256)])
def test_edge_lengths_raw(dtype, D):
    w = Workload(name="edge32", B=len(EDGE), q_len=1, Hq=8, Hkv=2, D=D, dtype=dtype, page_size=16,
                 causal=False, lengths="list:" + ",".join(map(str, EDGE)), seed=31)
    check(make_inputs(w))


@pytest.mark.parametrize("q_len,G", [(4, 4), (8, 2), (3, 16)])
def test_causal_small_q_raw(q_len, G):
    w = Workload(name="causal32", B=5, q_len=q_len, Hq=4 * G, Hkv=4, D=128, dtype="bf16", page_size=64,
                 causal=True, lengths="list:1,3,9,1025,3000", seed=41 + G)
    check(make_inputs(w))


def test_contiguous_cache_raw():
    w = Workload(name="contig32", B=4, q_len=1, Hq=4, Hkv=1, D=64, dtype="f16", page_size=0, causal=False,
                 lengths="list:1,77,300,513", seed=51)
    check(make_inputs(w, max_seqlen_k=600))


def test_f32out_refuses_bad_arguments():
    # the same checks as the 16-bit call, before any launch
    p = mxa.mxa_decode_params_t(2, 1, 8, 2, 96, 8, 16, 4, 64, mxa.MXA_BF16)
    plan = mxa.mxa_plan_t()
    st = mxa._lib.mxa_decode_fwd_f32out(None, None, None, None, None, p, 0.1, 0, plan, None, 0, None, None, None)
    assert st == mxa.MXA_ERR_UNSUPPORTED
    p.D = 128
    st = mxa._lib.mxa_decode_fwd_f32out(None, None, None, None, None, p, 0.1, 0, None, None, 0, None, None, None)
    assert st == mxa.MXA_ERR_INVALID_ARG


def test_head_dim_256_full_size_raw():
    from decode_attention_packed_b200.workloads import workload
    inp = make_inputs(workload("gqa_decode_hd256"))
    err, plan = check(inp)
    print(f"gqa_decode_hd256: raw max|err| (float32 O) = {err:.3e}, plan grid {plan.grid}")


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("f16", 64)])
def test_two_cache_segments_merge_through_combine(dtype, D):
    # Each row's keys are cut at a page boundary into two segments; each
    # segment is decoded on its own with a float32 output and its LSE, and
    # mxa_combine merges the two partial results into the decode of the
    # whole cache (the use the float32 output is offered for).
    w = Workload(name="segments", B=6, q_len=1, Hq=16, Hkv=4, D=D, dtype=dtype, page_size=16, causal=False,
                 lengths="list:1,31,40,300,1025,2048", seed=77)
    inp = make_inputs(w)
    ro, rl = oracle_of(inp)
    L = inp.cache_seqlens.numpy()
    bt = inp.block_table.numpy()
    first_pages = [(int(x) // 16) // 2 for x in L]  # segment A: the first half of the full pages
    la_len = np.array([p * 16 for p in first_pages], dtype=np.int32)
    lb_len = (L - la_len).astype(np.int32)
    bt_b = np.zeros_like(bt)
    for b, p in enumerate(first_pages):
        bt_b[b, :bt.shape[1] - p] = bt[b, p:]
    d = "cuda"
    q, k, v = inp.q.to(d), inp.k_cache.to(d), inp.v_cache.to(d)
    parts = []
    for table, lens in ((bt, la_len), (bt_b, lb_len)):
        o, l = mxa.decode(q, k, v, torch.from_numpy(table).to(d), torch.from_numpy(lens).to(d), scale=w.scale,
                          causal=False, max_seqlen_k=inp.max_seqlen_k, out_dtype=torch.float32)
        parts.append((o, l))
    o_part = torch.stack([parts[0][0], parts[1][0]])  # [2, B, q_len, Hq, D]
    lse_part = torch.stack([parts[0][1], parts[1][1]])  # [2, B, Hq, q_len]
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.q_len), dtype=torch.float32, device=d)
    mxa.mxa_combine(o_part, lse_part, out, lse)
    torch.cuda.synchronize()
    assert mxa.mxa_device_error(True) == mxa.MXA_OK
    from tests.tolerance import assert_out_close
    assert_out_close(out.cpu(), ro, dtype)
    assert_lse_close(lse.cpu(), rl)
