"""Rows with their own query counts (varlen queries): GPU parity.

The queries are packed as q [total_q, Hq, D] with offsets cu_seqlens_q
[B + 1]; the oracle's decode_varlen is the reference.  The cases mix rows
without queries, rows without keys, rows whose causal queries see no key,
one and two row tiles per KV head, both schedules, D = 64, 128 and 256, fp16
and bf16, paged and contiguous caches, and a full-size speculative batch with
counts drawn from {0, 1, 2, 4, 8}.
"""
import numpy as np
import pytest
import torch

import oracle
from decode_attention_packed_b200.workloads import Workload, make_inputs, make_varlen_queries
from tests.tolerance import assert_lse_close, assert_out_close

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from decode_attention_packed_b200 import mxa


@pytest.fixture(scope="module", autouse=True)
def _needs_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


CASES = [
    # speculative step with per-row draft lengths 0..4, groups of 4, pages of 16
    dict(q_lens=[1, 4, 0, 3, 2, 4], Hq=32, Hkv=8, D=128, dtype="bf16", page_size=16, causal=True,
         lengths=[5, 300, 77, 4096, 1, 1025]),
    # groups of 8: rows of 3 and 4 queries span two row tiles, rows of 1 and 2 one
    dict(q_lens=[4, 1, 2, 3, 4], Hq=16, Hkv=2, D=128, dtype="bf16", page_size=64, causal=True,
         lengths=[4, 67, 1025, 3000, 8192]),
    # D = 64, fp16, non-causal, contiguous cache
    dict(q_lens=[2, 0, 1, 2], Hq=8, Hkv=4, D=64, dtype="f16", page_size=0, causal=False,
         lengths=[2, 100, 0, 256]),
    # rows with queries but no keys, and with keys but no queries
    dict(q_lens=[3, 0, 2, 1], Hq=8, Hkv=2, D=128, dtype="bf16", page_size=16, causal=True,
         lengths=[0, 50, 0, 900]),
    # head dim 256, counts 0..8: a row of 8 queries in groups of 4 spans two row tiles
    dict(q_lens=[8, 1, 4, 0, 2], Hq=16, Hkv=4, D=256, dtype="bf16", page_size=32, causal=True,
         lengths=[9, 700, 2049, 40, 3000]),
    # counts 8 in groups of 2: exactly one full 16-row tile
    dict(q_lens=[8, 8, 1, 0], Hq=8, Hkv=4, D=64, dtype="f16", page_size=16, causal=False,
         lengths=[8, 513, 4096, 77]),
]


def draw(c, seed):
    B = len(c["q_lens"])
    w = Workload(name="varlen", B=B, q_len=1, Hq=c["Hq"], Hkv=c["Hkv"], D=c["D"], dtype=c["dtype"],
                 page_size=c["page_size"], causal=c["causal"],
                 lengths="list:" + ",".join(map(str, c["lengths"])), seed=seed)
    inp = make_inputs(w)
    q, cu = make_varlen_queries(c["q_lens"], c["Hq"], c["D"], c["dtype"], seed + 1)
    return w, inp, q, cu


def run_varlen(inp, q, cu, max_q, causal, num_splits=0):
    d = "cuda"
    bt = None if inp.block_table is None else inp.block_table.to(d)
    out, lse = mxa.decode_varlen(q.to(d), cu.to(d), inp.k_cache.to(d), inp.v_cache.to(d), bt,
                                 inp.cache_seqlens.to(d), max_seqlen_q=max_q, scale=inp.w.scale,
                                 causal=causal, num_splits=num_splits, max_seqlen_k=inp.max_seqlen_k)
    torch.cuda.synchronize()
    assert mxa.mxa_device_error(True) == mxa.MXA_OK
    return out.cpu(), lse.cpu()


@pytest.mark.parametrize("case", range(len(CASES)))
@pytest.mark.parametrize("num_splits", [0, 3])
def test_varlen_matches_oracle(case, num_splits):
    c = CASES[case]
    w, inp, q, cu = draw(c, 700 + 10 * case)
    out, lse = run_varlen(inp, q, cu, max(c["q_lens"]), c["causal"], num_splits)
    ro, rl = oracle.decode_varlen(q, cu.numpy(), inp.k_cache, inp.v_cache, inp.block_table, inp.cache_seqlens,
                                  Hkv=w.Hkv, page_size=inp.page_size, dtype=w.dtype, scale=w.scale,
                                  causal=c["causal"])
    assert_out_close(out, ro, w.dtype)
    assert_lse_close(lse, rl)


@pytest.mark.parametrize("causal", [False, True])
def test_full_size_speculative_batch_with_mixed_counts(causal):
    # the speculative workload's shape (16 rows, 32 query heads in groups of
    # 4, head dim 128, bf16, pages of 64, lengths 8192 / 1023 / 1025 / 1500 /
    # 3000) with per-row query counts drawn from {0, 1, 2, 4, 8}
    lengths = [[8192, 1023, 1025, 1500, 3000][b % 5] for b in range(16)]
    q_lens = np.random.default_rng(811).choice([0, 1, 2, 4, 8], size=16).tolist()
    c = dict(q_lens=q_lens, Hq=32, Hkv=8, D=128, dtype="bf16", page_size=64, causal=causal, lengths=lengths)
    w, inp, q, cu = draw(c, 810 + int(causal))
    ro, rl = oracle.decode_varlen(q, cu.numpy(), inp.k_cache, inp.v_cache, inp.block_table, inp.cache_seqlens,
                                  Hkv=w.Hkv, page_size=inp.page_size, dtype=w.dtype, scale=w.scale, causal=causal)
    for num_splits in (0, 4):
        out, lse = run_varlen(inp, q, cu, 8, causal, num_splits)
        assert_out_close(out, ro, w.dtype)
        assert_lse_close(lse, rl)


@pytest.mark.parametrize("causal", [False, True])
def test_equal_counts_are_bit_identical_to_fixed_q_len(causal):
    # the same problem through both entry points: same plan, same schedule
    B, q_len, Hq, D = 6, 3, 16, 128
    w = Workload(name="varlen_eq", B=B, q_len=q_len, Hq=Hq, Hkv=4, D=D, dtype="bf16", page_size=16,
                 causal=causal, lengths="list:3,40,700,1,2049,130", seed=760)
    inp = make_inputs(w)
    d = "cuda"
    args = (inp.k_cache.to(d), inp.v_cache.to(d), inp.block_table.to(d), inp.cache_seqlens.to(d))
    fo, fl = mxa.decode(inp.q.to(d), *args, scale=w.scale, causal=causal, max_seqlen_k=inp.max_seqlen_k)
    cu = torch.arange(0, (B + 1) * q_len, q_len, dtype=torch.int32)
    vo, vl = mxa.decode_varlen(inp.q.reshape(B * q_len, Hq, D).to(d), cu.to(d), *args, max_seqlen_q=q_len,
                               scale=w.scale, causal=causal, max_seqlen_k=inp.max_seqlen_k)
    torch.cuda.synchronize()
    assert mxa.mxa_device_error(True) == mxa.MXA_OK
    assert torch.equal(vo.cpu().view(torch.int16), fo.cpu().reshape(B * q_len, Hq, D).view(torch.int16))
    assert torch.equal(vl.cpu(), fl.cpu().permute(1, 0, 2).reshape(Hq, B * q_len))


def test_offsets_out_of_range_stay_in_bounds():
    # offsets that break the rules (past total_q, decreasing, a count above
    # max_seqlen_q) are clamped on the device: nothing outside out / lse is
    # written, the call completes, and the breach is reported
    c = CASES[0]
    w, inp, q, _ = draw(c, 780)
    total_q = q.shape[0]
    d = "cuda"
    cu = torch.tensor([0, 9, 3, total_q + 50, -7, total_q, total_q], dtype=torch.int32, device=d)
    pad = 64
    out_buf = torch.full((total_q + 2 * pad, w.Hq, w.D), 7.0, dtype=q.dtype, device=d)
    lse_buf = torch.full((w.Hq * total_q + 2 * pad,), 7.0, dtype=torch.float32, device=d)
    out = out_buf[pad:pad + total_q]
    lse = lse_buf[pad:pad + w.Hq * total_q].view(w.Hq, total_q)
    mxa.decode_varlen(q.to(d), cu, inp.k_cache.to(d), inp.v_cache.to(d), inp.block_table.to(d),
                      inp.cache_seqlens.to(d), max_seqlen_q=4, scale=w.scale, causal=True,
                      max_seqlen_k=inp.max_seqlen_k, out=out, lse=lse)
    torch.cuda.synchronize()
    assert mxa.mxa_device_error(True) == mxa.MXA_ERR_INVALID_ARG
    assert (out_buf[:pad] == 7).all() and (out_buf[pad + total_q:] == 7).all()
    assert (lse_buf[:pad] == 7).all() and (lse_buf[pad + w.Hq * total_q:] == 7).all()


def test_no_queries_writes_nothing():
    c = CASES[0]
    w, inp, _, _ = draw(c, 790)
    d = "cuda"
    q = torch.empty((0, w.Hq, w.D), dtype=torch.bfloat16, device=d)
    cu = torch.zeros(len(c["q_lens"]) + 1, dtype=torch.int32, device=d)
    out, lse = mxa.decode_varlen(q, cu, inp.k_cache.to(d), inp.v_cache.to(d), inp.block_table.to(d),
                                 inp.cache_seqlens.to(d), max_seqlen_q=1, scale=w.scale,
                                 max_seqlen_k=inp.max_seqlen_k)
    torch.cuda.synchronize()
    assert out.shape == (0, w.Hq, w.D) and lse.shape == (w.Hq, 0)
