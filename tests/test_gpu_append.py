"""Appending the new tokens' keys and values before decoding (GPU parity).

Each case draws a cache that already holds every row's L_b + q_len keys,
hands the last q_len of them to the call as k_new / v_new, and blanks them in
the cache the call receives. The call must write them back exactly: the
cache after the call equals the full cache bit for bit. It must then decode
as the oracle decodes the full cache.
"""
import numpy as np
import pytest
import torch

import oracle
from decode_attention_packed_b200.workloads import Workload, make_inputs
from tests.tolerance import assert_lse_close, assert_out_close

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from decode_attention_packed_b200 import mxa


@pytest.fixture(scope="module", autouse=True)
def _needs_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def split_off_new_tokens(inp, q_len):
    """(cache with the last q_len keys of each row blanked, k_new, v_new, L before)."""
    w = inp.w
    L_full = inp.cache_seqlens.numpy().astype(np.int64)
    L_before = L_full - q_len
    k_new = torch.zeros((w.B, q_len, w.Hkv, w.D), dtype=inp.k_cache.dtype)
    v_new = torch.zeros_like(k_new)
    k_blank, v_blank = inp.k_cache.clone(), inp.v_cache.clone()
    for b in range(w.B):
        for t in range(q_len):
            pos = int(L_before[b]) + t
            if inp.block_table is None:
                page, slot = b, pos
            else:
                page, slot = int(inp.block_table[b, pos // inp.page_size]), pos % inp.page_size
            k_new[b, t], v_new[b, t] = inp.k_cache[page, slot], inp.v_cache[page, slot]
            k_blank[page, slot] = 0
            v_blank[page, slot] = 0
    return k_blank, v_blank, k_new, v_new, torch.from_numpy(L_before.astype(np.int32))


def run_append(inp, q_len, num_splits=0):
    w = inp.w
    k_blank, v_blank, k_new, v_new, L_before = split_off_new_tokens(inp, q_len)
    d = "cuda"
    bt = None if inp.block_table is None else inp.block_table.to(d)
    kc, vc = k_blank.to(d), v_blank.to(d)
    out, lse = mxa.decode(inp.q.to(d), kc, vc, bt, L_before.to(d), scale=w.scale, causal=w.causal,
                          num_splits=num_splits, max_seqlen_k=inp.max_seqlen_k, k_new=k_new.to(d),
                          v_new=v_new.to(d))
    torch.cuda.synchronize()
    assert mxa.mxa_device_error(True) == mxa.MXA_OK
    return out.cpu(), lse.cpu(), kc.cpu(), vc.cpu()


def check_against_full_cache(inp, out, lse, kc, vc):
    w = inp.w
    assert torch.equal(kc.view(torch.int16), inp.k_cache.view(torch.int16))
    assert torch.equal(vc.view(torch.int16), inp.v_cache.view(torch.int16))
    ro, rl = oracle.decode(inp.q, inp.k_cache, inp.v_cache, inp.block_table, inp.cache_seqlens, Hkv=w.Hkv,
                           page_size=inp.page_size, dtype=w.dtype, scale=w.scale, causal=w.causal)
    assert_out_close(out, ro, w.dtype)
    assert_lse_close(lse, rl)


CASES = [
    # paged GQA decode, one new token per row, lengths U[1, 4096]
    dict(B=8, q_len=1, Hq=32, Hkv=8, D=128, dtype="bf16", page_size=16, causal=False,
         lengths="uniform:1:4096"),
    # speculative step: four draft tokens per row, causal among them, pages of 64
    dict(B=5, q_len=4, Hq=32, Hkv=8, D=128, dtype="bf16", page_size=64, causal=True,
         lengths="list:4,67,1025,3000,8192"),
    # head_dim 64, fp16, groups of 2, small pages; rows whose cache was empty
    dict(B=6, q_len=2, Hq=16, Hkv=8, D=64, dtype="f16", page_size=8, causal=True,
         lengths="list:2,3,17,130,2,900"),
    # 4 draft tokens x 8 query heads = 32 packed rows: two row tiles per KV head,
    # whose units both write the new tokens (the same bytes) before reading them
    dict(B=3, q_len=4, Hq=16, Hkv=2, D=128, dtype="bf16", page_size=16, causal=True,
         lengths="list:5,300,2049"),
]


@pytest.mark.parametrize("case", range(len(CASES)))
@pytest.mark.parametrize("num_splits", [0, 3])
def test_append_then_decode(case, num_splits):
    c = CASES[case]
    inp = make_inputs(Workload(name=f"append{case}", seed=500 + case, **c))
    out, lse, kc, vc = run_append(inp, c["q_len"], num_splits)
    check_against_full_cache(inp, out, lse, kc, vc)


def test_append_to_a_contiguous_cache():
    w = Workload(name="append_contig", B=3, q_len=2, Hq=4, Hkv=1, D=64, dtype="f16", page_size=0,
                 causal=False, lengths="list:2,100,256", seed=520)
    inp = make_inputs(w, max_seqlen_k=300)  # rows have spare capacity past their keys
    out, lse, kc, vc = run_append(inp, 2)
    check_against_full_cache(inp, out, lse, kc, vc)


def test_tokens_past_the_bound_are_not_written():
    # row 1 is already full (L = max_seqlen_k): its new token has no slot, the
    # cache keeps its bytes, and the row attends to max_seqlen_k keys
    w = Workload(name="append_full", B=2, q_len=1, Hq=8, Hkv=2, D=128, dtype="bf16", page_size=16,
                 causal=False, lengths="list:40,64", seed=530)
    inp = make_inputs(w)
    d = "cuda"
    L = torch.tensor([39, 64], dtype=torch.int32)
    k_new = torch.full((2, 1, 2, 128), 1.5, dtype=torch.bfloat16)
    v_new = torch.full((2, 1, 2, 128), -2.0, dtype=torch.bfloat16)
    kc, vc = inp.k_cache.to(d), inp.v_cache.to(d)
    out, lse = mxa.decode(inp.q.to(d), kc, vc, inp.block_table.to(d), L.to(d), scale=w.scale, causal=False,
                          max_seqlen_k=64, k_new=k_new.to(d), v_new=v_new.to(d))
    torch.cuda.synchronize()
    assert mxa.mxa_device_error(True) == mxa.MXA_OK
    kx, vx = oracle.append_kv(inp.k_cache, inp.v_cache, k_new[:1], v_new[:1], inp.block_table[:1],
                              L[:1].numpy(), page_size=16)  # row 0 only: row 1 has no room
    assert np.array_equal(kc.cpu().view(torch.int16).numpy().view(np.uint16), kx)
    assert np.array_equal(vc.cpu().view(torch.int16).numpy().view(np.uint16), vx)
    ro, rl = oracle.decode(inp.q, kx, vx, inp.block_table, np.array([40, 64], dtype=np.int32), Hkv=2,
                           page_size=16, dtype="bf16", scale=w.scale, causal=False)
    assert_out_close(out.cpu(), ro, "bf16")
    assert_lse_close(lse.cpu(), rl)


@pytest.mark.parametrize("bad_page", [10**6, -5])
def test_an_out_of_pool_page_id_is_reported_and_not_written(bad_page):
    # row 0's new token falls in a page whose id is not a page of the pool:
    # the token is skipped and reported; row 1's token is written as usual
    w = Workload(name="append_badpage", B=2, q_len=1, Hq=8, Hkv=2, D=128, dtype="bf16", page_size=16,
                 causal=False, lengths="list:40,20", seed=540)
    inp = make_inputs(w)
    d = "cuda"
    L = torch.tensor([39, 19], dtype=torch.int32)
    bt = inp.block_table.clone()
    bt[0, 39 // 16] = bad_page
    k_new = torch.full((2, 1, 2, 128), 1.5, dtype=torch.bfloat16)
    v_new = torch.full((2, 1, 2, 128), -2.0, dtype=torch.bfloat16)
    kc, vc = inp.k_cache.to(d), inp.v_cache.to(d)
    assert mxa.mxa_device_error(True) == mxa.MXA_OK
    mxa.decode(inp.q.to(d), kc, vc, bt.to(d), L.to(d), scale=w.scale, causal=False, max_seqlen_k=40,
               k_new=k_new.to(d), v_new=v_new.to(d))
    torch.cuda.synchronize()
    assert mxa.mxa_device_error(True) == mxa.MXA_ERR_INVALID_ARG
    kx, vx = oracle.append_kv(inp.k_cache, inp.v_cache, k_new[1:], v_new[1:], inp.block_table[1:], L[1:].numpy(),
                              page_size=16)  # row 1 only
    assert np.array_equal(kc.cpu().view(torch.int16).numpy().view(np.uint16), kx)
    assert np.array_equal(vc.cpu().view(torch.int16).numpy().view(np.uint16), vx)
