"""Pins for the oracle's varlen-query decode (rows with their own query count).

Row b's queries are the packed tokens cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1
(B + 1 running totals from 0, as the MLA metadata page's 参数说明 defines
cu_seqlens_q). Under causal masking, query t of a row with q_b queries sees
the first L_b - q_b + t + 1 keys.

The pins do not reuse the oracle's own row loop:

- zero keys give a closed-form LSE, ln(visible keys), per packed token. This
  fixes the per-row causal offset: using another row's q_len, the largest
  q_len or the packed index in place of t fails it;
- a per-token brute force finds each token's row with a search over the
  offsets;
- equal query counts reduce to the fixed-q_len decode;
- permuting the rows permutes the packed output;
- empty rows and malformed offsets are checked too.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from decode_attention_packed_b200.workloads import Workload, make_inputs


def caches(B, lengths, *, Hq=4, Hkv=2, D=8, page_size=4, dtype="bf16", seed=3):
    w = Workload(name="varlen_pin", B=B, q_len=1, Hq=Hq, Hkv=Hkv, D=D, dtype=dtype,
                 page_size=page_size, causal=False,
                 lengths="list:" + ",".join(str(int(x)) for x in lengths), seed=seed)
    return make_inputs(w)


def packed_q(q_lens, Hq, D, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    return torch.randn((int(sum(q_lens)), Hq, D), generator=g).to(tdt)


def offsets(q_lens):
    return np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)


def run(q, cu, inp, causal, scale=None):
    w = inp.w
    return oracle.decode_varlen(q, cu, inp.k_cache, inp.v_cache, inp.block_table, inp.cache_seqlens,
                                Hkv=w.Hkv, page_size=inp.page_size, dtype=w.dtype,
                                scale=w.scale if scale is None else scale, causal=causal)


def brute_varlen(q, cu, inp, scale, causal):
    """One packed token at a time; its row comes from a search over the offsets."""
    w = inp.w
    qd = q.double().numpy()
    kd = inp.k_cache.double().numpy()
    vd = inp.v_cache.double().numpy()
    L = inp.cache_seqlens.numpy().astype(np.int64)
    G = w.Hq // w.Hkv
    total = qd.shape[0]
    out = np.zeros((total, w.Hq, w.D))
    lse = np.full((w.Hq, total), -np.inf)
    for i in range(total):
        b = int(np.searchsorted(cu, i, side="right")) - 1
        t = i - int(cu[b])
        q_b = int(cu[b + 1] - cu[b])
        n = int(L[b])
        if causal:
            n = max(0, min(n, n - q_b + t + 1))
        if n == 0:
            continue
        j = np.arange(n)
        if inp.block_table is None:
            K, V = kd[b, j], vd[b, j]
        else:
            pages = inp.block_table.numpy()[b, j // inp.page_size]
            K, V = kd[pages, j % inp.page_size], vd[pages, j % inp.page_size]
        for h in range(w.Hq):
            s = K[:, h // G] @ qd[i, h] * scale
            e = np.exp(s)
            out[i, h] = e @ V[:, h // G] / e.sum()
            lse[h, i] = math.log(e.sum())
    return out, lse


@pytest.mark.parametrize("causal", [False, True])
def test_zero_keys_give_log_of_the_visible_count(causal):
    q_lens = [3, 1, 0, 5, 2]
    L = [9, 1, 4, 3, 17]
    inp = caches(len(L), L, seed=11)
    inp.k_cache.zero_()
    q = packed_q(q_lens, 4, 8, "bf16", 12)
    cu = offsets(q_lens)
    o, l = run(q, cu, inp, causal)
    for b, (qb, Lb) in enumerate(zip(q_lens, L)):
        for t in range(qb):
            i = int(cu[b]) + t
            n = max(0, min(Lb, Lb - qb + t + 1)) if causal else Lb   # written out per case below
            if n == 0:
                assert np.isneginf(l[:, i]).all() and (o[i] == 0).all()
            else:
                np.testing.assert_allclose(l[:, i], math.log(n), rtol=0, atol=1e-14)
    if causal:   # the same counts, by hand: row 3 (q=5, L=3) sees -1, 0, 1, 2, 3 keys
        assert np.isneginf(l[:, int(cu[3]) + 0]).all() and np.isneginf(l[:, int(cu[3]) + 1]).all()
        np.testing.assert_allclose(l[:, int(cu[3]) + 4], math.log(3), atol=1e-14)
        np.testing.assert_allclose(l[:, int(cu[0]) + 0], math.log(7), atol=1e-14)   # q=3, L=9
        np.testing.assert_allclose(l[:, int(cu[4]) + 1], math.log(17), atol=1e-14)  # q=2, L=17


def test_zero_keys_average_the_visible_values():
    q_lens = [2, 3]
    L = [5, 4]
    inp = caches(2, L, Hq=2, Hkv=1, D=4, page_size=2, seed=21)
    inp.k_cache.zero_()
    q = packed_q(q_lens, 2, 4, "bf16", 22)
    cu = offsets(q_lens)
    o, _ = run(q, cu, inp, True)
    vd = inp.v_cache.double().numpy()
    bt = inp.block_table.numpy()
    for b in range(2):
        for t in range(q_lens[b]):
            n = L[b] - q_lens[b] + t + 1
            rows = [vd[bt[b, j // 2], j % 2, 0] for j in range(n)]
            np.testing.assert_allclose(o[int(cu[b]) + t], np.mean(rows, axis=0)[None, :].repeat(2, 0),
                                       rtol=0, atol=1e-14)


@pytest.mark.parametrize("seed", range(8))
def test_brute_force_tiny(seed):
    rng = np.random.default_rng(900 + seed)
    B = int(rng.integers(1, 5))
    Hkv = int(rng.integers(1, 3))
    G = int(rng.integers(1, 4))
    D = int(rng.integers(1, 9))
    page = int(rng.choice([1, 2, 3, 0]))
    dtype = str(rng.choice(["f16", "bf16"]))
    L = rng.integers(0, 8, size=B)
    q_lens = rng.integers(0, 5, size=B)
    causal = bool(rng.integers(0, 2))
    inp = caches(B, L, Hq=Hkv * G, Hkv=Hkv, D=D, page_size=page, dtype=dtype, seed=seed)
    q = packed_q(q_lens, Hkv * G, D, dtype, 40 + seed)
    cu = offsets(q_lens)
    o, l = run(q, cu, inp, causal)
    bo, bl = brute_varlen(q, cu, inp, inp.w.scale, causal)
    np.testing.assert_allclose(o, bo, rtol=0, atol=1e-12)
    fin = np.isfinite(bl)
    assert (np.isfinite(l) == fin).all()
    np.testing.assert_allclose(l[fin], bl[fin], rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_equal_query_counts_reduce_to_fixed_q_len_decode(causal):
    B, q_len, Hq, D = 3, 4, 8, 16
    w = Workload(name="varlen_eq", B=B, q_len=q_len, Hq=Hq, Hkv=2, D=D, dtype="f16", page_size=8,
                 causal=causal, lengths="list:6,30,13", seed=31)
    inp = make_inputs(w)
    ro, rl = oracle.decode(inp.q, inp.k_cache, inp.v_cache, inp.block_table, inp.cache_seqlens, Hkv=2,
                           page_size=8, dtype="f16", scale=w.scale, causal=causal)
    o, l = run(inp.q.reshape(B * q_len, Hq, D), offsets([q_len] * B), inp, causal)
    assert np.array_equal(o, ro.reshape(B * q_len, Hq, D))
    assert np.array_equal(l, rl.transpose(1, 0, 2).reshape(Hq, B * q_len))


def test_row_permutation_permutes_the_packed_output():
    q_lens = [1, 4, 2, 3]
    L = [7, 12, 3, 20]
    inp = caches(4, L, seed=51)
    q = packed_q(q_lens, 4, 8, "bf16", 52)
    cu = offsets(q_lens)
    o, l = run(q, cu, inp, True)
    perm = [2, 0, 3, 1]
    q_p = torch.cat([q[int(cu[b]):int(cu[b + 1])] for b in perm])
    cu_p = offsets([q_lens[b] for b in perm])
    inp.block_table = inp.block_table[perm]
    inp.cache_seqlens = inp.cache_seqlens[perm]
    o_p, l_p = run(q_p, cu_p, inp, True)
    for k, b in enumerate(perm):
        assert np.array_equal(o_p[int(cu_p[k]):int(cu_p[k + 1])], o[int(cu[b]):int(cu[b + 1])])
        assert np.array_equal(l_p[:, int(cu_p[k]):int(cu_p[k + 1])], l[:, int(cu[b]):int(cu[b + 1])])


def test_all_rows_empty():
    inp = caches(3, [4, 0, 9], seed=61)
    q = packed_q([0, 0, 0], 4, 8, "bf16", 62)
    o, l = run(q, offsets([0, 0, 0]), inp, True)
    assert o.shape == (0, 4, 8) and l.shape == (4, 0)


@pytest.mark.parametrize("cu", [[1, 2, 3], [0, 3, 2], [0, 1, 5]])
def test_malformed_offsets_are_refused(cu):
    inp = caches(2, [4, 4], seed=71)
    q = packed_q([1, 2], 4, 8, "bf16", 72)   # total_q = 3
    with pytest.raises(ValueError):
        run(q, np.array(cu, dtype=np.int32), inp, False)
