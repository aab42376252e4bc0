"""Pins for the fp64 oracle: checks against things other than itself.

Closed forms (L = 1, identical keys, zero scale), a dominant-score special
case, the exact log-sum-exp merge of split results, invariances the
definition implies (page placement, paged vs contiguous, key order, GQA as
MHA with repeated KV heads, causal rows as truncated decodes), the exact
widening of every 16-bit input pattern, and an independent brute force on
tiny shapes.  Each is chosen so a plausible slip in the oracle (a dropped
term, a wrong sign, a wrong head/page/slot index, log2 for ln, an off-by-one
in the causal limit) fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from decode_attention_packed_b200.workloads import Workload, make_inputs
from tests.brute import brute_attention


def run_oracle(inp, causal=None, scale=None):
    w = inp.w
    return oracle.decode(inp.q, inp.k_cache, inp.v_cache, inp.block_table, inp.cache_seqlens,
                         Hkv=w.Hkv, page_size=inp.page_size, dtype=w.dtype,
                         scale=w.scale if scale is None else scale,
                         causal=w.causal if causal is None else causal)


def wl(**kw):
    base = dict(name="pin", B=2, q_len=1, Hq=4, Hkv=2, D=16, dtype="bf16", page_size=4,
                causal=False, lengths="const:9", seed=7)
    base.update(kw)
    return Workload(**base)


# --------------------------------------------------------------------------
# exact widening of the 16-bit storage formats
# --------------------------------------------------------------------------

def test_f16_widening_every_pattern():
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.f16_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert (np.isnan(got) == nan).all()
    assert (got[~nan] == ref[~nan]).all()


def test_bf16_widening_every_pattern():
    bits = np.arange(65536, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = np.array([oracle.bf16_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert (np.isnan(got) == nan).all()
    assert (got[~nan] == ref[~nan]).all()


# --------------------------------------------------------------------------
# closed forms
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_single_key_returns_its_value_row(dtype):
    """L = 1: softmax over one key is 1, so O = v_0 exactly and LSE = s_0."""
    inp = make_inputs(wl(dtype=dtype, lengths="const:1", B=3))
    out, lse = run_oracle(inp)
    w = inp.w
    for b in range(w.B):
        page = int(inp.block_table[b, 0])
        for h in range(w.Hq):
            kvh = h // w.G
            v0 = inp.v_cache[page, 0, kvh].double().numpy()
            k0 = inp.k_cache[page, 0, kvh].double().numpy()
            qv = inp.q[b, 0, h].double().numpy()
            assert (out[b, 0, h] == v0).all()
            assert lse[b, h, 0] == pytest.approx(w.scale * float(np.dot(qv, k0)), rel=0, abs=1e-12)


def test_identical_keys_average_the_values():
    """All keys equal: every weight is 1/n, O = mean of the value rows and
    LSE = s + ln n."""
    w = wl(lengths="const:13", page_size=4, Hq=6, Hkv=3)
    inp = make_inputs(w)
    inp.k_cache[:] = inp.k_cache[0:1, 0:1]          # one key row everywhere (per head too)
    out, lse = run_oracle(inp)
    n = 13
    for b in range(w.B):
        pages = inp.block_table[b, :4].tolist()
        for h in range(w.Hq):
            kvh = h // w.G
            V = torch.stack([inp.v_cache[pages[j // 4], j % 4, kvh] for j in range(n)]).double().numpy()
            np.testing.assert_allclose(out[b, 0, h], V.mean(0), rtol=0, atol=1e-13)
            s = w.scale * float(np.dot(inp.q[b, 0, h].double().numpy(), inp.k_cache[0, 0, kvh].double().numpy()))
            assert lse[b, h, 0] == pytest.approx(s + math.log(n), abs=1e-12)


def test_zero_scale_gives_uniform_weights():
    """scale = 0 makes every score 0: O = mean V, LSE = ln n."""
    w = wl(lengths="list:5,11", page_size=8)
    inp = make_inputs(w)
    out, lse = run_oracle(inp, scale=0.0)
    for b, n in enumerate([5, 11]):
        for h in range(w.Hq):
            kvh = h // w.G
            V = torch.stack([inp.v_cache[int(inp.block_table[b, j // 8]), j % 8, kvh] for j in range(n)])
            np.testing.assert_allclose(out[b, 0, h], V.double().numpy().mean(0), rtol=0, atol=1e-13)
            assert lse[b, h, 0] == pytest.approx(math.log(n), abs=1e-13)


def test_dominant_score_selects_its_value_row():
    """One key aligned with the query and scaled up dominates: O -> v_{j*}
    with error at most e^{-gap} * n * max|v|."""
    w = wl(lengths="const:40", page_size=8, Hq=2, Hkv=2, D=32, dtype="f16", B=1)
    inp = make_inputs(w)
    jstar = 23
    pg = int(inp.block_table[0, jstar // 8])
    for h in range(2):
        inp.k_cache[pg, jstar % 8, h] = (inp.q[0, 0, h].float() * 4).to(torch.float16)
    out, lse = run_oracle(inp)
    for h in range(2):
        qv = inp.q[0, 0, h].double().numpy()
        s = [w.scale * float(np.dot(qv, inp.k_cache[int(inp.block_table[0, j // 8]), j % 8, h].double().numpy()))
             for j in range(40)]
        gap = s[jstar] - max(s[j] for j in range(40) if j != jstar)
        assert gap > 15
        bound = math.exp(-gap) * 40 * float(inp.v_cache.abs().max()) * 2
        np.testing.assert_allclose(out[0, 0, h], inp.v_cache[pg, jstar % 8, h].double().numpy(), rtol=0, atol=bound)


# --------------------------------------------------------------------------
# the split / LSE-merge identity
# --------------------------------------------------------------------------

@pytest.mark.parametrize("cuts", [[8], [4, 20], [4, 8, 12, 16, 24]])
def test_merge_of_split_results_equals_full(cuts):
    """Running the oracle on disjoint key ranges and merging the partial
    (O, LSE) pairs with the log-sum-exp identity gives the full result."""
    w = wl(lengths="const:28", page_size=4, Hq=8, Hkv=2, D=24, B=3)
    inp = make_inputs(w)
    full_o, full_lse = run_oracle(inp)
    edges = [0] + cuts + [28]
    o_parts, l_parts = [], []
    for a, e in zip(edges[:-1], edges[1:]):
        sub = make_inputs(w)          # same draw; then view the range [a, e) of every row
        sub.block_table = inp.block_table[:, a // 4:].contiguous()
        sub.cache_seqlens = torch.full((w.B,), e - a, dtype=torch.int32)
        o, l = run_oracle(sub)
        o_parts.append(o.reshape(-1, w.D))
        l_parts.append(l.transpose(0, 2, 1).reshape(-1))
    o, l = oracle.combine(np.stack(o_parts), np.stack(l_parts))
    np.testing.assert_allclose(o, full_o.reshape(-1, w.D), rtol=0, atol=1e-12)
    np.testing.assert_allclose(l, full_lse.transpose(0, 2, 1).reshape(-1), rtol=0, atol=1e-12)


def test_combine_special_cases():
    rng = np.random.default_rng(3)
    o = rng.standard_normal((3, 5, 4))
    lse = rng.standard_normal((3, 5))
    # a single split is returned unchanged
    o1, l1 = oracle.combine(o[:1], lse[:1])
    np.testing.assert_array_equal(o1, o[0])
    np.testing.assert_array_equal(l1, lse[0])
    # empty splits (-inf) carry no weight
    lse2 = lse.copy()
    lse2[[0, 2]] = -np.inf
    o2, l2 = oracle.combine(o, lse2)
    np.testing.assert_allclose(o2, o[1], atol=1e-15)
    np.testing.assert_array_equal(l2, lse[1])
    # all empty -> O = 0, LSE = -inf
    o3, l3 = oracle.combine(o, np.full((3, 5), -np.inf))
    assert (o3 == 0).all() and np.isneginf(l3).all()
    # two equal splits: same O, LSE + ln 2
    o4, l4 = oracle.combine(np.stack([o[0], o[0]]), np.stack([lse[0], lse[0]]))
    np.testing.assert_allclose(o4, o[0], atol=1e-15)
    np.testing.assert_allclose(l4, lse[0] + math.log(2), atol=1e-15)


# --------------------------------------------------------------------------
# invariances
# --------------------------------------------------------------------------

def _relayout(inp, page_size, seed):
    """The same logical K/V rows placed in a fresh pool with another page
    size and a random page order."""
    w, L = inp.w, inp.cache_seqlens.tolist()
    rng = np.random.default_rng(seed)
    npp = [(l + page_size - 1) // page_size for l in L]
    total = max(sum(npp), 1)
    perm = rng.permutation(total)
    bt = np.zeros((w.B, max(max(npp), 1)), dtype=np.int32)
    k = torch.zeros((total, page_size, w.Hkv, w.D), dtype=inp.k_cache.dtype)
    v = torch.zeros_like(k)
    pos = 0
    for b in range(w.B):
        bt[b, :npp[b]] = perm[pos:pos + npp[b]]
        pos += npp[b]
        for j in range(L[b]):
            src_p = int(inp.block_table[b, j // inp.page_size]) if inp.block_table is not None else b
            k[bt[b, j // page_size], j % page_size] = inp.k_cache[src_p, j % inp.page_size]
            v[bt[b, j // page_size], j % page_size] = inp.v_cache[src_p, j % inp.page_size]
    out = make_inputs(w)
    out.k_cache, out.v_cache, out.block_table, out.page_size = k, v, torch.from_numpy(bt), page_size
    out.cache_seqlens = inp.cache_seqlens.clone()
    out.q = inp.q.clone()
    return out


@pytest.mark.parametrize("new_page", [1, 3, 16, 64])
def test_page_placement_does_not_change_result(new_page):
    inp = make_inputs(wl(lengths="list:17,30", page_size=4, D=8))
    o1, l1 = run_oracle(inp)
    o2, l2 = run_oracle(_relayout(inp, new_page, seed=new_page))
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_contiguous_layout_matches_paged():
    w = wl(lengths="list:21,6", page_size=4, D=8, q_len=2, causal=True)
    inp = make_inputs(w)
    o1, l1 = run_oracle(inp)
    cw = Workload(**{**w.__dict__, "page_size": 0})
    cont = make_inputs(cw, max_seqlen_k=24)
    cont.q = inp.q.clone()
    for b, n in enumerate([21, 6]):
        for j in range(n):
            cont.k_cache[b, j] = inp.k_cache[int(inp.block_table[b, j // 4]), j % 4]
            cont.v_cache[b, j] = inp.v_cache[int(inp.block_table[b, j // 4]), j % 4]
    o2, l2 = run_oracle(cont)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_key_order_does_not_change_result():
    """Non-causal attention is a function of the set of (k, v) pairs."""
    w = wl(page_size=0, lengths="const:37", B=1, D=16)
    inp = make_inputs(w)
    o1, l1 = run_oracle(inp)
    perm = torch.from_numpy(np.random.default_rng(5).permutation(37))
    inp.k_cache[0, :37] = inp.k_cache[0, perm]
    inp.v_cache[0, :37] = inp.v_cache[0, perm]
    o2, l2 = run_oracle(inp)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)


@pytest.mark.parametrize("G", [2, 3, 8])
def test_gqa_equals_mha_with_repeated_kv_heads(G):
    """Query head h reads KV head h // G: the same as MHA over KV heads
    repeated G times each (repeat_interleave on the head axis)."""
    w = wl(Hq=2 * G, Hkv=2, lengths="list:11,19", page_size=4, D=8, q_len=2, causal=True)
    inp = make_inputs(w)
    o1, l1 = run_oracle(inp)
    mha = make_inputs(Workload(**{**w.__dict__, "Hkv": w.Hq}))
    mha.q = inp.q.clone()
    mha.block_table = inp.block_table.clone()
    mha.cache_seqlens = inp.cache_seqlens.clone()
    mha.k_cache = inp.k_cache.repeat_interleave(G, dim=2)
    mha.v_cache = inp.v_cache.repeat_interleave(G, dim=2)
    o2, l2 = run_oracle(mha)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_causal_row_equals_truncated_decode():
    """Causal query t of qLen sees L - qLen + t + 1 keys: the same as a
    qLen = 1 decode of that query row against that many keys."""
    w = wl(q_len=4, causal=True, lengths="list:9,3", page_size=4, D=8)
    inp = make_inputs(w)
    o, l = run_oracle(inp)
    for t in range(4):
        one = make_inputs(Workload(**{**w.__dict__, "q_len": 1, "causal": False}))
        one.q = inp.q[:, t:t + 1].clone()
        one.k_cache, one.v_cache, one.block_table = inp.k_cache, inp.v_cache, inp.block_table
        one.cache_seqlens = torch.clamp(inp.cache_seqlens - 4 + t + 1, min=0).to(torch.int32)
        o1, l1 = run_oracle(one)
        np.testing.assert_array_equal(o[:, t], o1[:, 0])
        np.testing.assert_array_equal(l[:, :, t], l1[:, :, 0])


def test_rows_that_see_no_key():
    """L = 0, and causal rows with L - qLen + t + 1 <= 0: O = 0, LSE = -inf."""
    w = wl(q_len=4, causal=True, lengths="list:0,2", page_size=4, D=8)
    inp = make_inputs(w)
    o, l = run_oracle(inp)
    assert (o[0] == 0).all() and np.isneginf(l[0]).all()
    # L = 2, qLen = 4: rows t = 0, 1 see 2-4+t+1 <= 0 keys; t = 2 sees 1, t = 3 sees 2
    assert (o[1, :2] == 0).all() and np.isneginf(l[1, :, :2]).all()
    assert np.isfinite(l[1, :, 2:]).all()


# --------------------------------------------------------------------------
# independent brute force on tiny shapes
# --------------------------------------------------------------------------

@pytest.mark.parametrize("seed", range(12))
def test_brute_force_tiny(seed):
    rng = np.random.default_rng(100 + seed)
    Hkv = int(rng.integers(1, 3))
    G = int(rng.integers(1, 4))
    D = int(rng.integers(1, 9))
    q_len = int(rng.integers(1, 4))
    B = int(rng.integers(1, 4))
    page = int(rng.choice([1, 2, 3, 5, 0]))
    L = rng.integers(0, 6, size=B)
    w = Workload("tiny", B=B, q_len=q_len, Hq=Hkv * G, Hkv=Hkv, D=D,
                 dtype=str(rng.choice(["f16", "bf16"])), page_size=page,
                 causal=bool(rng.integers(0, 2)), lengths="list:" + ",".join(map(str, L)),
                 seed=seed)
    inp = make_inputs(w)
    o, l = run_oracle(inp)
    bo, bl = brute_attention(inp.q, inp.k_cache, inp.v_cache, inp.block_table, inp.cache_seqlens,
                             Hkv=Hkv, page_size=inp.page_size, scale=w.scale, causal=w.causal)
    np.testing.assert_allclose(o, bo, rtol=0, atol=1e-12)
    fin = np.isfinite(bl)
    assert (np.isfinite(l) == fin).all()
    np.testing.assert_allclose(l[fin], bl[fin], rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# appending new tokens to the cache (k / v of flash_attn_with_kvcache)
# --------------------------------------------------------------------------

def _labelled(shape, base):
    """bf16 tensor whose element values (small integers, exact in bf16) name their index."""
    idx = np.arange(int(np.prod(shape)), dtype=np.float32).reshape(shape) % 251 + base
    return torch.from_numpy(idx).to(torch.bfloat16)


def test_append_writes_each_token_to_its_page_and_slot():
    # two rows, pages of 4 slots; row 0 holds 2 keys, row 1 holds 5; 3 new tokens each
    bt = np.array([[3, 0], [1, 2]], dtype=np.int32)
    L = np.array([2, 5], dtype=np.int32)
    k_cache = torch.zeros((4, 4, 1, 2), dtype=torch.bfloat16)
    v_cache = torch.zeros((4, 4, 1, 2), dtype=torch.bfloat16)
    k_new = _labelled((2, 3, 1, 2), 1.0)
    v_new = _labelled((2, 3, 1, 2), 300.0)
    kb, vb = oracle.append_kv(k_cache, v_cache, k_new, v_new, bt, L, page_size=4)
    kf = torch.from_numpy(kb.view(np.int16)).view(torch.bfloat16).float()
    vf = torch.from_numpy(vb.view(np.int16)).view(torch.bfloat16).float()
    # written by hand: (row, new token) -> (page, slot)
    where = {(0, 0): (3, 2), (0, 1): (3, 3), (0, 2): (0, 0),
             (1, 0): (2, 1), (1, 1): (2, 2), (1, 2): (2, 3)}
    written = set()
    for (b, t), (page, slot) in where.items():
        assert torch.equal(kf[page, slot], k_new[b, t].float())
        assert torch.equal(vf[page, slot], v_new[b, t].float())
        written.add((page, slot))
    for page in range(4):
        for slot in range(4):
            if (page, slot) not in written:
                assert not kf[page, slot].any() and not vf[page, slot].any()


def test_append_then_decode_equals_decoding_the_full_cache():
    # a cache that already holds L + q_len keys per row, and the same cache
    # with its last q_len keys per row blanked and handed over as new tokens
    q_len = 3
    w = wl(B=3, q_len=q_len, Hq=8, Hkv=2, D=32, page_size=4, lengths="list:7,9,12", causal=True)
    full = make_inputs(w)
    L_before = full.cache_seqlens.numpy() - q_len
    k_new = torch.zeros((w.B, q_len, w.Hkv, w.D), dtype=full.k_cache.dtype)
    v_new = torch.zeros_like(k_new)
    k_blank, v_blank = full.k_cache.clone(), full.v_cache.clone()
    for b in range(w.B):
        for t in range(q_len):
            pos = int(L_before[b]) + t
            page, slot = int(full.block_table[b, pos // 4]), pos % 4
            k_new[b, t], v_new[b, t] = full.k_cache[page, slot], full.v_cache[page, slot]
            k_blank[page, slot] = 0
            v_blank[page, slot] = 0
    kb, vb = oracle.append_kv(k_blank, v_blank, k_new, v_new, full.block_table, L_before, page_size=4)
    assert np.array_equal(kb, oracle.oracle._bits(full.k_cache))
    assert np.array_equal(vb, oracle.oracle._bits(full.v_cache))
    ref_o, ref_l = run_oracle(full)
    got_o, got_l = oracle.decode(full.q, kb, vb, full.block_table, full.cache_seqlens, Hkv=w.Hkv,
                                 page_size=4, dtype=w.dtype, scale=w.scale, causal=True)
    assert np.array_equal(got_o, ref_o) and np.array_equal(got_l, ref_l)


def test_append_to_a_contiguous_cache():
    k_cache = torch.zeros((2, 8, 1, 2), dtype=torch.bfloat16)
    v_cache = torch.zeros_like(k_cache)
    k_new = _labelled((2, 2, 1, 2), 5.0)
    v_new = _labelled((2, 2, 1, 2), 77.0)
    kb, vb = oracle.append_kv(k_cache, v_cache, k_new, v_new, None, np.array([0, 6], dtype=np.int32),
                              page_size=8)
    kf = torch.from_numpy(kb.view(np.int16)).view(torch.bfloat16)
    assert torch.equal(kf[0, 0], k_new[0, 0]) and torch.equal(kf[0, 1], k_new[0, 1])
    assert torch.equal(kf[1, 6], k_new[1, 0]) and torch.equal(kf[1, 7], k_new[1, 1])
    assert int((kf != 0).sum()) == int((k_new != 0).sum())
