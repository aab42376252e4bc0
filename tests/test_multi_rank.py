"""Multi-process host logic on CPU: two `gloo` ranks.

Decode rows are independent, so spreading a batch over processes needs no
exchange on the data path: each rank computes its own rows, and gathering
the shards must give exactly the single-process result.  The benchmark's
multi-GPU mode gives each rank its own instance of the workload and takes
the slowest rank's time; both pieces of host logic are checked here with
the oracle standing in for the device (no GPU involved).
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from decode_attention_packed_b200.workloads import make_inputs, shard_rows, small_variant, workload  # noqa: E402

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _small_case():
    w = small_variant(workload("ragged_varlen"), B=7, lengths="loguniform:1:300")
    return make_inputs(w)


def _rank_main(rank: int, port: int, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=60))
    try:
        sys.path.insert(0, ROOT)
        import oracle
        inp = _small_case()
        w = inp.w
        rows = shard_rows(w.B, rank, WORLD)
        sl = slice(rows.start, rows.stop)
        out, lse = oracle.decode(inp.q[sl], inp.k_cache, inp.v_cache, inp.block_table[sl],
                                 inp.cache_seqlens[sl], Hkv=w.Hkv, page_size=inp.page_size,
                                 dtype=w.dtype, scale=w.scale, causal=w.causal)
        # shards differ in size when B is odd: pad to the largest, then trim
        n_max = len(shard_rows(w.B, 0, WORLD))
        pad_o = np.zeros((n_max,) + out.shape[1:])
        pad_l = np.full((n_max,) + lse.shape[1:], -np.inf)
        pad_o[:len(rows)], pad_l[:len(rows)] = out, lse
        go = [torch.zeros(pad_o.shape, dtype=torch.float64) for _ in range(WORLD)]
        gl = [torch.zeros(pad_l.shape, dtype=torch.float64) for _ in range(WORLD)]
        dist.all_gather(go, torch.from_numpy(pad_o))
        dist.all_gather(gl, torch.from_numpy(pad_l))
        # max over ranks of a per-rank time, as the benchmark reports it
        t = torch.tensor([1.0 + rank], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        if rank == 0:
            outs = [go[r][:len(shard_rows(w.B, r, WORLD))].numpy() for r in range(WORLD)]
            lses = [gl[r][:len(shard_rows(w.B, r, WORLD))].numpy() for r in range(WORLD)]
            results["out"] = np.concatenate(outs)
            results["lse"] = np.concatenate(lses)
            results["tmax"] = float(t.item())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("B", [0, 1, 2, 7, 32, 129])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_shard_rows_partition_the_batch(B, world):
    seen = []
    for r in range(world):
        rows = shard_rows(B, r, world)
        assert rows.step == 1
        seen.extend(rows)
    assert seen == list(range(B))
    sizes = [len(shard_rows(B, r, world)) for r in range(world)]
    assert max(sizes) - min(sizes) <= 1


def test_two_gloo_ranks_reproduce_the_single_process_result():
    import oracle
    inp = _small_case()
    w = inp.w
    ref_o, ref_l = oracle.decode(inp.q, inp.k_cache, inp.v_cache, inp.block_table,
                                 inp.cache_seqlens, Hkv=w.Hkv, page_size=inp.page_size,
                                 dtype=w.dtype, scale=w.scale, causal=w.causal)
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_rank_main, args=(_free_port(), results), nprocs=WORLD,
                           join=True, start_method="spawn")
        got_o, got_l, tmax = results["out"], results["lse"], results["tmax"]
    # every row is computed by exactly one rank from the same inputs: identical bits
    assert np.array_equal(got_o, ref_o)
    assert np.array_equal(got_l, ref_l)
    assert tmax == 2.0


def test_benchmark_ranks_draw_independent_instances_of_one_recipe():
    import importlib
    bench = importlib.import_module("bench")
    w = workload("gqa_decode")
    a, b = bench.shard_inputs(w, 0), bench.shard_inputs(w, 1)
    assert a.q.shape == b.q.shape and a.k_cache.shape[1:] == b.k_cache.shape[1:]
    assert not torch.equal(a.cache_seqlens, b.cache_seqlens)
    # rank 0 holds the canonical draw of the recipe
    assert torch.equal(a.cache_seqlens, make_inputs(w).cache_seqlens)
