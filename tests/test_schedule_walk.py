"""The split kernel's work schedule, walked on the CPU (tests/schedule_walk.py):
every KV block of every unit read by exactly one CTA, split pieces in
consecutive CTAs that agree on their count, every split unit tagged before
its pieces arrive; over random shapes, lengths (empty rows, rows of one
length), per-row query counts, grids and unit costs (quarter blocks, shared
out over the rows), and over the bench workloads' own lengths with the plans
the library makes for them.
"""
import random

import pytest

from decode_attention_packed_b200.workloads import make_inputs, workload
from tests.schedule_walk import Problem, check_launch, walk_cta

LENGTHS = [0, 1, 5, 63, 64, 65, 130, 1000, 4096]


def random_problem(rng):
    B = rng.randint(1, 12)
    q_len = rng.randint(1, 6)
    lens = [rng.choice(LENGTHS + [rng.randint(0, 3000)]) for _ in range(B)]
    if rng.random() < 0.3:
        lens = [lens[0]] * B  # rows all of one length
    kw = dict(B=B, Hkv=rng.choice([1, 2, 4, 8]), G=rng.choice([1, 2, 4, 8, 16]), q_len=q_len,
              D=rng.choice([64, 128, 256]), lens=lens, q_counts=[rng.randint(0, q_len) for _ in range(B)],
              varlen=rng.random() < 0.7)
    if rng.random() < 0.7:
        p = Problem(schedule="balanced", unit_cost_q=rng.choice([0, 1, 2, 3, 4, 5, 6, 16, 24, 256]), **kw)
        grid = rng.choice([1, 2, 3, 7, 148, 296, 1000])
    else:
        p = Problem(schedule="uniform", splits=rng.choice([1, 2, 3, 5]), **kw)
        grid = p.B * p.Hkv * p.RT * p.splits
    return p, grid


@pytest.mark.parametrize("seed", range(4))
def test_random_problems(seed):
    rng = random.Random(seed)
    for _ in range(500):
        p, grid = random_problem(rng)
        check_launch(p, grid)


def test_a_plan_past_the_blocks_leaves_ctas_idle():
    # more CTAs than KV blocks: the extra CTAs take no segment
    p = Problem(B=1, Hkv=1, G=1, q_len=1, D=128, lens=[100], q_counts=[1], varlen=False, schedule="balanced",
                unit_cost_q=4)
    assert check_launch(p, 50) == 2
    assert sum(len(walk_cta(p, bx, 50)[0]) for bx in range(50)) <= 2


@pytest.mark.parametrize("name,unit_cost_q", [("ragged_varlen", 4), ("gqa_decode", 6), ("spec_mtp_small_q", 24),
                                              ("long_context_split_kv", 16), ("gqa_decode_hd256", 4)])
def test_bench_workloads(name, unit_cost_q):
    # the workloads' own lengths, the balanced plan over one wave of
    # resident CTAs, and the fixed costs the planner sets for them
    w = workload(name)
    inp = make_inputs(w)
    p = Problem(B=w.B, Hkv=w.Hkv, G=w.Hq // w.Hkv, q_len=w.q_len, D=w.D, lens=[int(x) for x in inp.cache_seqlens],
                q_counts=[w.q_len] * w.B, varlen=False, schedule="balanced", unit_cost_q=unit_cost_q)
    grid = 148 if w.D == 256 else 296
    assert check_launch(p, grid) == sum((L + p.T - 1) // p.T for L in p.lens) * w.Hkv * p.RT
