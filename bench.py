"""Benchmark: paged GQA decode attention on B200 through libmxa.so.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mxa|reference]
                    [--workload NAME] [--num-splits S] [--append | --varlen]
                    [--no-suite] [--no-clocks]

One step = one decode call (one launch of the split kernel, which also
merges units split across CTAs) over the whole headline workload.  The
headline is ragged_varlen, the largest of the decode workloads: B = 128
rows, Hq = 16, Hkv = 8, head_dim 64, fp16, pages of 16 slots in a seeded
random permutation, KV lengths log-uniform in [1, 16384], keys scaled by 3.
Inputs are seeded synthetic data.  KV pools rotate over three device copies
(each larger than L2) so that no timed call reads KV left in L2 by the
previous one.  Each device-timed region opens behind about 100 us of a
device-side spin (outside the region), so that the first timed call does not
wait for the host's first launch; the end-to-end figure has no such spin.
Before the run's first timed region the device runs the first workload's
calls, untimed, for about 0.2 s, so that region does not catch the clocks
rising from idle.

Before the headline, the same run measures the other workloads that the
throughput target covers (gqa_decode, spec_mtp_small_q,
long_context_split_kv) the same way, each in its own timed region of K
calls after W warm-up calls, with its own roofline and CPU baseline, plus
per-call percentiles and, for long_context_split_kv, a table over
num_splits.  They are reported under "workloads"; --no-suite skips them,
and --workload NAME makes NAME the headline (and skips them too).

Prints one JSON line (rank 0).  `value` is KV-read throughput in GB/s
summed over ranks; `us_per_call` and the roofline block give the per-call
view.  Under torchrun every rank runs its own shard of independent decode
rows (weak scaling; no collective on the data path).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from decode_attention_packed_b200.workloads import make_inputs, make_varlen_queries, workload  # noqa: E402

METRIC = "decode-attn µs/call and KV-read GB/s as % of B200 HBM peak (1 GPU)"

# DRAM bytes (read + written) per launch of the split kernel, from one ncu
# capture per workload, keyed by a hash of the kernel sources the capture
# was taken on: once the kernel changes, the figures no longer apply and
# the bench reports null.  The captures and their commands are summarised
# under profiles/ (the median of three launches after five).
MEASURED_TRAFFIC = {
    ("dd2bfde320a38581", "ragged_varlen"): 518_542_592,
    ("dd2bfde320a38581", "gqa_decode"): 246_210_048,
    ("dd2bfde320a38581", "spec_mtp_small_q"): 216_960_256,
    ("dd2bfde320a38581", "long_context_split_kv"): 134_545_920,
    ("dd2bfde320a38581", "gqa_decode_hd256"): 315_172_352,
}
HEADLINE = "ragged_varlen"
SUITE = ("gqa_decode", "spec_mtp_small_q", "long_context_split_kv")
SPLIT_SWEEP = (1, 2, 4, 8, 16)
FALLBACK_HBM_GBS = 6650.0
N_POOLS = 3


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="mxa", choices=["mxa", "reference"])
    ap.add_argument("--workload", default=None,
                    help=f"headline workload (default {HEADLINE}, with the suite of the other gated workloads)")
    ap.add_argument("--num-splits", type=int, default=None)
    ap.add_argument("--no-suite", action="store_true", help="measure the headline workload only")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--append", action="store_true",
                    help="each step also appends the step's q_len new tokens per row to the cache "
                         "(mxa_decode_fwd_append) before attending")
    ap.add_argument("--varlen", action="store_true",
                    help="rows have their own query counts, drawn (seeded) from 1..q_len, packed with "
                         "cu_seqlens_q (mxa_decode_fwd_varlen)")
    ap.add_argument("--combine", action="store_true",
                    help="time the stand-alone merge (mxa_combine) of --num-splits float32 partial results of "
                         "the workload's shape, instead of the decode")
    args = ap.parse_args(argv)
    if args.warmup < 0 or args.steps < 1:
        ap.error("--steps must be at least 1 and --warmup at least 0")
    if args.append and args.varlen:
        ap.error("--append and --varlen do not combine")
    args.suite = args.workload is None and not args.no_suite
    if args.workload is None:
        args.workload = HEADLINE
    return args


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        try:
            with open(path) as f:
                return float(json.load(f)["hbm_gbs"]), "measured"
        except Exception:
            pass
    return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash() -> str:
    import glob
    import hashlib
    csrc = os.path.join(ROOT, "decode_attention_packed_b200", "csrc")
    files = sorted(glob.glob(os.path.join(csrc, "*.cu")) + glob.glob(os.path.join(csrc, "*.cuh")) +
                   glob.glob(os.path.join(csrc, "*.h")))
    h = hashlib.sha256()
    for f in files:
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def workload_config(w, nbytes: dict, world: int) -> dict:
    """The `config` object of the JSON line; both arms report the same one."""
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D, "q_len": w.q_len,
            "page_size": w.page_size, "lengths": w.lengths, "causal": w.causal,
            "kv_dtype": w.dtype, "kv_bytes_per_call": nbytes["kv"],
            "l2": f"KV rotates over {N_POOLS} device copies of {nbytes['kv'] / 1e6:.0f} MB (> L2)",
            "parallelism": f"dp{world} (independent decode rows per rank)"}


def algorithmic_bytes(inp) -> dict:
    """Bytes one decode call must move at minimum (read KV, Q, block table,
    lengths; write O and LSE)."""
    w = inp.w
    es = inp.q.element_size()
    L = inp.cache_seqlens.to(torch.int64)
    kv = int(L.sum()) * w.Hkv * 2 * w.D * es
    q = w.B * w.q_len * w.Hq * w.D * es
    o = q
    lse = w.B * w.Hq * w.q_len * 4
    bt = 0 if inp.block_table is None else int(((L + inp.page_size - 1) // inp.page_size).sum()) * 4
    return {"kv": kv, "total": kv + q + o + lse + bt + w.B * 4}


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the GPU works."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, enabled: bool):
        self.proc = None
        if enabled:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", "100"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except Exception:
                self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            text, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            text, _ = self.proc.communicate()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in text.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def setup_dist(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "mxa":
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available() and args.impl == "mxa":
        torch.cuda.set_device(local)
    return world, rank, local


def shard_inputs(w, rank):
    """Each rank owns an independent shard of decode rows of the same recipe
    (rank 0 holds the canonical draw)."""
    return make_inputs(w, seed=w.seed + 7919 * rank)


def oracle_cpu(inp, sample_rows=None):
    """Time the fp64 oracle on (a prefix of) the workload; returns seconds and KV bytes."""
    import oracle
    w = inp.w
    B = w.B if sample_rows is None else sample_rows
    bt = None if inp.block_table is None else inp.block_table[:B]
    t0 = time.perf_counter()
    oracle.decode(inp.q[:B], inp.k_cache, inp.v_cache, bt, inp.cache_seqlens[:B], Hkv=w.Hkv,
                  page_size=inp.page_size, dtype=w.dtype, scale=w.scale, causal=w.causal)
    dt = time.perf_counter() - t0
    kv = int(inp.cache_seqlens[:B].to(torch.int64).sum()) * w.Hkv * 2 * w.D * inp.q.element_size()
    return dt, kv


def omp_threads() -> int:
    try:
        import ctypes
        return int(ctypes.CDLL("libgomp.so.1").omp_get_max_threads())
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(inp, budget_s):
    """The oracle, as it stands, on the host cores: whole passes over the
    workload until about `budget_s` seconds of CPU work are done."""
    dt, kv = oracle_cpu(inp)
    reps, tot_t, tot_b = 1, dt, kv
    while tot_t < budget_s and reps < 200:
        dt, kv = oracle_cpu(inp)
        reps += 1
        tot_t += dt
        tot_b += kv
    return {"value": round(tot_b / tot_t / 1e9, 4), "unit": "GB/s", "cores": omp_threads(),
            "kind": "oracle",
            "sample": f"{reps} full pass(es) of {inp.w.name} (B={inp.w.B}), fp64, {tot_t:.1f} s"}


def run_reference(args, world, rank):
    if rank != 0:
        return
    w = workload(args.workload)
    inp = make_inputs(w)
    # one step = a bounded prefix of the workload's rows, sized so that all
    # warm-up and timed steps end within about two minutes
    t_row, _ = oracle_cpu(inp, sample_rows=1)
    per_step = 120.0 / max(args.steps + args.warmup, 1)
    rows = int(max(1, min(w.B, per_step / max(t_row, 1e-6))))
    for _ in range(args.warmup):
        oracle_cpu(inp, rows)
    tot_t = tot_b = 0.0
    for _ in range(args.steps):
        dt, kv = oracle_cpu(inp, rows)
        tot_t += dt
        tot_b += kv
    value = tot_b / tot_t / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(tot_t / args.steps * 1e3, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(workload_config(w, algorithmic_bytes(inp), world), append=False),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": omp_threads(),
                         "kind": "oracle", "sample": f"first {rows} of {w.B} rows per step"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


class Runner:
    """Device-side plumbing of one rank: stream, barriers, max over ranks."""

    def __init__(self, world, rank, local):
        self.world, self.rank, self.local = world, rank, local
        self.dev = torch.device("cuda", local)
        self.stream = torch.cuda.current_stream(self.dev)

    def barrier(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier(device_ids=[self.local])
        torch.cuda.synchronize(self.dev)

    def max_over_ranks(self, x: float) -> float:
        if self.world == 1:
            return x
        import torch.distributed as dist
        t = torch.tensor([x], dtype=torch.float64, device=self.dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def hold_device(self):
        """Keep the device busy for about 100 us (torch's spin kernel, outside
        any timed region) while the host enqueues the opening event and the
        first calls of a timed region.  Without it the region starts with the
        device idle, waiting for the host's first launch, and a short region
        of K calls counts that wait against the calls."""
        torch.cuda._sleep(200_000)

    def settle(self, call, seconds=0.2):
        """Before the run's first timed region only: untimed calls for about
        `seconds` of device time, so that the region does not catch the
        device's clocks still rising from idle (the first workload timed
        otherwise read up to 5 % slower over K = 20 calls than the same
        calls later in the run)."""
        if getattr(self, "_settled", False):
            return
        self._settled = True
        spent, i = 0.0, 0
        while spent < seconds:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(self.stream)
            for _ in range(100):
                call(i)
                i += 1
            e1.record(self.stream)
            e1.synchronize()
            spent += e0.elapsed_time(e1) / 1e3

    def timed(self, call, warmup, steps) -> float:
        """W untimed calls, then exactly `steps` calls between two events on
        the launching stream, barrier + synchronize on both sides; seconds,
        the max over ranks."""
        self.settle(call)
        for i in range(warmup):
            call(i)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        self.barrier()
        self.hold_device()
        e0.record(self.stream)
        for i in range(steps):
            call(i)
        e1.record(self.stream)
        self.barrier()
        return self.max_over_ranks(e0.elapsed_time(e1) / 1e3)

    def per_call(self, call, n) -> dict:
        """Spread of single calls: each call between its own pair of events,
        back to back (the events keep neighbouring calls from overlapping it)."""
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
        self.barrier()
        self.hold_device()
        ev[0].record(self.stream)
        for i in range(n):
            call(i)
            ev[i + 1].record(self.stream)
        self.barrier()
        each = sorted(ev[i].elapsed_time(ev[i + 1]) * 1e3 for i in range(n))
        pct = lambda f: round(each[min(n - 1, int(f * n))], 3)  # noqa: E731
        return {"p10": pct(0.10), "p50": pct(0.50), "p90": pct(0.90), "n": n, "unit": "us",
                "how": "each call between its own events, back to back"}


class Case:
    """One workload resident on the device, ready to be called."""

    def __init__(self, r: Runner, w, num_splits=None, append=False, varlen=False):
        from decode_attention_packed_b200 import mxa
        self.mxa, self.r, self.w = mxa, r, w
        self.append, self.varlen = append, varlen
        inp = self.inp = shard_inputs(w, r.rank)
        dev = r.dev
        self.q = inp.q.to(dev)
        self.bt = None if inp.block_table is None else inp.block_table.to(dev)
        self.sl = inp.cache_seqlens.to(dev)
        self.pools = [(inp.k_cache.to(dev), inp.v_cache.to(dev))]
        for _ in range(N_POOLS - 1):
            self.pools.append((self.pools[0][0].clone(), self.pools[0][1].clone()))
        self.splits = w.num_splits if num_splits is None else num_splits
        self.prep = mxa.prepare(self.q, self.pools[0][0], self.bt, max_seqlen_k=inp.max_seqlen_k,
                                num_splits=self.splits)
        self.cu = self.hcu = self.hqv = None
        if varlen:  # the plan above is for q_len queries per row, which bounds every row's count
            q_lens = np.random.default_rng(w.seed + 77).integers(1, w.q_len + 1, size=w.B)
            self.hqv, hcu = make_varlen_queries(q_lens, w.Hq, w.D, w.dtype, w.seed + 78)
            self.q, self.cu = self.hqv.to(dev), hcu.to(dev)
            self.hcu = hcu.pin_memory()
        self.out = torch.empty_like(self.q)
        self.lse = (torch.empty((w.Hq, self.q.shape[0]), dtype=torch.float32, device=dev) if varlen
                    else torch.empty((w.B, w.Hq, w.q_len), dtype=torch.float32, device=dev))
        self.nbytes = algorithmic_bytes(inp)
        if append:
            # the rows' last q_len keys arrive as this step's new tokens: the
            # call writes them (the same values each step) and attends to all
            # keys; the new tokens are read and written once more
            self.nbytes["total"] += 2 * 2 * w.B * w.q_len * w.Hkv * w.D * inp.q.element_size()
            self.sl_run = (self.sl - w.q_len).clamp(min=0)
            self.k_new = torch.randn((w.B, w.q_len, w.Hkv, w.D), device=dev).to(self.q.dtype)
            self.v_new = torch.randn_like(self.k_new)
        else:
            self.sl_run = self.sl

    def run(self, i, q, cu, bt, sl, out, lse):
        mxa, w, prep = self.mxa, self.w, self.prep
        k, v = self.pools[i % N_POOLS]
        if self.append:
            mxa.mxa_decode_fwd_append(q, k, v, self.k_new, self.v_new, bt, sl, prep.params, w.scale, w.causal,
                                      prep.plan, prep.workspace, out, lse, self.r.stream)
        elif self.varlen:
            mxa.mxa_decode_fwd_varlen(q, cu, k, v, bt, sl, prep.params, w.scale, w.causal, prep.plan,
                                      prep.workspace, out, lse, self.r.stream)
        else:
            mxa.mxa_decode_fwd_with_plan(q, k, v, bt, sl, prep.params, w.scale, w.causal, prep.plan,
                                         prep.workspace, out, lse, self.r.stream)

    def call(self, i):
        self.run(i, self.q, self.cu, self.bt, self.sl_run, self.out, self.lse)

    def check_clean(self):
        assert self.mxa.mxa_device_error(True) == self.mxa.MXA_OK, "device-side failure recorded during the bench"

    def roofline(self, per_call_s, peak, peak_kind):
        achieved = self.nbytes["total"] / per_call_s / 1e9
        key = (kernel_source_hash(), self.w.name)
        plain = not (self.append or self.varlen) and self.splits == self.w.num_splits
        return {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4),
                "traffic": MEASURED_TRAFFIC.get(key) if plain else None,
                "traffic_unit": "DRAM bytes read + written per launch (ncu)",
                "algorithmic_bytes": self.nbytes["total"],
                "peak_kind": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                else "fallback 6.65 TB/s",
                "kernel": "mxa_split_kernel (one launch per call; split units merged inside)"}

    def release(self):
        self.pools = self.q = self.out = self.lse = None


def measure(r: Runner, case: Case, args, peak, peak_kind, n_each):
    """Timed region, spread of single calls and roofline of one workload."""
    dev_s = r.timed(case.call, args.warmup, args.steps)
    case.check_clean()
    per_call_s = dev_s / args.steps
    kv_gbs = case.nbytes["kv"] / per_call_s / 1e9
    res = {
        "us_per_call": round(per_call_s * 1e6, 3),
        "kv_gbs": round(kv_gbs * r.world, 2),
        "kv_frac_of_hbm_peak": round(kv_gbs / peak, 4),
        "kv_bytes_per_call": case.nbytes["kv"],
        "roofline": case.roofline(per_call_s, peak, peak_kind),
        "plan": case.prep.plan.as_dict(),
        "steps": args.steps, "warmup": args.warmup,
    }
    # a longer back-to-back run of the same calls, for context
    n_long = max(args.steps, 2000)
    long_s = r.timed(case.call, args.warmup, n_long)
    res["sustained"] = {"us_per_call": round(long_s / n_long * 1e6, 3), "calls": n_long,
                        "kv_frac_of_hbm_peak": round(case.nbytes["kv"] / (long_s / n_long) / 1e9 / peak, 4)}
    res["per_call_us"] = r.per_call(case.call, n_each)
    case.check_clean()
    return res, dev_s


def split_sweep(r: Runner, case: Case, args, peak, n_calls):
    """µs per call over num_splits (uniform schedule) next to the automatic plan."""
    mxa = case.mxa
    rows = []
    auto = case.prep
    for s in (0,) + SPLIT_SWEEP:
        case.prep = mxa.prepare(case.q, case.pools[0][0], case.bt, max_seqlen_k=case.inp.max_seqlen_k,
                                num_splits=s)
        t = r.timed(case.call, args.warmup, n_calls) / n_calls
        case.check_clean()
        rows.append({"num_splits": s if s else "auto", "schedule": "uniform" if s else "balanced",
                     "grid": case.prep.plan.grid, "us_per_call": round(t * 1e6, 3),
                     "kv_frac_of_hbm_peak": round(case.nbytes["kv"] / t / 1e9 / peak, 4)})
    case.prep = auto
    return {"calls_per_entry": n_calls, "rows": rows}


def e2e(r: Runner, case: Case, args):
    """End to end through the C ABI: every step copies its inputs from pinned
    host memory (query, block table, lengths; the KV cache lives on the
    device) and reads its result back (output and LSE).  As in a serving
    loop the copies run on their own streams and overlap the previous and
    next steps' kernels: inputs and outputs are double buffered, and events
    order each buffer's copy-in, decode and copy-out."""
    w, inp, dev, stream = case.w, case.inp, r.dev, r.stream
    hq = (case.hqv if case.varlen else inp.q).pin_memory()
    hbt = None if inp.block_table is None else inp.block_table.pin_memory()
    hsl = ((inp.cache_seqlens - w.q_len).clamp(min=0) if case.append else inp.cache_seqlens).pin_memory()
    hcu = case.hcu
    h2d = (hq.numel() * hq.element_size() + hsl.numel() * 4 + (0 if hbt is None else hbt.numel() * 4)
           + (0 if hcu is None else hcu.numel() * 4))
    d2h = case.out.numel() * case.out.element_size() + case.lse.numel() * 4
    steps = args.steps
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    slots = []
    for _ in range(2):
        slots.append(dict(
            q=torch.empty_like(case.q), sl=torch.empty_like(case.sl),
            bt=None if case.bt is None else torch.empty_like(case.bt),
            cu=None if case.cu is None else torch.empty_like(case.cu),
            out=torch.empty_like(case.out), lse=torch.empty_like(case.lse),
            hout=torch.empty(case.out.shape, dtype=case.out.dtype, pin_memory=True),
            hlse=torch.empty(case.lse.shape, dtype=case.lse.dtype, pin_memory=True),
            copied=torch.cuda.Event(), decoded=torch.cuda.Event(), read=torch.cuda.Event()))
    for sd in slots:  # every buffer starts out free
        sd["decoded"].record(stream)
        sd["read"].record(s_out)

    def step(i):
        sd = slots[i % 2]
        with torch.cuda.stream(s_in):
            s_in.wait_event(sd["decoded"])  # the decode two steps back is done with these inputs
            sd["q"].copy_(hq, non_blocking=True)
            sd["sl"].copy_(hsl, non_blocking=True)
            if hbt is not None:
                sd["bt"].copy_(hbt, non_blocking=True)
            if hcu is not None:
                sd["cu"].copy_(hcu, non_blocking=True)
            sd["copied"].record(s_in)
        stream.wait_event(sd["copied"])
        stream.wait_event(sd["read"])  # the read-back two steps back is done with these outputs
        case.run(i, sd["q"], sd["cu"], sd["bt"], sd["sl"], sd["out"], sd["lse"])
        sd["decoded"].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(sd["decoded"])
            sd["hout"].copy_(sd["out"], non_blocking=True)
            sd["hlse"].copy_(sd["lse"], non_blocking=True)
            sd["read"].record(s_out)

    for i in range(args.warmup):
        step(i)
    r.barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(s_in)
    for i in range(steps):
        step(i)
    s_out.wait_event(slots[(steps - 1) % 2]["read"])
    f1.record(s_out)
    r.barrier()
    e2e_s = r.max_over_ranks(f0.elapsed_time(f1) / 1e3)
    for sd in slots:  # the last results arrived intact
        assert torch.equal(sd["hout"], sd["out"].cpu())
    case.check_clean()
    return {"value": round(case.nbytes["kv"] * r.world / (e2e_s / steps) / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "us_per_step": round(e2e_s / steps * 1e6, 3),
            "copies": "pinned host buffers on their own streams, double buffered, overlapping the "
                      "neighbouring steps' kernels"}


def run_combine(args, r: Runner):
    """The stand-alone merge of S float32 partial results (mxa_combine) for the
    rows of the workload's shape: synthetic partials (N(0,1) rows, LSEs
    N(0, 4^2) with some splits empty), W warm-up calls, then K timed calls.
    Bytes per call: S partial rows and LSEs read, one output row and LSE
    written per (b, t, h)."""
    from decode_attention_packed_b200 import mxa
    w = workload(args.workload)
    S = args.num_splits or 16
    g = torch.Generator(device="cpu").manual_seed(w.seed + 31)
    rows = w.B * w.q_len * w.Hq
    o = torch.randn((S, w.B, w.q_len, w.Hq, w.D), generator=g).to(r.dev)
    lse_p = (torch.randn((S, w.B, w.Hq, w.q_len), generator=g) * 4).to(r.dev)
    lse_p[S // 2] = float("-inf")  # an empty split
    out = torch.empty((w.B, w.q_len, w.Hq, w.D), dtype=torch.bfloat16 if w.dtype == "bf16" else torch.float16,
                      device=r.dev)
    lse = torch.empty((w.B, w.Hq, w.q_len), dtype=torch.float32, device=r.dev)
    call = lambda i: mxa.mxa_combine(o, lse_p, out, lse, r.stream)  # noqa: E731
    dev_s = r.timed(call, args.warmup, args.steps)
    nbytes = S * rows * (w.D + 1) * 4 + rows * (w.D * out.element_size() + 4)
    per = dev_s / args.steps
    peak, peak_kind = measured_peak()
    if r.rank == 0:
        print(json.dumps({
            "metric": "mxa_combine µs/call and GB/s (1 GPU)", "value": round(nbytes / per / 1e9, 2), "unit": "GB/s",
            "n_gpus": r.world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(per * 1e3, 5),
            "us_per_call": round(per * 1e6, 3), "higher_is_better": True, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "num_splits": S, "rows": rows, "D": w.D, "bytes_per_call": nbytes},
            "roofline": {"bound": "hbm", "achieved": round(nbytes / per / 1e9, 2), "peak": peak, "unit": "GB/s",
                         "frac": round(nbytes / per / 1e9 / peak, 4), "peak_kind": peak_kind,
                         "kernel": "mxa_combine_kernel"},
            "gpu_launches": args.steps}), flush=True)


def main(argv=None):
    args = parse(argv)
    world, rank, local = setup_dist(args)
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    if args.combine:
        run_combine(args, Runner(world, rank, local))
        return

    r = Runner(world, rank, local)
    peak, peak_kind = measured_peak()
    n_each = max(200, min(2000, args.steps))
    clocks = ClockSampler(local, enabled=not args.no_clocks)

    # ---- the other gated workloads, each in its own timed region ----
    suite = {}
    cases = []
    if args.suite:
        for name in SUITE:
            case = Case(r, workload(name))
            res, _ = measure(r, case, args, peak, peak_kind, n_each)
            if name == "long_context_split_kv":
                res["split_sweep"] = split_sweep(r, case, args, peak, n_calls=max(args.steps, 500))
            res["config"] = workload_config(case.w, case.nbytes, world)
            suite[name] = res
            cases.append(case)

    # ---- the headline workload: W warm-up calls, then exactly K timed calls ----
    w = workload(args.workload)
    head = Case(r, w, num_splits=args.num_splits, append=args.append, varlen=args.varlen)
    res, dev_s = measure(r, head, args, peak, peak_kind, n_each)
    e2e_res = e2e(r, head, args)
    clk = clocks.stop()

    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    if world == 1:  # the oracle on the host cores, after all GPU timing
        res["cpu_baseline"] = cpu_baseline(head.inp, budget_s=10.0)
        for case in cases:
            suite[case.w.name]["cpu_baseline"] = cpu_baseline(case.inp, budget_s=4.0)
    per_call_s = dev_s / args.steps
    kv_gbs = head.nbytes["kv"] / per_call_s / 1e9
    line = {
        "metric": METRIC,
        "value": round(kv_gbs * world, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(per_call_s * 1e3, 5),
        "us_per_call": res["us_per_call"],
        "per_call_us": res["per_call_us"],
        "sustained": res["sustained"],
        "kv_frac_of_hbm_peak": res["kv_frac_of_hbm_peak"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic",
        "config": dict(workload_config(w, head.nbytes, world), append=bool(args.append),
                       **({"varlen": {"q_lens": "U{1..%d} per row, seeded" % w.q_len,
                                      "total_q": int(head.q.shape[0])}} if args.varlen else {})),
        "plan": res["plan"],
        "roofline": res["roofline"],
        "e2e": e2e_res,
        "gpu_launches": args.steps,
        "clocks": clk,
    }
    if "cpu_baseline" in res:
        line["cpu_baseline"] = res["cpu_baseline"]
    if suite:
        line["workloads"] = suite
        fracs = {name: v["kv_frac_of_hbm_peak"] for name, v in suite.items()}
        fracs[w.name] = res["kv_frac_of_hbm_peak"]
        line["gate"] = {"kv_frac_of_hbm_peak": fracs, "target": 0.70,
                        "all_met": all(f >= 0.70 for f in fracs.values())}
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
