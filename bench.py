"""Benchmark: paged GQA decode attention on B200 through libmxa.so.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mxa|reference]
                    [--workload gqa_decode] [--num-splits S]

One step = one decode call (one launch of the split kernel, which also merges
units split across CTAs) over the whole workload:
B = 32 rows, Hq = 32, Hkv = 8, head_dim 128, bf16, pages of 16 slots in a
seeded random permutation, KV lengths uniform in [1, 4096].  Inputs are
seeded synthetic data.  KV pools rotate over three copies (each larger than
L2) so no timed call reads KV from L2 left by the previous one.

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

from decode_attention_packed_b200.workloads import WORKLOADS, make_inputs, make_varlen_queries, workload  # noqa: E402

METRIC = "decode-attn µs/call and KV-read GB/s as % of B200 HBM peak (1 GPU)"

# DRAM bytes (read + written) per launch of the split kernel on the default
# workload, from an ncu capture (profiles/mxa_split_kernel_gqa_decode.md),
# keyed by a hash of the kernel sources it was taken on: once the kernel
# changes the number no longer applies and the bench reports null.
MEASURED_TRAFFIC = {"b7634f37e38a8462": 248863488}
DEFAULT_WORKLOAD = "gqa_decode"
FALLBACK_HBM_GBS = 6650.0
N_POOLS = 3


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", default="mxa", choices=["mxa", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--num-splits", type=int, default=None)
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--append", action="store_true",
                    help="each step also appends the step's q_len new tokens per row to the cache "
                         "(mxa_decode_fwd_append) before attending")
    ap.add_argument("--varlen", action="store_true",
                    help="rows have their own query counts, drawn (seeded) from 1..q_len, packed with "
                         "cu_seqlens_q (mxa_decode_fwd_varlen)")
    return ap.parse_args()


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
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, enabled: bool):
        self.proc = None
        self.gpu = gpu_index
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


def cpu_baseline(inp, budget_s=12.0):
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


def main():
    args = parse()
    world, rank, local = setup_dist(args)
    if args.impl == "reference":
        run_reference(args, world, rank)
        return

    from decode_attention_packed_b200 import mxa

    w = workload(args.workload)
    inp = shard_inputs(w, rank)
    if args.append and args.varlen:
        raise SystemExit("--append and --varlen do not combine")
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    q = inp.q.to(dev)
    bt = None if inp.block_table is None else inp.block_table.to(dev)
    sl = inp.cache_seqlens.to(dev)
    pools = [(inp.k_cache.to(dev), inp.v_cache.to(dev))]
    for _ in range(N_POOLS - 1):
        pools.append((pools[0][0].clone(), pools[0][1].clone()))
    splits = w.num_splits if args.num_splits is None else args.num_splits
    prep = mxa.prepare(q, pools[0][0], bt, max_seqlen_k=inp.max_seqlen_k, num_splits=splits)
    cu = hcu = None
    if args.varlen:  # the plan above is for q_len queries per row, which bounds every row's count
        q_lens = np.random.default_rng(w.seed + 77).integers(1, w.q_len + 1, size=w.B)
        hqv, hcu = make_varlen_queries(q_lens, w.Hq, w.D, w.dtype, w.seed + 78)
        q, cu = hqv.to(dev), hcu.to(dev)
        hcu = hcu.pin_memory()
    out = torch.empty_like(q)
    lse = (torch.empty((w.Hq, q.shape[0]), dtype=torch.float32, device=dev) if args.varlen
           else torch.empty((w.B, w.Hq, w.q_len), dtype=torch.float32, device=dev))
    nbytes = algorithmic_bytes(inp)
    if args.append:  # the new tokens are read and written once more
        nbytes["total"] += 2 * 2 * w.B * w.q_len * w.Hkv * w.D * inp.q.element_size()
    launches_per_call = 1  # the split kernel merges split units itself

    if args.append:
        # the rows' last q_len keys arrive as this step's new tokens: the call
        # writes them (the same values each step) and attends to all keys
        sl_before = (sl - w.q_len).clamp(min=0)
        k_new = torch.randn((w.B, w.q_len, w.Hkv, w.D), device=dev).to(q.dtype)
        v_new = torch.randn_like(k_new)

    def run(i, q, cu, bt, sl, out, lse):
        k, v = pools[i % N_POOLS]
        if args.append:
            mxa.mxa_decode_fwd_append(q, k, v, k_new, v_new, bt, sl, prep.params, w.scale, w.causal,
                                      prep.plan, prep.workspace, out, lse, stream)
        elif args.varlen:
            mxa.mxa_decode_fwd_varlen(q, cu, k, v, bt, sl, prep.params, w.scale, w.causal, prep.plan,
                                      prep.workspace, out, lse, stream)
        else:
            mxa.mxa_decode_fwd_with_plan(q, k, v, bt, sl, prep.params, w.scale, w.causal, prep.plan,
                                         prep.workspace, out, lse, stream)

    def call(i):
        run(i, q, cu, bt, sl_before if args.append else sl, out, lse)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier(device_ids=[local])
        torch.cuda.synchronize(dev)

    def max_over_ranks(x: float) -> float:
        if world == 1:
            return x
        import torch.distributed as dist
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    # ---- device-timed region: inputs resident in HBM ----
    for i in range(args.warmup):
        call(i)
    barrier()
    clocks = ClockSampler(local, enabled=not args.no_clocks)
    time.sleep(0.25 if not args.no_clocks else 0)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    e0.record(stream)
    for i in range(args.steps):
        call(i)
    e1.record(stream)
    barrier()
    clk = clocks.stop()
    dev_s = max_over_ranks(e0.elapsed_time(e1) / 1e3)
    assert mxa.mxa_device_error(True) == mxa.MXA_OK, "device-side wait ran out during the bench"

    # ---- spread of single calls: each call between its own pair of events
    # (so neighbouring calls do not overlap it), after the timed region ----
    n_each = max(1, min(args.steps, 2000))
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(n_each + 1)]
    barrier()
    ev[0].record(stream)
    for i in range(n_each):
        call(i)
        ev[i + 1].record(stream)
    barrier()
    each_us = sorted(ev[i].elapsed_time(ev[i + 1]) * 1e3 for i in range(n_each))
    pct = lambda f: round(each_us[min(n_each - 1, int(f * n_each))], 3)
    per_call = {"p10": pct(0.10), "p50": pct(0.50), "p90": pct(0.90), "n": n_each, "unit": "us",
                "how": "each call between its own events, back to back; the headline value is the mean "
                       "over the timed region"}

    # ---- end to end through the C ABI: every step copies its inputs from
    # pinned host memory (query, block table, lengths; the KV cache lives on
    # the device) and reads its result back (output and LSE).  As in a
    # serving loop the copies run on their own streams and overlap the
    # previous and next steps' kernels: inputs and outputs are double
    # buffered, and events order each buffer's copy-in, decode and copy-out.
    hq = (hqv if args.varlen else inp.q).pin_memory()
    hbt = None if inp.block_table is None else inp.block_table.pin_memory()
    hsl = ((inp.cache_seqlens - w.q_len).clamp(min=0) if args.append else inp.cache_seqlens).pin_memory()
    h2d = (hq.numel() * hq.element_size() + hsl.numel() * 4 + (0 if hbt is None else hbt.numel() * 4)
           + (0 if hcu is None else hcu.numel() * 4))
    d2h = out.numel() * out.element_size() + lse.numel() * 4
    e2e_steps = max(1, min(args.steps, 2000))
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    slots = []
    for _ in range(2):
        slots.append(dict(
            q=torch.empty_like(q), sl=torch.empty_like(sl), bt=None if bt is None else torch.empty_like(bt),
            cu=None if cu is None else torch.empty_like(cu),
            out=torch.empty_like(out), lse=torch.empty_like(lse),
            hout=torch.empty(out.shape, dtype=out.dtype, pin_memory=True),
            hlse=torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True),
            copied=torch.cuda.Event(), decoded=torch.cuda.Event(), read=torch.cuda.Event()))
    for sd in slots:  # every buffer starts out free
        sd["decoded"].record(stream)
        sd["read"].record(s_out)

    def e2e_step(i):
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
        run(i, sd["q"], sd["cu"], sd["bt"], sd["sl"], sd["out"], sd["lse"])
        sd["decoded"].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(sd["decoded"])
            sd["hout"].copy_(sd["out"], non_blocking=True)
            sd["hlse"].copy_(sd["lse"], non_blocking=True)
            sd["read"].record(s_out)

    for i in range(min(args.warmup, 50)):
        e2e_step(i)
    barrier()
    torch.cuda.synchronize(dev)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(s_in)
    for i in range(e2e_steps):
        e2e_step(i)
    s_out.wait_event(slots[(e2e_steps - 1) % 2]["read"])
    f1.record(s_out)
    barrier()
    torch.cuda.synchronize(dev)
    e2e_s = max_over_ranks(f0.elapsed_time(f1) / 1e3)
    for sd in slots:  # the last step's result arrived intact
        assert torch.equal(sd["hout"], sd["out"].cpu())

    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    peak, peak_kind = measured_peak()
    per_call_s = dev_s / args.steps
    kv_gbs = nbytes["kv"] / per_call_s / 1e9
    achieved = nbytes["total"] / per_call_s / 1e9
    line = {
        "metric": METRIC,
        "value": round(kv_gbs * world, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(dev_s / args.steps * 1e3, 5),
        "us_per_call": round(per_call_s * 1e6, 3),
        "per_call_us": per_call,
        "kv_frac_of_hbm_peak": round(kv_gbs / peak, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic",
        "config": dict(workload_config(w, nbytes, world), append=bool(args.append),
                       **({"varlen": {"q_lens": "U{1..%d} per row, seeded" % w.q_len,
                                      "total_q": int(q.shape[0])}} if args.varlen else {})),
        "plan": prep.plan.as_dict(),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4),
                     "traffic": MEASURED_TRAFFIC.get(kernel_source_hash())
                     if w.name == DEFAULT_WORKLOAD and not (args.append or args.varlen) else None,
                     "peak_kind": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                     else "fallback 6.65 TB/s",
                     "kernel": "mxa_split_kernel (one launch per call; split units merged inside)"},
        "e2e": {"value": round(nbytes["kv"] * world / (e2e_s / e2e_steps) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "copies": "pinned host buffers on their own streams, double buffered, overlapping the "
                          "neighbouring steps' kernels"},
        "gpu_launches": args.steps * launches_per_call,
        "clocks": clk,
    }
    if world == 1:
        line["cpu_baseline"] = cpu_baseline(inp)
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
