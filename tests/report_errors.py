"""Raw parity figures per workload against the fp64 oracle (needs a CUDA device).

For each full-size workload, with the plan the benchmark uses, it prints:

- max |out - oracle| of the 16-bit output;
- the largest ratio of that error to the test bound, 2e-3 + half an output ulp;
- the share of 16-bit elements within a raw 2e-3;
- max |out - oracle| of the float32 output (mxa_decode_fwd_f32out: O before
  its one rounding), which the tests hold to a raw 2e-3;
- max |lse - oracle|.

Run from the repository root:

    python -m tests.report_errors
"""
import numpy as np
import torch

import oracle
from decode_attention_packed_b200 import mxa
from decode_attention_packed_b200.workloads import WORKLOADS, make_inputs
from tests.tolerance import out_errors


def main():
    print("| workload | max abs err (16-bit out) | max err / bound | share within raw 2e-3 "
          "| max abs err (float32 out) | max abs err (lse) |")
    print("|---|---|---|---|---|---|")
    for w in WORKLOADS:
        inp = make_inputs(w)
        ro, rl = oracle.decode(inp.q, inp.k_cache, inp.v_cache, inp.block_table, inp.cache_seqlens, Hkv=w.Hkv,
                               page_size=inp.page_size, dtype=w.dtype, scale=w.scale, causal=w.causal)
        d = "cuda"
        bt = None if inp.block_table is None else inp.block_table.to(d)
        args = (inp.q.to(d), inp.k_cache.to(d), inp.v_cache.to(d), bt, inp.cache_seqlens.to(d))
        kw = dict(scale=w.scale, causal=w.causal, num_splits=w.num_splits, max_seqlen_k=inp.max_seqlen_k)
        out, lse = mxa.decode(*args, **kw)
        o32, _ = mxa.decode(*args, **kw, out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert mxa.mxa_device_error(True) == mxa.MXA_OK
        err, bound = out_errors(out, ro, w.dtype)
        raw32 = float(np.abs(o32.cpu().double().numpy() - ro).max())
        g = lse.cpu().double().numpy()
        fin = np.isfinite(rl)
        lse_err = float(np.abs(g[fin] - rl[fin]).max()) if fin.any() else 0.0
        print(f"| {w.name} | {err.max():.3e} | {(err / bound).max():.3f} | {(err <= 2e-3).mean():.6f} "
              f"| {raw32:.3e} | {lse_err:.3e} |")


if __name__ == "__main__":
    main()
