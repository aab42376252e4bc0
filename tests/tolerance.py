"""Parity tolerance between the CUDA output and the fp64 oracle.

The bar is |gpu - oracle| <= 2e-3 + ulp_out(|oracle|) / 2 per element for
16-bit outputs: 2e-3 absolute for the computation, plus the half unit in the
last place that rounding an exact result to the output type costs by itself
(a bf16 output of magnitude 1 already carries up to 2^-9 of rounding).  LSE
(fp32) within 1e-4 absolute, with identical -inf positions.

A float32 output (mxa_decode_fwd_f32out: O before its one rounding) is held
to the raw 2e-3 with no rounding allowance (assert_out_raw).
"""
import numpy as np
import torch

ABS_TOL = 2e-3
LSE_TOL = 1e-4


def ulp(x: np.ndarray, dtype: str) -> np.ndarray:
    """Spacing of the 16-bit output type at |x| (normal and subnormal ranges)."""
    mant, emin = (7, -126) if dtype == "bf16" else (10, -14)
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    e = np.maximum(e, emin)
    return np.exp2(e - mant)


def out_errors(gpu: torch.Tensor, ref: np.ndarray, dtype: str):
    g = gpu.detach().float().cpu().double().numpy()
    err = np.abs(g - ref)
    bound = ABS_TOL + 0.5 * ulp(ref, dtype)
    return err, bound


def assert_out_close(gpu: torch.Tensor, ref: np.ndarray, dtype: str, what: str = "out"):
    err, bound = out_errors(gpu, ref, dtype)
    assert np.isfinite(err).all(), f"{what}: non-finite output"
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {err.size} elements out of tolerance; worst at {i}: "
                             f"gpu={gpu.flatten()[np.ravel_multi_index(i, err.shape)].item()} "
                             f"ref={ref[i]} err={err[i]:.3e} bound={bound[i]:.3e}")
    return float(err.max()) if err.size else 0.0


def assert_out_raw(gpu: torch.Tensor, ref: np.ndarray, what: str = "out", tol: float = ABS_TOL):
    """|gpu - oracle| <= tol element by element, with no allowance for output
    rounding: for outputs that carry the computation's own float32 result."""
    g = gpu.detach().cpu().double().numpy()
    err = np.abs(g - ref)
    assert np.isfinite(err).all(), f"{what}: non-finite output"
    if err.size and err.max() > tol:
        i = np.unravel_index(np.argmax(err), err.shape)
        raise AssertionError(f"{what}: {(err > tol).sum()} of {err.size} elements above {tol}; worst at {i}: "
                             f"gpu={g[i]} ref={ref[i]} err={err[i]:.3e}")
    return float(err.max()) if err.size else 0.0


def assert_lse_close(gpu: torch.Tensor, ref: np.ndarray, what: str = "lse"):
    g = gpu.detach().cpu().double().numpy()
    assert (np.isneginf(g) == np.isneginf(ref)).all(), f"{what}: -inf pattern differs"
    fin = np.isfinite(ref)
    assert np.isfinite(g[fin]).all(), f"{what}: non-finite values"
    if fin.any():
        d = np.abs(g[fin] - ref[fin])
        assert d.max() <= LSE_TOL, f"{what}: max |diff| {d.max():.3e} > {LSE_TOL}"
        return float(d.max())
    return 0.0
