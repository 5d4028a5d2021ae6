"""Element-by-element comparison of CUDA results with the float64 oracle.

Tolerances:

* float32 output: |gpu - ref| <= 2e-3 (absolute);
* LSE (natural log): |gpu - ref| <= 1e-3 (absolute); -inf must match -inf exactly;
* bf16 output: at most one bf16 ulp at the value's magnitude, where the ulp of x is
  2^(floor(log2 |x|) - 7) (bf16 keeps 8 significant bits). At an exact-cancellation point the
  reference is far smaller than the row's typical value and the plain gate would demand more
  precision than any fp32-accumulating kernel has, so the magnitude used is
  max(|ref|, 2^-8 * max over the row of |ref|). The strict count (magnitude |ref| alone) is
  reported too, as is how many elements needed the floor.

Every comparison prints one ``PARITY`` line with its counts (pytest shows it with ``-rP`` or
``-s``); with FD_PARITY_LOG set to a file path the same record is appended there as JSON.
"""

from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

F32_TOL = 2e-3
LSE_TOL = 1e-3
ROW_FLOOR = 2.0 ** -8


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = x > 0
    out[nz] = np.exp2(np.floor(np.log2(x[nz])) - 7.0)
    return out


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def record(what: str, stats: dict) -> None:
    """Print one comparison's counts and append them to $FD_PARITY_LOG when it is set."""
    rec = {"what": what, **stats}
    print(f"PARITY {json.dumps(rec)}")
    path = os.environ.get("FD_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(rec) + "\n")


def check_out(gpu: torch.Tensor, ref: np.ndarray, what: str = "out") -> dict:
    """Compare outputs [..., D]. Rows of ref that are NaN (not computed) are skipped."""
    g = to_f64(gpu)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, f"{what}: shape {g.shape} vs {r.shape}"
    rows = ~np.isnan(r).any(axis=-1)
    g, r = g[rows], r[rows]
    assert np.isfinite(g).all(), f"{what}: non-finite GPU values"
    err = np.abs(g - r)
    if gpu.dtype == torch.float32:
        m = float(err.max()) if err.size else 0.0
        stats = {"dtype": "f32", "max_abs_err": m, "n": int(err.size)}
        record(what, stats)
        assert m <= F32_TOL, f"{what}: max abs err {m:.3e} > {F32_TOL}"
        return stats
    rowmax = np.abs(r).max(axis=-1, keepdims=True)
    mag = np.maximum(np.abs(r), ROW_FLOOR * rowmax)
    tol = bf16_ulp(mag)
    bad = err > tol
    strict_bad = err > bf16_ulp(np.abs(r))
    floor_used = np.abs(r) < ROW_FLOOR * rowmax
    stats = {"dtype": "bf16", "n": int(err.size), "fail": int(bad.sum()),
             "strict_fail": int(strict_bad.sum()), "floor_used": int(floor_used.sum()),
             "max_err_in_ulps": float((err / np.where(tol > 0, tol, np.inf)).max()) if err.size else 0.0}
    record(what, stats)
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {stats['fail']} of {stats['n']} elements beyond 1 bf16 ulp; "
                             f"first at {tuple(i)}: gpu {g[tuple(i)]!r} ref {r[tuple(i)]!r} "
                             f"tol {tol[tuple(i)]!r}; {stats}")
    return stats


def check_lse(gpu: torch.Tensor, ref: np.ndarray, what: str = "lse") -> dict:
    g = to_f64(gpu)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape
    sel = ~np.isnan(r)
    g, r = g[sel], r[sel]
    ninf = np.isneginf(r)
    assert np.array_equal(np.isneginf(g), ninf), f"{what}: -inf pattern differs"
    fin = ~ninf
    assert np.isfinite(g[fin]).all(), f"{what}: non-finite GPU LSE"
    m = float(np.abs(g[fin] - r[fin]).max()) if fin.any() else 0.0
    stats = {"dtype": "lse", "max_abs_err": m, "n": int(fin.sum()), "neg_inf": int(ninf.sum())}
    record(what, stats)
    assert m <= LSE_TOL, f"{what}: max abs err {m:.3e} > {LSE_TOL}"
    return stats
