"""Shared test helpers: tolerances, golden-file reader, comparison report.

Tolerances (absolute + relative to the unrounded fp64 oracle value):
  * fp16 output: |out - ref| <= 1e-2 + 2e-3 * |ref|
  * fp32 output: |out - ref| <= 1e-3 + 1e-4 * |ref|
  * bf16 output: |out - ref| <= 1e-2 + 4e-3 * |ref|.  bf16 keeps 8 significand
    bits, so the cast alone may move a value by up to 2^-8 = 3.9e-3 of its
    magnitude; the fp16 bound's 2e-3 relative term would be tighter than the
    format can represent, and 4e-3 covers the half-ulp of the cast.
"""
from __future__ import annotations

import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

TOL = {
    torch.float16: (1e-2, 2e-3),
    torch.float32: (1e-3, 1e-4),
    torch.bfloat16: (1e-2, 4e-3),
}


def tolerance(ref: np.ndarray, out_dtype: torch.dtype) -> np.ndarray:
    atol, rtol = TOL[out_dtype]
    return atol + rtol * np.abs(ref)


def check_close(out, ref: np.ndarray, out_dtype: torch.dtype, relu: bool, what: str = ""):
    """Assert element-wise parity; return (max_abs_err, max_err_over_tol)."""
    o = np.asarray(out.float().cpu().numpy() if isinstance(out, torch.Tensor) else out,
                   dtype=np.float64)
    assert o.shape == ref.shape, (o.shape, ref.shape)
    assert np.all(np.isfinite(o)), f"{what}: non-finite output"
    if relu:
        assert np.all(o >= 0), f"{what}: negative output with relu"
    err = np.abs(o - ref)
    tol = tolerance(ref, out_dtype)
    bad = err > tol
    if bad.any():
        idx = np.argwhere(bad)[:5]
        details = [(tuple(int(v) for v in i), float(o[tuple(i)]), float(ref[tuple(i)]))
                   for i in idx]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; "
                             f"first (index, out, ref): {details}")
    return float(err.max(initial=0.0)), float((err / tol).max(initial=0.0))


def read_golden(name: str) -> dict[str, np.ndarray]:
    """Parse a golden text file: '# comments', then blocks 'NAME rows cols' + rows."""
    out: dict[str, np.ndarray] = {}
    with open(os.path.join(GOLDEN, name)) as f:
        lines = [ln.strip() for ln in f if ln.strip() and not ln.lstrip().startswith("#")]
    i = 0
    while i < len(lines):
        key, r, c = lines[i].split()
        r, c = int(r), int(c)
        rows = [[float(v) for v in lines[i + 1 + k].split()] for k in range(r)]
        arr = np.array(rows, dtype=np.float64)
        assert arr.shape == (r, c), (key, arr.shape)
        out[key] = arr
        i += 1 + r
    return out
