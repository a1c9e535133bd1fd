"""Tolerance of attention outputs against the fp64 oracle.

Bound: max abs error <= 1e-2 and mean abs error <= 1e-3 (bf16/fp16 output,
fp32 accumulation). Where the output format itself cannot meet 1e-2 -- a bf16
value of magnitude >= 4 is spaced 2^-5 apart, so even the correctly rounded
result can be 0.0156 away -- an element may instead be within one unit in the
last place of the output format at the reference value. The number of
elements that needed that allowance is reported.
"""
from __future__ import annotations

import numpy as np

ATOL = 1e-2
MEAN_TOL = 1e-3


def out_ulp(ref: np.ndarray, dtype: str) -> np.ndarray:
    a = np.abs(np.asarray(ref, dtype=np.float64))
    if dtype == "f16":
        e = np.floor(np.log2(np.maximum(a, 2.0 ** -14)))
        return 2.0 ** (e - 10)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def compare(got: np.ndarray, ref: np.ndarray, dtype: str) -> dict:
    got = np.asarray(got, dtype=np.float64)
    err = np.abs(got - ref)
    tol = np.maximum(ATOL, out_ulp(ref, dtype))
    finite = np.isfinite(got)
    bad = (err > tol) | ~finite
    floor = np.abs(_round_like(ref, dtype) - ref)
    return {
        "n": int(err.size),
        "max_abs": float(err.max()) if err.size else 0.0,
        "mean_abs": float(err.mean()) if err.size else 0.0,
        "n_bad": int(bad.sum()),
        "n_ulp_branch": int(((err > ATOL) & ~bad).sum()),
        "rounding_floor_mean": float(floor.mean()) if floor.size else 0.0,
    }


def assert_close(got, ref, dtype, what=""):
    s = compare(got, ref, dtype)
    assert s["n_bad"] == 0, f"{what}: {s['n_bad']} elements outside tolerance; {s}"
    assert s["mean_abs"] <= MEAN_TOL, f"{what}: mean abs error {s['mean_abs']}; {s}"
    return s


def _round_like(x, dtype):
    import torch
    t = torch.from_numpy(np.asarray(x, dtype=np.float64))
    return t.to(torch.float16 if dtype == "f16" else torch.bfloat16).to(torch.float64).numpy()
