"""Shared helpers of the GPU parity tests: run a workload through the library (C ABI via
the ctypes binding) and through the float64 oracle, and compare them.

Tolerance, per output tensor, over valid rows: max|err| <= 1e-2 * max|ref| + 1e-3
(bf16 inputs, fp32 accumulation, bf16 outputs).  Pad rows must be exactly zero.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import attention as A
from padded_variable_length_b200 import workloads as W

RTOL_MAX = 1e-2
ATOL = 1e-3


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def oracle_bias(w: W.Workload, epilogue: int) -> np.ndarray:
    if epilogue == A.SIGMOID:
        return A.bias_from_counts(w.counts)
    return np.zeros((w.B, w.Nq))


def device_setup(w: W.Workload, t: dict, dev="cuda"):
    """Uploads inputs; builds the plan and the bias with the library's own kernels."""
    from padded_variable_length_b200 import binding as Bd
    Bd.set_wait_limit_ns(500_000_000)  # no legitimate wait inside one CTA comes near this
    d = {k: v.to(dev) for k, v in t.items()}
    if w.lengths is not None:
        lengths = torch.from_numpy(w.lengths.astype(np.int32)).to(dev)
        plan = Bd.Plan.from_lengths(lengths, w.Nq)
    else:
        mask = torch.from_numpy(w.mask).to(dev)
        plan = Bd.Plan.from_mask(mask)
    counts = torch.from_numpy(np.ascontiguousarray(w.counts, dtype=np.int32)).to(dev)
    bias = Bd.bias_from_counts(counts)
    return d, plan, bias


def valid_rows_q(w: W.Workload) -> np.ndarray:
    """bool [B, Nq]: rows that are not padding (for element masks: all rows)."""
    if w.lengths is not None:
        return np.arange(w.Nq)[None, :] < w.lengths[:, None]
    return np.ones((w.B, w.Nq), dtype=bool)


def valid_rows_k(w: W.Workload) -> np.ndarray:
    if w.lengths is not None:
        return np.arange(w.Nk)[None, :] < w.lengths[:, None]
    return np.ones((w.B, w.Nk), dtype=bool)


def check_close(got: np.ndarray, ref: np.ndarray, name: str, rows=None):
    """got/ref [B, N, H, d]; rows: bool [B, N] selecting rows to compare."""
    if rows is not None:
        got = got[rows]
        ref = ref[rows]
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    err = float(np.max(np.abs(got - ref))) if got.size else 0.0
    mref = float(np.max(np.abs(ref))) if ref.size else 0.0
    tol = RTOL_MAX * mref + ATOL
    assert err <= tol, f"{name}: max|err| {err:.3e} > tol {tol:.3e} (max|ref| {mref:.3e})"
    return err, tol


def check_pad_zero(got: np.ndarray, w: W.Workload, name: str, side="q"):
    if w.lengths is None:
        return
    valid = valid_rows_q(w) if side == "q" else valid_rows_k(w)
    pad = got[~valid]
    assert np.all(pad == 0), f"{name}: pad rows not exactly zero"
