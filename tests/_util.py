"""Helpers shared by the GPU parity tests (no method arithmetic here)."""
from __future__ import annotations

import os

import numpy as np
import torch

import oracle

# |gpu - oracle| <= 1e-2 * max|oracle| + 2^-7 * |oracle|, per element, with the
# max taken over the compared output of the call.
TOL_ABS_OF_MAX = 1e-2
TOL_REL = 2.0 ** -7


def set_oracle_threads():
    oracle.set_threads(os.cpu_count() or 1)


def to_dev_bf16(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def to_dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_within_tolerance(gpu: np.ndarray, ref: np.ndarray, what: str = "") -> float:
    """Checks the per-element bound; returns the worst ratio err / bound."""
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(ref)), f"{what}: oracle produced non-finite values"
    amax = float(np.abs(ref).max()) if ref.size else 0.0
    bound = TOL_ABS_OF_MAX * amax + TOL_REL * np.abs(ref)
    err = np.abs(gpu - ref)
    bad = ~(err <= bound)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(
            f"{what}: {int(bad.sum())}/{bad.size} elements out of tolerance; max|ref|={amax:.4g}; first "
            + ", ".join(f"{tuple(i)}: gpu={gpu[tuple(i)]:.6g} ref={ref[tuple(i)]:.6g}" for i in idx))
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(bound > 0, err / bound, 0.0)
    return float(ratio.max()) if ratio.size else 0.0


def offsets_from_counts(counts) -> np.ndarray:
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)


def sample_rows(offsets: np.ndarray, per_group: int = 2, extra=(), seed: int = 0, limit: int | None = None):
    """First and last row of up to `per_group`-sampled non-empty groups plus `extra` rows."""
    rng = np.random.default_rng(seed)
    rows = set(int(r) for r in extra)
    E = offsets.shape[0] - 1
    nonempty = [e for e in range(E) if offsets[e + 1] > offsets[e]]
    for e in nonempty:
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        rows.add(lo)
        rows.add(hi - 1)
        if hi - lo > 2:
            rows.update(int(x) for x in rng.integers(lo, hi, size=min(per_group, hi - lo)))
    rows = np.array(sorted(rows), np.int64)
    if limit is not None and rows.size > limit:
        keep = np.unique(np.concatenate([rows[:limit // 4], rows[-limit // 4:],
                                         rng.choice(rows, size=limit // 2, replace=False)]))
        rows = keep
    return rows
