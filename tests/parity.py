"""Comparison helpers for GPU-vs-oracle parity tests.

Tolerances (stated once, used by every parity test):
  * selection: kept-tile sets bit-exact, except rows whose differing tiles all
    score within TIE_REL (relative, in the oracle's fp64) of the row's k-th
    score -- a near-tie the fp32 kernels may legitimately order either way;
    every such row is reported.
  * selector projections q̂, k̂ (fp32 on the device): each element within
    the forward error bound of fp32 summation (Higham, "Accuracy and
    Stability of Numerical Algorithms", section 3.1: a sum of n terms in any
    order is off by at most gamma_(n-1) times the sum of the terms' magnitudes,
    gamma_n = n u / (1 - n u), u = 2^-24).  The tile mean (T terms, one
    division) and the projection (d multiply-adds) together give
    |err_c| <= (gamma_(T+1) + gamma_(d+1)) * sum_e |W[e, c]| * mean_t |x[t, e]|.
  * attention, fp32 problems: max-abs <= 1e-4 and relative L2 <= 1e-4.
  * attention, bf16 problems: max-abs <= 2e-2 and relative L2 <= 5e-3
    (the output itself is rounded to bf16, 2^-9 relative).
"""
from __future__ import annotations

import warnings
from dataclasses import dataclass, field
from typing import List

import numpy as np
import torch

TIE_REL = 1e-4
TOL = {torch.float32: (1e-4, 1e-4), torch.bfloat16: (2e-2, 5e-3)}


U32 = 2.0 ** -24


def gamma(n: int) -> float:
    return n * U32 / (1.0 - n * U32)


def assert_projection_within_bound(oracle_mod, got: np.ndarray, want: np.ndarray, x: torch.Tensor,
                                   w: torch.Tensor, T: int, what: str = ""):
    """got: the device's fp32 projection [B,H,n,r]; want: the oracle's fp64;
    x: the pooled input [B,N,H,d]; w: the weights [H,d,r]."""
    d = x.shape[-1]
    mag = oracle_mod.project(oracle_mod.pool(x.abs(), T), w.abs())
    bound = (gamma(T + 1) + gamma(d + 1)) * mag
    err = np.abs(got - want)
    worst = float(np.max(err / np.maximum(bound, 1e-300)))
    assert worst <= 1.0, f"{what}: projection error {worst:.3g} x the fp32 summation bound"


@dataclass
class SelectionReport:
    rows: int
    mismatched: int = 0
    tie_band: List[int] = field(default_factory=list)
    violations: List[int] = field(default_factory=list)


class TieBandReport(UserWarning):
    """A kept-tile row that differs from the oracle only inside the tie band
    (reported, as the selection contract requires, not a failure)."""


def compare_selection(oracle_mod, gpu_idx: np.ndarray, ref_idx: np.ndarray, kth: np.ndarray,
                      qhat: np.ndarray, khat: np.ndarray) -> SelectionReport:
    """Rows of kept tiles from the GPU against the oracle's.

    A row is valid only when it holds `budget` distinct in-range indices in
    strictly ascending order.  A valid row that differs from the oracle's is
    inside the tie band when every tile in the symmetric difference scores
    within TIE_REL (relative, oracle fp64) of the row's k-th score; anything
    else -- an invalid row, a row with the oracle's set in another order, or a
    swap outside the band -- is a violation."""
    g = gpu_idx.reshape(-1, gpu_idx.shape[-1])
    o = ref_idx.reshape(-1, ref_idx.shape[-1])
    rep = SelectionReport(rows=g.shape[0])
    nk = khat.shape[2]
    ascending = (np.diff(g, axis=1) > 0).all(axis=1) if g.shape[1] > 1 else np.ones(g.shape[0], bool)
    in_range = ((g >= 0) & (g < nk)).all(axis=1)
    invalid = ~(ascending & in_range)
    rep.violations.extend(int(x) for x in np.nonzero(invalid)[0])
    bad = np.nonzero((g != o).any(axis=1) & ~invalid)[0]
    rep.mismatched = int(len(bad) + invalid.sum())
    if len(bad) == 0:
        return rep
    s = oracle_mod.scores(qhat, khat, bad)
    kth_flat = kth.reshape(-1)
    for q, row in enumerate(bad):
        diff = set(g[row].tolist()) ^ set(o[row].tolist())
        if not diff:                     # same set, another order: cannot happen for a valid row
            rep.violations.append(int(row))
            continue
        sk = kth_flat[row]
        ok = all(abs(s[q, j] - sk) <= TIE_REL * max(abs(s[q, j]), abs(sk)) for j in diff)
        (rep.tie_band if ok else rep.violations).append(int(row))
    rep.violations.sort()
    return rep


def assert_selection(rep: SelectionReport, what: str = ""):
    assert not rep.violations, (f"{what}: {len(rep.violations)} rows differ outside the tie band or are not "
                                f"strictly ascending in-range lists (first {rep.violations[:5]})")
    if rep.tie_band:
        warnings.warn(f"{what}: {len(rep.tie_band)} of {rep.rows} kept-tile rows differ from the oracle only "
                      f"inside the {TIE_REL:g} relative tie band (rows {rep.tie_band[:10]})", TieBandReport)


def errors(got: np.ndarray, want: np.ndarray):
    m = ~np.isnan(want)
    d = got[m] - want[m]
    max_abs = float(np.abs(d).max()) if d.size else 0.0
    rel_l2 = float(np.linalg.norm(d) / max(np.linalg.norm(want[m]), 1e-30)) if d.size else 0.0
    return max_abs, rel_l2


def assert_close(got: np.ndarray, want: np.ndarray, dtype, what: str = ""):
    tol_abs, tol_rel = TOL[dtype]
    max_abs, rel_l2 = errors(got, want)
    assert np.isfinite(got[~np.isnan(want)]).all(), f"{what}: non-finite output"
    assert max_abs <= tol_abs and rel_l2 <= tol_rel, \
        f"{what}: max-abs {max_abs:.3g} (<= {tol_abs}), rel-L2 {rel_l2:.3g} (<= {tol_rel})"
    return max_abs, rel_l2


def gather_units(out: torch.Tensor, units, T: int) -> np.ndarray:
    """GPU output [B, N, H, d] -> [n_units, T, d] fp64 (NaN past the end)."""
    B, N, H, d = out.shape
    res = np.full((len(units), T, d), np.nan)
    host = {}
    for u, (b, h, i) in enumerate(units):
        t0, t1 = i * T, min(N, (i + 1) * T)
        res[u, :t1 - t0] = out[b, t0:t1, h].float().cpu().double().numpy()
    return res


def gather_lse(lse: torch.Tensor, units, T: int) -> np.ndarray:
    B, H, N = lse.shape
    res = np.full((len(units), T), np.nan)
    for u, (b, h, i) in enumerate(units):
        t0, t1 = i * T, min(N, (i + 1) * T)
        res[u, :t1 - t0] = lse[b, h, t0:t1].cpu().double().numpy()
    return res
