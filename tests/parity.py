"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (from the hot path's specification):
  * selected block sets identical, except swaps between blocks whose oracle
    scores differ by less than 1e-4 relative (each such swap is reported);
  * sketched scores within 1e-3 relative, read as
    |S_gpu - S_oracle| <= 1e-3 * max(|S_oracle|, rms of the row), because a
    pure relative error is meaningless for entries near zero;
  * attention outputs within 2e-2 max-abs and 5e-3 mean-abs of the oracle
    computed with the same mask (the GPU's selection fed to the oracle).
"""
from __future__ import annotations

import math

import numpy as np
import torch

TIE_REL = 1e-4
SCORE_REL = 1e-3
ATTN_MAX_ABS = 2e-2
ATTN_MEAN_ABS = 5e-3


# Tolerated near-tie swaps per test, filled by record_ties and summarised at the
# end of the session (conftest.py prints the counts and writes them as JSON).
TIE_REPORT: dict = {}


def record_ties(swaps, compared: int = 0, name: str = None):
    """Adds a test's tolerated swaps (each a tuple ending in the oracle's relative
    gap) and the number of selections it compared to the session's tie report,
    under the running test's id unless a name is given."""
    if name is None:
        import os
        name = os.environ.get("PYTEST_CURRENT_TEST", "unnamed").rsplit(" (", 1)[0].split("::", 1)[-1]
    e = TIE_REPORT.setdefault(name, {"swaps": 0, "selections_compared": 0, "largest_gap": 0.0, "examples": []})
    e["swaps"] += len(swaps)
    e["selections_compared"] += int(compared)
    for s in swaps:
        e["largest_gap"] = max(e["largest_gap"], float(s[-1]))
        if len(e["examples"]) < 5:
            e["examples"].append([float(x) if isinstance(x, float) else int(x) for x in s])


class LazyHeads:
    """Indexable view of a [H, n, d] tensor that widens one head at a time to fp64 numpy."""

    def __init__(self, t: torch.Tensor):
        self.t = t
        self.shape = tuple(t.shape)

    def __getitem__(self, h):
        return self.t[h].to(torch.float64).cpu().numpy()


def check_csr_valid(row_ptr: np.ndarray, col_idx: np.ndarray, b: int, num: int, den: int):
    assert row_ptr[0] == 0
    for i in range(b):
        tau = -(-(i + 1) * num // den)
        cols = col_idx[row_ptr[i]:row_ptr[i + 1]]
        assert len(cols) == tau, (i, len(cols), tau)
        assert np.all(np.diff(cols) > 0), (i, cols)
        assert cols.min() >= 0 and cols.max() <= i, (i, cols)


def compare_selection(gpu_sel, oracle_sel, score_row, rel=TIE_REL, log_domain=False):
    """Returns the list of tolerated swaps (gpu_only, oracle_only, rel_gap); raises on a real mismatch."""
    g, o = set(int(x) for x in gpu_sel), set(int(x) for x in oracle_sel)
    if g == o:
        return []
    go, og = sorted(g - o), sorted(o - g)
    assert len(go) == len(og), (go, og)
    swaps = []
    for a, c in zip(go, og):
        if log_domain:
            gap = abs(1.0 - math.exp(-abs(score_row[a] - score_row[c])))
        else:
            m = max(abs(score_row[a]), abs(score_row[c]))
            gap = abs(score_row[a] - score_row[c]) / m if m > 0 else 0.0
        assert gap < rel, f"selection differs beyond the tie tolerance: gpu-only {a}, oracle-only {c}, gap {gap:.3e}"
        swaps.append((a, c, gap))
    return swaps


def compare_csr(gpu_rp, gpu_ci, oracle_rp, oracle_ci, R, rows=None):
    swaps = []
    b = len(oracle_rp) - 1
    for i in (range(b) if rows is None else rows):
        s = compare_selection(gpu_ci[gpu_rp[i]:gpu_rp[i + 1]], oracle_ci[oracle_rp[i]:oracle_rp[i + 1]], R[i])
        swaps += [(i,) + x for x in s]
    return swaps


def compare_scores(S_gpu: np.ndarray, S_oracle: np.ndarray):
    b = S_oracle.shape[0]
    low = np.tril(np.ones((b, b), dtype=bool))
    So = np.where(low, S_oracle, 0.0)
    rms = np.sqrt((So ** 2).sum(axis=1) / np.arange(1, b + 1))
    bound = SCORE_REL * np.maximum(np.abs(So), rms[:, None])
    err = np.abs(np.where(low, S_gpu, 0.0) - So)
    assert np.all(err <= bound), f"sketch scores: worst ratio {(err / np.maximum(bound, 1e-300)).max():.3e}"
    return float((err / np.maximum(np.maximum(np.abs(So), rms[:, None]), 1e-300)).max())


def compare_walk(R_gpu: np.ndarray, R_oracle: np.ndarray, rel=1e-6):
    low = np.tril(np.ones(R_oracle.shape, dtype=bool))
    assert np.all(R_gpu[~low] == 0.0)
    m = low & (R_oracle > 1e-280)
    err = np.abs(R_gpu[m] - R_oracle[m]) / R_oracle[m]
    assert err.max() <= rel, f"walk state relative error {err.max():.3e}"
    return float(err.max())


def compare_attention(O_gpu: np.ndarray, O_oracle: np.ndarray):
    d = np.abs(np.asarray(O_gpu, dtype=np.float64) - O_oracle)
    assert np.isfinite(O_gpu).all()
    assert d.max() <= ATTN_MAX_ABS, f"attention max-abs {d.max():.3e}"
    assert d.mean() <= ATTN_MEAN_ABS, f"attention mean-abs {d.mean():.3e}"
    return float(d.max()), float(d.mean())
