"""Helpers for the GPU-vs-oracle parity tests (CPU side only)."""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence

import numpy as np

import oracle as O

# Output tolerances for bf16 I/O (and f32 inputs rounded to bf16 for the
# tensor-core products): maximum absolute error and relative Frobenius error.
MAX_ABS_TOL = 2e-2
REL_FRO_TOL = 1e-2

# Selection: a swap between the GPU's and the oracle's exact sets is a
# rounding tie when every swapped block's fp64 score lies within this
# relative bound (times the sum of |terms| of its score) of the k-th score.
# The GPU's float32 score has error <= ~ (d + 2 * block_size) * 2^-24 * sum|terms|
# (dot product of d terms plus the rounding of the float32 block means).
TIE_REL = 2e-5


def to64(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def score_magnitude(qbar, kbar, scale, cov=None, cov_weight=0.0, rows=None):
    qb = qbar if rows is None else qbar[np.asarray(rows)]
    mag = abs(scale) * (np.abs(qb) @ np.abs(kbar).T)
    if cov_weight != 0.0:
        mag = mag + abs(cov_weight) * np.abs(cov)[None, :]
    return mag


@dataclass
class SelectionReport:
    rows: int = 0
    exact_rows: int = 0
    tie_rows: List[int] = field(default_factory=list)
    bad_rows: List[int] = field(default_factory=list)


def compare_selection(gpu_idx: np.ndarray, orc: Dict, scale: float, cov_weight: float,
                      sink_idx: Optional[int]) -> SelectionReport:
    """gpu_idx: [rows, k_sel] for the rows orc['rows'] of one head."""
    rep = SelectionReport()
    sc = orc["scores"]
    mag = score_magnitude(orc["qbar"], orc["kbar"], scale, orc["cov"], cov_weight, orc["rows"])
    N = orc["kbar"].shape[0]
    sink = None if sink_idx is None else (0 if sink_idx == 0 else N - 1)
    for r, i in enumerate(orc["rows"]):
        rep.rows += 1
        g = set(int(x) for x in gpu_idx[r])
        o = set(int(x) for x in orc["idx"][r])
        if g == o and len(g) == gpu_idx.shape[1]:
            rep.exact_rows += 1
            continue
        if len(g) != gpu_idx.shape[1] or (sink is not None and sink not in g):
            rep.bad_rows.append(int(i))
            continue
        cand = [j for j in o if j != sink]
        if not cand:
            rep.bad_rows.append(int(i))
            continue
        thr = min(sc[r, j] for j in cand)
        swapped = (g ^ o) - ({sink} if sink is not None else set())
        ok = all(abs(sc[r, j] - thr) <= TIE_REL * max(mag[r, j], 1e-30) for j in swapped)
        (rep.tie_rows if ok else rep.bad_rows).append(int(i))
    return rep


def output_errors(gpu_out: np.ndarray, ref: np.ndarray):
    d = gpu_out - ref
    max_abs = float(np.abs(d).max()) if d.size else 0.0
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-30)) if d.size else 0.0
    return max_abs, rel


def block_rows(L: int, block_size: int, blocks: Sequence[int]) -> np.ndarray:
    rows = []
    for i in blocks:
        rows.extend(range(i * block_size, min((i + 1) * block_size, L)))
    return np.asarray(rows, dtype=np.int64)
