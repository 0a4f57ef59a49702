"""Per-head threshold calibration for synthetic inputs (test infrastructure only).

The paper calibrates a threshold table offline: per query position it sorts the
off-diagonal block maxima and takes the value that keeps exactly the top-k
blocks, averaged over calibration samples ("Block Sparse Flash Attention",
§4.2 "Threshold Calibration" and App. B.3 "Threshold tensor").

The workloads here use one threshold per query head, so the same rule is taken
per head over every gated (visible, off-diagonal) block of that head: sort the
block maxima ascending, and for a target skip fraction p put tau in the gap
near the n-th value, n = round(p * count): among the ranks within 0.2% of n it
takes the widest gap between neighbouring maxima and puts tau at its midpoint,
rounded to float32, so that tau sits as far as it can from every block maximum.
The achieved skip fraction is reported, not assumed.
"""
from __future__ import annotations

import numpy as np

from .bsfa_oracle import CODE_SKIPPED, block_maxima

RANK_WINDOW = 0.002


def tau_for_skip(values: np.ndarray, p: float, window: float = RANK_WINDOW) -> float:
    """Threshold that skips a fraction ~p of ``values`` (block maxima), as a float32 value.

    With the values sorted ascending and n = round(p * count), tau is the midpoint
    of the widest gap a[m-1] < tau <= a[m] among the ranks m within
    +-round(window * count) of n (ties go to the rank nearest n). This keeps the
    skipped fraction within ``window`` of p while keeping tau as far as possible
    from every block maximum.
    """
    a = np.sort(np.asarray(values, dtype=np.float64))
    n_total = len(a)
    if n_total == 0:
        return float(np.float32(-np.inf))
    n = int(round(p * n_total))
    if n <= 0:
        return float(np.float32(a[0] - 1.0))
    if n >= n_total:
        return float(np.float32(a[-1] + 1.0))
    w = int(round(window * n_total))
    ranks = range(max(1, n - w), min(n_total - 1, n + w) + 1)
    order = sorted(ranks, key=lambda m: (-(a[m] - a[m - 1]), abs(m - n), m))
    for m in order:
        t = float(np.float32(0.5 * (a[m - 1] + a[m])))
        if a[m - 1] < t <= a[m]:
            return t
    return float(np.float32(0.5 * (a[n - 1] + a[n])))


def gated_maxima(maxima: dict, Hq: int) -> list[np.ndarray]:
    """Collect, per head, the block maxima of every gated block from ``block_maxima`` output."""
    per_head = [[] for _ in range(Hq)]
    for (b, hq, i), (codes, smax) in maxima.items():
        sel = codes == CODE_SKIPPED           # at tau=+inf every gated block reads "skipped"
        per_head[hq].append(smax[sel])
    return [np.concatenate(v) if v else np.zeros(0) for v in per_head]


def calibrate(q_bits, k_bits, Bq: int, Bk: int, causal: bool, skips, tiles=None) -> dict:
    """{p: [tau_h for each head]} for each target skip fraction p."""
    Hq = q_bits.shape[2]
    maxima = block_maxima(q_bits, k_bits, Bq, Bk, causal, tiles)
    vals = gated_maxima(maxima, Hq)
    return {float(p): [tau_for_skip(vals[h], p) for h in range(Hq)] for p in skips}
