"""Threshold calibration for synthetic inputs (test infrastructure only).

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

The per-position table of the paper is built too (``topk_threshold``,
``fixed_k_table``): for one query tile of one calibration sample, sort the
tile's off-diagonal (gated) block maxima and put tau between the k-th and the
(k+1)-th largest, so that exactly the top k are kept; average that value over
the calibration samples; one table column per query tile, one table per
sparsity level k (§4.2; App. B.3 "Threshold tensor"). Sequences that do not
fill their last tile are padded by repeating the last token before their
maxima are taken (App. B.3 "Practical considerations", ``pad_repeat_last``).
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


def topk_threshold(values, k: int) -> float:
    """The float32 threshold that keeps exactly the k largest of ``values`` (§4.2).

    With the values sorted descending, a[0] >= a[1] >= ..., it returns the midpoint
    of a[k] and a[k-1] when float32 can hold a value t with a[k] < t <= a[k-1],
    else the smallest such float32; the gate's ``s_max >= tau`` then keeps
    a[0..k-1] and skips the rest. When a[k] == a[k-1] no threshold separates them
    and every tied value is kept. With at most k values every block is kept
    (-inf); with k = 0, none is (just above a[0]).
    """
    a = np.sort(np.asarray(values, dtype=np.float64))[::-1]
    if k >= len(a):
        return float(-np.inf)
    up = np.float32(np.inf)
    if k <= 0:
        t = np.float32(a[0])
        return float(t if t > a[0] else np.nextafter(t, up))
    hi, lo = a[k - 1], a[k]
    t = np.float32(0.5 * (lo + hi))
    if lo < t <= hi:
        return float(t)
    t = np.float32(lo)
    if t <= lo:
        t = np.nextafter(t, up)
    if t <= hi:
        return float(t)
    t = np.float32(hi)                       # a tie at the cut: keep all of it
    return float(t if t <= hi else np.nextafter(t, np.float32(-np.inf)))


def pad_repeat_last(bits: np.ndarray, multiple: int) -> np.ndarray:
    """[B, N, H, D] -> [B, N', H, D] with N' the next multiple of ``multiple``, the
    new positions holding copies of token N-1 (App. B.3 "Practical considerations")."""
    N = bits.shape[1]
    pad = (-N) % multiple
    if pad == 0:
        return bits
    tail = np.repeat(bits[:, N - 1:N], pad, axis=1)
    return np.concatenate([bits, tail], axis=1)


def tile_gated_maxima(q_bits, k_bits, Bq: int, Bk: int, causal: bool) -> dict:
    """{(b, hq, i): gated block maxima of that query tile} for one calibration sample.

    A sequence that does not fill its last query tile or key block is first padded
    by repeating its last token, so the tile has no artificial rows or keys. Tiles
    and blocks made of padding only are not part of the sequence and are dropped.
    """
    N = q_bits.shape[1]
    mq, mkv = -(-N // Bq), -(-N // Bk)
    multiple = int(np.lcm(Bq, Bk))
    qp, kp = pad_repeat_last(q_bits, multiple), pad_repeat_last(k_bits, multiple)
    maxima = block_maxima(qp, kp, Bq, Bk, causal)
    return {key: smax[:mkv][codes[:mkv] == CODE_SKIPPED] for key, (codes, smax) in maxima.items() if key[2] < mq}


def fixed_k_table(samples, Bq: int, Bk: int, causal: bool, ks) -> np.ndarray:
    """T[level, hq, i] (float32) for one layer: the top-k threshold of every query
    tile, averaged over the calibration samples (§4.2; App. B.3 "Threshold tensor").

    samples: a list of (q_bits, k_bits) pairs of one length; every batch entry of a
    sample counts as a calibration sample. ks: the retained-block counts, one table
    level each. A tile with at most k gated blocks keeps them all (-inf).
    """
    per_sample = [tile_gated_maxima(q, k, Bq, Bk, causal) for (q, k) in samples]
    _, N, Hq, _ = samples[0][0].shape
    T = np.zeros((len(ks), Hq, -(-N // Bq)), dtype=np.float32)
    for li, k in enumerate(ks):
        cuts = {}
        for m in per_sample:
            for (b, hq, i), vals in m.items():
                cuts.setdefault((hq, i), []).append(topk_threshold(vals, k))
        for (hq, i), v in cuts.items():
            T[li, hq, i] = np.float32(np.mean(v))
    return T
