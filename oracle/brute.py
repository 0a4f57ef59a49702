"""Scalar brute force of the BSFA definition (test infrastructure only).

A second statement of the same definition as ``bsfa_oracle``, written as plain
Python loops with no BLAS and no vectorisation, for tiny inputs only. It does
not reuse the oracle's geometry helpers: block visibility, the forced
("diagonal") blocks and the block maxima are found here by enumerating the
(query, key) pairs of each block.

Source: "Block Sparse Flash Attention" (paperpeel.com/paper/2512.07011),
§4.1 "Gating Mechanism" (gate on the exact block maximum; diagonal blocks bypass
it), §4.4 (skipped blocks stay out of the running statistics), App. B.2 (scaled
scores, softmax), App. B.3 (bidirectional case).
"""
from __future__ import annotations

import math


def _is_valid(r: int, c: int, causal: bool) -> bool:
    return c <= r if causal else True


def _threshold(tau, hq: int, i: int) -> float:
    """tau[hq] when it is a number; else the per-tile list tau[hq], whose last
    entry serves every tile past its end (§4.1, App. B.3 "Threshold tensor")."""
    t = tau[hq]
    if isinstance(t, (list, tuple)):
        return t[i] if i < len(t) else t[len(t) - 1]
    return t


def brute_forward(q, k, v, tau, Bq: int, Bk: int, causal: bool):
    """q: float [B][N][Hq][D]; k, v: float [B][N][Hkv][D]; tau: [Hq] numbers, or
    [Hq] lists of per-query-tile thresholds.

    Returns (out [B][N][Hq][D], lse [B][Hq][N], codes {(b, hq, i, j): code}).
    """
    B, N, Hq, D = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    Hkv = len(k[0][0])
    per_kv = Hq // Hkv
    inv = 1.0 / math.sqrt(D)
    mq = (N + Bq - 1) // Bq
    mkv = (N + Bk - 1) // Bk
    out = [[[[0.0] * D for _ in range(Hq)] for _ in range(N)] for _ in range(B)]
    lse = [[[0.0] * N for _ in range(Hq)] for _ in range(B)]
    codes = {}
    for b in range(B):
        for hq in range(Hq):
            g = hq // per_kv
            s = [[0.0] * N for _ in range(N)]
            for r in range(N):
                for c in range(N):
                    acc = 0.0
                    for d in range(D):
                        acc += q[b][r][hq][d] * k[b][c][g][d]
                    s[r][c] = acc * inv
            for i in range(mq):
                rows = range(i * Bq, min((i + 1) * Bq, N))
                for j in range(mkv):
                    cols = range(j * Bk, min((j + 1) * Bk, N))
                    any_valid = False
                    best = -math.inf
                    for r in rows:
                        for c in cols:
                            if _is_valid(r, c, causal):
                                any_valid = True
                                if s[r][c] > best:
                                    best = s[r][c]
                    if not any_valid:
                        codes[(b, hq, i, j)] = 3
                        continue
                    # Forced blocks are found on the full-size tile and block, as if
                    # the sequence were padded to whole tiles.
                    full_rows = range(i * Bq, (i + 1) * Bq)
                    full_cols = range(j * Bk, (j + 1) * Bk)
                    if causal:
                        forced = any(not _is_valid(r, c, True) for r in full_rows for c in full_cols)
                    else:
                        forced = any(c in full_rows for c in full_cols)
                    if forced:
                        codes[(b, hq, i, j)] = 2
                    elif best >= _threshold(tau, hq, i):
                        codes[(b, hq, i, j)] = 1
                    else:
                        codes[(b, hq, i, j)] = 0
            for r in range(N):
                i = r // Bq
                kept = [c for c in range(N)
                        if _is_valid(r, c, causal) and codes[(b, hq, i, c // Bk)] in (1, 2)]
                m = max(s[r][c] for c in kept)
                weights = [math.exp(s[r][c] - m) for c in kept]
                total = sum(weights)
                for d in range(D):
                    out[b][r][hq][d] = sum(w * v[b][c][g][d] for w, c in zip(weights, kept)) / total
                lse[b][hq][r] = m + math.log(total)
    return out, lse, codes


def brute_gap_codes(q, k, gamma, Bq: int, Bk: int, causal: bool):
    """Block codes under the gap-to-running-maximum gate, by plain loops.

    For each query tile the visible key blocks are visited in increasing order.
    Row r's running maximum starts at -inf and takes in every score of every kept
    block. A block that is not forced is kept when some row with a valid entry in
    it has no kept block yet or reaches at least (running maximum - gamma[hq]). Forced and visible blocks
    are found by enumerating the full-size tile and block, as in ``brute_forward``.
    Returns {(b, hq, i, j): code}.
    """
    B, N, Hq, D = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    Hkv = len(k[0][0])
    per_kv = Hq // Hkv
    inv = 1.0 / math.sqrt(D)
    mq = (N + Bq - 1) // Bq
    mkv = (N + Bk - 1) // Bk
    codes = {}
    for b in range(B):
        for hq in range(Hq):
            g = hq // per_kv
            for i in range(mq):
                rows = list(range(i * Bq, min((i + 1) * Bq, N)))
                run = {r: -math.inf for r in rows}
                for j in range(mkv):
                    cols = list(range(j * Bk, min((j + 1) * Bk, N)))
                    best = {}
                    for r in rows:
                        for c in cols:
                            if _is_valid(r, c, causal):
                                acc = 0.0
                                for d in range(D):
                                    acc += q[b][r][hq][d] * k[b][c][g][d]
                                val = acc * inv
                                if r not in best or val > best[r]:
                                    best[r] = val
                    if not best:
                        codes[(b, hq, i, j)] = 3
                        continue
                    full_rows = range(i * Bq, (i + 1) * Bq)
                    full_cols = range(j * Bk, (j + 1) * Bk)
                    if causal:
                        forced = any(not _is_valid(r, c, True) for r in full_rows for c in full_cols)
                    else:
                        forced = any(c in full_rows for c in full_cols)
                    if forced:
                        code = 2
                    else:
                        code = 1 if any(run[r] == -math.inf or best[r] >= run[r] - gamma[hq] for r in best) else 0
                    codes[(b, hq, i, j)] = code
                    if code != 0:
                        for r, val in best.items():
                            if val > run[r]:
                                run[r] = val
    return codes
