"""CPU oracle for the BSFA prefill forward (test infrastructure only).

This is the plain, slow, float64 statement of what Block Sparse Flash Attention
computes. Only the test suite, the smoke check and the bench's CPU-baseline leg
use it; the product path never imports it, and it shares no code with the CUDA
kernels.

Source: "Block Sparse Flash Attention" (paperpeel.com/paper/2512.07011):
  * §2 "FlashAttention" and App. B.2: queries are split into M_Q = ceil(N/B_M)
    tiles and keys/values into M_KV = ceil(N/B_N) blocks; the score tile is
    S_ij = Q_i K_j^T / sqrt(d).
  * §4.1 "Gating Mechanism": block (i, j) is skipped when its maximum score
    s_max^(i,j) is below the threshold; diagonal blocks bypass the gate.
  * §4.4 "Algorithm and Implementation": a skipped block loads no values, does
    no PV product and does not enter the running statistics (m_i, l_i, O_i).
  * App. B.3 "Practical considerations": the method also applies to the
    bidirectional (non-causal) case.

Because a skipped block never enters (m, l, O), the streamed result equals a
softmax taken over the kept key set only. The oracle therefore evaluates that
definition directly, per query tile, with no streaming and no rescaling:

    C_r   = { c : c valid for row r, and block(c) kept for r's tile }
    m_r   = max_{c in C_r} s_rc
    l_r   = sum_{c in C_r} exp(s_rc - m_r)
    out_r = sum_{c in C_r} exp(s_rc - m_r) v_c / l_r
    lse_r = m_r + ln l_r

Readings taken where the pages are silent or garbled:
  * the score carries the 1/sqrt(d) factor of App. B.2 step (3), and tau is in
    the units of that scaled score;
  * "below the threshold" skips, so a block whose maximum equals tau is kept;
  * s_max is one scalar per (query tile, key block), the maximum over every
    valid entry of the block;
  * causal: a block is visible when some entry is valid (key <= query); it is
    "diagonal" when it is visible and also holds an invalid entry, the tile and
    block taken at full size (as if padded, App. B.3);
    non-causal: a block is "diagonal" when its key range overlaps the tile's
    query range;
  * tau is one float per query head, or a per-position table [Hq, M] (one
    value per query tile; tiles past the table's end reuse its last column);
  * GQA: query head h reads KV head h // (Hq / Hkv);
  * lse is the natural-log logsumexp, laid out [B, Hq, N];
  * keys at index >= N are invalid (an unaligned tail is never read).

Block codes: 0 = skipped by the gate, 1 = kept by the gate, 2 = forced keep
(diagonal), 3 = not visible (causally masked out entirely).

A second gate is provided for comparison (``gate="gap"``): the gap to the
running maximum, which the page attributes to BLASST and SpargeAttention (§3
Related Work, paragraphs "Gating after scoring" and "Predicting importance
before scoring"): a block is skipped when it lies far below the running maximum. The
pages give no formula, so the reading here is: the query tile visits its
visible key blocks in increasing order; each row r keeps M_r, the maximum of
its scores over the blocks kept so far (-inf at first); a non-diagonal block
is kept when some row with a valid entry in it has no kept block yet or has
rowmax_r(block) >= M_r - gamma (gamma per head, in scaled-score units, of either
sign); kept blocks (diagonal ones included) then raise M_r. Skipped blocks leave M_r alone, as they leave
the softmax statistics alone in BSFA.
"""
from __future__ import annotations

import math

import numpy as np

CODE_SKIPPED = 0
CODE_KEPT = 1
CODE_FORCED = 2
CODE_INVISIBLE = 3


def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact float64 values."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def score_scale(D: int) -> float:
    """The 1/sqrt(d) factor of the scaled score (App. B.2, step 3)."""
    return 1.0 / math.sqrt(D)


def gate_keep(smax: float, tau: float) -> bool:
    """§4.1: skip when the block maximum is below tau, so equality keeps."""
    return smax >= tau


def tile_tau(tau, hq: int, i: int) -> float:
    """Threshold of query tile i of head hq.

    §4.1 gates block (i, j) against a threshold indexed by layer, head and query
    position; App. B.3 "Threshold tensor" stores ceil(N_max / B_M) positions per
    head, and a sequence longer than N_max reuses the threshold of the last
    calibrated position. ``tau`` is one layer's slice: either [Hq] (one value per
    head) or [Hq, M] (one value per head and query tile).
    """
    t = np.asarray(tau, dtype=np.float64)
    if t.ndim == 1:
        return float(t[hq])
    return float(t[hq, min(i, t.shape[1] - 1)])


def kv_head(hq: int, Hq: int, Hkv: int) -> int:
    """GQA: contiguous groups of Hq/Hkv query heads share one KV head."""
    return hq // (Hq // Hkv)


def tile_rows(i: int, Bq: int, N: int) -> tuple[int, int]:
    return i * Bq, min((i + 1) * Bq, N)


def block_cols(j: int, Bk: int, N: int) -> tuple[int, int]:
    return j * Bk, min((j + 1) * Bk, N)


def block_visible(i: int, j: int, Bq: int, Bk: int, N: int, causal: bool) -> bool:
    """A block is visible when at least one of its entries is a valid (query, key) pair."""
    r0, r1 = tile_rows(i, Bq, N)
    c0, c1 = block_cols(j, Bk, N)
    if c0 >= c1 or r0 >= r1:
        return False
    return (not causal) or c0 <= r1 - 1


def block_diagonal(i: int, j: int, Bq: int, Bk: int, N: int, causal: bool) -> bool:
    """The blocks that bypass the gate (§4.1, "Diagonal blocks bypass the gate").

    Judged on the full tile and block, [i*Bq, (i+1)*Bq) x [j*Bk, (j+1)*Bk), as if an
    unaligned sequence were padded to whole tiles (App. B.3 "Practical
    considerations"): a visible block is diagonal when it holds, or would hold, a
    key later than the tile's first query (causal), or when its key range overlaps
    the tile's query range (bidirectional). The block holding a row's own key is
    therefore always forced, also for a last tile cut down to a single row.
    """
    if not block_visible(i, j, Bq, Bk, N, causal):
        return False
    r0, c0 = i * Bq, j * Bk
    if causal:
        return c0 + Bk - 1 > r0
    return c0 < r0 + Bq and c0 + Bk > r0


def valid_mask(r0: int, r1: int, ncols: int, causal: bool) -> np.ndarray:
    rows = np.arange(r0, r1)[:, None]
    cols = np.arange(ncols)[None, :]
    if causal:
        return cols <= rows
    return np.ones((r1 - r0, ncols), dtype=bool)


def tile_scores(qi: np.ndarray, kmat: np.ndarray, D: int) -> np.ndarray:
    """S = Q_i K^T / sqrt(d) in float64 (App. B.2, step 3)."""
    return (qi @ kmat.T) * score_scale(D)


def tile_block_codes(S: np.ndarray, valid: np.ndarray, i: int, tau: float, Bq: int, Bk: int,
                     N: int, causal: bool, flip=()) -> tuple[np.ndarray, np.ndarray]:
    """Block codes and block maxima of one query tile against every key block.

    ``flip`` names gated (non-forced, visible) blocks whose decision is inverted;
    tests use it to evaluate the other admissible result for a block whose
    maximum lies within rounding of tau.
    """
    mkv = -(-N // Bk)
    codes = np.full(mkv, CODE_INVISIBLE, dtype=np.uint8)
    smax = np.full(mkv, np.nan)
    # Maximum over the valid entries of every block the tile's columns reach.
    ncols = S.shape[1]
    nb = -(-ncols // Bk)
    Sm = np.full((S.shape[0], nb * Bk), -np.inf)
    Sm[:, :ncols] = np.where(valid, S, -np.inf)
    bmax = Sm.reshape(S.shape[0], nb, Bk).max(axis=(0, 2))
    for j in range(mkv):
        if not block_visible(i, j, Bq, Bk, N, causal):
            continue
        smax[j] = float(bmax[j])
        if block_diagonal(i, j, Bq, Bk, N, causal):
            codes[j] = CODE_FORCED
        else:
            keep = gate_keep(smax[j], tau)
            if j in flip:
                keep = not keep
            codes[j] = CODE_KEPT if keep else CODE_SKIPPED
    return codes, smax


def tile_block_codes_gap(S: np.ndarray, valid: np.ndarray, i: int, gamma: float, Bq: int, Bk: int,
                         N: int, causal: bool, flip=()) -> tuple[np.ndarray, np.ndarray]:
    """Block codes of one query tile under the gap-to-running-maximum gate.

    Returns (codes, margin): margin[j] is, for a gated block, the largest over its
    rows with a valid entry of rowmax_r - (M_r - gamma) (kept iff >= 0); NaN for
    forced and invisible blocks. ``flip`` inverts the decision of the named gated
    blocks, and later blocks follow the flipped running maxima.
    """
    mkv = -(-N // Bk)
    codes = np.full(mkv, CODE_INVISIBLE, dtype=np.uint8)
    margin = np.full(mkv, np.nan)
    ncols = S.shape[1]
    M = np.full(S.shape[0], -np.inf)
    for j in range(mkv):
        if not block_visible(i, j, Bq, Bk, N, causal):
            continue
        c0, c1 = j * Bk, min((j + 1) * Bk, ncols)
        blk = np.where(valid[:, c0:c1], S[:, c0:c1], -np.inf) if c0 < ncols else np.full((S.shape[0], 1), -np.inf)
        rowmax = blk.max(axis=1)
        if block_diagonal(i, j, Bq, Bk, N, causal):
            codes[j] = CODE_FORCED
        else:
            part = np.isfinite(rowmax)
            # a row with no kept block yet (M = -inf) always qualifies
            with np.errstate(invalid="ignore"):      # -inf - (-inf) in the branch not taken
                gaps = np.where(np.isneginf(M[part]), np.inf, rowmax[part] - (M[part] - gamma))
            margin[j] = float(gaps.max()) if gaps.size else -np.inf
            keep = bool(gaps.size) and margin[j] >= 0.0
            if j in flip:
                keep = not keep
            codes[j] = CODE_KEPT if keep else CODE_SKIPPED
        if codes[j] in (CODE_KEPT, CODE_FORCED):
            M = np.maximum(M, rowmax)
    return codes, margin


def tile_softmax(S: np.ndarray, valid: np.ndarray, codes: np.ndarray, vmat: np.ndarray,
                 Bk: int) -> tuple[np.ndarray, np.ndarray]:
    """Softmax over the kept key set only (§4.4: skipped blocks never enter m, l, O)."""
    ncols = S.shape[1]
    col_block = np.arange(ncols) // Bk
    kept_col = np.isin(codes[col_block], (CODE_KEPT, CODE_FORCED))
    C = valid & kept_col[None, :]
    Sm = np.where(C, S, -np.inf)
    m = Sm.max(axis=1)
    w = np.where(C, np.exp(Sm - m[:, None]), 0.0)
    l = w.sum(axis=1)
    out = (w @ vmat[:ncols]) / l[:, None]
    lse = m + np.log(l)
    return out, lse


def forward_tile(q_bits, k_bits, v_bits, tau, b: int, hq: int, i: int, Bq: int, Bk: int,
                 causal: bool, flip=(), with_output: bool = True, gate: str = "tau") -> dict:
    """The BSFA result for one query tile (b, hq, i).

    q_bits: uint16 [B, N, Hq, D]; k_bits, v_bits: uint16 [B, N, Hkv, D]; tau: [Hq] or [Hq, M]
    (see ``tile_tau``).
    Returns out [rows, D], lse [rows], codes [M_KV], smax [M_KV] (NaN where not visible).
    """
    B, N, Hq, D = q_bits.shape
    Hkv = k_bits.shape[2]
    g = kv_head(hq, Hq, Hkv)
    r0, r1 = tile_rows(i, Bq, N)
    ncols = r1 if causal else N           # keys past the last row of the tile are never valid
    qi = widen_bf16(q_bits[b, r0:r1, hq, :])
    kmat = widen_bf16(k_bits[b, :ncols, g, :])
    S = tile_scores(qi, kmat, D)
    valid = valid_mask(r0, r1, ncols, causal)
    if gate == "gap":
        codes, margin = tile_block_codes_gap(S, valid, i, tile_tau(tau, hq, i), Bq, Bk, N, causal, flip)
        res = {"codes": codes, "margin": margin, "rows": (r0, r1)}
    else:
        codes, smax = tile_block_codes(S, valid, i, tile_tau(tau, hq, i), Bq, Bk, N, causal, flip)
        res = {"codes": codes, "smax": smax, "rows": (r0, r1)}
    if with_output:
        vmat = widen_bf16(v_bits[b, :ncols, g, :])
        res["out"], res["lse"] = tile_softmax(S, valid, codes, vmat, Bk)
    return res


def forward(q_bits, k_bits, v_bits, tau, Bq: int, Bk: int, causal: bool, gate: str = "tau") -> dict:
    """The whole BSFA forward: out [B,N,Hq,D], lse [B,Hq,N], codes/smax [B,Hq,M_Q,M_KV].

    gate="gap" uses the gap-to-running-maximum gate with ``tau`` holding gamma;
    "smax" then holds each gated block's margin instead.
    """
    B, N, Hq, D = q_bits.shape
    mq, mkv = -(-N // Bq), -(-N // Bk)
    out = np.zeros((B, N, Hq, D))
    lse = np.zeros((B, Hq, N))
    codes = np.zeros((B, Hq, mq, mkv), dtype=np.uint8)
    smax = np.zeros((B, Hq, mq, mkv))
    tau = np.asarray(tau, dtype=np.float64)
    for b in range(B):
        for hq in range(Hq):
            for i in range(mq):
                t = forward_tile(q_bits, k_bits, v_bits, tau, b, hq, i, Bq, Bk, causal, gate=gate)
                r0, r1 = t["rows"]
                out[b, r0:r1, hq, :] = t["out"]
                lse[b, hq, r0:r1] = t["lse"]
                codes[b, hq, i] = t["codes"]
                smax[b, hq, i] = t["margin" if gate == "gap" else "smax"]
    return {"out": out, "lse": lse, "codes": codes, "smax": smax}


def block_maxima(q_bits, k_bits, Bq: int, Bk: int, causal: bool, tiles=None) -> dict:
    """Block maxima and forced/visible flags only (no softmax), for threshold calibration.

    tiles: optional iterable of (b, hq, i); default is every query tile.
    Returns {(b, hq, i): (codes_at_tau_plus_inf, smax)} where code 0 marks gated blocks.
    """
    B, N, Hq, D = q_bits.shape
    mq = -(-N // Bq)
    if tiles is None:
        tiles = [(b, hq, i) for b in range(B) for hq in range(Hq) for i in range(mq)]
    tau_inf = np.full(Hq, np.inf)
    res = {}
    for (b, hq, i) in tiles:
        t = forward_tile(q_bits, k_bits, None, tau_inf, b, hq, i, Bq, Bk, causal, with_output=False)
        res[(b, hq, i)] = (t["codes"], t["smax"])
    return res


def forward_varlen(q_bits, k_bits, v_bits, cu_seqlens, tau, Bq: int, Bk: int, causal: bool) -> dict:
    """A packed batch of sequences of different lengths: each sequence
    [cu[e], cu[e+1]) of q [total, Hq, D] and k, v [total, Hkv, D] is its own
    forward (App. B.2 tiling starts at its first row). Returns out [total, Hq, D],
    lse [Hq, total] and, per sequence, its codes [Hq, M_Q, M_KV]."""
    total, Hq, D = q_bits.shape
    out = np.zeros((total, Hq, D))
    lse = np.zeros((Hq, total))
    codes = []
    for e in range(len(cu_seqlens) - 1):
        r0, r1 = int(cu_seqlens[e]), int(cu_seqlens[e + 1])
        if r1 <= r0:
            codes.append(None)
            continue
        r = forward(q_bits[None, r0:r1], k_bits[None, r0:r1], v_bits[None, r0:r1], tau, Bq, Bk, causal)
        out[r0:r1] = r["out"][0]
        lse[:, r0:r1] = r["lse"][0]
        codes.append(r["codes"][0])
    return {"out": out, "lse": lse, "codes": codes}
