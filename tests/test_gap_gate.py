"""The gap-to-running-maximum gate of the oracle (a comparison gate; §3 Related
Work, on BLASST and SpargeAttention), pinned against things other than itself:

* the scalar brute force (``oracle.brute.brute_gap_codes``), which enumerates
  every (query, key) pair and keeps its own running maxima, on aligned and ragged
  sequences, causal and bidirectional, GQA, Bq != Bk;
* limits: gamma = +inf keeps every block (dense attention); a gamma below every
  margin skips every gated block that does not raise a row's maximum;
* the softmax over the kept set is the same function as for the BSFA gate: the
  gap gate only changes which blocks are kept;
* planted mistakes (running maxima that take in skipped blocks, one maximum for
  the whole tile, forced blocks that leave the maxima alone) fail the
  brute-force pins; a strict comparison fails an exact-tie case.
"""
import math

import numpy as np
import pytest

from oracle import bsfa_oracle as O
from oracle import brute
from threshold_gated_block_b200.inputs import custom_config, make_inputs

CASES = [
    # N, D, Hq, Hkv, Bq, Bk, causal, kind
    (64, 8, 2, 1, 16, 16, True, "normal"),
    (96, 8, 4, 2, 16, 32, True, "normal"),
    (81, 8, 2, 1, 32, 16, True, "normal"),
    (64, 8, 2, 2, 16, 16, False, "normal"),
    (70, 8, 4, 2, 32, 16, False, "normal"),
    (128, 16, 2, 1, 16, 16, True, "planted"),
]
GAMMAS = [-2.0, -1.0, -0.4, 0.0]


def _codes_match(x, gam, Bq, Bk, causal):
    r = O.forward(x["q"], x["k"], x["v"], gam, Bq, Bk, causal, gate="gap")
    qf, kf = (O.widen_bf16(x[n]).tolist() for n in "qk")
    codes = brute.brute_gap_codes(qf, kf, gam, Bq, Bk, causal)
    return r, all(r["codes"][key] == c for key, c in codes.items())


@pytest.mark.parametrize("N,D,Hq,Hkv,Bq,Bk,causal,kind", CASES)
def test_gap_codes_match_brute_force(N, D, Hq, Hkv, Bq, Bk, causal, kind):
    x = make_inputs(custom_config(N=N, D=D, Hq=Hq, Hkv=Hkv, Bq=Bq, Bk=Bk, causal=causal, kind=kind, seed=N + Bq))
    skipped = kept = 0
    for g in GAMMAS:
        gam = [g + 0.05 * h for h in range(Hq)]
        r, ok = _codes_match(x, gam, Bq, Bk, causal)
        assert ok, (g, gam)
        skipped += int((r["codes"] == O.CODE_SKIPPED).sum())
        kept += int((r["codes"] == O.CODE_KEPT).sum())
    assert skipped > 0 and kept > 0


def test_gap_output_is_the_softmax_over_the_kept_set():
    """Same kept set -> same output as the BSFA path evaluated with those codes."""
    x = make_inputs(custom_config(N=128, D=16, Hq=2, Hkv=1, Bq=32, Bk=32, causal=True, seed=4))
    r = O.forward(x["q"], x["k"], x["v"], [-0.5, -0.2], 32, 32, True, gate="gap")
    for hq in range(2):
        for i in range(4):
            t = O.forward_tile(x["q"], x["k"], x["v"], [np.inf, np.inf], 0, hq, i, 32, 32, True)
            flip = tuple(int(j) for j in np.nonzero(r["codes"][0, hq, i] == O.CODE_KEPT)[0])
            t = O.forward_tile(x["q"], x["k"], x["v"], [np.inf, np.inf], 0, hq, i, 32, 32, True, flip=flip)
            assert np.array_equal(t["codes"], r["codes"][0, hq, i])
            r0, r1 = t["rows"]
            np.testing.assert_array_equal(t["out"], r["out"][0, r0:r1, hq])
            np.testing.assert_array_equal(t["lse"], r["lse"][0, hq, r0:r1])


@pytest.mark.parametrize("causal", [True, False])
def test_gap_limits(causal):
    x = make_inputs(custom_config(N=160, D=8, Hq=2, Hkv=1, Bq=32, Bk=32, causal=causal, seed=8))
    dense = O.forward(x["q"], x["k"], x["v"], [-np.inf, -np.inf], 32, 32, causal)
    wide = O.forward(x["q"], x["k"], x["v"], [np.inf, np.inf], 32, 32, causal, gate="gap")
    assert not (wide["codes"] == O.CODE_SKIPPED).any()
    np.testing.assert_array_equal(wide["out"], dense["out"])
    # gamma = -inf: a gated block is kept only while some row still has no kept block
    narrow = O.forward(x["q"], x["k"], x["v"], [-np.inf, -np.inf], 32, 32, causal, gate="gap")
    for hq in range(2):
        for i in range(5):
            c = narrow["codes"][0, hq, i]
            gated = np.nonzero(np.isin(c, (O.CODE_SKIPPED, O.CODE_KEPT)))[0]
            first_kept = [j for j in range(len(c)) if c[j] in (O.CODE_KEPT, O.CODE_FORCED)]
            # after the first kept block every row has a finite running maximum
            assert all(c[j] == O.CODE_SKIPPED for j in gated if j > first_kept[0])


# ----------------------------------------------------------------------------- planted mistakes

def _gap_taking_in_skipped_blocks(S, valid, i, gamma, Bq, Bk, N, causal, flip=()):
    mkv = -(-N // Bk)
    codes = np.full(mkv, O.CODE_INVISIBLE, dtype=np.uint8)
    M = np.full(S.shape[0], -np.inf)
    for j in range(mkv):
        if not O.block_visible(i, j, Bq, Bk, N, causal):
            continue
        c0, c1 = j * Bk, min((j + 1) * Bk, S.shape[1])
        rowmax = np.where(valid[:, c0:c1], S[:, c0:c1], -np.inf).max(axis=1)
        if O.block_diagonal(i, j, Bq, Bk, N, causal):
            codes[j] = O.CODE_FORCED
        else:
            part = np.isfinite(rowmax)
            ok = np.isneginf(M[part]) | (rowmax[part] >= M[part] - gamma)
            codes[j] = O.CODE_KEPT if ok.any() else O.CODE_SKIPPED
        M = np.maximum(M, rowmax)                      # mistake: skipped blocks raise M too
    return codes, np.full(mkv, np.nan)


def _gap_with_one_tile_maximum(S, valid, i, gamma, Bq, Bk, N, causal, flip=()):
    mkv = -(-N // Bk)
    codes = np.full(mkv, O.CODE_INVISIBLE, dtype=np.uint8)
    M = -np.inf
    for j in range(mkv):
        if not O.block_visible(i, j, Bq, Bk, N, causal):
            continue
        c0, c1 = j * Bk, min((j + 1) * Bk, S.shape[1])
        bmax = np.where(valid[:, c0:c1], S[:, c0:c1], -np.inf).max()
        if O.block_diagonal(i, j, Bq, Bk, N, causal):
            codes[j] = O.CODE_FORCED
        else:
            codes[j] = O.CODE_KEPT if bmax >= M - gamma else O.CODE_SKIPPED
        if codes[j] != O.CODE_SKIPPED:
            M = max(M, bmax)                           # mistake: one maximum for the whole tile
    return codes, np.full(mkv, np.nan)


_real_gap = O.tile_block_codes_gap


def _gap_strict(S, valid, i, gamma, Bq, Bk, N, causal, flip=()):
    codes, margin = _real_gap(S, valid, i, gamma, Bq, Bk, N, causal, flip)
    codes = codes.copy()
    codes[(codes == O.CODE_KEPT) & (margin == 0.0)] = O.CODE_SKIPPED
    return codes, margin


def _gap_forced_blocks_do_not_raise(S, valid, i, gamma, Bq, Bk, N, causal, flip=()):
    mkv = -(-N // Bk)
    codes = np.full(mkv, O.CODE_INVISIBLE, dtype=np.uint8)
    M = np.full(S.shape[0], -np.inf)
    for j in range(mkv):
        if not O.block_visible(i, j, Bq, Bk, N, causal):
            continue
        c0, c1 = j * Bk, min((j + 1) * Bk, S.shape[1])
        rowmax = np.where(valid[:, c0:c1], S[:, c0:c1], -np.inf).max(axis=1)
        if O.block_diagonal(i, j, Bq, Bk, N, causal):
            codes[j] = O.CODE_FORCED
            continue                                   # mistake: the forced block leaves M alone
        part = np.isfinite(rowmax)
        ok = np.isneginf(M[part]) | (rowmax[part] >= M[part] - gamma)
        codes[j] = O.CODE_KEPT if ok.any() else O.CODE_SKIPPED
        if codes[j] == O.CODE_KEPT:
            M = np.maximum(M, rowmax)
    return codes, np.full(mkv, np.nan)


GAP_MUTATIONS = {
    "running maxima take in skipped blocks": _gap_taking_in_skipped_blocks,
    "one running maximum for the whole tile": _gap_with_one_tile_maximum,
    "forced blocks do not raise the running maxima": _gap_forced_blocks_do_not_raise,
}


def _gap_battery() -> bool:
    for (N, D, Hq, Hkv, Bq, Bk, causal, kind) in CASES:
        x = make_inputs(custom_config(N=N, D=D, Hq=Hq, Hkv=Hkv, Bq=Bq, Bk=Bk, causal=causal, kind=kind, seed=N + Bq))
        for g in GAMMAS:
            if not _codes_match(x, [g + 0.05 * h for h in range(Hq)], Bq, Bk, causal)[1]:
                return False
    return True


@pytest.mark.parametrize("name", list(GAP_MUTATIONS))
def test_gap_pins_catch_planted_mistake(name, monkeypatch):
    monkeypatch.setattr(O, "tile_block_codes_gap", GAP_MUTATIONS[name])
    assert not _gap_battery(), name


def test_gap_keeps_an_exact_tie_and_a_strict_comparison_would_not():
    """A block whose row maximum equals the running maximum minus gamma is kept."""
    scale = 1.0 / math.sqrt(2)
    # row 2 of a 3-token bidirectional sequence, one-row tiles and one-key blocks:
    # blocks 0 and 1 are gated, block 2 is its diagonal
    S = np.array([[2.0 * scale, 1.0 * scale, 0.5 * scale]])
    valid = np.ones((1, 3), dtype=bool)
    gamma = 2.0 * scale - 1.0 * scale
    codes, margin = O.tile_block_codes_gap(S, valid, 2, gamma, 1, 1, 3, False)
    assert list(codes) == [O.CODE_KEPT, O.CODE_KEPT, O.CODE_FORCED] and margin[1] == 0.0
    codes_strict, _ = _gap_strict(S, valid, 2, gamma, 1, 1, 3, False)
    assert codes_strict[1] == O.CODE_SKIPPED
