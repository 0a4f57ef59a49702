"""Plant plausible mistakes in the oracle (on the CPU) and check the pins catch each one.

Every mutation below swaps one helper of ``oracle.bsfa_oracle`` for a wrong
version (a dropped or wrong score scale, a strict comparison at the gate, an
inverted gate, no diagonal bypass, a diagonal judged on the cut-down last tile,
a wrong GQA head map, a normaliser that counts skipped blocks, a gate on unscaled
scores or on the block minimum, a per-position threshold table read at the wrong
column). The pin battery (hand-derived closed forms, the scalar brute force on
aligned and ragged sequences with per-head and per-tile thresholds, and the
tau = -inf library case) must fail for each of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import bsfa_oracle as O
from oracle import brute
from threshold_gated_block_b200.inputs import custom_config, make_inputs, f32_to_bf16_bits


def _battery(golden_dir) -> bool:
    """True when every pin holds."""
    with open(os.path.join(golden_dir, "hand_example.json")) as f:
        g = json.load(f)
    ev = lambda e: float(eval(e, {"__builtins__": {}}, {"e": math.e, "ln": math.log}))
    q = f32_to_bf16_bits(np.array(g["q"], dtype=np.float32))[None, :, None, :]
    k = f32_to_bf16_bits(np.array(g["k"], dtype=np.float32))[None, :, None, :]
    v = f32_to_bf16_bits(np.array(g["v"], dtype=np.float32))[None, :, None, :]
    with np.errstate(all="ignore"):
        for case in g["cases"]:
            r = O.forward(q, k, v, [case["tau"]], 2, 2, case["causal"])
            want = np.array([[ev(x) for x in row] for row in case["out"]])
            if r["codes"][0, 0].tolist() != case["codes"]:
                return False
            if not np.allclose(r["out"][0, :, 0, :], want, atol=1e-12, rtol=0):
                return False
        for (N, D, Hq, Hkv, Bq, Bk, causal) in [(64, 8, 4, 2, 16, 16, True), (48, 8, 4, 2, 16, 16, False)]:
            x = make_inputs(custom_config(N=N, D=D, Hq=Hq, Hkv=Hkv, Bq=Bq, Bk=Bk, causal=causal, seed=99))
            tau = [2.6, 2.8, 3.0, 2.7]
            r = O.forward(x["q"], x["k"], x["v"], tau, Bq, Bk, causal)
            qf, kf, vf = (O.widen_bf16(x[n]).tolist() for n in "qkv")
            out, lse, codes = brute.brute_forward(qf, kf, vf, tau, Bq, Bk, causal)
            if any(r["codes"][key] != c for key, c in codes.items()):
                return False
            if not (np.allclose(r["out"], out, atol=1e-12, rtol=0) and np.allclose(r["lse"], lse, atol=1e-12, rtol=0)):
                return False
            # tau = -inf against torch SDPA (float64, GQA by repeat_interleave)
            r = O.forward(x["q"], x["k"], x["v"], [-np.inf] * Hq, Bq, Bk, causal)
            tq, tk, tv = (torch.from_numpy(O.widen_bf16(x[n])).permute(0, 2, 1, 3) for n in "qkv")
            tk = tk.repeat_interleave(Hq // Hkv, 1)
            tv = tv.repeat_interleave(Hq // Hkv, 1)
            ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal)
            if not np.allclose(r["out"], ref.permute(0, 2, 1, 3).numpy(), atol=1e-12, rtol=0):
                return False
        # ragged end (last tile of one row) with a per-tile table shorter than M_Q
        x = make_inputs(custom_config(N=65, D=8, Hq=2, Hkv=1, Bq=16, Bk=16, causal=True, seed=98))
        table = [[2.9, 2.2, 2.6], [2.4, 3.0, 2.5]]
        r = O.forward(x["q"], x["k"], x["v"], table, 16, 16, True)
        qf, kf, vf = (O.widen_bf16(x[n]).tolist() for n in "qkv")
        out, lse, codes = brute.brute_forward(qf, kf, vf, table, 16, 16, True)
        if any(r["codes"][key] != c for key, c in codes.items()):
            return False
        if not (np.allclose(r["out"], out, atol=1e-12, rtol=0) and np.allclose(r["lse"], lse, atol=1e-12, rtol=0)):
            return False
    return True


def test_unmutated_oracle_passes_the_battery(golden_dir):
    assert _battery(golden_dir)


def _strict_gate(smax, tau):
    return smax > tau


def _inverted_gate(smax, tau):
    return smax < tau


def _no_diagonal(i, j, Bq, Bk, N, causal):
    return False


def _diagonal_on_clipped_tile(i, j, Bq, Bk, N, causal):
    if not O.block_visible(i, j, Bq, Bk, N, causal):
        return False
    r0, r1 = O.tile_rows(i, Bq, N)
    c0, c1 = O.block_cols(j, Bk, N)
    return (c1 - 1 > r0) if causal else (c0 < r1 and c1 > r0)


def _table_wraps(tau, hq, i):
    t = np.asarray(tau, dtype=np.float64)
    return float(t[hq]) if t.ndim == 1 else float(t[hq, i % t.shape[1]])


def _table_first_column(tau, hq, i):
    t = np.asarray(tau, dtype=np.float64)
    return float(t[hq]) if t.ndim == 1 else float(t[hq, 0])


def _wrong_gqa(hq, Hq, Hkv):
    return hq % Hkv


def _normaliser_counts_skipped(S, valid, codes, vmat, Bk):
    ncols = S.shape[1]
    kept_col = np.isin(codes[np.arange(ncols) // Bk], (1, 2))
    C = valid & kept_col[None, :]
    Sm = np.where(valid, S, -np.inf)
    m = Sm.max(axis=1)
    w_all = np.where(valid, np.exp(Sm - m[:, None]), 0.0)
    w = np.where(C, w_all, 0.0)
    l = w_all.sum(axis=1)
    return (w @ vmat[:ncols]) / l[:, None], m + np.log(l)


_real_codes = O.tile_block_codes


def _gate_on_unscaled_scores(S, valid, i, tau, Bq, Bk, N, causal, flip=()):
    D = 8  # the battery's head dimension
    return _real_codes(S * math.sqrt(D), valid, i, tau, Bq, Bk, N, causal, flip)


def _gate_on_block_minimum(S, valid, i, tau, Bq, Bk, N, causal, flip=()):
    return _real_codes(-np.where(valid, S, np.inf), valid, i, -tau, Bq, Bk, N, causal, flip)


MUTATIONS = {
    "dropped score scale": ("score_scale", lambda D: 1.0),
    "scale 1/d instead of 1/sqrt(d)": ("score_scale", lambda D: 1.0 / D),
    "strict comparison at the gate": ("gate_keep", _strict_gate),
    "inverted gate": ("gate_keep", _inverted_gate),
    "no diagonal bypass": ("block_diagonal", _no_diagonal),
    "diagonal judged on the cut-down last tile": ("block_diagonal", _diagonal_on_clipped_tile),
    "threshold table wraps instead of reusing its last column": ("tile_tau", _table_wraps),
    "threshold table read at its first column only": ("tile_tau", _table_first_column),
    "wrong GQA head map": ("kv_head", _wrong_gqa),
    "normaliser counts skipped blocks": ("tile_softmax", _normaliser_counts_skipped),
    "gate compares the unscaled score": ("tile_block_codes", _gate_on_unscaled_scores),
    "gate on the block minimum": ("tile_block_codes", _gate_on_block_minimum),
}


@pytest.mark.parametrize("name", list(MUTATIONS))
def test_battery_catches_planted_mistake(name, monkeypatch, golden_dir):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(O, attr, fn)
    try:
        ok = _battery(golden_dir)
    except (ValueError, IndexError, ZeroDivisionError, FloatingPointError):
        ok = False
    assert not ok, f"pins missed the planted mistake: {name}"
