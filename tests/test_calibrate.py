"""The per-head threshold rule and the stored threshold table (CPU only)."""
import json
import os

import numpy as np
import pytest

from oracle import bsfa_oracle as O
from oracle.calibrate import calibrate, fixed_k_table, tau_for_skip, tile_gated_maxima, topk_threshold
from threshold_gated_block_b200.inputs import CONFIGS, custom_config, make_inputs


def test_tau_sits_in_the_gap_at_the_target_rank():
    assert tau_for_skip([4.0, 1.0, 3.0, 2.0], 0.5) == 2.5
    assert tau_for_skip([1.0, 2.0, 3.0, 4.0], 0.25) == 1.5


def test_widest_gap_within_the_rank_window():
    # 2000 maxima 1e-5 apart with one 1e-3 gap two ranks above the target rank
    a = np.cumsum(np.full(2000, 1e-5)) + 3.0
    a[1002:] += 1e-3
    t = tau_for_skip(a, 0.5)                 # window = round(0.002 * 2000) = 4 ranks
    assert a[1001] < t < a[1002]
    assert (a < t).sum() == 1002


def test_small_counts_cut_at_the_exact_rank():
    t = tau_for_skip([1.0, 1.0001, 2.0, 3.0], 0.25)
    assert 1.0 < t < 1.0001


def test_extreme_fractions():
    assert tau_for_skip([1.0, 2.0], 0.0) < 1.0
    assert tau_for_skip([1.0, 2.0], 1.0) > 2.0
    assert tau_for_skip([], 0.5) == -np.inf


def test_tau_is_float32_representable():
    t = tau_for_skip(np.random.default_rng(0).normal(size=1000), 0.3)
    assert float(np.float32(t)) == t


def test_stored_table_matches_recomputation_for_the_small_workload(golden_dir):
    with open(os.path.join(golden_dir, "taus.json")) as f:
        table = json.load(f)
    cfg = CONFIGS["c1"]
    x = make_inputs(cfg)
    fresh = calibrate(x["q"], x["k"], cfg.Bq, cfg.Bk, cfg.causal, cfg.skips)
    for p, taus in fresh.items():
        assert table["c1"]["taus"][str(p)] == taus
    r = O.forward(x["q"], x["k"], x["v"], fresh[0.5], cfg.Bq, cfg.Bk, cfg.causal)
    gated = np.isin(r["codes"], (O.CODE_SKIPPED, O.CODE_KEPT))
    assert abs((r["codes"] == O.CODE_SKIPPED).sum() / gated.sum() - 0.5) < 0.02


def test_table_covers_every_workload(golden_dir):
    with open(os.path.join(golden_dir, "taus.json")) as f:
        table = json.load(f)
    for name, cfg in CONFIGS.items():
        if name not in table:
            pytest.skip(f"{name} not calibrated yet")
        for p in cfg.skips:
            assert len(table[name]["taus"][str(float(p))]) == cfg.Hq


# ----------------------------------------------------------------------------- per-position (fixed-k) table

def test_topk_threshold_keeps_exactly_k():
    rng = np.random.default_rng(7)
    for n in (1, 2, 5, 63, 500):
        v = rng.normal(size=n) * 3
        for k in range(0, min(n, 12) + 1):
            t = topk_threshold(v, k)
            assert float(np.float32(t)) == t
            assert (v >= t).sum() == min(k, n), (n, k)


def test_topk_threshold_edges():
    assert topk_threshold([], 3) == -np.inf
    assert topk_threshold([1.0, 2.0], 2) == -np.inf
    assert topk_threshold([4.0, 1.0, 3.0, 2.0], 2) == 2.5
    assert topk_threshold([1.0, 2.0], 0) > 2.0
    assert topk_threshold([1.0, 1.0, 3.0], 2) <= 1.0      # tie at the cut keeps every tied block


def test_padding_by_repetition_leaves_the_gated_maxima_unchanged():
    """App. B.3 pads an unaligned sequence with copies of its last token; on the real
    tiles the padded view has the same gated block maxima as masking past N."""
    for causal in (True, False):
        for (N, Bq, Bk) in ((200, 64, 64), (130, 128, 64), (100, 64, 128), (257, 128, 128)):
            cfg = custom_config(N=N, D=16, Hq=2, Hkv=1, Bq=Bq, Bk=Bk, causal=causal, seed=N + Bq)
            x = make_inputs(cfg)
            padded = tile_gated_maxima(x["q"], x["k"], Bq, Bk, causal)
            plain = O.block_maxima(x["q"], x["k"], Bq, Bk, causal)
            for key, (codes, smax) in plain.items():
                np.testing.assert_array_equal(np.sort(padded[key]), np.sort(smax[codes == O.CODE_SKIPPED]))


def test_fixed_k_table_keeps_k_blocks_on_its_own_sample():
    """On the sample it was calibrated on, level k keeps exactly k gated blocks in
    every tile that has more than k (counted from the oracle's gate decisions)."""
    cfg = custom_config(N=1024, D=32, Hq=4, Hkv=2, Bq=64, Bk=64, causal=True, kind="planted", seed=77)
    x = make_inputs(cfg)
    ks = (2, 5, 9)
    T = fixed_k_table([(x["q"], x["k"])], 64, 64, True, ks)
    assert T.shape == (3, 4, 16) and T.dtype == np.float32
    assert (T[0] >= T[1]).all() and (T[1] >= T[2]).all()          # more blocks kept, lower threshold
    for li, k in enumerate(ks):
        r = O.forward(x["q"], x["k"], x["v"], T[li], 64, 64, True)
        for hq in range(4):
            for i in range(16):
                c = r["codes"][0, hq, i]
                gated = np.isin(c, (O.CODE_SKIPPED, O.CODE_KEPT)).sum()
                assert (c == O.CODE_KEPT).sum() == min(k, gated), (k, hq, i)
                assert np.isfinite(T[li, hq, i]) == (gated > k)


def test_fixed_k_table_averages_the_samples():
    cfg = custom_config(N=512, D=32, Hq=2, Hkv=1, Bq=64, Bk=64, causal=False, seed=5)
    xs = [make_inputs(cfg, seed=s) for s in (11, 12)]
    T = fixed_k_table([(x["q"], x["k"]) for x in xs], 64, 64, False, [3])
    each = [fixed_k_table([(x["q"], x["k"])], 64, 64, False, [3]) for x in xs]
    np.testing.assert_allclose(T, (each[0].astype(np.float64) + each[1]) / 2, rtol=0, atol=1e-6)
