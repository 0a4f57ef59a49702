"""The per-head threshold rule and the stored threshold table (CPU only)."""
import json
import os

import numpy as np
import pytest

from oracle import bsfa_oracle as O
from oracle.calibrate import tau_for_skip, calibrate
from threshold_gated_block_b200.inputs import CONFIGS, make_inputs


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
