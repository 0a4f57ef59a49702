"""The bench line's cpu_baseline (bench.cpu_baseline) on the CPU: the oracle's
dense-equivalent FLOPs are counted per visible (query tile, key block) pair, the
exact-count sample holds the seeded tiles it names, and the extrapolated layer
time is the layer's FLOPs at the sample's rate."""
import json
import os

import numpy as np

import bench
from threshold_gated_block_b200.inputs import CONFIGS, make_inputs, sample_tiles

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _c1():
    cfg = CONFIGS["c1"]
    with open(os.path.join(ROOT, "tests", "golden", "taus.json")) as f:
        taus = json.load(f)["c1"]["taus"]["0.5"]
    return cfg, make_inputs(cfg), taus


def test_exact_count_sample_and_extrapolation():
    cfg, x, taus = _c1()
    layer = 3.0e9
    r = bench.cpu_baseline(cfg, x, taus, "tau", layer, 6, 0.0)
    tiles = sample_tiles(cfg, 6, seed=cfg.seed + 5)
    mq = -(-cfg.N // cfg.Bq)
    assert len(tiles) == 6 and (0, 0, 0) in tiles and (0, 0, mq - 1) in tiles
    assert r["sample"].startswith("6 seeded query tiles of c1 (exact count")
    assert r["kind"] == "oracle" and r["cores"] >= 1
    # c1 is causal with N a multiple of Bq = Bk: query tile i sees blocks 0..i,
    # each 2 * Bq * Bk * D FLOPs of QK^T and as many of PV (dense-equivalent).
    flops = sum(2 * bench.tile_flop(cfg) * (i + 1) for (_, _, i) in tiles)
    seconds = r["seconds_per_tile"] * len(tiles)
    assert np.isclose(r["value"] * 1e12 * seconds, flops, rtol=1e-9)
    assert np.isclose(r["extrapolated_layer_s"], layer / (r["value"] * 1e12), rtol=1e-12)


def test_budget_sample_runs_at_least_one_tile():
    cfg, x, taus = _c1()
    r = bench.cpu_baseline(cfg, x, taus, "tau", 3.0e9, 0, 0.0)
    n = int(r["sample"].split()[0])
    assert n >= 1 and r["value"] > 0 and "extrapolated_layer_s" not in r
