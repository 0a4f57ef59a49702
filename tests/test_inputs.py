"""The seeded input generators: reproducible bits, the stated layout, and the
structure each recipe promises (sink, needles, grid-local DiT scores).

Both the oracle and the CUDA path consume these bits, so a silent change here
would move every parity case and stored threshold at once.
"""
import math

import numpy as np
import pytest

from threshold_gated_block_b200.inputs import (NEEDLE_COSINE, NEEDLES_PER_HEAD, QUERIES_PER_NEEDLE, SINK_KEYS,
                                               CONFIGS, bf16_bits_to_f32, custom_config, make_inputs, sample_tiles)


@pytest.mark.parametrize("kind", ["normal", "planted"])
def test_same_seed_same_bits_other_seed_other_bits(kind):
    cfg = custom_config(N=320, D=64, Hq=4, Hkv=2, kind=kind, seed=11)
    a, b, c = make_inputs(cfg), make_inputs(cfg), make_inputs(cfg, seed=12)
    for n in "qkv":
        assert a[n].dtype == np.uint16
        assert np.array_equal(a[n], b[n])
        assert not np.array_equal(a[n], c[n])
    assert a["recipe"]["seed"] == 11 and c["recipe"]["seed"] == 12


def test_layout_is_b_n_h_d():
    cfg = custom_config(B=2, N=100, D=64, Hq=6, Hkv=3, kind="normal", seed=3)
    x = make_inputs(cfg)
    assert x["q"].shape == (2, 100, 6, 64)
    assert x["k"].shape == x["v"].shape == (2, 100, 3, 64)
    assert all(x[n].flags.c_contiguous for n in "qkv")
    q = bf16_bits_to_f32(x["q"]).astype(np.float64)
    assert abs(q.mean()) < 0.02 and abs(q.std() - 1.0) < 0.02


def _planted(N=768, D=64, Hq=4, Hkv=2, seed=5):
    cfg = custom_config(N=N, D=D, Hq=Hq, Hkv=Hkv, kind="planted", seed=seed)
    x = make_inputs(cfg)
    return cfg, {n: bf16_bits_to_f32(x[n]).astype(np.float64) for n in "qkv"}


def test_needles_are_matched_by_later_queries():
    """Every needle key has norm sqrt(D); each q-head of its group has rows at
    cosine NEEDLE_COSINE to it, at most QUERIES_PER_NEEDLE of them and all at or
    after the needle (visible to it under the causal mask). A later needle may take
    over a row an earlier one had claimed, so the total is a little under
    NEEDLES_PER_HEAD * QUERIES_PER_NEEDLE."""
    cfg, x = _planted(N=2048)
    D, g = cfg.D, cfg.group
    qn = x["q"] / np.linalg.norm(x["q"], axis=-1, keepdims=True)
    for kv in range(cfg.Hkv):
        keys = x["k"][0, :, kv, :]
        kn = keys / np.linalg.norm(keys, axis=-1, keepdims=True)
        for h in range(kv * g, (kv + 1) * g):
            cos = qn[0, :, h, :] @ kn.T                        # [query, key]
            rows, cols = np.nonzero(np.abs(cos - NEEDLE_COSINE) < 0.01)
            needles = np.unique(cols)
            assert len(needles) == NEEDLES_PER_HEAD
            assert (needles >= SINK_KEYS).all()
            assert np.allclose(np.linalg.norm(keys[needles], axis=-1), math.sqrt(D), rtol=1e-2)
            assert (rows >= cols).all()
            per_needle = np.bincount(cols, minlength=cfg.N)[needles]
            assert per_needle.max() <= QUERIES_PER_NEEDLE
            assert per_needle.sum() >= 0.75 * NEEDLES_PER_HEAD * QUERIES_PER_NEEDLE


def test_sink_keys_are_shifted_by_two_sqrt_d():
    """The first SINK_KEYS keys of each KV head carry a common shift of norm
    2 sqrt(D) (their mean has that norm, up to the noise of 64 N(0,1) draws);
    other keys carry none."""
    cfg, x = _planted(seed=6)
    shift = 2.0 * math.sqrt(cfg.D)
    for kv in range(cfg.Hkv):
        k = x["k"][0, :, kv, :]
        assert abs(np.linalg.norm(k[:SINK_KEYS].mean(axis=0)) - shift) < 0.15 * shift
        assert np.linalg.norm(k[SINK_KEYS:].mean(axis=0)) < 0.1 * shift


def test_dit_scores_are_local_on_the_grid():
    """Q and K share a smooth, per-channel standardised field: the q.k/D
    covariance is about 1 at a query's own grid cell, almost as large at the
    next cell (Gaussian blur, sigma 4 cells) and small half the grid away."""
    side, D = 32, 64
    cfg = custom_config(N=side * side, D=D, Hq=2, Hkv=2, causal=False, kind="dit", seed=9)
    x = make_inputs(cfg)
    q = bf16_bits_to_f32(x["q"])[0, :, 0, :].astype(np.float64).reshape(side, side, D)
    k = bf16_bits_to_f32(x["k"])[0, :, 0, :].astype(np.float64).reshape(side, side, D)
    cov = lambda a, b: float(np.mean(np.sum(a * b, axis=-1)) / D)
    assert 0.85 < cov(q, k) < 1.15
    assert cov(q[:, :-1], k[:, 1:]) > 0.8
    assert cov(q[:-1], k[1:]) > 0.8
    # half the grid away: near 0, a little negative (each channel's grid mean is removed)
    assert abs(cov(q[:, : side // 2], k[:, side // 2:])) < 0.3


def test_dit_needs_a_square_grid_and_mha():
    with pytest.raises(ValueError):
        make_inputs(custom_config(N=1000, D=64, Hq=2, Hkv=2, causal=False, kind="dit"))
    with pytest.raises(ValueError):
        make_inputs(custom_config(N=1024, D=64, Hq=4, Hkv=2, causal=False, kind="dit"))


def test_sampled_tiles_are_seeded_and_hold_the_ends():
    cfg = CONFIGS["c4"]
    a, b = sample_tiles(cfg, 64), sample_tiles(cfg, 64)
    mq = -(-cfg.N // cfg.Bq)
    assert a == b and len(a) == 64 and len(set(a)) == 64
    assert (0, 0, 0) in a and (0, 0, mq - 1) in a
    assert all(0 <= h < cfg.Hq and 0 <= i < mq for (_, h, i) in a)
    assert sample_tiles(cfg, 64, seed=1) != a
