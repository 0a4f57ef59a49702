"""Pins for the CPU oracle: checks against things other than the oracle itself.

* hand-derived closed forms (tests/golden/hand_example.json);
* the scalar brute force, a loop-form statement of the same definition that
  finds visibility, forced blocks and block maxima by enumeration;
* tau = -inf is dense softmax attention (torch SDPA in float64, a library routine);
* tau = +inf with Bq = Bk is block-local attention (SDPA with a block-diagonal mask);
* invariants: attention weights form a convex combination over the kept keys,
  out and lse agree with each other, permuting keys inside a fully valid
  off-diagonal block or queries inside a bidirectional tile changes nothing but
  the order, scaling V scales out, the kept set shrinks monotonically as tau grows.

Sources: "Block Sparse Flash Attention" §4.1 (gate, diagonal bypass), §4.4
(skipped blocks stay out of the statistics), App. B.2 (scaled scores, online
softmax), App. B.3 (bidirectional case).
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


def _eval(expr: str) -> float:
    return float(eval(expr, {"__builtins__": {}}, {"e": math.e, "ln": math.log}))


def _bits(a) -> np.ndarray:
    bits = f32_to_bf16_bits(np.asarray(a, dtype=np.float32))
    assert np.array_equal(O.widen_bf16(bits), np.asarray(a, dtype=np.float64)), "not bf16-exact"
    return bits


# ----------------------------------------------------------------------------- bf16 widening

def test_widen_bf16_known_patterns():
    pats = np.array([0x3F80, 0xC000, 0x3F81, 0x0000, 0x8000, 0x3E00, 0x4049, 0x0001], dtype=np.uint16)
    want = [1.0, -2.0, 1.0078125, 0.0, -0.0, 0.125, 3.140625, 2.0 ** -133]
    got = O.widen_bf16(pats)
    assert got.tolist() == want
    assert math.copysign(1.0, got[4]) == -1.0


# ----------------------------------------------------------------------------- closed forms

def _hand_cases(golden_dir):
    with open(os.path.join(golden_dir, "hand_example.json")) as f:
        g = json.load(f)
    q = _bits(g["q"])[None, :, None, :]
    k = _bits(g["k"])[None, :, None, :]
    v = _bits(g["v"])[None, :, None, :]
    return g, q, k, v


def test_hand_example_closed_forms(golden_dir):
    g, q, k, v = _hand_cases(golden_dir)
    for case in g["cases"]:
        r = O.forward(q, k, v, [case["tau"]], g["Bq"], g["Bk"], case["causal"])
        assert r["codes"][0, 0].tolist() == case["codes"], case["name"]
        want_out = np.array([[_eval(x) for x in row] for row in case["out"]])
        want_lse = np.array([_eval(x) for x in case["lse"]])
        np.testing.assert_allclose(r["out"][0, :, 0, :], want_out, rtol=0, atol=1e-14, err_msg=case["name"])
        np.testing.assert_allclose(r["lse"][0, 0], want_lse, rtol=0, atol=1e-14, err_msg=case["name"])


# ----------------------------------------------------------------------------- brute force

BRUTE_CASES = [
    # N, D, Hq, Hkv, Bq, Bk, causal
    (64, 8, 2, 1, 16, 16, True),
    (64, 16, 4, 2, 16, 32, True),
    (64, 8, 4, 2, 32, 16, True),
    (48, 8, 2, 2, 16, 16, False),
    (64, 8, 4, 2, 32, 16, False),
    (128, 8, 2, 1, 32, 32, True),
    # ragged sequence ends: a last tile of one row, partial key blocks
    (65, 8, 2, 1, 16, 16, True),
    (81, 8, 4, 2, 32, 16, True),
    (50, 8, 2, 1, 16, 32, False),
    (97, 16, 2, 2, 32, 32, False),
]


def _calibrated_taus(x, Bq, Bk, causal, p=0.5):
    from oracle.calibrate import calibrate
    return calibrate(x["q"], x["k"], Bq, Bk, causal, [p])[p]


@pytest.mark.parametrize("N,D,Hq,Hkv,Bq,Bk,causal", BRUTE_CASES)
def test_oracle_matches_scalar_brute_force(N, D, Hq, Hkv, Bq, Bk, causal):
    cfg = custom_config(N=N, D=D, Hq=Hq, Hkv=Hkv, Bq=Bq, Bk=Bk, causal=causal, seed=N + D + Bq)
    x = make_inputs(cfg)
    tau = _calibrated_taus(x, Bq, Bk, causal)
    r = O.forward(x["q"], x["k"], x["v"], tau, Bq, Bk, causal)
    qf, kf, vf = (O.widen_bf16(x[n]).tolist() for n in "qkv")
    out, lse, codes = brute.brute_forward(qf, kf, vf, tau, Bq, Bk, causal)
    for key, c in codes.items():
        assert r["codes"][key] == c, key
    assert (r["codes"] == O.CODE_SKIPPED).any() and (r["codes"] == O.CODE_KEPT).any()
    np.testing.assert_allclose(r["out"], np.array(out), rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["lse"], np.array(lse), rtol=0, atol=1e-12)


@pytest.mark.parametrize("N,causal", [(96, True), (81, True), (70, False)])
def test_per_tile_thresholds_match_brute_force(N, causal):
    """A [Hq, T] table: tile i of head h uses column min(i, T-1) (§4.1, App. B.3)."""
    Bq = Bk = 16
    cfg = custom_config(N=N, D=8, Hq=2, Hkv=1, Bq=Bq, Bk=Bk, causal=causal, seed=N)
    x = make_inputs(cfg)
    mq = -(-N // Bq)
    rng = np.random.default_rng(N)
    table = rng.uniform(2.0, 3.2, size=(2, mq - 2))          # shorter than M_Q: the last column is reused
    r = O.forward(x["q"], x["k"], x["v"], table, Bq, Bk, causal)
    qf, kf, vf = (O.widen_bf16(x[n]).tolist() for n in "qkv")
    out, lse, codes = brute.brute_forward(qf, kf, vf, [list(row) for row in table], Bq, Bk, causal)
    for key, c in codes.items():
        assert r["codes"][key] == c, key
    assert (r["codes"] == O.CODE_SKIPPED).any() and (r["codes"] == O.CODE_KEPT).any()
    np.testing.assert_allclose(r["out"], np.array(out), rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["lse"], np.array(lse), rtol=0, atol=1e-12)
    # a per-head vector and a one-column table are the same thresholds
    per_head = O.forward(x["q"], x["k"], x["v"], table[:, 0], Bq, Bk, causal)
    one_col = O.forward(x["q"], x["k"], x["v"], table[:, :1], Bq, Bk, causal)
    assert np.array_equal(per_head["codes"], one_col["codes"])


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("N", [33, 65, 97])
def test_every_row_keeps_its_own_key_at_ragged_ends(N, causal):
    """At tau=+inf only forced blocks remain; with N = 1 (mod Bq) the last tile has
    one row, and the block holding that row's key must still be forced."""
    cfg = custom_config(N=N, D=8, Hq=1, Hkv=1, Bq=32, Bk=32, causal=causal, seed=N)
    x = make_inputs(cfg)
    r = O.forward(x["q"], x["k"], x["v"], [np.inf], 32, 32, causal)
    assert np.isfinite(r["lse"]).all() and np.isfinite(r["out"]).all()
    for row in range(N):
        assert r["codes"][0, 0, row // 32, row // 32] == O.CODE_FORCED


# ----------------------------------------------------------------------------- library special cases

def _sdpa(x, mask_fn, Hq, Hkv, D):
    """Textbook attention via torch SDPA in float64 with an explicit boolean mask."""
    q = torch.from_numpy(O.widen_bf16(x["q"])).permute(0, 2, 1, 3)      # B,H,N,D
    k = torch.from_numpy(O.widen_bf16(x["k"])).permute(0, 2, 1, 3)
    v = torch.from_numpy(O.widen_bf16(x["v"])).permute(0, 2, 1, 3)
    k = k.repeat_interleave(Hq // Hkv, dim=1)
    v = v.repeat_interleave(Hq // Hkv, dim=1)
    N = q.shape[2]
    mask = torch.tensor([[mask_fn(r, c) for c in range(N)] for r in range(N)])
    out = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask)
    s = (q @ k.transpose(-1, -2)) / math.sqrt(D)
    lse = torch.logsumexp(s.masked_fill(~mask, -math.inf), dim=-1)
    return out.permute(0, 2, 1, 3).numpy(), lse.numpy()


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("Bq,Bk", [(32, 32), (64, 32), (32, 64)])
def test_tau_minus_inf_is_dense_attention(causal, Bq, Bk):
    N, D, Hq, Hkv = 256, 32, 4, 2
    x = make_inputs(custom_config(N=N, D=D, Hq=Hq, Hkv=Hkv, Bq=Bq, Bk=Bk, causal=causal, seed=11))
    r = O.forward(x["q"], x["k"], x["v"], [-np.inf] * Hq, Bq, Bk, causal)
    out, lse = _sdpa(x, (lambda a, b: b <= a) if causal else (lambda a, b: True), Hq, Hkv, D)
    assert not (r["codes"] == O.CODE_SKIPPED).any()
    np.testing.assert_allclose(r["out"], out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["lse"], lse, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_tau_plus_inf_is_block_local_attention(causal):
    N, D, Hq, Hkv, B_ = 256, 32, 2, 1, 32
    x = make_inputs(custom_config(N=N, D=D, Hq=Hq, Hkv=Hkv, Bq=B_, Bk=B_, causal=causal, seed=12))
    r = O.forward(x["q"], x["k"], x["v"], [np.inf] * Hq, B_, B_, causal)
    if causal:
        local = lambda a, b: (a // B_ == b // B_) and b <= a
    else:
        local = lambda a, b: a // B_ == b // B_
    out, lse = _sdpa(x, local, Hq, Hkv, D)
    assert not (r["codes"] == O.CODE_KEPT).any()
    np.testing.assert_allclose(r["out"], out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["lse"], lse, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- invariants

def test_weights_are_a_convex_combination_over_the_kept_set():
    # V = identity, so out[r] is row r's weight vector over the keys.
    N, D, Bq, Bk = 32, 32, 8, 8
    for causal in (True, False):
        x = make_inputs(custom_config(N=N, D=D, Hq=2, Hkv=1, Bq=Bq, Bk=Bk, causal=causal, seed=5))
        x["v"] = _bits(np.eye(N, D)[None, :, None, :])
        tau = _calibrated_taus(x, Bq, Bk, causal)
        r = O.forward(x["q"], x["k"], x["v"], tau, Bq, Bk, causal)
        qf, kf = O.widen_bf16(x["q"]), O.widen_bf16(x["k"])
        for h in range(2):
            s = qf[0, :, h, :] @ kf[0, :, 0, :].T / math.sqrt(D)
            for row in range(N):
                w = r["out"][0, row, h, :N]
                codes = r["codes"][0, h, row // Bq]
                kept = np.array([(c <= row or not causal) and codes[c // Bk] in (1, 2) for c in range(N)])
                assert (w >= 0).all()
                assert abs(w.sum() - 1.0) < 1e-13
                assert (w[~kept] == 0).all()
                # each kept weight is exp(s - lse): out and lse describe the same distribution
                np.testing.assert_allclose(w[kept], np.exp(s[row, kept] - r["lse"][0, h, row]), atol=1e-13)
                assert r["lse"][0, h, row] >= s[row, kept].max() - 1e-13
                assert r["lse"][0, h, row] <= s[row, kept].max() + math.log(kept.sum()) + 1e-13


def test_key_permutation_inside_an_offdiagonal_block():
    N, D, Bq, Bk = 128, 16, 32, 32
    x = make_inputs(custom_config(N=N, D=D, Hq=2, Hkv=1, Bq=Bq, Bk=Bk, causal=True, seed=21))
    tau = _calibrated_taus(x, Bq, Bk, True)
    r0 = O.forward(x["q"], x["k"], x["v"], tau, Bq, Bk, True)
    j = 1                                     # block 1 is fully valid for tiles 2 and 3
    perm = np.arange(N)
    rng = np.random.default_rng(3)
    perm[j * Bk:(j + 1) * Bk] = j * Bk + rng.permutation(Bk)
    y = dict(x, k=x["k"][:, perm], v=x["v"][:, perm])
    r1 = O.forward(y["q"], y["k"], y["v"], tau, Bq, Bk, True)
    rows = slice((j + 1) * Bq, N)
    assert np.array_equal(r0["codes"][:, :, j + 1:], r1["codes"][:, :, j + 1:])
    np.testing.assert_allclose(r1["out"][:, rows], r0["out"][:, rows], atol=1e-13)
    np.testing.assert_allclose(r1["lse"][:, :, rows], r0["lse"][:, :, rows], atol=1e-13)


def test_query_permutation_inside_a_bidirectional_tile():
    N, D, Bq, Bk = 128, 16, 32, 32
    x = make_inputs(custom_config(N=N, D=D, Hq=2, Hkv=2, Bq=Bq, Bk=Bk, causal=False, seed=22))
    tau = _calibrated_taus(x, Bq, Bk, False)
    r0 = O.forward(x["q"], x["k"], x["v"], tau, Bq, Bk, False)
    perm = np.arange(N)
    perm[Bq:2 * Bq] = Bq + np.random.default_rng(4).permutation(Bq)
    r1 = O.forward(x["q"][:, perm], x["k"], x["v"], tau, Bq, Bk, False)
    assert np.array_equal(r0["codes"], r1["codes"])
    np.testing.assert_allclose(r1["out"], r0["out"][:, perm], atol=1e-13)
    np.testing.assert_allclose(r1["lse"], r0["lse"][:, :, perm], atol=1e-13)


@pytest.mark.parametrize("alpha", [2.0, 0.5, -1.0])
def test_value_scaling(alpha):
    N, D, Bq, Bk = 128, 16, 32, 32
    x = make_inputs(custom_config(N=N, D=D, Hq=2, Hkv=1, Bq=Bq, Bk=Bk, causal=True, seed=23))
    tau = _calibrated_taus(x, Bq, Bk, True)
    r0 = O.forward(x["q"], x["k"], x["v"], tau, Bq, Bk, True)
    v2 = _bits(O.widen_bf16(x["v"]) * alpha)
    r1 = O.forward(x["q"], x["k"], v2, tau, Bq, Bk, True)
    np.testing.assert_allclose(r1["out"], alpha * r0["out"], atol=1e-13)
    np.testing.assert_array_equal(r1["lse"], r0["lse"])


def test_kept_set_shrinks_as_tau_grows():
    N, D, Bq, Bk = 256, 16, 32, 32
    x = make_inputs(custom_config(N=N, D=D, Hq=2, Hkv=1, Bq=Bq, Bk=Bk, causal=True, seed=24))
    prev = None
    for t in np.linspace(-1.0, 6.0, 15):
        codes = O.forward(x["q"], x["k"], x["v"], [t, t], Bq, Bk, True)["codes"]
        kept = codes == O.CODE_KEPT
        if prev is not None:
            assert not (kept & ~prev).any()
        prev = kept
        assert ((codes == O.CODE_FORCED).sum(axis=-1) >= 1).all()


def test_bf16_round_to_nearest_even():
    x = np.array([1.00390625, 1.01171875, -1.00390625, 1.0], dtype=np.float32)
    assert f32_to_bf16_bits(x).tolist() == [0x3F80, 0x3F82, 0xBF80, 0x3F80]


# ----------------------------------------------------------------------------- packed mixed-length batches

def test_varlen_oracle_is_each_sequence_alone():
    """A packed batch is the per-sequence forward on each [cu[e], cu[e+1]) slice,
    checked here against the scalar brute force of each slice; empty sequences
    produce nothing and rows of one sequence never see another's keys."""
    lengths = [17, 0, 40, 1, 33]
    cfg = custom_config(N=sum(lengths), D=8, Hq=2, Hkv=1, Bq=16, Bk=16, causal=True, seed=3)
    x = make_inputs(cfg)
    packed = {n: x[n][0] for n in "qkv"}
    cu = np.concatenate([[0], np.cumsum(lengths)])
    tau = [2.0, 2.4]
    r = O.forward_varlen(packed["q"], packed["k"], packed["v"], cu, tau, 16, 16, True)
    assert r["out"].shape == (sum(lengths), 2, 8) and r["lse"].shape == (2, sum(lengths))
    assert r["codes"][1] is None
    for e, n in enumerate(lengths):
        if n == 0:
            continue
        r0, r1 = int(cu[e]), int(cu[e + 1])
        qf, kf, vf = (O.widen_bf16(packed[m][r0:r1])[None].tolist() for m in "qkv")
        out, lse, codes = brute.brute_forward(qf, kf, vf, tau, 16, 16, True)
        np.testing.assert_allclose(r["out"][r0:r1], np.array(out)[0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(r["lse"][:, r0:r1], np.array(lse)[0], rtol=0, atol=1e-12)
        for (b, hq, i, j), c in codes.items():
            assert r["codes"][e][hq, i, j] == c
