"""Randomised agreement of the oracle with the scalar brute force.

Hypothesis draws small shapes (ragged N, Bq != Bk, GQA, both masks, both
gates, per-head and per-tile thresholds) and seeds; the numpy oracle and the
loop-form brute force must agree on every block code and, to 1e-12, on every
output and lse value. A shrunk counterexample names the shape that breaks.
"""
import numpy as np
from hypothesis import given, settings, strategies as st, HealthCheck

from oracle import bsfa_oracle as O
from oracle import brute
from threshold_gated_block_b200.inputs import custom_config, make_inputs

shapes = st.tuples(
    st.integers(1, 70),                    # N
    st.sampled_from([4, 8]),               # D
    st.sampled_from([(1, 1), (2, 1), (2, 2), (4, 2)]),   # (Hq, Hkv)
    st.sampled_from([8, 16, 32]),          # Bq
    st.sampled_from([8, 16, 32]),          # Bk
    st.booleans(),                         # causal
    st.integers(0, 10_000),                # seed
)


@settings(max_examples=120, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(shape=shapes, level=st.floats(1.0, 3.0), per_tile=st.booleans())
def test_threshold_gate_matches_brute_force(shape, level, per_tile):
    N, D, (Hq, Hkv), Bq, Bk, causal, seed = shape
    x = make_inputs(custom_config(N=N, D=D, Hq=Hq, Hkv=Hkv, Bq=Bq, Bk=Bk, causal=causal, seed=seed))
    rng = np.random.default_rng(seed)
    mq = -(-N // Bq)
    if per_tile:
        tau = level + rng.uniform(-0.5, 0.5, size=(Hq, max(1, mq - 1)))
        tau_b = [list(row) for row in tau]
    else:
        tau = level + rng.uniform(-0.5, 0.5, size=Hq)
        tau_b = list(tau)
    r = O.forward(x["q"], x["k"], x["v"], tau, Bq, Bk, causal)
    qf, kf, vf = (O.widen_bf16(x[n]).tolist() for n in "qkv")
    out, lse, codes = brute.brute_forward(qf, kf, vf, tau_b, Bq, Bk, causal)
    for key, c in codes.items():
        assert r["codes"][key] == c, key
    np.testing.assert_allclose(r["out"], np.array(out), rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["lse"], np.array(lse), rtol=0, atol=1e-12)


@settings(max_examples=120, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(shape=shapes, gamma=st.floats(-2.0, 0.5))
def test_gap_gate_matches_brute_force(shape, gamma):
    N, D, (Hq, Hkv), Bq, Bk, causal, seed = shape
    x = make_inputs(custom_config(N=N, D=D, Hq=Hq, Hkv=Hkv, Bq=Bq, Bk=Bk, causal=causal, seed=seed))
    gam = [gamma + 0.1 * h for h in range(Hq)]
    r = O.forward(x["q"], x["k"], x["v"], gam, Bq, Bk, causal, gate="gap")
    qf, kf = (O.widen_bf16(x[n]).tolist() for n in "qk")
    codes = brute.brute_gap_codes(qf, kf, gam, Bq, Bk, causal)
    for key, c in codes.items():
        assert r["codes"][key] == c, key
