"""GPU parity for packed mixed-length batches (bsfa_forward_varlen).

Sequences of different lengths (one token, ragged ends, whole tiles, a long
one, an empty one) are packed along the row dimension. Each sequence is its own
attention problem, so the oracle runs on each sequence alone; the comparison
and tolerances are those of parity.py. The packed result must also equal,
bit for bit, the fixed-length entry point run on each sequence alone.
"""
import numpy as np
import pytest
import torch

from oracle.calibrate import calibrate
from threshold_gated_block_b200 import bsfa
from threshold_gated_block_b200.build import build
from threshold_gated_block_b200.inputs import custom_config, make_inputs

from parity import Report, all_tiles, compare_tiles, to_device

pytestmark = pytest.mark.gpu

LENGTHS = [300, 1, 129, 0, 640, 63, 1000, 128]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build()
    bsfa.load()


def _packed(lengths, D, Hq, Hkv, kind, seed):
    total = sum(lengths)
    cfg = custom_config(B=1, N=total, D=D, Hq=Hq, Hkv=Hkv, Bq=64, Bk=64, causal=True, kind=kind, seed=seed)
    x = make_inputs(cfg)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return {n: x[n][0] for n in "qkv"}, cu


def _run_varlen(x, cu, tau, Bq, Bk, causal):
    q, k, v = (to_device(x[n]) for n in "qkv")
    t = torch.tensor(np.asarray(tau, dtype=np.float32), device="cuda")
    cu_d = torch.tensor(cu, dtype=torch.int32, device="cuda")
    max_len = int(np.diff(cu).max())
    out, lse, mask = bsfa.forward_varlen(q, k, v, cu_d, max_len, t, Bq=Bq, Bk=Bk, causal=causal, want_mask=True)
    torch.cuda.synchronize()
    assert bsfa.bsfa_get_status(None) == bsfa.BSFA_OK, bsfa.bsfa_last_error()
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64), mask.cpu().numpy()


def _compare(x, cu, tau, Bq, Bk, causal, out, lse, mask):
    rep = Report()
    for e in range(len(cu) - 1):
        r0, r1 = int(cu[e]), int(cu[e + 1])
        n = r1 - r0
        if n == 0:
            assert (mask[e] == 3).all()
            continue
        xe = {name: x[name][None, r0:r1] for name in "qkv"}
        mq, mkv = -(-n // Bq), -(-n // Bk)
        ge = {"out": out[None, r0:r1], "lse": lse[None, :, r0:r1], "mask": mask[e][None, :, :mq, :mkv]}
        assert (mask[e][:, mq:, :] == 3).all() and (mask[e][:, :, mkv:] == 3).all()
        compare_tiles(xe, tau, Bq, Bk, causal, ge, all_tiles(1, x["q"].shape[1], n, Bq), rep)
    return rep.check()


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("Bq,Bk", [(128, 128), (64, 64), (128, 64), (64, 128)])
@pytest.mark.parametrize("D", [64, 128])
def test_varlen_every_variant(D, Bq, Bk, causal):
    x, cu = _packed(LENGTHS, D, 4, 2, "planted", seed=D + Bq + Bk)
    tau = calibrate(x["q"][None, 1133:2133], x["k"][None, 1133:2133], Bq, Bk, causal, [0.5])[0.5]
    out, lse, mask = _run_varlen(x, cu, tau, Bq, Bk, causal)
    stats = _compare(x, cu, tau, Bq, Bk, causal, out, lse, mask)
    assert (mask == 0).any() and (mask == 1).any()
    print(stats)


@pytest.mark.parametrize("Hq,Hkv", [(4, 2), (3, 3)])
def test_varlen_equals_each_sequence_alone(Hq, Hkv):
    x, cu = _packed(LENGTHS, 128, Hq, Hkv, "normal", seed=7 + Hq)
    tau = calibrate(x["q"][None, 1133:2133], x["k"][None, 1133:2133], 128, 128, True, [0.5])[0.5]
    out, lse, mask = _run_varlen(x, cu, tau, 128, 128, True)
    t = torch.tensor(np.asarray(tau, dtype=np.float32), device="cuda")
    for e in range(len(cu) - 1):
        r0, r1 = int(cu[e]), int(cu[e + 1])
        if r1 == r0:
            continue
        q, k, v = (to_device(x[n][None, r0:r1]) for n in "qkv")
        o1, l1, m1 = bsfa.forward(q, k, v, t, Bq=128, Bk=128, causal=True, want_mask=True)
        torch.cuda.synchronize()
        assert np.array_equal(o1.float().cpu().numpy()[0], out[r0:r1]), e
        assert np.array_equal(l1.cpu().numpy()[0], lse[:, r0:r1]), e
        n = r1 - r0
        assert np.array_equal(m1.cpu().numpy()[0], mask[e][:, : -(-n // 128), : -(-n // 128)]), e


def test_packed_total_beyond_the_per_sequence_block_limit():
    """A packed batch whose total (about 283,000 rows) exceeds 4096 blocks of 64 keys,
    made of many short sequences: the limit applies per sequence, so it runs.
    Checked against the oracle on a seeded sample of sequences, the last among them."""
    rng = np.random.default_rng(77)
    lengths = [int(n) for n in rng.integers(1, 1200, size=460)]
    total = sum(lengths)
    assert total > 4096 * 64 and max(lengths) <= 4096 * 64
    Hq, Hkv, D, Bq, Bk = 2, 1, 64, 64, 64
    cfg = custom_config(B=1, N=total, D=D, Hq=Hq, Hkv=Hkv, Bq=Bq, Bk=Bk, causal=True, kind="normal", seed=78)
    xx = make_inputs(cfg)
    x = {n: xx[n][0] for n in "qkv"}
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    tau = calibrate(x["q"][None, :2048], x["k"][None, :2048], Bq, Bk, True, [0.5])[0.5]
    out, lse, mask = _run_varlen(x, cu, tau, Bq, Bk, True)
    pick = sorted(set(int(e) for e in rng.choice(len(lengths) - 1, size=12, replace=False)) | {len(lengths) - 1})
    rep = Report()
    for e in pick:
        r0, r1 = int(cu[e]), int(cu[e + 1])
        n = r1 - r0
        xe = {name: x[name][None, r0:r1] for name in "qkv"}
        mq, mkv = -(-n // Bq), -(-n // Bk)
        ge = {"out": out[None, r0:r1], "lse": lse[None, :, r0:r1], "mask": mask[e][None, :, :mq, :mkv]}
        compare_tiles(xe, tau, Bq, Bk, True, ge, all_tiles(1, Hq, n, Bq), rep)
    stats = rep.check()
    assert (mask == 0).any() and (mask == 1).any()
    print(stats)
