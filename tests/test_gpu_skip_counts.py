"""The skip itself, counted on the device ("Block Sparse Flash Attention" §4.3
Complexity Analysis, §4.4: a skipped block's values are not loaded and its PV
product is not issued).

A launch that writes the block mask also counts, per device, the V tiles it
loaded and the PV products it issued (bsfa_get_debug_counts). Both numbers are
fixed by the mask and by how the kernel groups query tiles: a CTA owns two
128-row slots that read the same key blocks (two query heads of one KV group
on the same rows when the group size is even, else two adjacent row blocks of
one head), so it loads block j's V tile once if either slot kept j, and issues
one PV product per (slot, kept block). A slot keeps j when any of its query
tiles (one at Bq = 128, two at Bq = 64) has code 1 or 2 at j.
"""
import numpy as np
import pytest
import torch

from oracle.calibrate import calibrate
from threshold_gated_block_b200 import bsfa
from threshold_gated_block_b200.build import build
from threshold_gated_block_b200.inputs import CONFIGS, custom_config, make_inputs

from parity import run_gpu, stored_taus

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build()
    bsfa.load()


def expected_counts(mask: np.ndarray, Bq: int, Hq: int, Hkv: int):
    """(V tiles, PV products) a launch must have issued, from its block codes."""
    B, _, MQ, MKV = mask.shape
    kept = np.isin(mask, (1, 2))
    per = 128 // Bq                                   # query tiles per 128-row slot
    rows128 = -(-MQ // per)                           # 128-row blocks of the sequence

    def slot(b, h, r):                                # keep flags of the slot holding 128-row block r of head h
        ts = [t for t in range(r * per, (r + 1) * per) if t < MQ]
        return kept[b, h, ts].any(axis=0) if ts else np.zeros(MKV, dtype=bool)

    v = pv = 0
    for b in range(B):
        if (Hq // Hkv) % 2 == 0:                      # two heads of a KV group on the same rows
            pairs = [((b, 2 * hp, r), (b, 2 * hp + 1, r)) for hp in range(Hq // 2) for r in range(rows128)]
        else:                                         # two adjacent row blocks of one head
            pairs = [((b, h, 2 * rp), (b, h, 2 * rp + 1)) for h in range(Hq) for rp in range(-(-rows128 // 2))]
        for a, c in pairs:
            s0, s1 = slot(*a), slot(*c)
            v += int((s0 | s1).sum())
            pv += int(s0.sum() + s1.sum())
    return v, pv


def _counted_run(x, tau, Bq, Bk, causal):
    bsfa.debug_counts()                               # start from zero
    gpu = run_gpu(x, tau, Bq, Bk, causal, want_mask=True)
    return gpu["mask"], bsfa.debug_counts()


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (6, 6), (3, 1)])
@pytest.mark.parametrize("Bq,Bk", [(128, 128), (64, 64), (64, 128), (128, 64)])
@pytest.mark.parametrize("causal", [True, False])
def test_counts_follow_the_mask_small(Hq, Hkv, Bq, Bk, causal):
    N = 900
    cfg = custom_config(B=2, N=N, D=64, Hq=Hq, Hkv=Hkv, Bq=Bq, Bk=Bk, causal=causal, kind="planted", seed=80 + Hq)
    x = make_inputs(cfg)
    tau = calibrate(x["q"], x["k"], Bq, Bk, causal, [0.6])[0.6]
    mask, (v, pv) = _counted_run(x, tau, Bq, Bk, causal)
    ev, epv = expected_counts(mask, Bq, Hq, Hkv)
    assert (mask == 0).any(), "the case must skip some blocks"
    assert (v, pv) == (ev, epv)
    # and a dense launch of the same layer loads every visible block
    dmask, (dv, dpv) = _counted_run(x, [-np.inf] * Hq, Bq, Bk, causal)
    assert (dv, dpv) == expected_counts(dmask, Bq, Hq, Hkv)
    assert dv > v and dpv > pv


def test_counts_on_the_8k_layer():
    cfg = CONFIGS["c2"]
    x = make_inputs(cfg)
    tau = stored_taus("c2", 0.5)
    mask, (v, pv) = _counted_run(x, tau, cfg.Bq, cfg.Bk, cfg.causal)
    ev, epv = expected_counts(mask, cfg.Bq, cfg.Hq, cfg.Hkv)
    print({"v_tiles": v, "pv_products": pv, "visible_tiles": int((mask != 3).sum())})
    assert (v, pv) == (ev, epv)
    # PV products: exactly the kept (head, tile, block) entries at Bq = 128
    assert pv == int(np.isin(mask, (1, 2)).sum())


def test_launches_without_a_mask_count_nothing():
    cfg = custom_config(B=1, N=512, D=128, Hq=4, Hkv=2, Bq=128, Bk=128, causal=True, kind="normal", seed=3)
    x = make_inputs(cfg)
    bsfa.debug_counts()
    run_gpu(x, [0.0] * 4, 128, 128, True, want_mask=False)
    assert bsfa.debug_counts() == (0, 0)
