"""GPU parity of the BSFA forward against the CPU oracle, through the C ABI.

Every case compares element by element with the oracle on the same seeded
bf16 inputs (see parity.py for the tolerances). The small cases span several
tiles, every kernel variant (D, Bq, Bk, causal) and GQA group sizes; the
workload configurations run at their full sizes with the thresholds stored in
tests/golden/taus.json, compared on every tile (c1, c2) or on seeded samples of
tiles (c3, c4, c5).
"""
import numpy as np
import pytest
import torch

from oracle.calibrate import calibrate
from threshold_gated_block_b200 import bsfa
from threshold_gated_block_b200.build import build
from threshold_gated_block_b200.inputs import CONFIGS, custom_config, make_inputs, sample_tiles

from parity import Report, all_tiles, compare_tiles, run_gpu, stored_taus

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build()
    bsfa.load()


def _small(D, Bq, Bk, causal, N=512, Hq=4, Hkv=2, B=1, kind="normal", seed=3):
    cfg = custom_config(B=B, N=N, D=D, Hq=Hq, Hkv=Hkv, Bq=Bq, Bk=Bk, causal=causal, kind=kind, seed=seed)
    return cfg, make_inputs(cfg)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("Bk", [64, 128])
@pytest.mark.parametrize("Bq", [64, 128])
@pytest.mark.parametrize("D", [64, 128])
def test_every_variant_small(D, Bq, Bk, causal):
    cfg, x = _small(D, Bq, Bk, causal, N=640 if causal else 512, seed=D + Bq + Bk + causal)
    tau = calibrate(x["q"], x["k"], Bq, Bk, causal, [0.5])[0.5]
    gpu = run_gpu(x, tau, Bq, Bk, causal)
    rep = compare_tiles(x, tau, Bq, Bk, causal, gpu, all_tiles(cfg.B, cfg.Hq, cfg.N, Bq))
    stats = rep.check()
    codes = gpu["mask"]
    assert (codes == 0).any() and (codes == 1).any() and (codes == 2).any()
    if causal:
        assert (codes == 3).any()
    print(stats)


@pytest.mark.parametrize("group", [1, 4, 8])
def test_gqa_groups_and_batch(group):
    Hkv = 2
    cfg, x = _small(128, 128, 128, True, N=1024, Hq=Hkv * group, Hkv=Hkv, B=2, kind="planted", seed=40 + group)
    tau = calibrate(x["q"], x["k"], 128, 128, True, [0.6])[0.6]
    gpu = run_gpu(x, tau, 128, 128, True)
    compare_tiles(x, tau, 128, 128, True, gpu, all_tiles(cfg.B, cfg.Hq, cfg.N, 128)).check()


@pytest.mark.parametrize("causal", [True, False])
def test_dense_and_block_local_limits(causal):
    cfg, x = _small(128, 128, 64, causal, N=768, Hq=4, Hkv=2, seed=9)
    for t in (-np.inf, np.inf):
        tau = [t] * cfg.Hq
        gpu = run_gpu(x, tau, 128, 64, causal)
        compare_tiles(x, tau, 128, 64, causal, gpu, all_tiles(cfg.B, cfg.Hq, cfg.N, 128)).check()
        assert not (gpu["mask"] == (0 if t == -np.inf else 1)).any()


def test_dense_limit_matches_torch_attention():
    """tau = -inf is plain attention: compare with torch SDPA in fp32 on the GPU."""
    cfg, x = _small(128, 128, 128, True, N=1024, Hq=8, Hkv=2, seed=10)
    gpu = run_gpu(x, [-np.inf] * cfg.Hq, 128, 128, True, want_mask=False)
    q, k, v = (torch.from_numpy(x[n].view(np.int16)).view(torch.bfloat16).cuda().float().transpose(1, 2) for n in "qkv")
    k = k.repeat_interleave(4, dim=1)
    v = v.repeat_interleave(4, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True).transpose(1, 2)
    d = np.abs(gpu["out"] - ref.cpu().numpy())
    assert d.max() <= 2e-2 and d.mean() <= 2e-3


def test_mixed_per_head_thresholds():
    cfg, x = _small(64, 64, 64, True, N=512, Hq=4, Hkv=4, seed=12)
    tau = calibrate(x["q"], x["k"], 64, 64, True, [0.5])[0.5]
    tau = [-np.inf, tau[1], np.inf, tau[3]]
    gpu = run_gpu(x, tau, 64, 64, True)
    compare_tiles(x, tau, 64, 64, True, gpu, all_tiles(cfg.B, cfg.Hq, cfg.N, 64)).check()


def test_optional_outputs_and_determinism():
    cfg, x = _small(128, 128, 128, True, N=1024, Hq=4, Hkv=1, kind="planted", seed=13)
    tau = calibrate(x["q"], x["k"], 128, 128, True, [0.5])[0.5]
    a = run_gpu(x, tau, 128, 128, True, want_mask=True)
    b = run_gpu(x, tau, 128, 128, True, want_mask=False)
    assert np.array_equal(a["out"], b["out"]) and np.array_equal(a["lse"], b["lse"])
    c = run_gpu(x, tau, 128, 128, True, want_mask=True)
    assert np.array_equal(a["mask"], c["mask"]) and np.array_equal(a["out"], c["out"])


# ----------------------------------------------------------------------------- the workloads at full size

def _workload(name, p, sampled=None):
    cfg = CONFIGS[name]
    x = make_inputs(cfg)
    tau = stored_taus(name, p)
    gpu = run_gpu(x, tau, cfg.Bq, cfg.Bk, cfg.causal)
    tiles = sample_tiles(cfg, sampled) if sampled else all_tiles(cfg.B, cfg.Hq, cfg.N, cfg.Bq)
    stats = compare_tiles(x, tau, cfg.Bq, cfg.Bk, cfg.causal, gpu, tiles).check()
    m = gpu["mask"]
    gated = np.isin(m, (0, 1))
    stats["skip_fraction"] = float((m == 0).sum() / max(gated.sum(), 1))
    print(name, p, stats)
    return stats


def test_workload_c1_small_causal():
    s = _workload("c1", 0.5)
    assert abs(s["skip_fraction"] - 0.5) < 0.02


def test_workload_c2_gqa_layer_8k():
    s = _workload("c2", 0.5)
    assert abs(s["skip_fraction"] - 0.5) < 0.02


@pytest.mark.parametrize("p", [0.5, 0.8])
def test_workload_c5_dit_bidirectional(p):
    s = _workload("c5", p, sampled=96)
    assert abs(s["skip_fraction"] - p) < 0.02


@pytest.mark.parametrize("p", [0.3, 0.5, 0.7, 0.9])
def test_workload_c3_gqa_layer_32k(p):
    s = _workload("c3", p, sampled=48)
    assert abs(s["skip_fraction"] - p) < 0.02


@pytest.mark.parametrize("p", [0.7, 0.9])
def test_workload_c4_gqa_layer_128k(p):
    s = _workload("c4", p, sampled=64)
    assert abs(s["skip_fraction"] - p) < 0.05
