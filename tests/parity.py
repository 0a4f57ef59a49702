"""Shared parity machinery for the GPU tests: run the CUDA path through the C ABI
and compare it with the oracle tile by tile.

Tolerances (bf16 inputs, fp32 accumulation, bf16 output):
  out: max |gpu - oracle| <= 2e-2 and mean |gpu - oracle| <= 2e-3;
  lse: max |gpu - oracle| <= 1e-3;
  block mask: bit-exact, except gated blocks whose oracle maximum lies within
  NEAR_TAU of tau. Those are counted; where the GPU took the other decision on
  such a block, the oracle evaluates the tile with that block's decision flipped
  (both results are correct readings of the method), and the GPU must match it.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch

from oracle import bsfa_oracle as O
from threshold_gated_block_b200 import bsfa

OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3
LSE_MAX_ABS = 1e-3
NEAR_TAU = 1e-4

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def stored_taus(name: str, p: float) -> list:
    with open(os.path.join(GOLDEN, "taus.json")) as f:
        return json.load(f)[name]["taus"][str(float(p))]


def to_device(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def run_gpu(x: dict, tau, Bq: int, Bk: int, causal: bool, want_mask: bool = True, gate: str = "tau"):
    q, k, v = (to_device(x[n]) for n in "qkv")
    t = torch.tensor(np.asarray(tau, dtype=np.float32), device="cuda")
    out, lse, mask = bsfa.forward(q, k, v, t, Bq=Bq, Bk=Bk, causal=causal, want_lse=True, want_mask=want_mask,
                                  gate=gate)
    torch.cuda.synchronize()
    assert bsfa.bsfa_get_status(None) == bsfa.BSFA_OK, bsfa.bsfa_last_error()
    res = {
        "out": out.float().cpu().numpy().astype(np.float64),
        "lse": lse.cpu().numpy().astype(np.float64),
        "mask": mask.cpu().numpy() if mask is not None else None,
    }
    del q, k, v, out, lse, mask
    return res


class Report:
    def __init__(self):
        self.tiles = 0
        self.rows = 0
        self.max_abs = 0.0
        self.sum_abs = 0.0
        self.count = 0
        self.lse_max = 0.0
        self.near_tau = 0
        self.flipped = 0
        self.mask_mismatch = 0

    def check(self):
        mean = self.sum_abs / max(self.count, 1)
        assert self.mask_mismatch == 0, f"{self.mask_mismatch} block codes differ from the oracle"
        assert self.max_abs <= OUT_MAX_ABS, f"out max abs {self.max_abs:.3e}"
        assert mean <= OUT_MEAN_ABS, f"out mean abs {mean:.3e}"
        assert self.lse_max <= LSE_MAX_ABS, f"lse max abs {self.lse_max:.3e}"
        return {"tiles": self.tiles, "out_max_abs": self.max_abs, "out_mean_abs": mean, "lse_max_abs": self.lse_max,
                "near_tau": self.near_tau, "flipped": self.flipped}


def compare_tiles(x: dict, tau, Bq: int, Bk: int, causal: bool, gpu: dict, tiles, report: Report | None = None,
                  gate: str = "tau"):
    """Compare the GPU result with the oracle on the given (b, hq, i) tiles.

    gate="gap": the gap gate with tau holding gamma; a gated block is near the
    boundary when its margin (largest row excess over M_r - gamma) is within
    NEAR_TAU of zero.
    """
    rep = report or Report()
    tau = np.asarray(tau, dtype=np.float64)
    for (b, hq, i) in tiles:
        tau_i = O.tile_tau(tau, hq, i)
        t = O.forward_tile(x["q"], x["k"], x["v"], tau, b, hq, i, Bq, Bk, causal, gate=gate)
        flip = ()
        if gpu["mask"] is not None:
            gm = gpu["mask"][b, hq, i]
            gated = np.isin(t["codes"], (O.CODE_SKIPPED, O.CODE_KEPT))
            dist = np.abs(t["margin"]) if gate == "gap" else np.abs(t["smax"] - tau_i)
            near = gated & (dist <= NEAR_TAU)
            rep.near_tau += int(near.sum())
            differ = gm != t["codes"]
            flip = tuple(int(j) for j in np.nonzero(differ & near)[0])
            rep.mask_mismatch += int((differ & ~near).sum())
            if flip:
                rep.flipped += len(flip)
                t = O.forward_tile(x["q"], x["k"], x["v"], tau, b, hq, i, Bq, Bk, causal, flip=flip, gate=gate)
        r0, r1 = t["rows"]
        d = np.abs(gpu["out"][b, r0:r1, hq, :] - t["out"])
        rep.max_abs = max(rep.max_abs, float(d.max()))
        rep.sum_abs += float(d.sum())
        rep.count += d.size
        rep.lse_max = max(rep.lse_max, float(np.abs(gpu["lse"][b, hq, r0:r1] - t["lse"]).max()))
        rep.tiles += 1
        rep.rows += r1 - r0
    return rep


def all_tiles(B, Hq, N, Bq):
    return [(b, h, i) for b in range(B) for h in range(Hq) for i in range(-(-N // Bq))]
