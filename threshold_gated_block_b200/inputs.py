"""Seeded synthetic inputs for the BSFA prefill forward.

This module only draws random tensors and rounds them to bf16. It holds none of
the attention arithmetic (no scores, no block maxima, no softmax), so that both
the CPU oracle and the CUDA path can consume the same bits without sharing any
of the method's code.

Workloads (shapes from the Block Sparse Flash Attention paper's setting: a
Llama-3.1-8B attention layer with 32 query heads, 8 KV heads, head dimension
128, §5.1 "Models and datasets"; and the bidirectional extension of App. B.3
"Practical considerations"). The long-context suites the paper measures on are
not available, so these generators stand in for them:

* ``normal``  : Q, K, V ~ N(0, 1).
* ``planted`` : Q, K, V ~ N(0, 1) plus an attention sink on the first 64 keys
                (shifted along the group's mean query direction) and 16 planted
                needle keys per KV head, each matched by 16 queries per q-head
                at cosine 0.9 (the "sink" and "heavy hitter" structure of §2
                "Empirical sparsity patterns").
* ``dit``     : tokens on a sqrt(N) x sqrt(N) latent grid; Q and K share a
                spatially smooth component (Gaussian-blurred noise, sigma 4
                cells), so score mass is local on the grid.

All tensors are returned as uint16 arrays holding bf16 bit patterns in the
layout [B, N, H, D] (row-major, D fastest).
"""
from __future__ import annotations

from dataclasses import dataclass, field
import math

import numpy as np

__all__ = ["Config", "CONFIGS", "make_inputs", "custom_config", "f32_to_bf16_bits", "bf16_bits_to_f32"]


@dataclass(frozen=True)
class Config:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    N: int
    Bq: int
    Bk: int
    causal: bool
    kind: str                      # "normal" | "planted" | "dit"
    skips: tuple = (0.5,)          # target off-diagonal skip fractions
    seed: int = 1000
    description: str = ""
    sampled_tiles: int = 0         # >0: parity/calibration on sampled query tiles
    extra: dict = field(default_factory=dict, hash=False, compare=False)

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv


CONFIGS = {
    "c1": Config("c1", B=1, Hq=2, Hkv=2, D=64, N=512, Bq=64, Bk=64, causal=True,
                 kind="normal", skips=(0.5,), seed=1000,
                 description="small causal MHA case, D=64, 64x64 tiles"),
    "c2": Config("c2", B=1, Hq=32, Hkv=8, D=128, N=8192, Bq=128, Bk=128, causal=True,
                 kind="planted", skips=(0.5,), seed=1001,
                 description="Llama-3.1-8B-shaped GQA attention layer prefill, N=8192"),
    "c3": Config("c3", B=1, Hq=32, Hkv=8, D=128, N=32768, Bq=128, Bk=128, causal=True,
                 kind="planted", skips=(0.3, 0.5, 0.7, 0.9), seed=1002,
                 description="same GQA layer, N=32768, skip sweep"),
    "c4": Config("c4", B=1, Hq=32, Hkv=8, D=128, N=131072, Bq=128, Bk=128, causal=True,
                 kind="planted", skips=(0.7, 0.9), seed=1003, sampled_tiles=512,
                 description="same GQA layer, N=131072, sampled-tile parity"),
    "c5": Config("c5", B=1, Hq=24, Hkv=24, D=128, N=16384, Bq=128, Bk=128, causal=False,
                 kind="dit", skips=(0.5, 0.8), seed=1004,
                 description="non-causal DiT-shaped MHA on a 128x128 latent grid"),
}

# Planted-structure parameters (recorded by the bench next to every result).
SINK_KEYS = 64
SINK_ALPHA = 2.0
NEEDLES_PER_HEAD = 16
QUERIES_PER_NEEDLE = 16
NEEDLE_COSINE = 0.9
DIT_SIGMA = 4.0
DIT_RADIUS = 12


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); return uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).copy()
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    u += np.uint32(0x7FFF)
    u += lsb
    u >>= np.uint32(16)
    return u.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _unit(rng: np.random.Generator, d: int) -> np.ndarray:
    v = rng.standard_normal(d).astype(np.float64)
    return v / np.linalg.norm(v)


def _normal(rng: np.random.Generator, shape) -> np.ndarray:
    return rng.standard_normal(shape, dtype=np.float32)


def _plant(q: np.ndarray, k: np.ndarray, group: int, rng: np.random.Generator) -> None:
    """Add the sink and the needles in place (float32 tensors [B, N, H, D])."""
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    root_d = math.sqrt(D)
    for b in range(B):
        for g in range(Hkv):
            heads = range(g * group, (g + 1) * group)
            # Sink: first keys pushed along the group's mean query direction.
            mean_q = np.zeros(D, dtype=np.float64)
            for h in heads:
                mean_q += q[b, :, h, :].astype(np.float64).sum(axis=0)
            u = mean_q / np.linalg.norm(mean_q)
            k[b, :SINK_KEYS, g, :] += (SINK_ALPHA * root_d * u).astype(np.float32)
            # Needles.
            if N <= SINK_KEYS:
                continue
            n_needles = min(NEEDLES_PER_HEAD, N - SINK_KEYS)
            positions = np.sort(rng.choice(np.arange(SINK_KEYS, N), size=n_needles, replace=False))
            for p in positions:
                nhat = _unit(rng, D)
                k[b, p, g, :] = (root_d * nhat).astype(np.float32)
                for h in heads:
                    count = min(QUERIES_PER_NEEDLE, N - p)
                    rows = rng.choice(np.arange(p, N), size=count, replace=False)
                    for r in rows:
                        w = rng.standard_normal(D)
                        w -= w.dot(nhat) * nhat
                        w /= np.linalg.norm(w)
                        norm_q = np.linalg.norm(q[b, r, h, :].astype(np.float64))
                        direction = NEEDLE_COSINE * nhat + math.sqrt(1.0 - NEEDLE_COSINE ** 2) * w
                        q[b, r, h, :] = (norm_q * direction).astype(np.float32)


def _blur_axis(x: np.ndarray, axis: int, weights: np.ndarray) -> np.ndarray:
    r = (len(weights) - 1) // 2
    pad = [(0, 0)] * x.ndim
    pad[axis] = (r, r)
    xp = np.pad(x, pad, mode="reflect")
    out = np.zeros_like(x)
    n = x.shape[axis]
    for t, wt in enumerate(weights):
        sl = [slice(None)] * x.ndim
        sl[axis] = slice(t, t + n)
        out += np.float32(wt) * xp[tuple(sl)]
    return out


def _dit_smooth(rng: np.random.Generator, side: int, D: int) -> np.ndarray:
    """Gaussian-blurred, per-channel standardised noise on a side x side grid -> [side*side, D]."""
    f = _normal(rng, (side, side, D))
    taps = np.arange(-DIT_RADIUS, DIT_RADIUS + 1, dtype=np.float64)
    wts = np.exp(-0.5 * (taps / DIT_SIGMA) ** 2)
    wts /= wts.sum()
    f = _blur_axis(f, 0, wts)
    f = _blur_axis(f, 1, wts)
    f = f.reshape(side * side, D)
    f -= f.mean(axis=0, keepdims=True)
    f /= f.std(axis=0, keepdims=True)
    return f


def make_inputs(cfg: Config, seed: int | None = None) -> dict:
    """Draw Q, K, V for ``cfg`` and return bf16 bit arrays plus the recipe record."""
    seed = cfg.seed if seed is None else seed
    ss = np.random.SeedSequence(seed)
    rq, rk, rv, rs = [np.random.Generator(np.random.PCG64(s)) for s in ss.spawn(4)]
    B, N, Hq, Hkv, D = cfg.B, cfg.N, cfg.Hq, cfg.Hkv, cfg.D
    if cfg.kind == "dit":
        side = math.isqrt(N)
        if side * side != N or Hq != Hkv:
            raise ValueError("dit generator needs a square token grid and MHA")
        q = np.empty((B, N, Hq, D), dtype=np.float32)
        k = np.empty((B, N, Hkv, D), dtype=np.float32)
        for b in range(B):
            for h in range(Hq):
                f = _dit_smooth(rs, side, D)
                q[b, :, h, :] = _normal(rq, (N, D)) + f
                k[b, :, h, :] = _normal(rk, (N, D)) + f
        v = _normal(rv, (B, N, Hkv, D))
    else:
        q = _normal(rq, (B, N, Hq, D))
        k = _normal(rk, (B, N, Hkv, D))
        v = _normal(rv, (B, N, Hkv, D))
        if cfg.kind == "planted":
            _plant(q, k, Hq // Hkv, rs)
        elif cfg.kind != "normal":
            raise ValueError(f"unknown generator kind {cfg.kind!r}")
    recipe = {"kind": cfg.kind, "seed": seed, "dist": "N(0,1) fp32 rounded to bf16 (RNE)"}
    if cfg.kind == "planted":
        recipe.update(sink_keys=SINK_KEYS, sink_alpha=SINK_ALPHA, needles_per_kv_head=NEEDLES_PER_HEAD,
                      queries_per_needle_per_q_head=QUERIES_PER_NEEDLE, needle_cosine=NEEDLE_COSINE)
    if cfg.kind == "dit":
        recipe.update(grid=math.isqrt(N), blur_sigma_cells=DIT_SIGMA, blur_radius=DIT_RADIUS)
    out = {"q": f32_to_bf16_bits(q)}
    del q
    out["k"] = f32_to_bf16_bits(k)
    del k
    out["v"] = f32_to_bf16_bits(v)
    out["recipe"] = recipe
    return out


def custom_config(name="custom", *, B=1, Hq=2, Hkv=2, D=64, N=256, Bq=64, Bk=64, causal=True,
                  kind="normal", seed=7) -> Config:
    """A small configuration for tests (same generators, arbitrary shape)."""
    return Config(name, B=B, Hq=Hq, Hkv=Hkv, D=D, N=N, Bq=Bq, Bk=Bk, causal=causal, kind=kind, seed=seed)


def sample_tiles(cfg: Config, count: int, seed: int | None = None) -> list:
    """Seeded sample of query tiles (b, hq, i), spread over heads, always holding the
    first and last tile of head 0."""
    seed = (cfg.seed if seed is None else seed) + 77
    rng = np.random.Generator(np.random.PCG64(seed))
    mq = -(-cfg.N // cfg.Bq)
    tiles = {(0, 0, 0), (0, 0, mq - 1)}
    while len(tiles) < min(count, cfg.B * cfg.Hq * mq):
        b = int(rng.integers(cfg.B))
        h = int(rng.integers(cfg.Hq))
        i = int(rng.integers(mq))
        tiles.add((b, h, i))
    return sorted(tiles)
