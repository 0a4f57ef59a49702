"""Cycle trace of the BSFA forward kernel (profiling aid).

    python -m threshold_gated_block_b200.trace [--config c2] [--skip 0.5] [--ctas 16] [--dense]

Builds the trace variant of the library (libbsfa_trace.so: the same kernels
compiled with BSFA_TRACE, which stamp the SM clock at fixed points of every
role; include/bsfa_trace.h), runs one forward of the workload with the first
``--ctas`` CTAs traced, and prints the median length in SM cycles of each phase
of a step, separately for kept and skipped steps of the steady state (the first
two and the last step of each slot left out):

  fence      S-ready barrier passed -> tcgen05 fence done
  load       -> the 128 (or 64) scores of the row loaded from TMEM
  max        -> masked and the row maximum taken
  gate       -> gate barrier passed (waits for the slowest row of the tile)
  exp        -> exponentials and row sums done (kept steps)
  P store    -> P written to TMEM and the write waited for
  announce   -> p_full arrival (after the O rescale when due, and the fence)
  to MMA     p_full arrival -> the MMA thread sees it
  V wait     P seen -> V ready (kept steps; the decision read on skipped ones)
  PV issue   -> the PV MMAs issued
  QK issue   -> the next QK^T MMAs issued and committed
  to S       -> the waiter sees that S complete (the tensor core's time)
  to softmax waiter sees S -> the warpgroup passes the S-ready barrier
  period     one S-ready to the next, for the same slot

Stamps of different warps are put on one clock with the per-warp offsets the
kernel records right after its first __syncthreads.

The process must not have loaded libbsfa.so before: the trace library takes its
place for the whole process.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

STEPS = 64
SOFTMAX = 16
MMA = SOFTMAX + 2 * STEPS * 8
WAIT = MMA + 2 * STEPS * 4
VPROD = WAIT + 2 * STEPS
KPROD = VPROD + 2 * STEPS
EPI = KPROD + STEPS
# Warps of the roles: the softmax stamps come from warp 4s (the row-0 thread of
# slot s), the MMA stamps of both slots from the issuing warp 9 and the S-wait
# stamps from the waiter warp 11.
K_WARP, MMA_WARP, V_WARP, WAIT_WARP = 8, 9, 10, 11


def load_trace_lib(path: str | None = None):
    from threshold_gated_block_b200 import bsfa
    from threshold_gated_block_b200.build import build
    path = path or build(trace=True)
    lib = bsfa.load(path)
    if os.path.abspath(lib._name) != os.path.abspath(path):
        raise RuntimeError("another BSFA library was loaded before the trace library in this process")
    lib.bsfa_trace_attach.argtypes = [ctypes.c_void_p, ctypes.c_int]
    lib.bsfa_trace_attach.restype = ctypes.c_int
    lib.bsfa_trace_stride.argtypes = []
    lib.bsfa_trace_stride.restype = ctypes.c_int
    return lib


def phases(tr: np.ndarray, nblk: list[int]):
    """Per-step phase lengths of one CTA's trace: a list of dicts (slot, step, kept, phases)."""
    off = lambda w: int(tr[3 + w]) - int(tr[3])          # warp w's clock minus warp 0's
    rows = []
    for s in range(2):
        n = min(nblk[s], STEPS)
        sm = lambda j, e: int(tr[SOFTMAX + (s * STEPS + j) * 8 + e]) - off(4 * s)
        mm = lambda j, e: int(tr[MMA + (s * STEPS + j) * 4 + e]) - off(MMA_WARP)
        wt = lambda j: int(tr[WAIT + s * STEPS + j]) - off(WAIT_WARP)
        for j in range(n):
            kept = tr[SOFTMAX + (s * STEPS + j) * 8 + 5] != 0
            ph = {"fence": sm(j, 1) - sm(j, 0), "load": sm(j, 2) - sm(j, 1), "max": sm(j, 3) - sm(j, 2),
                  "gate": sm(j, 4) - sm(j, 3)}
            if kept:
                ph.update({"exp": sm(j, 5) - sm(j, 4), "P store": sm(j, 6) - sm(j, 5),
                           "announce": sm(j, 7) - sm(j, 6)})
            else:
                ph["announce"] = sm(j, 7) - sm(j, 4)
            ph["to MMA"] = mm(j, 0) - sm(j, 7)
            if tr[MMA + (s * STEPS + j) * 4 + 2] != 0:
                ph["V wait"] = mm(j, 1) - mm(j, 0)
                ph["PV issue"] = mm(j, 2) - mm(j, 1)
                ph["QK issue"] = mm(j, 3) - mm(j, 2)
            else:
                ph["QK issue"] = mm(j, 3) - mm(j, 0)
            if j + 1 < n:
                ph["to S"] = wt(j + 1) - mm(j, 3)
                ph["to softmax"] = sm(j + 1, 0) - wt(j + 1)
                ph["period"] = sm(j + 1, 0) - sm(j, 0)
            rows.append({"slot": s, "step": j, "kept": kept, "n": n, "ph": ph})
    return rows


ORDER = ("fence", "load", "max", "gate", "exp", "P store", "announce", "to MMA", "V wait", "PV issue", "QK issue",
         "to S", "to softmax", "period")


def summarize(all_rows):
    """Median of each phase over the steady-state steps, kept and skipped apart."""
    out = {}
    for kept in (True, False):
        sel = [r for r in all_rows if r["kept"] == kept and 2 <= r["step"] < r["n"] - 1]
        if not sel:
            continue
        med = {"steps": len(sel)}
        for k in ORDER:
            vals = [r["ph"][k] for r in sel if k in r["ph"]]
            if vals:
                med[k] = float(np.median(vals))
        out["kept" if kept else "skipped"] = med
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", default="c2")
    ap.add_argument("--skip", type=float, default=None)
    ap.add_argument("--ctas", type=int, default=16)
    ap.add_argument("--dense", action="store_true", help="tau = -inf (every block kept)")
    ap.add_argument("--lib", default=None, help="a prebuilt trace library (default: build libbsfa_trace.so)")
    ap.add_argument("--dump", default=None, help="also write the raw stamps of every traced CTA (.npy)")
    args = ap.parse_args()

    lib = load_trace_lib(args.lib)
    import torch
    from threshold_gated_block_b200 import bsfa
    from threshold_gated_block_b200.inputs import CONFIGS, make_inputs

    cfg = CONFIGS[args.config]
    p = cfg.skips[0] if args.skip is None else args.skip
    with open(os.path.join(ROOT, "tests", "golden", "taus.json")) as f:
        taus = json.load(f)[cfg.name]["taus"][str(float(p))]
    if args.dense:
        taus = [float("-inf")] * cfg.Hq
    x = make_inputs(cfg)
    dev = torch.device("cuda", 0)
    to_dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    q, k, v = to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"])
    tau = torch.tensor(taus, dtype=torch.float32, device=dev)
    stride = lib.bsfa_trace_stride()
    buf = torch.zeros(args.ctas * stride, dtype=torch.int64, device=dev)
    for _ in range(3):
        bsfa.forward(q, k, v, tau, Bq=cfg.Bq, Bk=cfg.Bk, causal=cfg.causal)
    torch.cuda.synchronize()
    if lib.bsfa_trace_attach(buf.data_ptr(), args.ctas) != 0:
        raise RuntimeError(bsfa.bsfa_last_error())
    bsfa.forward(q, k, v, tau, Bq=cfg.Bq, Bk=cfg.Bk, causal=cfg.causal)
    torch.cuda.synchronize()
    lib.bsfa_trace_attach(None, 0)
    if bsfa.bsfa_get_status(None) != bsfa.BSFA_OK:
        raise RuntimeError(bsfa.bsfa_last_error())
    tr = buf.view(args.ctas, stride).cpu().numpy().astype(np.int64)
    if args.dump:
        np.save(args.dump, tr)

    # The first CTAs of a causal layer hold the last (heaviest) query rows.
    tiles = -(-cfg.N // 128)
    nblk_full = -(-cfg.N // cfg.Bk)
    rows = []
    for c in range(args.ctas):
        nb = [sum(1 for j in range(STEPS) if tr[c, SOFTMAX + (s * STEPS + j) * 8] != 0) for s in range(2)]
        rows += phases(tr[c], nb)
    summary = summarize(rows)
    cta_cycles = [int(tr[c, 2] - tr[c, 0]) for c in range(args.ctas)]
    print(json.dumps({"config": cfg.name, "tau": "dense" if args.dense else f"skip {p}", "ctas": args.ctas,
                      "query_tiles": tiles, "key_blocks": nblk_full,
                      "cta_cycles_median": float(np.median(cta_cycles)), "phases": summary}, indent=1))


if __name__ == "__main__":
    main()
