#!/usr/bin/env python
"""Throughput of the BSFA prefill forward (one attention layer per step) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config c2] [--skip 0.5]
    python bench.py --impl reference ...      # the CPU oracle on a bounded sample

A step is one ``bsfa_forward`` call over every head of the layer (all rows of the
hot path: QK^T, block maxima, gate, online softmax, PV for kept blocks,
epilogue), on synthetic inputs already resident in HBM; L2 is flushed with a
256 MB memset between steps, outside the timed events. The metric is
dense-equivalent TFLOP/s: the FLOPs the same tiles would cost with every
visible block kept (2*Bq*Bk*D for QK^T plus 2*Bq*Bk*D for PV per visible tile),
divided by the kernel time. Executed TFLOP/s counts PV only for kept tiles.
The same kernel at tau = -inf gives the dense comparator. ``e2e`` repeats the
measurement through the host-buffer call (pinned host inputs copied in, out and
lse copied back, inside the timed region).

For N > 1 (torchrun) every rank runs its own copy of the layer (independent
problems, no data-path collective): weak scaling, value = all ranks' FLOPs over
the slowest rank's time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from threshold_gated_block_b200.inputs import CONFIGS, make_inputs, sample_tiles  # noqa: E402

METRIC = "prefill-attention TFLOP/s (dense-equivalent)"
UNIT = "TFLOP/s"
TAUS = os.path.join(ROOT, "tests", "golden", "taus.json")
TAU_TABLES = os.path.join(ROOT, "tests", "golden", "tau_tables.json")
# Workloads that share one layer type share its per-position threshold table.
TABLE_FOR = {"c2": "c2", "c3": "c2", "c4": "c2"}
PEAKS = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC = os.path.join(ROOT, "profiles", "bsfa_fwd_c2_traffic.txt")
KERNEL_SOURCES = ["ptx.cuh", "bsfa_fwd_kernel.cuh", "bsfa_launch.cuh", "bsfa_fwd_d64.cu", "bsfa_fwd_d128.cu",
                  "bsfa_api.cu"]
FALLBACK_BF16_TFLOPS = 1590.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="c2")
    ap.add_argument("--skip", type=float, default=None, help="target skip fraction (a stored calibration)")
    ap.add_argument("--tau-table", type=int, default=None, metavar="K",
                    help="gate with the stored per-position (fixed-k) table level that keeps K blocks per tile")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the CPU-oracle baseline")
    ap.add_argument("--cpu-tiles", type=int, default=None,
                    help="run the CPU-oracle baseline on exactly this many seeded query tiles (no time budget) and "
                         "extrapolate to the full layer; default 64 for c4, else the --cpu-seconds budget")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-sweep", action="store_true",
                    help="leave out the skip sweep (the default c2 line also times the 32K layer at 30/50/70/90%% "
                         "skip and dense, one GPU)")
    ap.add_argument("--sweep-config", default="c3", help="workload of the skip sweep")
    ap.add_argument("--gate", choices=["tau", "gap"], default="tau",
                    help="tau: the BSFA gate; gap: the gap-to-running-maximum gate, for comparison")
    ap.add_argument("--gamma", type=float, default=-1.0, help="gamma of the gap gate (scaled-score units)")
    ap.add_argument("--shard", choices=["replica", "heads"], default="replica",
                    help="multi-GPU layout: replica = every rank runs the whole layer (weak scaling); heads = the "
                         "layer's KV groups are split across the ranks (strong scaling, no exchange needed)")
    ap.add_argument("--curve", action="store_true",
                    help="instead of the bench line: error against dense attention, skip fraction and time for "
                         "several settings of each gate (one JSON line each)")
    return ap.parse_args()


def workload(args):
    """(config, threshold description, thresholds): per head [Hq] or per position [Hq, T]."""
    cfg = CONFIGS[args.config]
    if args.gate == "gap":
        return cfg, {"gate": "gap to the running row maximum", "gamma": args.gamma}, [args.gamma] * cfg.Hq
    if args.tau_table is not None:
        with open(TAU_TABLES) as f:
            spec = json.load(f)[TABLE_FOR[cfg.name]]
        level = spec["ks"].index(args.tau_table)
        desc = {"tau": "per-position table", "k": args.tau_table, "table_n_max": spec["n_max"],
                "calib_seeds": spec["calib_seeds"]}
        return cfg, desc, spec["table"][level]
    p = cfg.skips[0] if args.skip is None else args.skip
    with open(TAUS) as f:
        taus = json.load(f)[cfg.name]["taus"][str(float(p))]
    return cfg, {"tau": "per head", "target_skip": p}, taus


def config_record(cfg, tau_desc, achieved=None):
    rec = {"workload": f"{cfg.name}: {cfg.description}", "B": cfg.B, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "D": cfg.D,
           "N": cfg.N, "Bq": cfg.Bq, "Bk": cfg.Bk, "causal": cfg.causal, "inputs": cfg.kind,
           **tau_desc, "l2": "flushed between steps (256 MB memset outside the timed events)"}
    if achieved is not None:
        rec["achieved_skip"] = achieved
    return rec


def tile_flop(cfg) -> float:
    return 2.0 * cfg.Bq * cfg.Bk * cfg.D


def mask_flops(mask: np.ndarray, cfg):
    """(executed, dense-equivalent) FLOPs of one layer from the block codes."""
    visited = int((mask != 3).sum())
    kept = int(np.isin(mask, (1, 2)).sum())
    f = tile_flop(cfg)
    return (visited + kept) * f, 2 * visited * f


def cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"), default=0)
        if n:
            return n
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_sample(cfg, x, taus, budget_s, tiles, gate="tau"):
    """Run the oracle on sampled tiles until the budget is spent: (dense FLOPs, seconds, tiles)."""
    from oracle import bsfa_oracle as O
    tau = np.asarray(taus, dtype=np.float64)
    f = tile_flop(cfg)
    flops, done, t0 = 0.0, 0, time.perf_counter()
    for (b, h, i) in tiles:
        t = O.forward_tile(x["q"], x["k"], x["v"], tau, b, h, i, cfg.Bq, cfg.Bk, cfg.causal, gate=gate)
        flops += 2 * int((t["codes"] != O.CODE_INVISIBLE).sum()) * f
        done += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    return flops, time.perf_counter() - t0, done


def cpu_baseline(cfg, x, taus, gate, layer_dense_flops, count, budget_s):
    """The oracle timed on the host cores: the bench line's cpu_baseline object.

    count > 0: exactly that many seeded query tiles (spread over heads, the first
    and last tile of head 0 among them), no time budget, extrapolated to the
    layer by dense-equivalent FLOPs. Otherwise: shuffled seeded tiles until
    budget_s seconds of oracle work are spent."""
    if count > 0:
        tiles = sample_tiles(cfg, count, seed=cfg.seed + 5)
        f, t, n = oracle_sample(cfg, x, taus, float("inf"), tiles, gate)
        return {"value": f / t / 1e12, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                "sample": f"{n} seeded query tiles of {cfg.name} (exact count, {t:.1f} s of oracle work), "
                          f"dense-equivalent FLOPs of those tiles",
                "seconds_per_tile": t / n,
                "extrapolated_layer_s": layer_dense_flops / (f / t),
                "extrapolated": "full-layer time = the layer's dense-equivalent FLOPs / the sample's FLOP rate"}
    tiles = sample_tiles(cfg, 4096, seed=cfg.seed + 5)
    np.random.default_rng(0).shuffle(tiles)
    f, t, n = oracle_sample(cfg, x, taus, budget_s, tiles, gate)
    return {"value": f / t / 1e12, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
            "sample": f"{n} seeded query tiles of {cfg.name} (about {t:.1f} s of oracle work), "
                      f"dense-equivalent FLOPs of those tiles"}


def head_shard(rank: int, world: int, Hkv: int) -> tuple[int, int]:
    """(first KV head, KV head count) of ``rank`` when a layer's KV groups are split
    evenly across ``world`` ranks."""
    if Hkv % world != 0:
        raise ValueError(f"{Hkv} KV heads do not split evenly across {world} ranks")
    per = Hkv // world
    return rank * per, per


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """The largest of each rank's value (every rank gets it); with no process group, the value."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(flops_per_rank: float, world: int, slowest_ms: float) -> float:
    """Whole-job TFLOP/s: every rank's FLOPs over the slowest rank's time."""
    return world * flops_per_rank / (slowest_ms * 1e-3) / 1e12


def kernel_hash() -> str:
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "threshold_gated_block_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic(cfg, tau_desc):
    """DRAM bytes per launch from the committed ncu summary, if it matches this kernel and workload
    (the per-head threshold gate it was captured with)."""
    if tau_desc.get("tau") != "per head":
        return None
    if not os.path.exists(TRAFFIC):
        return None
    kv = {}
    with open(TRAFFIC) as f:
        for line in f:
            if ":" in line:
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
    if kv.get("kernel_hash") != kernel_hash() or kv.get("config") != cfg.name:
        return None
    try:
        return float(kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the GPU works."""
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device_index: int, bus_id: str | None):
        self.proc = None
        target = bus_id or str(device_index)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={target}", "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            parts = [s.strip() for s in line.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- reference arm (CPU oracle)

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cfg, p, taus = workload(args)
    x = make_inputs(cfg)
    tiles = sample_tiles(cfg, 4096, seed=cfg.seed + 5)
    rng = np.random.default_rng(0)
    rng.shuffle(tiles)
    per_step = max(0.05, min(2.0, 150.0 / max(args.steps + args.warmup, 1)))
    pos = 0
    for _ in range(args.warmup):
        _, _, n = oracle_sample(cfg, x, taus, per_step, tiles[pos:] + tiles[:pos], args.gate)
        pos = (pos + n) % len(tiles)
    tot_f, tot_t, tot_n = 0.0, 0.0, 0
    for _ in range(args.steps):
        f, t, n = oracle_sample(cfg, x, taus, per_step, tiles[pos:] + tiles[:pos], args.gate)
        pos = (pos + n) % len(tiles)
        tot_f, tot_t, tot_n = tot_f + f, tot_t + t, tot_n + n
    value = tot_f / tot_t / 1e12
    cores = cpu_cores()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_record(cfg, p),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{tot_n} query tiles of {cfg.name} (about {per_step:.2f} s of oracle work per "
                                   f"step), dense-equivalent FLOPs of those tiles"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- skip sweep (extra keys of the line)

def skip_sweep(cfg_name, dev, steps, warmup, flush, peak):
    """Time one layer of ``cfg_name`` at every stored per-head skip level and at
    tau = -inf (the dense comparator), with L2 flushed between launches: the
    evidence that wall time falls with the skip fraction. One JSON object."""
    import torch
    from threshold_gated_block_b200 import bsfa
    cfg = CONFIGS[cfg_name]
    with open(TAUS) as f:
        levels = json.load(f)[cfg.name]["taus"]
    x = make_inputs(cfg)
    to_dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    q, k, v = to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"])
    del x
    out = torch.empty_like(q)
    lse = torch.empty((cfg.B, cfg.Hq, cfg.N), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def run(t):
        st = bsfa.bsfa_forward(q, k, v, t, out, lse, None, cfg.B, cfg.Hq, cfg.Hkv, cfg.N, cfg.D, cfg.Bq, cfg.Bk,
                               cfg.causal, stream)
        if st != bsfa.BSFA_OK:
            raise RuntimeError(bsfa.bsfa_last_error())

    def timed_ms(t):
        for _ in range(warmup):
            run(t)
        ev = []
        for _ in range(steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            run(t)
            b.record(stream)
            ev.append((a, b))
        torch.cuda.synchronize(dev)
        return sum(a.elapsed_time(b) for a, b in ev) / steps

    sampler = ClockSampler(dev.index or 0, None)
    time.sleep(0.2)
    dense = torch.full((cfg.Hq,), float("-inf"), dtype=torch.float32, device=dev)
    dense_ms = timed_ms(dense)
    points = []
    for p_s, taus in sorted(levels.items(), key=lambda kv: float(kv[0])):
        t = torch.tensor(taus, dtype=torch.float32, device=dev)
        _, _, mask = bsfa.forward(q, k, v, t, Bq=cfg.Bq, Bk=cfg.Bk, causal=cfg.causal, want_lse=False,
                                  want_mask=True)
        m = mask.cpu().numpy()
        del mask
        exec_f, dense_f = mask_flops(m, cfg)
        ms = timed_ms(t)
        gated = np.isin(m, (0, 1))
        points.append({"target_skip": float(p_s), "achieved_skip": float((m == 0).sum() / max(gated.sum(), 1)),
                       "ms": ms, "speedup_vs_dense": dense_ms / ms,
                       "exec_tflops": exec_f / (ms * 1e-3) / 1e12, "dense_equiv_tflops": dense_f / (ms * 1e-3) / 1e12,
                       "frac": exec_f / (ms * 1e-3) / 1e12 / peak})
    clocks = sampler.stop()
    if bsfa.bsfa_get_status(stream) != bsfa.BSFA_OK:
        raise RuntimeError(f"device status: {bsfa.bsfa_last_error()}")
    del q, k, v, out, lse
    torch.cuda.empty_cache()
    ms_list = [pt["ms"] for pt in points]
    return {"workload": f"{cfg.name}: {cfg.description}", "steps": steps, "warmup": warmup, "dense_ms": dense_ms,
            "points": points, "monotone": all(a > b for a, b in zip(ms_list, ms_list[1:])), "clocks": clocks}


# ----------------------------------------------------------------------------- our arm

def run_ours(args):
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    from threshold_gated_block_b200 import bsfa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=180), device_id=dev)
    bsfa.load()

    cfg, p, taus = workload(args)
    heads = args.shard == "heads"
    if heads and (args.gate != "tau" or args.tau_table is not None):
        raise SystemExit("--shard heads runs the per-head threshold gate only")
    kv_begin, kv_count = head_shard(rank, world, cfg.Hkv) if heads else (0, cfg.Hkv)
    x = make_inputs(cfg)
    to_dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    q, k, v = to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"])
    tau = torch.tensor(taus, dtype=torch.float32, device=dev)
    tau_dense = torch.full_like(tau, float("-inf"))
    out = torch.empty_like(q)
    lse = torch.empty((cfg.B, cfg.Hq, cfg.N), dtype=torch.float32, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(t):
        if heads:
            st = bsfa.bsfa_forward_heads(q, k, v, t, out, lse, None, cfg.B, cfg.Hq, cfg.Hkv, cfg.N, cfg.D, cfg.Bq,
                                         cfg.Bk, cfg.causal, kv_begin, kv_count, stream)
        elif args.gate == "gap" and t is not tau_dense:
            st = bsfa.bsfa_forward_gap(q, k, v, t, out, lse, None, cfg.B, cfg.Hq, cfg.Hkv, cfg.N, cfg.D, cfg.Bq, cfg.Bk,
                                       cfg.causal, stream)
        elif t.dim() == 1:
            st = bsfa.bsfa_forward(q, k, v, t, out, lse, None, cfg.B, cfg.Hq, cfg.Hkv, cfg.N, cfg.D, cfg.Bq, cfg.Bk,
                                   cfg.causal, stream)
        else:
            st = bsfa.bsfa_forward_tau_table(q, k, v, t, t.shape[1], out, lse, None, cfg.B, cfg.Hq, cfg.Hkv, cfg.N,
                                             cfg.D, cfg.Bq, cfg.Bk, cfg.causal, stream)
        if st != bsfa.BSFA_OK:
            raise RuntimeError(bsfa.bsfa_last_error())

    # Block codes of this layer (untimed) give the executed and dense-equivalent FLOPs.
    _, _, mask = bsfa.forward(q, k, v, tau, Bq=cfg.Bq, Bk=cfg.Bk, causal=cfg.causal, want_lse=False, want_mask=True,
                              gate=args.gate)
    m = mask.cpu().numpy()
    del mask
    layer_dense_flops = mask_flops(m, cfg)[1]
    g = cfg.Hq // cfg.Hkv
    m = m[:, kv_begin * g:(kv_begin + kv_count) * g]      # this rank's heads (all of them unless head-sharded)
    exec_flops, dense_flops = mask_flops(m, cfg)
    gated = np.isin(m, (0, 1))
    achieved_skip = float((m == 0).sum() / max(gated.sum(), 1))
    kv_bytes = cfg.B * cfg.N * cfg.Hkv * cfg.D * 2

    def timed(t, steps):
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        for i in range(steps):
            flush.zero_()
            starts[i].record(stream)
            step(t)
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
        return [s.elapsed_time(e) for s, e in zip(starts, ends)]

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()

    props = torch.cuda.get_device_properties(dev)
    bus = None
    if hasattr(props, "pci_bus_id"):
        bus = f"{getattr(props, 'pci_domain_id', 0):08X}:{props.pci_bus_id:02X}:{getattr(props, 'pci_device_id', 0):02X}.0"
    sampler = ClockSampler(local, bus)
    time.sleep(0.3)

    for _ in range(args.warmup):
        step(tau)
    barrier()
    times = timed(tau, args.steps)                     # the timed region: exactly K steps
    barrier()
    t_total = max_over_ranks(sum(times), dist, dev)
    ms = t_total / args.steps

    # Dense comparator: the same kernel at tau = -inf.
    for _ in range(args.warmup):
        step(tau_dense)
    barrier()
    dense_ms = max_over_ranks(sum(timed(tau_dense, args.steps)), dist, dev) / args.steps

    e2e = None
    if not args.no_e2e and not heads:
        hq = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=True)
        hk = torch.empty(k.shape, dtype=torch.bfloat16, pin_memory=True)
        hv = torch.empty(v.shape, dtype=torch.bfloat16, pin_memory=True)
        ht = torch.tensor(taus, dtype=torch.float32).pin_memory()
        hq.copy_(q.cpu()); hk.copy_(k.cpu()); hv.copy_(v.cpu())
        bufs = bsfa.device_buffers(q.shape, k.shape, dev)
        ke = max(3, min(args.steps, 30))
        for _ in range(max(1, min(args.warmup, 3))):
            bsfa.forward_host(hq, hk, hv, ht, Bq=cfg.Bq, Bk=cfg.Bk, causal=cfg.causal, device=dev, stream=stream,
                              bufs=bufs, gate=args.gate)
        barrier()
        et = []
        for _ in range(ke):
            s0 = torch.cuda.Event(enable_timing=True)
            s1 = torch.cuda.Event(enable_timing=True)
            s0.record(stream)
            bsfa.forward_host(hq, hk, hv, ht, Bq=cfg.Bq, Bk=cfg.Bk, causal=cfg.causal, device=dev, stream=stream,
                              bufs=bufs, gate=args.gate)
            s1.record(stream)
            torch.cuda.synchronize(dev)
            et.append(s0.elapsed_time(s1))
        e2e_ms = max_over_ranks(sum(et), dist, dev) / ke
        h2d = (hq.numel() + hk.numel() + hv.numel()) * 2 + ht.numel() * 4
        d2h = bufs["out_host"].numel() * 2 + bufs["lse_host"].numel() * 4
        e2e = {"value": weak_scaling_value(dense_flops, world, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": ke}

    clocks = sampler.stop()
    status = bsfa.bsfa_get_status(stream)
    if status != bsfa.BSFA_OK:
        raise RuntimeError(f"device status: {bsfa.bsfa_last_error()}")

    exec_tflops = exec_flops / (ms * 1e-3) / 1e12
    dense_tflops = dense_flops / (ms * 1e-3) / 1e12
    peak, peak_src = FALLBACK_BF16_TFLOPS, "fallback"
    if os.path.exists(PEAKS):
        with open(PEAKS) as f:
            peaks = json.load(f)
        if peaks.get("bf16_tflops"):
            peak, peak_src = float(peaks["bf16_tflops"]), "measured (MEASURED_PEAKS.json bf16_tflops, burst)"
    traffic = measured_traffic(cfg, p)
    sweep = None
    if world == 1 and not args.no_sweep and not heads and args.config == "c2" and args.gate == "tau" \
            and args.tau_table is None:
        sweep = skip_sweep(args.sweep_config, dev, max(3, min(args.steps, 10)), 3, flush, peak)

    line = None
    if rank == 0:
        line = {
            "metric": METRIC,
            "value": layer_dense_flops / (ms * 1e-3) / 1e12 if heads else weak_scaling_value(dense_flops, world, ms),
            "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "strong" if heads else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {**config_record(cfg, p, achieved_skip),
                       **({"parallelism": f"KV heads split across {world} GPUs"} if heads else {})},
            "exec_tflops": world * exec_tflops, "dense_equiv_tflops": world * dense_tflops,
            "ms_per_layer": ms, "dense_ms_per_layer": dense_ms, "speedup_vs_dense": dense_ms / ms,
            "exec_flops_per_layer": exec_flops, "dense_flops_per_layer": dense_flops,
            "roofline": {"bound": "tensor", "achieved": exec_tflops, "peak": peak, "unit": UNIT,
                         "frac": exec_tflops / peak, "traffic": traffic, "peak_source": peak_src,
                         "kernel": "bsfa_fwd_kernel", "kv_bytes_per_head_tensor": kv_bytes},
            "gpu_launches": args.steps,
            "clocks": clocks,
        }
        if e2e is not None:
            line["e2e"] = e2e
        if sweep is not None:
            line["skip_sweep"] = sweep
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        if world == 1:
            count = args.cpu_tiles if args.cpu_tiles is not None else (64 if cfg.name == "c4" else 0)
            line["cpu_baseline"] = cpu_baseline(cfg, x, taus, args.gate, layer_dense_flops, count, args.cpu_seconds)
        print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- gate comparison sweep

GAMMA_SWEEP = (0.0, -0.25, -0.5, -0.75, -1.0, -1.5, -2.0, -3.0)


def run_curve(args):
    """Error against dense attention, skip fraction and kernel time for every
    stored per-head threshold, every stored fixed-k table level and a sweep of
    the gap gate's gamma, on one workload. The dense reference is the same
    kernel at tau = -inf. One JSON line per setting."""
    import torch
    from threshold_gated_block_b200 import bsfa

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    bsfa.load()
    cfg = CONFIGS[args.config]
    x = make_inputs(cfg)
    to_dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    q, k, v = to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"])
    f32 = lambda a: torch.tensor(np.asarray(a, dtype=np.float32), device=dev)
    points = []
    with open(TAUS) as f:
        for p, t in sorted(json.load(f)[cfg.name]["taus"].items(), key=lambda kv: float(kv[0])):
            points.append(("tau per head", f"target skip {p}", "tau", f32(t)))
    if cfg.name in TABLE_FOR:
        with open(TAU_TABLES) as f:
            spec = json.load(f)[TABLE_FOR[cfg.name]]
        for level, kk in enumerate(spec["ks"]):
            points.append(("tau per position (fixed k)", f"k = {kk}", "tau", f32(spec["table"][level])))
    for g in GAMMA_SWEEP:
        points.append(("gap to running max", f"gamma = {g}", "gap", f32([g] * cfg.Hq)))
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def timed_ms(t, gate, reps=20):
        run = lambda: bsfa.forward(q, k, v, t, Bq=cfg.Bq, Bk=cfg.Bk, causal=cfg.causal, want_lse=True, gate=gate,
                                   out=out_buf, lse=lse_buf, stream=stream)
        for _ in range(3):
            run()
        ts = []
        for _ in range(reps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            run()
            e1.record(stream)
            ts.append((e0, e1))
        torch.cuda.synchronize(dev)
        return float(np.median([a.elapsed_time(b) for a, b in ts]))

    out_buf = torch.empty_like(q)
    lse_buf = torch.empty((cfg.B, cfg.Hq, cfg.N), dtype=torch.float32, device=dev)
    dense_tau = f32([float("-inf")] * cfg.Hq)
    ref_out, ref_lse, _ = bsfa.forward(q, k, v, dense_tau, Bq=cfg.Bq, Bk=cfg.Bk, causal=cfg.causal, want_lse=True)
    ref64 = ref_out.double()
    ref_norm = float(ref64.norm())
    dense_ms = timed_ms(dense_tau, "tau")
    for (method, setting, gate, t) in points:
        o, l, m = bsfa.forward(q, k, v, t, Bq=cfg.Bq, Bk=cfg.Bk, causal=cfg.causal, want_lse=True, want_mask=True,
                               gate=gate)
        mm = m.cpu().numpy()
        gated = int(np.isin(mm, (0, 1)).sum())
        d = o.double() - ref64
        line = {"curve": cfg.name, "method": method, "setting": setting,
                "skip": float((mm == 0).sum() / max(gated, 1)),
                "out_rel_l2": float(d.norm()) / ref_norm, "out_max_abs": float(d.abs().max()),
                "lse_mean_abs": float((l - ref_lse).abs().mean()), "ms": timed_ms(t, gate), "dense_ms": dense_ms}
        print(json.dumps(line), flush=True)
    if bsfa.bsfa_get_status(stream) != bsfa.BSFA_OK:
        raise RuntimeError(bsfa.bsfa_last_error())
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.curve:
        return run_curve(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
