"""Write tests/golden/taus.json: per-head thresholds for every workload.

The thresholds are inputs of both the CUDA path and the oracle, so they come
from the oracle alone: the seeded generator draws Q and K, the oracle takes the
block maxima, and the calibration rule (per head, sorted gated block maxima,
midpoint of a gap around the target skip fraction) picks tau. Nothing here runs
on the GPU.

Usage: python tests/golden/make_taus.py [config ...]
"""
import json
import os
import sys
import time

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from threshold_gated_block_b200.inputs import CONFIGS, make_inputs, sample_tiles  # noqa: E402
from oracle.calibrate import calibrate  # noqa: E402

OUT = os.path.join(HERE, "taus.json")

# Extra skip targets beyond a workload's own, for the gate comparison sweep.
EXTRA_SKIPS = {"c2": (0.3, 0.7, 0.9)}


def main(names):
    table = {}
    if os.path.exists(OUT):
        with open(OUT) as f:
            table = json.load(f)
    for name in names:
        cfg = CONFIGS[name]
        t0 = time.time()
        x = make_inputs(cfg)
        tiles = sample_tiles(cfg, cfg.sampled_tiles) if cfg.sampled_tiles else None
        skips = tuple(sorted(set(cfg.skips) | set(EXTRA_SKIPS.get(name, ()))))
        taus = calibrate(x["q"], x["k"], cfg.Bq, cfg.Bk, cfg.causal, skips, tiles)
        table[name] = {
            "taus": {str(p): t for p, t in taus.items()},
            "calibrated_on": "sampled tiles" if tiles else "all tiles",
            "n_tiles": len(tiles) if tiles else None,
            "seed": cfg.seed,
        }
        print(f"{name}: {time.time() - t0:.1f} s", flush=True)
        with open(OUT, "w") as f:
            json.dump(table, f, indent=1, sort_keys=True)


if __name__ == "__main__":
    main(sys.argv[1:] or list(CONFIGS))
