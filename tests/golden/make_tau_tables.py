"""Write tests/golden/tau_tables.json: per-position (fixed-k) threshold tables.

Each table is one layer's slice of the paper's threshold tensor, one level per
retained-block count k: T[level, head, query tile] (§4.2 "Threshold
Calibration"; App. B.3 "Threshold tensor"). It is calibrated on seeds other
than the workload's own (the workload seed is held out, as the paper
calibrates and evaluates on disjoint samples), from the oracle alone: the
seeded generator draws Q and K, the oracle takes the block maxima, and the
top-k rule of ``oracle.calibrate.fixed_k_table`` averages the per-sample cuts.
Nothing here runs on the GPU.

Usage: python tests/golden/make_tau_tables.py
"""
import json
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from threshold_gated_block_b200.inputs import CONFIGS, make_inputs  # noqa: E402
from oracle.calibrate import fixed_k_table  # noqa: E402

OUT = os.path.join(HERE, "tau_tables.json")

# workload -> retained-block counts (levels) and calibration seeds
TABLES = {
    "c2": {"ks": [8, 16, 32], "calib_seeds": [3001, 3002]},
}


def main():
    res = {}
    for name, spec in TABLES.items():
        cfg = CONFIGS[name]
        t0 = time.time()
        samples = []
        for s in spec["calib_seeds"]:
            x = make_inputs(cfg, seed=s)
            samples.append((x["q"], x["k"]))
        T = fixed_k_table(samples, cfg.Bq, cfg.Bk, cfg.causal, spec["ks"])
        res[name] = {
            "ks": spec["ks"],
            "calib_seeds": spec["calib_seeds"],
            "n_max": cfg.N,
            "Bq": cfg.Bq,
            "Bk": cfg.Bk,
            # float32 values written exactly; -Infinity marks tiles that keep every block
            "table": [[[float(v) for v in row] for row in level] for level in T.astype(np.float64)],
        }
        print(f"{name}: {time.time() - t0:.1f} s", flush=True)
    with open(OUT, "w") as f:
        json.dump(res, f, separators=(",", ":"))


if __name__ == "__main__":
    main()
