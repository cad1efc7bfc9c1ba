"""Writes tests/golden/lm_oracle_losses.json: the loss curve of the LM oracle
(oracle/lm_ref.py) over the seeded workload of workloads/lm.py. Calls only the
oracle and the seeded input generators.

    python tests/golden/make_lm_golden.py                 # fp64 (the reference curve)
    python tests/golden/make_lm_golden.py --dtype fp32    # lm_oracle_losses_fp32.json: the same
                                                          # oracle with an fp32 model around BitLinear
"""

import argparse
import json
import os
import sys
import time

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import lm_ref  # noqa: E402
from workloads.lm import LM_CONFIG, lm_batches, lm_init  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--dtype", choices=["fp64", "fp32"], default="fp64")
    args = ap.parse_args()
    cfg = LM_CONFIG
    t0 = time.time()
    dtype = torch.float64 if args.dtype == "fp64" else torch.float32
    losses, _ = lm_ref.train(lm_init(cfg, seed=0), lm_batches(cfg, seed=0), cfg, dtype=dtype)
    out = {"config": cfg.__dict__, "seed": 0, "dtype": args.dtype, "losses": losses,
           "note": "oracle/lm_ref.py train() on workloads/lm.py lm_init(seed=0), lm_batches(seed=0); "
                   "loss of each step's forward pass, before that step's update"}
    name = "lm_oracle_losses.json" if args.dtype == "fp64" else "lm_oracle_losses_fp32.json"
    with open(os.path.join(HERE, name), "w") as f:
        json.dump(out, f, indent=1)
    print(f"{len(losses)} steps in {time.time() - t0:.0f} s; first {losses[0]:.6f} last {losses[-1]:.6f}")


if __name__ == "__main__":
    main()
