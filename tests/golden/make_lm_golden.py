"""Writes tests/golden/lm_oracle_losses.json: the loss curve of the LM oracle
(oracle/lm_ref.py) over the seeded workload of workloads/lm.py. Calls only the
oracle and the seeded input generators.

    python tests/golden/make_lm_golden.py
"""

import json
import os
import sys
import time

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import lm_ref  # noqa: E402
from workloads.lm import LM_CONFIG, lm_batches, lm_init  # noqa: E402


def main():
    cfg = LM_CONFIG
    t0 = time.time()
    losses, _ = lm_ref.train(lm_init(cfg, seed=0), lm_batches(cfg, seed=0), cfg)
    out = {"config": cfg.__dict__, "seed": 0, "losses": losses,
           "note": "oracle/lm_ref.py train() on workloads/lm.py lm_init(seed=0), lm_batches(seed=0); "
                   "loss of each step's forward pass, before that step's update"}
    with open(os.path.join(HERE, "lm_oracle_losses.json"), "w") as f:
        json.dump(out, f, indent=1)
    print(f"{len(losses)} steps in {time.time() - t0:.0f} s; first {losses[0]:.6f} last {losses[-1]:.6f}")


if __name__ == "__main__":
    main()
