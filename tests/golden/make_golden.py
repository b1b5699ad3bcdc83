"""Write tests/golden/oracle_tiny_seed0.txt: sampled oracle outputs for the
tiny workload (B=1, Cc=4, H=W=16, fp32, seed 0).

Calls only the oracle and the seeded input generator.  The file guards the
oracle against unintended changes; any change to it must come with the
passage (or the reading of it) that justifies the change.
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from spatial_propagation_vision_b200.workloads import WORKLOADS, workload_inputs  # noqa: E402


def main():
    inp = workload_inputs(WORKLOADS["tiny"], seed=0)
    t = {k: v.double().numpy() for k, v in inp.items()}
    y = oracle.prop2d(t["x"], t["lam"], t["wlogit"], t["u"])
    rng = np.random.default_rng(0)
    idx = [(0, c, i, j) for c in range(4) for (i, j) in [(0, 0), (0, 15), (15, 0), (15, 15), (7, 8)]]
    idx += [tuple([0] + list(rng.integers(0, [4, 16, 16]))) for _ in range(44)]
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny_seed0.txt")
    with open(out, "w") as f:
        f.write("# b c i j y  -- oracle output, tiny workload, seed 0 (tests/golden/make_golden.py)\n")
        for (b, c, i, j) in idx:
            f.write(f"{b} {c} {i} {j} {y[b, c, i, j]:.17e}\n")


if __name__ == "__main__":
    main()
