"""Writes oracle_tiny_fp32_sample.json: oracle outputs (fp64) on sampled tokens
of the tiny fp32 workload. Calls only the oracle and the input generator."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from static_token_routed_b200 import workloads as wl  # noqa: E402


def main():
    w = wl.WORKLOADS["tiny_fp32"]
    t = wl.make_tables(w)
    b = wl.make_batch(w)
    tokens = [0, 1, 2, 3, 100, 255, 256, 511]
    eps = 1e-5
    y = oracle.forward(b.ids, t.offsets, b.x, t.W_K, t.W_V, t.W_up, t.ln_gamma, t.ln_beta,
                       t.W_mix, eps, select=np.array(tokens))
    out = {"workload": w.name, "eps": eps, "tokens": tokens,
           "ids": [int(b.ids[i]) for i in tokens],
           "y": [[float(v) for v in row] for row in y]}
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny_fp32_sample.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
