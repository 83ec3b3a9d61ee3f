"""Writes tests/golden/tiny_oracle.json from the CPU oracle alone.

The pages print no worked numbers for this method, so this fixture is a
regression record of the oracle on the seeded tiny workload (B=1, H=2, Hkv=1,
N=256, d=64, w=64, seed 0): delta as float32 bit patterns, the eviction
index e of every key, and O/LSE of a few query rows.  It is produced by this
script only (never from the CUDA path); rerun it only together with an oracle
change whose commit message names the passage that justifies the change.

Usage: python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from workloads import get, make_inputs  # noqa: E402

ROWS = [0, 1, 63, 64, 65, 127, 200, 255]


def main():
    wl = get("tiny")
    I = make_inputs(wl)
    _, delta = oracle.gate(I.V, I.Delta, I.A)
    d32 = delta.astype(np.float32)
    e = np.stack([oracle.topw_eviction(d32[0, h], wl.w) for h in range(wl.H)])[None]
    O, LSE = oracle.attn_fwd(I.Q, I.K, I.V, d32.astype(np.float64), e, rows=np.array(ROWS))
    out = {
        "source": "oracle/dma_oracle.py on workload 'tiny' (seed 0); see make_golden.py",
        "workload": {"B": wl.B, "H": wl.H, "Hkv": wl.Hkv, "N": wl.N, "d": wl.d, "w": wl.w, "seed": wl.seed},
        "delta_f32_bits": [[int(v) for v in d32[0, h].view(np.uint32)] for h in range(wl.H)],
        "evict": [[int(v) for v in e[0, h]] for h in range(wl.H)],
        "rows": ROWS,
        "LSE": [[float(LSE[0, h, r]) for r in ROWS] for h in range(wl.H)],
        "O_row_sums": [[float(O[0, h, r].sum()) for r in ROWS] for h in range(wl.H)],
    }
    with open(os.path.join(HERE, "tiny_oracle.json"), "w") as f:
        json.dump(out, f, indent=0)


if __name__ == "__main__":
    main()
