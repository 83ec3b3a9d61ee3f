"""Regression record of the oracle on the tiny workload (written by
tests/golden/make_golden.py, which calls only the oracle)."""
import json
import os

import numpy as np

import oracle
from workloads import get, make_inputs

GOLD = os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle.json")


def test_oracle_matches_its_golden_record():
    g = json.load(open(GOLD))
    wl = get("tiny")
    I = make_inputs(wl)
    _, delta = oracle.gate(I.V, I.Delta, I.A)
    d32 = delta.astype(np.float32)
    np.testing.assert_array_equal(d32[0].view(np.uint32), np.array(g["delta_f32_bits"], dtype=np.uint32))
    e = np.stack([oracle.topw_eviction(d32[0, h], wl.w) for h in range(wl.H)])
    np.testing.assert_array_equal(e, np.array(g["evict"]))
    rows = np.array(g["rows"])
    O, LSE = oracle.attn_fwd(I.Q, I.K, I.V, d32.astype(np.float64), e[None], rows=rows)
    np.testing.assert_allclose(LSE[0][:, rows], np.array(g["LSE"]), rtol=1e-12)
    np.testing.assert_allclose(O[0][:, rows].sum(-1), np.array(g["O_row_sums"]), rtol=1e-10, atol=1e-12)
