"""Golden cases of the dual-window search (tests/golden/search_cases.json):
loading, and the per-offset masses each case states."""
import json
import os

import numpy as np

import oracle as O

UNIT = 1 << 16  # integer mass of one fixture unit
FIELDS = ("moves", "windows", "covered_units", "total_units", "pairs")


def load(golden_dir):
    return json.load(open(os.path.join(golden_dir, "search_cases.json")))["cases"]


def mass(case):
    """[Nt, Nt] masses: every pair of tiles at offset (|dt|, |dy|, |dx|)
    carries f * 2^16 / 2^24 (f from the case, 0 if absent); exact in fp32."""
    T, H, W = case["grid"]
    nh, nw, nt, _ = O.tile_grid(T, H, W)
    idx = np.arange(nt)
    t, y, x = idx // (nh * nw), (idx // nw) % nh, idx % nw
    m = np.zeros((nt, nt))
    for q in range(nt):
        for k in range(nt):
            key = f"{abs(t[q] - t[k])},{abs(y[q] - y[k])},{abs(x[q] - x[k])}"
            m[q, k] = case["f"].get(key, 0) * UNIT / 2.0 ** 24
    return m
