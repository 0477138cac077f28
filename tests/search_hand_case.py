"""The hand-worked layer-search case of tests/golden/search_layer_hand.txt:
its inputs and its expected table, read from the file (shared by the oracle
pin and the GPU test; no method arithmetic here)."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "search_layer_hand.txt")
ALPHAS = (0.25, 0.5, 0.75)
KS = (0, 1, 2)
PAIR_SUM_Y2 = 4418.0


def inputs():
    X = np.ones((1, 32), np.float32)
    X[0, 0] = 16.0
    A = np.full(32, 0.5, np.float32)
    A[:2] = (1.0, 16.0)
    B = np.ones(32, np.float32)
    W = np.stack([A if n % 2 == 0 else B for n in range(16)])
    return X, W


def expected():
    table, best = {}, None
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        parts = [p.strip() for p in line.split("|")]
        if parts[0] == "best":
            best = (float(parts[1]), int(parts[2]), int(parts[3]))
        else:
            table[(float(parts[0]), int(parts[1]), int(parts[2]))] = \
                float(np.sqrt(float(parts[3]) / PAIR_SUM_Y2))
    return table, best
