"""Reader for the hand-worked fixtures under tests/golden: one `name = v1 v2 ...` line per array
(values in row-major order), `#` starts a comment (the derivation and its citation)."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read(name: str) -> dict:
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = (s.strip() for s in line.split("=", 1))
            out[key] = np.array([float(x) for x in val.split()], dtype=np.float64)
    return out
