"""Reader for the hand-worked fixtures under tests/golden/."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _num(s):
    s = s.strip()
    return float(s)


def verify_cases():
    out = []
    with open(os.path.join(GOLDEN, "verify_cases.txt"), encoding="utf-8") as f:
        for line in f:
            if not line.strip() or line.lstrip().startswith("#"):
                continue
            name, bv, rows, drafts, res = [p.strip() for p in line.split("|")]
            B, V = (int(t) for t in bv.split())
            z = np.array([[_num(t) for t in r.split(",")] for r in rows.split(";")], dtype=np.float32)
            assert z.shape == (B, V), name
            d = [] if drafts == "-" else [int(t) for t in drafts.split(",")]
            assert len(d) == B - 1, name
            a, nxt = (int(t) for t in res.split())
            out.append((name, z, np.array(d, dtype=np.int64), a, nxt))
    return out
