"""Parser for the hand-written fixtures under tests/golden/."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _hex_bytes(tokens):
    out = []
    for t in tokens:
        if "*" in t:
            b, n = t.split("*")
            out.extend([int(b, 16)] * int(n))
        else:
            out.append(int(t, 16))
    return out


def load_hfq4_cases(name="hfq4_handpacked.txt"):
    cases = []
    cur = None
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        head, _, rest = line.partition(" ")
        if head == "case":
            f = rest.split()
            cur = {"name": f[0], "rows": int(f[2]), "cols": int(f[4]), "bytes": [], "expect": []}
            cases.append(cur)
        elif head == "hex":
            cur["bytes"].extend(_hex_bytes(rest.split()))
        elif head == "expect":
            n, _, vals = rest.partition(":")
            assert n.startswith("repeat")
            cur["expect"].extend([float(v) for v in vals.split()] * int(n.split()[1]))
    for c in cases:
        c["bytes"] = np.array(c["bytes"], dtype=np.uint8)
        c["expect"] = np.array(c["expect"], dtype=np.float64).reshape(c["rows"], c["cols"])
    return cases


def load_placement_cases(name="placement_auto.txt"):
    """Rows of the hand-worked placement fixture as dicts."""
    keys = ["name", "resident", "hot", "budget", "ok", "N", "hbm", "host", "deficit"]
    out = []
    for line in open(os.path.join(GOLDEN, name)):
        if line.startswith("case "):
            f = line.split()[1:]
            d = dict(zip(keys, [f[0]] + [int(v) for v in f[1:]]))
            d["ok"] = bool(d["ok"])
            out.append(d)
    return out
