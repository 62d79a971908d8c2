"""Reader for the hand-worked fixtures under tests/golden (name = values lines)."""
import os

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read(name):
    out = {}
    with open(os.path.join(HERE, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = (s.strip() for s in line.split("=", 1))
            out.setdefault(key, []).append(val.split())
    return out


def floats(vals):
    return [float(v) for v in vals]


def ints(vals):
    return [int(v, 0) for v in vals]
