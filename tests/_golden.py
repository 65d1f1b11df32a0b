"""Readers for the hand-worked fixtures in tests/golden/."""
import os

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line


def e2m1_points():
    out = []
    for line in rows("e2m1_rne_points.txt"):
        v, code = line.split()
        out.append((float(v), int(code, 16)))
    return out


def nvfp4_groups():
    out = []
    for line in rows("nvfp4_groups.txt"):
        name, gs, xs, sfb, codes = [p.strip() for p in line.split("|")]
        out.append((name, float(gs), [float(t) for t in xs.split()], int(sfb, 16),
                    [int(t, 16) for t in codes.split()]))
    return out
