"""Seeded choice of the (sample, head) pairs a full-size parity test compares.

The full-size workloads have too many (sample, head) pairs for the float64
oracle to check them all in seconds, so those tests compare a seeded subset:
`per_class` distinct pairs of every head class (local, literal, hybrid),
drawn without replacement (all of a class's pairs when it has fewer)."""
import numpy as np


def class_pairs(S: int, head_classes, per_class: int, seed: int):
    hc = [int(c) for c in head_classes]
    rng = np.random.default_rng(seed)
    out = set()
    for c in (0, 1, 2):
        cand = [(s, h) for s in range(S) for h in range(len(hc)) if hc[h] == c]
        if not cand:
            continue
        take = min(per_class, len(cand))
        for i in rng.choice(len(cand), size=take, replace=False):
            out.add(cand[int(i)])
    return out
