"""Independent numpy lattice helpers for tests (no oracle or library code)."""
import itertools

import numpy as np


def e8_points(max_n2=48, min_n2=0):
    """All doubled E8 points with min_n2 <= |P|^2 <= max_n2, sorted by
    (|P|^2, lexicographic)."""
    lim = int(np.floor(np.sqrt(max_n2)))
    pts = []
    for start in (0, 1):
        vals = np.array([v for v in range(-lim, lim + 1) if (v - start) % 2 == 0])
        grid = np.array(list(itertools.product(vals, repeat=4)), np.int32)
        n2h = (grid * grid).sum(1)
        sh = grid.sum(1)
        ok = n2h <= max_n2
        grid, n2h, sh = grid[ok], n2h[ok], sh[ok]
        for i in range(len(grid)):
            rem = max_n2 - n2h[i]
            sel = (n2h <= rem) & (n2h >= min_n2 - n2h[i]) & (((sh[i] + sh) % 4) == 0)
            if sel.any():
                pts.append(np.concatenate([np.repeat(grid[i:i + 1], sel.sum(), 0), grid[sel]], 1))
    P = np.concatenate(pts, 0)
    n2 = (P * P).sum(1)
    order = np.lexsort(tuple(P[:, k] for k in range(7, -1, -1)) + (n2,))
    return P[order], n2[order]


def is_e8(P):
    P = np.asarray(P)
    par = P[..., :1] & 1
    return ((P & 1) == par).all(-1) & (P.sum(-1) % 4 == 0)
