"""Local nearest-neighbour distogram of residue positions: a plain CPU oracle.

TEST INFRASTRUCTURE ONLY: imported by tests/, never by the product path.
Shares no code with the CUDA library.

Flash Invariant Point Attention (TL;DR) builds its pair information from "a
local nearest-neighbor distogram" but fixes neither the number of neighbours,
nor the distance bins, nor how the result becomes pair factors.  This module
computes the one part those words do fix, with every open choice a
parameter:

  for batch b and valid residue i (mask[b, i]):
    neighbours  the k valid residues j != i closest to i, by the Euclidean
                distance |x_j - x_i| of their positions (C-alpha / frame
                origins), nearest first, equal distances in increasing j;
                slots beyond the number of valid other residues hold -1
    bins        bin of each neighbour's distance against the caller's
                increasing edges e_0 < ... < e_{nb-2} (Angstrom):
                bin(d) = #{m : d >= e_m}, in [0, nb - 1]; -1 for empty slots
    histogram   hist[b, i, c] = number of the i's neighbours in bin c
                (the local distogram of residue i; all 0 for a masked i)

Distances are compared as squared distances evaluated in float32 in a fixed
order -- dx = x_j - x_i per axis, d2 = (dx*dx + dy*dy) + dz*dz, edges squared
as e*e -- so that the integer results are defined by one precision (the
kernel's) and can be compared bit for bit.
"""
from __future__ import annotations

import numpy as np

__all__ = ["knn_distogram", "squared_distances_f32"]


def squared_distances_f32(x_b: np.ndarray, i: int) -> np.ndarray:
    """Squared distances from residue i to every residue, float32, in the
    order (dx*dx + dy*dy) + dz*dz."""
    x = np.asarray(x_b, dtype=np.float32)
    d = x - x[i]
    dx, dy, dz = d[:, 0], d[:, 1], d[:, 2]
    return (dx * dx + dy * dy) + dz * dz


def knn_distogram(x, mask, k: int, edges):
    """(idx [B, L, k] int32, bins [B, L, k] int32, hist [B, L, nb] float32)."""
    x = np.asarray(x, dtype=np.float32)
    mask = np.asarray(mask, dtype=bool)
    e = np.asarray(edges, dtype=np.float32)
    e2 = e * e
    nb = len(e) + 1
    B, L, _ = x.shape
    idx = np.full((B, L, k), -1, dtype=np.int32)
    bins = np.full((B, L, k), -1, dtype=np.int32)
    hist = np.zeros((B, L, nb), dtype=np.float32)
    for b in range(B):
        for i in range(L):
            if not mask[b, i]:
                continue
            d2 = squared_distances_f32(x[b], i)
            cand = [j for j in range(L) if j != i and mask[b, j]]
            # nearest first, equal distances in increasing index
            cand.sort(key=lambda j: (float(d2[j]), j))
            for s, j in enumerate(cand[:k]):
                idx[b, i, s] = j
                c = int(np.sum(d2[j] >= e2))
                bins[b, i, s] = c
                hist[b, i, c] += 1.0
    return idx, bins, hist
