"""Pins of the local nearest-neighbour distogram oracle: a lattice with known
neighbour distances, exact bin counts, brute-force selection against a full
sort, tie order, masks, and fewer valid residues than k."""
import itertools

import numpy as np

from oracle.distogram import knn_distogram
from rna_structure_models_b200.synth import random_walk


def test_cubic_lattice_neighbours_and_bins():
    # points on a 4 x 4 x 4 grid of spacing 2 A: an interior point has 6
    # neighbours at 2 A, 12 at 2 sqrt(2), 8 at 2 sqrt(3); with edges
    # (2.5, 3.0, 3.6) those fall in bins 0, 1 and 2 exactly
    pts = np.array(list(itertools.product(range(4), repeat=3)), dtype=np.float32) * 2.0
    x = pts[None]
    mask = np.ones((1, 64), bool)
    i = 1 * 16 + 1 * 4 + 1                           # grid point (1, 1, 1): interior
    idx, bins, hist = knn_distogram(x, mask, 26, [2.5, 3.0, 3.6])
    d = np.linalg.norm(pts[idx[0, i]] - pts[i], axis=1)
    assert np.allclose(d[:6], 2.0) and np.allclose(d[6:18], 2 * np.sqrt(2)) and np.allclose(d[18:], 2 * np.sqrt(3))
    assert hist[0, i].tolist() == [6.0, 12.0, 8.0, 0.0]
    assert bins[0, i].tolist() == [0] * 6 + [1] * 12 + [2] * 8
    # equal distances come in increasing index
    for lo, hi in ((0, 6), (6, 18), (18, 26)):
        assert list(idx[0, i, lo:hi]) == sorted(idx[0, i, lo:hi])


def test_brute_force_selection_and_counts():
    rng = np.random.default_rng(3)
    L = 57
    x = np.stack([random_walk(rng, L) for _ in range(2)]).astype(np.float32)
    mask = np.ones((2, L), bool)
    mask[1, 40:] = False
    mask[0, 7] = False
    edges = [3.0, 5.0, 8.0, 12.0, 20.0]
    idx, bins, hist = knn_distogram(x, mask, 10, edges)
    for b in range(2):
        for i in range(L):
            if not mask[b, i]:
                assert np.all(idx[b, i] == -1) and np.all(hist[b, i] == 0)
                continue
            # float64 distances decide everything except near-ties (consecutive
            # walk residues sit 3.8 A apart, equal after float32 rounding), so
            # compare the selected distances, not the order of equal ones
            others = [j for j in range(L) if j != i and mask[b, j]]
            dist = {j: float(np.linalg.norm(x[b, j].astype(np.float64) - x[b, i])) for j in others}
            best = sorted(dist[j] for j in others)[:10]
            got = [dist[int(j)] for j in idx[b, i]]
            assert np.allclose(got, best, atol=1e-5), (got, best)
            assert all(got[s] <= got[s + 1] + 1e-5 for s in range(len(got) - 1))
            assert len(set(idx[b, i].tolist())) == 10 and i not in idx[b, i]
            assert hist[b, i].sum() == len(best)
            for s, j in enumerate(idx[b, i]):
                d = dist[int(j)]
                if all(abs(d - e) > 1e-5 for e in edges):
                    assert bins[b, i, s] == sum(d >= e for e in edges)


def test_fewer_valid_residues_than_k():
    x = np.zeros((1, 5, 3), np.float32)
    x[0, :, 0] = [0.0, 1.0, 3.0, 6.0, 10.0]
    mask = np.array([[True, True, False, True, False]])
    idx, bins, hist = knn_distogram(x, mask, 4, [2.0, 5.0])
    assert idx[0, 0].tolist() == [1, 3, -1, -1]
    assert bins[0, 0].tolist() == [0, 2, -1, -1]
    assert hist[0, 0].tolist() == [1.0, 0.0, 1.0]
    assert idx[0, 3].tolist() == [1, 0, -1, -1]     # distances 5 and 6: 5 >= edge 5.0 -> bin 2
    assert bins[0, 3].tolist() == [2, 2, -1, -1]
