"""The local nearest-neighbour distogram on the GPU (C ABI) against the
oracle on the same seeded positions: neighbour indices, bins and histograms
bit for bit (both sides decide in float32), on ragged and masked inputs,
every supported neighbour-count class, strided positions, and a lattice
with exact ties."""
import itertools

import numpy as np
import pytest
import torch

from oracle.distogram import knn_distogram
from rna_structure_models_b200 import api
from rna_structure_models_b200.synth import random_walk

pytestmark = pytest.mark.gpu

EDGES = [2.0, 3.5, 5.0, 6.5, 8.0, 10.0, 12.0, 15.0, 20.0]


def walk(B, L, seed, jitter=0.0):
    rng = np.random.default_rng(seed)
    x = np.stack([random_walk(rng, L) for _ in range(B)])
    if jitter:
        x = x + jitter * rng.standard_normal(x.shape)
    return x.astype(np.float32)


def run(x, mask, k, edges):
    xd = torch.from_numpy(x).cuda()
    md = torch.from_numpy(mask).cuda()
    idx, bins, hist = api.knn_distogram(xd, md, k, edges)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), bins.cpu().numpy(), hist.cpu().numpy()


@pytest.mark.parametrize("k", [1, 8, 9, 16, 17, 32])
@pytest.mark.parametrize("L", [1, 2, 33, 130, 517])
def test_matches_oracle_bit_for_bit(cuda_device, L, k):
    x = walk(2, L, 7 * L + k, jitter=0.3)
    mask = np.ones((2, L), bool)
    if L > 4:
        mask[1, L // 3:] = False
        mask[0, 2] = False
    got = run(x, mask, k, EDGES)
    ref = knn_distogram(x, mask, k, EDGES)
    for g, r, name in zip(got, ref, ("idx", "bins", "hist")):
        assert np.array_equal(g, r), name


def test_exact_ties_on_a_lattice(cuda_device):
    pts = np.array(list(itertools.product(range(5), repeat=3)), dtype=np.float32) * 1.5
    x = pts[None]
    mask = np.ones((1, len(pts)), bool)
    got = run(x, mask, 32, [1.6, 2.2, 2.7, 3.1])
    ref = knn_distogram(x, mask, 32, [1.6, 2.2, 2.7, 3.1])
    for g, r, name in zip(got, ref, ("idx", "bins", "hist")):
        assert np.array_equal(g, r), name


def test_strided_positions_and_no_edges(cuda_device):
    x = walk(1, 300, 3)
    big = np.zeros((1, 300, 7), np.float32)
    big[..., 2:5] = x
    xd = torch.from_numpy(big).cuda()[..., 2:5]
    assert not xd.is_contiguous()
    md = torch.ones((1, 300), dtype=torch.bool, device="cuda")
    idx, bins, hist = api.knn_distogram(xd, md, 12, [])
    ref = knn_distogram(x, np.ones((1, 300), bool), 12, [])
    assert np.array_equal(idx.cpu().numpy(), ref[0])
    assert np.all(bins.cpu().numpy() == 0) and np.all(hist.cpu().numpy() == 12)


def test_long_sequence_sampled_rows(cuda_device):
    L = 4096
    x = walk(1, L, 11, jitter=0.5)
    mask = np.ones((1, L), bool)
    got = run(x, mask, 16, EDGES)
    rows = np.random.default_rng(2).choice(L, 48, replace=False)
    from oracle.distogram import squared_distances_f32
    e2 = np.asarray(EDGES, np.float32) ** 2
    for i in rows:
        d2 = squared_distances_f32(x[0], i)
        order = sorted((j for j in range(L) if j != i), key=lambda j: (float(d2[j]), j))[:16]
        assert list(got[0][0, i]) == order
        assert list(got[1][0, i]) == [int(np.sum(d2[j] >= e2)) for j in order]
