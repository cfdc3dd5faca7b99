"""Pins of the float64 geometric-attention oracle ("Geometric
direction-and-distance attention", Required behavior) against invariances,
special cases and library routines."""
import math

import numpy as np
import pytest

from oracle import geo_dense, geo_dense_blocked, softplus_stable
from rna_structure_models_b200.synth import GeoDims, geo_inputs, random_rotations


def small(seed=0, N=10, **kw):
    return geo_inputs(GeoDims(B=2, N=N, H=3, M=2, Cout=5), seed, **kw)


def close(a, b, tol):
    a, b = np.asarray(a), np.asarray(b)
    scale = max(1.0, float(np.max(np.abs(b))))
    assert np.max(np.abs(a - b)) <= tol * scale, np.max(np.abs(a - b))


def test_softplus_stable_matches_library_and_does_not_overflow():
    x = np.linspace(-30, 30, 121)
    close(softplus_stable(x), np.logaddexp(0.0, x), 1e-14)
    assert softplus_stable(1000.0) == 1000.0
    assert 0.0 <= softplus_stable(-1000.0) < 1e-300


@pytest.mark.parametrize("seed", [0, 1])
def test_invariance_under_global_rigid_motion(seed):
    inp = small(seed)
    v0, a0, o0 = geo_dense(inp)
    rng = np.random.default_rng(10 + seed)
    G = random_rotations(rng, 1)[0]
    s = rng.normal(size=3) * 40.0
    mv = dict(inp)
    mv["rotation"] = np.einsum("xy,bnyz->bnxz", G, inp["rotation"].astype(float))
    mv["translation"] = inp["translation"].astype(float) @ G.T + s
    v1, a1, o1 = geo_dense(mv)
    close(v1, v0, 1e-10)
    close(a1, a0, 1e-10)
    close(o1, o0, 1e-10)


def test_identity_frames_match_library_attention():
    # identity rotations and zero translations: scores are
    # (a q.k - b |q - k|) / sqrt(3), i.e. SDPA with scale a/sqrt(3) and an
    # additive bias -b cdist(q, k)/sqrt(3) (torch routines, float64).
    torch = pytest.importorskip("torch")
    inp = small(2, with_pair_mask=False)
    B, N, H, M = 2, 10, 3, 2
    inp["rotation"] = np.broadcast_to(np.eye(3), (B, N, 3, 3)).copy()
    inp["translation"] = np.zeros((B, N, 3))
    inp["frame_mask"] = np.ones((B, N), bool)
    vec, att, _ = geo_dense(inp)
    a = softplus_stable(inp["direction_scale"])
    b = softplus_stable(inp["distance_scale"])
    for h in range(H):
        q = torch.tensor(inp["q_direction"][:, :, h], dtype=torch.float64)
        k = torch.tensor(inp["k_direction"][:, :, h], dtype=torch.float64)
        qp = torch.tensor(inp["q_point"][:, :, h], dtype=torch.float64)
        kp = torch.tensor(inp["k_point"][:, :, h], dtype=torch.float64)
        val = torch.tensor(inp["values"][:, :, h].reshape(B, N, M * 3), dtype=torch.float64)
        bias = -float(b[h]) * torch.cdist(qp, kp) / math.sqrt(3.0)
        ref = torch.nn.functional.scaled_dot_product_attention(
            q, k, val, attn_mask=bias, scale=float(a[h]) / math.sqrt(3.0))
        close(vec[:, :, h].reshape(B, N, M * 3), ref.numpy(), 1e-12)
        w = torch.softmax(float(a[h]) / math.sqrt(3.0) * q @ k.transpose(1, 2) + bias, -1)
        close(att[:, h], w.numpy(), 1e-12)


def test_single_residue():
    # N = 1: attention 1, vectors = R^T R values = values (exactly orthogonal R)
    inp = small(3, N=1, with_pair_mask=False)
    inp["frame_mask"] = np.ones((2, 1), bool)
    inp["rotation"] = random_rotations(np.random.default_rng(3), 2).reshape(2, 1, 3, 3)
    vec, att, out = geo_dense(inp)
    close(att, np.ones_like(att), 1e-15)
    close(vec, inp["values"].astype(float), 1e-12)
    flat = inp["values"].astype(float).reshape(2, 1, -1)
    close(out, flat @ inp["output_weight"].astype(float) + inp["output_bias"], 1e-12)


def test_masks_rows_and_outputs():
    inp = small(4)
    fm = np.ones((2, 10), bool)
    fm[0, 3] = False                      # invalid frame: query row empty in every head
    inp["frame_mask"] = fm
    pm = np.ones((2, 3, 10, 10), bool)
    pm[1, 2, 6, :] = False                # one head row of (b=1, i=6) fully excluded
    inp["pair_mask"] = pm
    vec, att, out = geo_dense(inp)
    # invalid query: everything zero, including the readout despite the bias
    assert np.all(vec[0, 3] == 0) and np.all(att[0, :, 3] == 0) and np.all(out[0, 3] == 0)
    # invalid key: zero weight everywhere
    assert np.all(att[0, :, :, 3] == 0)
    # one head row excluded: that head's vectors are exact zeros, the others not,
    # and the readout keeps its bias (some head has an allowed key)
    assert np.all(vec[1, 6, 2] == 0) and np.all(att[1, 2, 6] == 0)
    assert np.any(vec[1, 6, 0] != 0)
    flat = vec[1, 6].reshape(-1)
    close(out[1, 6], flat @ inp["output_weight"].astype(float) + inp["output_bias"], 1e-12)
    # rows that have keys sum to one
    s = att.sum(-1)
    live = s > 0
    close(s[live], np.ones(live.sum()), 1e-12)


def test_all_heads_masked_forces_zero_output():
    inp = small(5)
    pm = np.ones((2, 3, 10, 10), bool)
    pm[0, :, 2, :] = False
    inp["pair_mask"] = pm
    _, _, out = geo_dense(inp)
    assert np.all(out[0, 2] == 0.0)


def test_pair_mask_broadcast_equals_expanded():
    inp = small(6)
    pm = np.random.default_rng(6).random((1, 1, 10, 10)) > 0.3
    inp["pair_mask"] = pm
    r1 = geo_dense(inp)
    inp["pair_mask"] = np.broadcast_to(pm, (2, 3, 10, 10)).copy()
    r2 = geo_dense(inp)
    for x, y in zip(r1, r2):
        close(x, y, 1e-14)


def test_distance_is_unsquared():
    # two keys: one at distance 1, one at distance 2 from the query point, all
    # directions zero; scores are -b*1/sqrt(3) and -b*2/sqrt(3), so the weight
    # ratio is exp(b/sqrt(3)) (a squared distance would give exp(3b/sqrt(3))).
    inp = geo_inputs(GeoDims(B=1, N=3, H=1, M=1, Cout=1), 0, with_pair_mask=False)
    inp["rotation"] = np.broadcast_to(np.eye(3), (1, 3, 3, 3)).copy()
    inp["translation"] = np.zeros((1, 3, 3))
    inp["frame_mask"] = np.ones((1, 3), bool)
    inp["q_direction"] = np.zeros((1, 3, 1, 3))
    inp["k_direction"] = np.zeros((1, 3, 1, 3))
    inp["q_point"] = np.zeros((1, 3, 1, 3))
    kp = np.zeros((1, 3, 1, 3))
    kp[0, 1, 0, 0] = 1.0
    kp[0, 2, 0, 0] = 2.0
    kp[0, 0, 0, 0] = 50.0
    inp["k_point"] = kp
    _, att, _ = geo_dense(inp)
    b = float(softplus_stable(inp["distance_scale"])[0])
    ratio = att[0, 0, 0, 1] / att[0, 0, 0, 2]
    close(ratio, math.exp(b / math.sqrt(3.0)), 1e-12)


def test_values_rotate_without_translation():
    # One allowed key j for query i: vectors_i = R_i^T R_j values_j, with no
    # translation term.
    inp = small(7, N=2, with_pair_mask=False)
    inp["frame_mask"] = np.ones((2, 2), bool)
    pm = np.zeros((2, 3, 2, 2), bool)
    pm[:, :, 0, 1] = True
    pm[:, :, 1, 0] = True
    inp["pair_mask"] = pm
    vec, _, _ = geo_dense(inp)
    R = inp["rotation"].astype(float)
    val = inp["values"].astype(float)
    for b in range(2):
        for h in range(3):
            exp = (R[b, 0].T @ R[b, 1] @ val[b, 1, h].T).T
            close(vec[b, 0, h], exp, 1e-12)


def test_blocked_equals_full():
    inp = small(8, N=33)
    v0, a0, o0 = geo_dense(inp)
    v1, a1, o1 = geo_dense_blocked(inp, block=8)
    close(v1, v0, 1e-14)
    close(a1, a0, 1e-14)
    close(o1, o0, 1e-14)
