"""Pins of the backbone-frame oracle (Flash Invariant Point Attention,
Figure 1: Gram-Schmidt frame on C_alpha from C_alpha->N and C_alpha->C):
recovery of the frames the atoms were built from, orthonormality and
handedness, rigid-motion equivariance, axis construction."""
import numpy as np
import pytest

from oracle import frames_from_backbone
from rna_structure_models_b200.synth import backbone_inputs, random_rotations


def test_recovers_the_frames_the_atoms_were_built_from():
    bb = backbone_inputs(2, 50, 0)
    R, t = frames_from_backbone(bb["n"].astype(np.float64), bb["ca"].astype(np.float64), bb["c"].astype(np.float64))
    # atoms were stored as float32: compare at float32 resolution
    assert np.allclose(R, bb["rot"], atol=2e-5)
    assert np.allclose(t, bb["trans"], atol=1e-4)


def test_orthonormal_right_handed_for_noisy_atoms():
    bb = backbone_inputs(3, 40, 1, jitter=0.3)
    R, _ = frames_from_backbone(bb["n"], bb["ca"], bb["c"])
    eye = np.einsum("blxi,blxj->blij", R, R)
    assert np.allclose(eye, np.eye(3), atol=1e-12)
    assert np.allclose(np.linalg.det(R), 1.0, atol=1e-12)


def test_equivariant_under_rigid_motion():
    bb = backbone_inputs(1, 30, 2, jitter=0.2)
    rng = np.random.default_rng(4)
    G = random_rotations(rng, 1)[0]
    s = rng.normal(size=3) * 20
    R, t = frames_from_backbone(bb["n"], bb["ca"], bb["c"])
    mv = lambda a: a.astype(np.float64) @ G.T + s  # noqa: E731
    R2, t2 = frames_from_backbone(mv(bb["n"]), mv(bb["ca"]), mv(bb["c"]))
    assert np.allclose(R2, np.einsum("xy,blyz->blxz", G, R), atol=1e-12)
    assert np.allclose(t2, t.astype(np.float64) @ G.T + s, atol=1e-10)


def test_axis_construction():
    rng = np.random.default_rng(5)
    ca = rng.normal(size=(20, 3))
    c = ca + rng.normal(size=(20, 3))
    n = ca + rng.normal(size=(20, 3))
    R, t = frames_from_backbone(n, ca, c)
    e1, e2, e3 = R[..., 0], R[..., 1], R[..., 2]
    v1, v2 = c - ca, n - ca
    assert np.allclose(np.cross(e1, v1), 0.0, atol=1e-12) and np.all(np.sum(e1 * v1, -1) > 0)
    assert np.allclose(np.sum(e3 * v2, -1), 0.0, atol=1e-12)          # N lies in the e1-e2 plane
    assert np.all(np.sum(e2 * v2, -1) > 0)                            # on the positive e2 side
    assert np.allclose(np.cross(e1, e2), e3, atol=1e-12)
    assert np.allclose(t, ca)
    # positive rescaling of the bond vectors leaves the frame unchanged
    R2, _ = frames_from_backbone(ca + 3.0 * (n - ca), ca, ca + 0.5 * (c - ca))
    assert np.allclose(R2, R, atol=1e-12)
