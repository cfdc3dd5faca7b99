"""Pins of the float64 gradient oracle of the geometric attention variant
("Geometric direction-and-distance attention", Required behavior: gradients,
zero derivative of the distance at a zero displacement): central finite
differences of the forward oracle, covariance under a rigid motion, masked
frames, the zero-displacement rule, and float64 autograd of a torch
restatement of the forward."""
import math

import numpy as np
import pytest
import torch

from oracle import geo_dense, geo_grad
from rna_structure_models_b200.synth import GeoDims, geo_inputs, geo_upstream, random_rotations

FLOAT_KEYS = ["q_direction", "k_direction", "q_point", "k_point", "values", "direction_scale",
              "distance_scale", "output_weight", "output_bias", "rotation", "translation"]


def as64(inp):
    return {k: (np.asarray(v, dtype=np.float64) if isinstance(v, np.ndarray) and v.dtype != bool else v)
            for k, v in inp.items()}


def loss(inp, up):
    vec, att, out = geo_dense(inp)
    total = float(np.sum(out * up["g_output"]))
    if up["g_attention"] is not None:
        total += float(np.sum(att * up["g_attention"]))
    if up["g_vectors"] is not None:
        total += float(np.sum(vec * up["g_vectors"]))
    return total


def fd_grad(inp, up, key, h=1e-6):
    base = inp[key]
    g = np.zeros_like(base)
    for idx in np.ndindex(base.shape):
        for sgn in (1, -1):
            x = base.copy()
            x[idx] += sgn * h
            g[idx] += sgn * loss(dict(inp, **{key: x}), up)
        g[idx] /= 2 * h
    return g


def tiny(seed, **kw):
    dims = GeoDims(B=1, N=5, H=2, M=2, Cout=3)
    inp = as64(geo_inputs(dims, seed, pair_drop=0.3, **kw))
    up = {k: (None if v is None else v.astype(np.float64)) for k, v in geo_upstream(dims, seed + 100).items()}
    return inp, up


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_matches_central_differences_of_the_forward(seed):
    inp, up = tiny(seed, frame_drop=0.2)
    g = geo_grad(inp, **up)
    for key in FLOAT_KEYS:
        fd = fd_grad(inp, up, key)
        scale = max(1.0, float(np.max(np.abs(fd))))
        assert np.max(np.abs(g[key] - fd)) <= 2e-6 * scale, key


def test_dead_query_and_masked_frame():
    inp, up = tiny(3)
    inp["frame_mask"] = inp["frame_mask"].copy()
    inp["frame_mask"][0, 1] = False                        # frame 1 takes no part
    pm = np.ones((1, 2, 5, 5), dtype=bool)
    pm[0, :, 3, :] = False                                 # query 3 has no allowed key in any head
    inp["pair_mask"] = pm
    g = geo_grad(inp, **up)
    for key in ("q_direction", "k_direction", "q_point", "k_point", "values"):
        assert np.all(g[key][0, 1] == 0.0), key
    assert np.all(g["q_direction"][0, 3] == 0.0) and np.all(g["q_point"][0, 3] == 0.0)
    for key in FLOAT_KEYS:
        fd = fd_grad(inp, up, key)
        assert np.max(np.abs(g[key] - fd)) <= 2e-6 * max(1.0, float(np.max(np.abs(fd)))), key


def test_zero_displacement_has_zero_distance_derivative():
    # put key point (j=2, h=0) exactly on query point (i=0, h=0): the central
    # difference of |x| at x = 0 is 0 in every direction, the page's rule
    inp, up = tiny(4, frame_drop=0.0, with_pair_mask=False)
    # identity frames on residues 0 and 2 make the coincidence exact in float64
    inp["rotation"] = inp["rotation"].copy()
    inp["translation"] = inp["translation"].copy()
    inp["rotation"][0, 0] = np.eye(3)
    inp["rotation"][0, 2] = np.eye(3)
    inp["translation"][0, 2] = 0.0
    inp["k_point"] = inp["k_point"].copy()
    inp["k_point"][0, 2, 0] = inp["q_point"][0, 0, 0] + inp["translation"][0, 0]
    g = geo_grad(inp, **up)
    assert all(np.all(np.isfinite(v)) for v in g.values() if v is not None)
    for key in ("q_point", "k_point", "translation", "rotation", "distance_scale"):
        fd = fd_grad(inp, up, key, h=1e-7)
        assert np.max(np.abs(g[key] - fd)) <= 1e-5 * max(1.0, float(np.max(np.abs(fd)))), key


def test_covariant_under_a_rigid_motion():
    dims = GeoDims(B=2, N=12, H=3, M=2, Cout=4)
    inp = as64(geo_inputs(dims, 5))
    up = geo_upstream(dims, 6)
    g = geo_grad(inp, **up)
    rng = np.random.default_rng(7)
    G = random_rotations(rng, 1)[0]
    s = rng.normal(size=3) * 10
    moved = dict(inp, rotation=np.einsum("xy,bnyz->bnxz", G, inp["rotation"]),
                 translation=inp["translation"] @ G.T + s)
    gm = geo_grad(moved, **up)
    for key in ("q_direction", "k_direction", "q_point", "k_point", "values", "direction_scale",
                "distance_scale", "output_weight", "output_bias"):
        assert np.allclose(gm[key], g[key], atol=1e-9, rtol=1e-9), key
    assert np.allclose(gm["rotation"], np.einsum("xy,bnyz->bnxz", G, g["rotation"]), atol=1e-9)
    assert np.allclose(gm["translation"], g["translation"] @ G.T, atol=1e-9)


def torch_forward(t, pair_mask, frame_mask):
    """The page's forward restated with torch float64 ops (distance with a
    zero gradient at zero displacement) for autograd."""
    R, T = t["rotation"], t["translation"]
    qd = torch.einsum("bnxy,bnhy->bnhx", R, t["q_direction"])
    kd = torch.einsum("bnxy,bnhy->bnhx", R, t["k_direction"])
    qp = torch.einsum("bnxy,bnhy->bnhx", R, t["q_point"]) + T[:, :, None]
    kp = torch.einsum("bnxy,bnhy->bnhx", R, t["k_point"]) + T[:, :, None]
    A = torch.nn.functional.softplus(t["direction_scale"])
    Bd = torch.nn.functional.softplus(t["distance_scale"])
    dot = torch.einsum("bihx,bjhx->bhij", qd, kd)
    d = qp.permute(0, 2, 1, 3)[:, :, :, None] - kp.permute(0, 2, 1, 3)[:, :, None]
    d2 = (d * d).sum(-1)
    pos = d2 > 0
    dist = torch.where(pos, torch.sqrt(torch.where(pos, d2, torch.ones_like(d2))), torch.zeros_like(d2))
    s = (A[:, None, None] * dot - Bd[:, None, None] * dist) / math.sqrt(3.0)
    allowed = (frame_mask[:, :, None] & frame_mask[:, None, :])[:, None] & pair_mask
    s = s.masked_fill(~allowed, float("-inf"))
    live_h = allowed.any(-1, keepdim=True)
    a = torch.where(live_h, torch.softmax(torch.where(live_h, s, torch.zeros_like(s)), -1), torch.zeros_like(s))
    a = torch.where(allowed, a, torch.zeros_like(a))
    vr = torch.einsum("bjxy,bjhmy->bjhmx", R, t["values"])
    agg = torch.einsum("bhij,bjhmx->bihmx", a, vr)
    vec = torch.einsum("bixy,bihmx->bihmy", R, agg)
    B, N = vec.shape[:2]
    out = vec.reshape(B, N, -1) @ t["output_weight"] + t["output_bias"]
    live = allowed.any(-1).any(1)
    out = torch.where(live[..., None], out, torch.zeros_like(out))
    return vec, a, out


def test_matches_float64_autograd_of_a_torch_restatement():
    dims = GeoDims(B=2, N=24, H=3, M=2, Cout=5)
    inp = as64(geo_inputs(dims, 8))
    for key in ("rotation", "translation", "k_point"):
        inp[key] = inp[key].copy()
    inp["rotation"][1, 4] = np.eye(3)                       # exact zero displacement of (i=9, j=4, h=2)
    inp["rotation"][1, 9] = np.eye(3)
    inp["translation"][1, 4] = 0.0
    inp["k_point"][1, 4, 2] = inp["q_point"][1, 9, 2] + inp["translation"][1, 9]
    up = geo_upstream(dims, 9)
    t = {k: torch.tensor(inp[k], dtype=torch.float64, requires_grad=True) for k in FLOAT_KEYS}
    vec, att, out = torch_forward(t, torch.tensor(inp["pair_mask"]), torch.tensor(inp["frame_mask"]))
    L = (out * torch.tensor(up["g_output"], dtype=torch.float64)).sum() \
        + (att * torch.tensor(up["g_attention"], dtype=torch.float64)).sum() \
        + (vec * torch.tensor(up["g_vectors"], dtype=torch.float64)).sum()
    L.backward()
    g = geo_grad(inp, **up)
    for key in FLOAT_KEYS:
        ref = t[key].grad.numpy()
        assert np.allclose(g[key], ref, atol=1e-10 * max(1.0, float(np.abs(ref).max())), rtol=1e-9), key
