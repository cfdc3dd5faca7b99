"""Pins of the float64 gradient oracle of the IPA core (the core is trained,
Flash Invariant Point Attention, TL;DR): central finite differences of the
forward oracle for every element of every input, the zero-norm convention,
rigid-motion covariance, and float64 autograd of an independent torch
restatement of the forward."""
import math

import numpy as np
import pytest
import torch

from oracle import ipa_dense, ipa_grad
from rna_structure_models_b200.synth import IpaDims, ipa_inputs, random_rotations

KEYS = ["q", "k", "v", "q_pts", "k_pts", "v_pts", "rot", "trans", "z1", "z2", "w_bias", "gamma"]


def as64(inp):
    return {k: (np.asarray(v, dtype=np.float64) if isinstance(v, np.ndarray) and v.dtype != bool else v)
            for k, v in inp.items()}


def upstream(inp, seed):
    out = ipa_dense(inp)
    return np.random.default_rng(seed).standard_normal(out.shape)


def fd(inp, g, key, h=1e-6):
    base = inp[key]
    res = np.zeros_like(base)
    for idx in np.ndindex(base.shape):
        for sgn in (1, -1):
            x = base.copy()
            x[idx] += sgn * h
            res[idx] += sgn * float(np.sum(ipa_dense(dict(inp, **{key: x})) * g))
        res[idx] /= 2 * h
    return res


def close(a, b, tol, what):
    scale = max(1.0, float(np.max(np.abs(b))))
    assert np.max(np.abs(a - b)) <= tol * scale, (what, float(np.max(np.abs(a - b))))


@pytest.mark.parametrize("seed", [0, 1])
def test_matches_central_differences(seed):
    inp = as64(ipa_inputs(IpaDims(B=1, L=5, H=2, C=4, Pq=2, Pv=3, R=2, Cz=3), seed, jitter=0.5))
    inp["mask"] = inp["mask"].copy()
    inp["mask"][0, 3] = False                      # a masked residue: no key, and a dead query row
    g = upstream(inp, seed + 10)
    grads = ipa_grad(inp, g)
    for key in KEYS:
        close(grads[key], fd(inp, g, key), 2e-6, key)
    assert np.all(grads["q"][0, 3] == 0) and np.all(grads["k"][0, 3] == 0)


def test_zero_norm_has_zero_derivative():
    # one residue with zero value points: o_pt = R^T (R 0 + t - t) = 0 exactly,
    # and the central difference of |x| at 0 vanishes
    inp = as64(ipa_inputs(IpaDims(B=1, L=1, H=2, C=4, Pq=2, Pv=3, R=1, Cz=2), 3))
    inp["v_pts"] = inp["v_pts"].copy()
    inp["v_pts"][0, 0, 1, 2] = 0.0
    g = upstream(inp, 4)
    grads = ipa_grad(inp, g)
    assert all(np.all(np.isfinite(x)) for x in grads.values())
    close(grads["v_pts"], fd(inp, g, "v_pts", h=1e-7), 1e-6, "v_pts")


def test_covariant_under_a_rigid_motion():
    inp = as64(ipa_inputs(IpaDims(B=2, L=12, H=3, C=8, Pq=2, Pv=2, R=2, Cz=4), 5, masked_tail_frac=0.2))
    g = upstream(inp, 6)
    base = ipa_grad(inp, g)
    rng = np.random.default_rng(7)
    G = random_rotations(rng, 1)[0]
    moved = dict(inp, rot=np.einsum("xy,blyz->blxz", G, inp["rot"]), trans=inp["trans"] @ G.T + rng.normal(size=3) * 9)
    mv = ipa_grad(moved, g)
    for key in ("q", "k", "v", "q_pts", "k_pts", "v_pts", "z1", "z2", "w_bias", "gamma"):
        close(mv[key], base[key], 1e-9, key)
    close(mv["rot"], np.einsum("xy,blyz->blxz", G, base["rot"]), 1e-9, "rot")
    close(mv["trans"], base["trans"] @ G.T, 1e-9, "trans")


def torch_ipa(t, mask, w_L, w_C, ss):
    """The dense IPA core restated with torch float64 ops for autograd."""
    R, T = t["rot"], t["trans"]
    gq = torch.einsum("blxy,blhpy->blhpx", R, t["q_pts"]) + T[:, :, None, None]
    gk = torch.einsum("blxy,blhpy->blhpx", R, t["k_pts"]) + T[:, :, None, None]
    gv = torch.einsum("blxy,blhpy->blhpx", R, t["v_pts"]) + T[:, :, None, None]
    z = torch.einsum("birc,bjrc->bijc", t["z1"], t["z2"])
    d = gq[:, :, None] - gk[:, None]
    d2 = (d * d).sum((-1, -2)).permute(0, 3, 1, 2)
    lg = w_L * (ss * torch.einsum("bihc,bjhc->bhij", t["q"], t["k"]) + torch.einsum("bijc,ch->bhij", z, t["w_bias"])
                - (t["gamma"] * w_C / 2)[None, :, None, None] * d2)
    allowed = (mask[:, :, None] & mask[:, None, :])[:, None]
    lg = lg.masked_fill(~allowed, float("-inf"))
    live = allowed.any(-1, keepdim=True)
    a = torch.where(live, torch.softmax(torch.where(live, lg, torch.zeros_like(lg)), -1), torch.zeros_like(lg))
    a = torch.where(allowed, a, torch.zeros_like(a))
    o = torch.einsum("bhij,bjhc->bihc", a, t["v"])
    og = torch.einsum("bhij,bjhpx->bihpx", a, gv)
    o_pt = torch.einsum("bixy,bihpx->bihpy", R, og - T[:, :, None, None])
    n = torch.sqrt((o_pt * o_pt).sum(-1))
    op = torch.einsum("bhij,bijc->bihc", a, z)
    B, L, H = o.shape[:3]
    out = torch.cat([o, o_pt.reshape(B, L, H, -1), n, op], -1)
    return torch.where(live.permute(0, 2, 1, 3), out, torch.zeros_like(out))


def test_matches_float64_autograd_of_a_torch_restatement():
    dims = IpaDims(B=2, L=20, H=3, C=8, Pq=3, Pv=2, R=2, Cz=5)
    inp = as64(ipa_inputs(dims, 8, masked_tail_frac=0.15, jitter=1.0))
    g = upstream(inp, 9)
    t = {k: torch.tensor(inp[k], requires_grad=True) for k in KEYS}
    w_L, w_C, ss = math.sqrt(1 / 3), math.sqrt(2 / (9 * 3)), 1 / math.sqrt(8)
    out = torch_ipa(t, torch.tensor(inp["mask"]), w_L, w_C, ss)
    (out * torch.tensor(g)).sum().backward()
    grads = ipa_grad(inp, g)
    for key in KEYS:
        close(grads[key], t[key].grad.numpy(), 1e-10, key)


def test_blocked_gradient_equals_the_dense_gradient():
    # the row-blocked oracle (bounded memory, for long sequences) sums the
    # same per-row steps; it must reproduce ipa_grad, including masked and
    # dead rows and a ragged last block
    from oracle.ipa_grad_blocked import ipa_grad_blocked
    inp = as64(ipa_inputs(IpaDims(B=2, L=23, H=3, C=4, Pq=2, Pv=3, R=2, Cz=5), 7, jitter=0.5))
    inp["mask"] = inp["mask"].copy()
    inp["mask"][0, 4] = False
    inp["mask"][1, :] = False
    inp["mask"][1, 9] = True
    g = upstream(inp, 17)
    ref = ipa_grad(inp, g)
    for block in (1, 5, 8, 64):
        got = ipa_grad_blocked(inp, g, block=block)
        for key in KEYS:
            assert np.allclose(got[key], ref[key], rtol=1e-10, atol=1e-12), (block, key)


# ---- the d gamma tolerance scale (root-sum-square of the summed terms' magnitudes)

def test_gamma_scale_one_residue_closed_form():
    # one live residue: the softmax has the single key j = i, a = 1 and D = da,
    # so the one term's magnitude is w_L w_C |da| d2_ii, with d2_ii =
    # sum_p |R (q_p - k_p)|^2 (R as stored: orthonormal to float32 precision
    # only, so the rotation is kept).  With the translation at
    # zero every output (o_pt = R^T a gv included) is homogeneous of degree 1
    # in a, so da = <g, out>.  A second, masked residue contributes nothing.
    from oracle import ipa_grad_gamma_scale
    from oracle.ipa_dense import ipa_constants
    inp = as64(ipa_inputs(IpaDims(B=1, L=2, H=3, C=4, Pq=2, Pv=3, R=2, Cz=3), 5, jitter=0.5))
    inp["mask"] = inp["mask"].copy()
    inp["mask"][0, 1] = False
    inp["trans"] = np.zeros_like(inp["trans"])
    g = upstream(inp, 6)
    got = ipa_grad_gamma_scale(inp, g)
    cst = ipa_constants(4, 2)
    out = ipa_dense(inp)
    for h in range(3):
        da = float(np.sum(g[0, 0, h] * out[0, 0, h]))
        d2 = float(np.sum((inp["rot"][0, 0] @ (inp["q_pts"][0, 0, h] - inp["k_pts"][0, 0, h]).T) ** 2))
        want = cst["w_L"] * cst["w_C"] * abs(da) * d2
        assert abs(got[h] - want) <= 1e-10 * max(1.0, want), (h, got[h], want)


def test_gamma_scale_bounds_the_gradient_and_is_invariant():
    # |d gamma_h| <= sum |terms| <= sqrt(n_h) * scale_h (Cauchy-Schwarz, since
    # |dl| <= a (|da| + |D|)); the scale is even and of degree 1 in g_out and
    # unchanged by a global rigid motion
    from oracle import ipa_grad_gamma_scale
    inp = as64(ipa_inputs(IpaDims(B=2, L=9, H=3, C=4, Pq=2, Pv=3, R=2, Cz=3), 7, jitter=0.5))
    inp["mask"] = inp["mask"].copy()
    inp["mask"][1, 5:] = False
    g = upstream(inp, 8)
    sc = ipa_grad_gamma_scale(inp, g)
    n = int(sum(int(m.sum()) ** 2 for m in inp["mask"]))
    dg = ipa_grad(inp, g)["gamma"]
    assert np.all(sc > 0)
    assert np.all(np.abs(dg) <= math.sqrt(n) * sc * (1 + 1e-12))
    assert np.allclose(ipa_grad_gamma_scale(inp, -2.5 * g), 2.5 * sc, rtol=1e-12)
    rng = np.random.default_rng(9)
    G = random_rotations(rng, 1)[0]
    moved = dict(inp)
    moved["rot"] = np.einsum("xy,blyz->blxz", G, inp["rot"])
    moved["trans"] = inp["trans"] @ G.T + rng.normal(size=3) * 5.0
    assert np.allclose(ipa_grad_gamma_scale(moved, g), sc, rtol=1e-9)
