"""Pins of the float64 IPA oracle against facts fixed by the pages and by
mathematics -- never against the oracle itself.

Sources: Flash Invariant Point Attention (TL;DR: SE(3) invariance, exact
factorisation z_ij = z1_i^T z2_j); MEET, section 2.2 eq. (7)-(8) (the squared
distance as an augmented dot product); closed forms and a library routine
(torch scaled_dot_product_attention) for the special cases.
"""
import math

import numpy as np
import pytest

from oracle import ipa_constants, ipa_dense, ipa_dense_blocked
from rna_structure_models_b200.synth import IpaDims, ipa_inputs, random_rotations

RTOL = 1e-10


def small(seed=0, **kw):
    dims = IpaDims(B=2, L=kw.pop("L", 12), H=3, C=4, Pq=2, Pv=3, R=2, Cz=5)
    return ipa_inputs(dims, seed, **kw)


def close(a, b, tol=RTOL):
    a, b = np.asarray(a), np.asarray(b)
    scale = max(1.0, float(np.max(np.abs(b))))
    assert np.max(np.abs(a - b)) <= tol * scale, np.max(np.abs(a - b))


# ---------------------------------------------------------------- softmax facts
def test_rows_sum_to_one_and_masked_rows_zero():
    inp = small(masked_tail_frac=0.25)
    out, a = ipa_dense(inp, return_attn=True)
    mask = inp["mask"]
    s = a.sum(axis=-1)                                    # [B, H, L]
    for b in range(2):
        for i in range(12):
            if mask[b, i]:
                assert abs(s[b, :, i] - 1).max() < 1e-12
                # masked keys get exactly zero weight
                assert np.all(a[b, :, i, ~mask[b]] == 0.0)
            else:
                assert np.all(a[b, :, i] == 0.0)
                assert np.all(out[b, i] == 0.0)


def test_all_masked_batch_gives_zero():
    inp = small()
    inp["mask"][1, :] = False
    out = ipa_dense(inp)
    assert np.all(out[1] == 0.0)
    assert np.any(out[0] != 0.0)


# ------------------------------------------------------- SE(3) invariance (p.1)
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_invariance_under_global_rigid_motion(seed):
    inp = small(seed)
    ref = ipa_dense(inp)
    rng = np.random.default_rng(100 + seed)
    G = random_rotations(rng, 1)[0]
    s = rng.normal(size=3) * 50.0
    moved = dict(inp)
    moved["rot"] = np.einsum("xy,blyz->blxz", G, inp["rot"].astype(np.float64))
    moved["trans"] = inp["trans"].astype(np.float64) @ G.T + s
    close(ipa_dense(moved), ref, 1e-9)


def test_not_invariant_to_local_frame_change():
    # Control for the invariance test: rotating ONE residue's frame must change
    # the outputs (points are expressed in local frames).
    inp = small(3)
    ref = ipa_dense(inp)
    mod = dict(inp)
    rot = inp["rot"].astype(np.float64).copy()
    rot[0, 5] = random_rotations(np.random.default_rng(7), 1)[0]
    mod["rot"] = rot
    assert np.max(np.abs(ipa_dense(mod) - ref)) > 1e-3


# ----------------------------------------- squared distance as a dot product (MEET eq. 7-8)
def meet_phi(x, s):
    # phi_s(x) = s (+)_k [x_k^2, 1, -2 x_k]
    return s * np.concatenate([np.stack([xk ** 2, np.ones_like(xk), -2 * xk], -1)
                               for xk in np.moveaxis(x, -1, 0)], -1)


def meet_psi(x, s):
    # psi_s(x) = s (+)_k [1, x_k^2, x_k]
    return s * np.concatenate([np.stack([np.ones_like(xk), xk ** 2, xk], -1)
                               for xk in np.moveaxis(x, -1, 0)], -1)


def test_meet_identity_itself():
    rng = np.random.default_rng(0)
    xi, xj = rng.normal(size=(5, 3)) * 30, rng.normal(size=(7, 3)) * 30
    s = 0.37
    lhs = meet_phi(xi, s) @ meet_psi(xj, s).T
    rhs = s * s * ((xi[:, None, :] - xj[None, :, :]) ** 2).sum(-1)
    close(lhs, rhs, 1e-12)


def test_point_term_equals_augmented_dot_product():
    # Identity frames and zero translations: global points are the local ones.
    # Scalar and pair terms switched off; then
    #   logit_ij = -w_L * sum_p <phi_s(q_p), psi_s(k_p)>,  s^2 = gamma w_C / 2.
    inp = small(4)
    B, L, H = 2, 12, 3
    inp["rot"] = np.broadcast_to(np.eye(3), (B, L, 3, 3)).copy()
    inp["trans"] = np.zeros((B, L, 3))
    inp["q"] = np.zeros_like(inp["q"])
    inp["w_bias"] = np.zeros_like(inp["w_bias"])
    c = ipa_constants(4, 2)
    _, a = ipa_dense(inp, return_attn=True)
    qp = inp["q_pts"].astype(np.float64)
    kp = inp["k_pts"].astype(np.float64)
    for b in range(B):
        for h in range(H):
            s = math.sqrt(float(inp["gamma"][h]) * c["w_C"] / 2.0)
            aq = np.concatenate([meet_phi(qp[b, :, h, p], s) for p in range(2)], -1)
            ak = np.concatenate([meet_psi(kp[b, :, h, p], s) for p in range(2)], -1)
            lg = -c["w_L"] * (aq @ ak.T)
            e = np.exp(lg - lg.max(-1, keepdims=True))
            close(a[b, h], e / e.sum(-1, keepdims=True), 1e-12)


def test_point_term_prefers_near_keys():
    # The point term is a penalty: with everything else off, a key whose point
    # coincides with the query's point gets the largest weight.
    inp = small(5)
    inp["q"] = np.zeros_like(inp["q"])
    inp["w_bias"] = np.zeros_like(inp["w_bias"])
    inp["rot"] = np.broadcast_to(np.eye(3), inp["rot"].shape).copy()
    inp["trans"] = np.zeros_like(inp["trans"])
    kp = inp["k_pts"].copy()
    kp[:, 7] = inp["q_pts"][:, 2]
    inp["k_pts"] = kp
    _, a = ipa_dense(inp, return_attn=True)
    assert np.all(np.argmax(a[:, :, 2, :], axis=-1) == 7)


# ------------------------------------------------- factorised pair term (p.1)
def test_factorised_bias_and_pair_value_equal_dense():
    # scalar and point terms off: logits = w_L * b_ij, with the bias and the
    # pair value computed in factorised form (never forming z_ij).
    inp = small(6)
    inp["q"] = np.zeros_like(inp["q"])
    inp["gamma"] = np.zeros_like(inp["gamma"])
    out, a = ipa_dense(inp, return_attn=True)
    z1 = inp["z1"].astype(np.float64)
    z2 = inp["z2"].astype(np.float64)
    w = inp["w_bias"].astype(np.float64)
    c = ipa_constants(4, 2)
    for b in range(2):
        for h in range(3):
            qa = (z1[b] * w[None, None, :, h]).reshape(12, -1)     # [L, R*Cz]
            ka = z2[b].reshape(12, -1)
            lg = c["w_L"] * qa @ ka.T
            e = np.exp(lg - lg.max(-1, keepdims=True))
            ab = e / e.sum(-1, keepdims=True)
            close(a[b, h], ab, 1e-12)
            pz = ab @ ka                                           # [L, R*Cz]
            pair = (z1[b] * pz.reshape(12, 2, 5)).sum(1)           # sum_r z1 (a z2)
            close(out[b, :, h, -5:], pair, 1e-12)


def test_pair_value_brute_force_loops():
    # tiny case, pure-python triple loop over j, r, c for o_pair
    inp = small(7, L=5)
    out, a = ipa_dense(inp, return_attn=True)
    z1, z2 = inp["z1"].astype(float), inp["z2"].astype(float)
    for b in range(2):
        for i in range(5):
            for h in range(3):
                for c in range(5):
                    acc = 0.0
                    for j in range(5):
                        zij = 0.0
                        for r in range(2):
                            zij += z1[b, i, r, c] * z2[b, j, r, c]
                        acc += a[b, h, i, j] * zij
                    assert abs(out[b, i, h, -5 + c] - acc) < 1e-12


# ------------------------------------------------------------- closed forms
def test_single_residue_returns_own_values():
    # L = 1: the only key is the query itself, a = 1, so the point output is
    # R^T (R v + t - t) = v and the pair output is z_ii = sum_r z1 z2.
    inp = small(8, L=1)
    # exactly orthogonal float64 frames (float32-rounded ones are orthogonal
    # only to ~1e-7, which R^T R = I would expose)
    inp["rot"] = random_rotations(np.random.default_rng(8), 2).reshape(2, 1, 3, 3)
    out = ipa_dense(inp)
    H, C, Pv = 3, 4, 3
    v = inp["v"].astype(float)
    vp = inp["v_pts"].astype(float)
    close(out[..., :C], v, 1e-12)
    close(out[..., C:C + 3 * Pv], vp.reshape(2, 1, H, 3 * Pv), 1e-12)
    close(out[..., C + 3 * Pv:C + 4 * Pv], np.linalg.norm(vp, axis=-1), 1e-12)
    pair = (inp["z1"].astype(float) * inp["z2"].astype(float)).sum(2)   # [B, 1, Cz]
    close(out[..., -5:], np.broadcast_to(pair[:, :, None, :], (2, 1, H, 5)), 1e-12)


def test_one_dominant_key_maps_its_point_into_query_frame():
    # Two residues; the scalar term makes a_01 = 1 to double precision.  Then
    # o_pt(0) = R_0^T (R_1 v_pts(1) + t_1 - t_0).
    dims = IpaDims(B=1, L=2, H=1, C=1, Pq=1, Pv=2, R=1, Cz=1)
    inp = ipa_inputs(dims, 9)
    inp["gamma"] = np.zeros(1)
    inp["w_bias"] = np.zeros((1, 1))
    inp["q"] = np.array([[[[60.0]], [[0.0]]]])
    inp["k"] = np.array([[[[-60.0]], [[60.0]]]])
    out = ipa_dense(inp)
    R = inp["rot"][0].astype(float)
    t = inp["trans"][0].astype(float)
    vp = inp["v_pts"][0, 1, 0].astype(float)                       # [Pv, 3]
    expect = (R[0].T @ (R[1] @ vp.T + t[1][:, None] - t[0][:, None])).T
    close(out[0, 0, 0, 1:7], expect.reshape(-1), 1e-12)
    close(out[0, 0, 0, 0], inp["v"][0, 1, 0, 0], 1e-12)


def test_hand_worked_two_residue_case():
    # Hand-derived (w_L = 1, w_C = 2, scalar_scale = 1 so the logit is
    # q.k + b - gamma |dq - dk|^2), identity frames:
    #   q_0 = 0 (scalar term off), gamma = 1, w_bias = 1, z1_0 = 1,
    #   z2_0 = 0, z2_1 = 1 + ln 3, t_0 = 0, t_1 = (1, 0, 0), all points 0.
    #   logit_00 = 0 + 0 - 0 = 0;  logit_01 = 0 + (1 + ln 3) - 1 = ln 3
    #   => a_0 = (1/4, 3/4).
    #   v = (2, 6)            => o_0 = 2/4 + 18/4 = 5
    #   gv_0 = 0, gv_1 = t_1  => o_pt_0 = R_0^T (3/4, 0, 0); with R_0 a 90 deg
    #                            turn about z this is (0, -3/4, 0), norm 3/4
    #   z_00 = 0, z_01 = 1 + ln 3 => o_pair_0 = 3/4 (1 + ln 3)
    dims = IpaDims(B=1, L=2, H=1, C=1, Pq=1, Pv=1, R=1, Cz=1)
    inp = ipa_inputs(dims, 0)
    Rz = np.array([[0.0, -1.0, 0.0], [1.0, 0.0, 0.0], [0.0, 0.0, 1.0]])
    inp.update({
        "q": np.zeros((1, 2, 1, 1)), "k": np.ones((1, 2, 1, 1)),
        "v": np.array([2.0, 6.0]).reshape(1, 2, 1, 1),
        "q_pts": np.zeros((1, 2, 1, 1, 3)), "k_pts": np.zeros((1, 2, 1, 1, 3)),
        "v_pts": np.zeros((1, 2, 1, 1, 3)),
        "rot": np.stack([Rz, np.eye(3)])[None],
        "trans": np.array([[[0.0, 0, 0], [1.0, 0, 0]]]),
        "z1": np.ones((1, 2, 1, 1)),
        "z2": np.array([0.0, 1.0 + math.log(3.0)]).reshape(1, 2, 1, 1),
        "w_bias": np.ones((1, 1)), "gamma": np.ones(1),
        "mask": np.ones((1, 2), bool),
    })
    out, a = ipa_dense(inp, w_L=1.0, w_C=2.0, scalar_scale=1.0, return_attn=True)
    close(a[0, 0, 0], [0.25, 0.75], 1e-14)
    row = out[0, 0, 0]
    close(row[0], 5.0, 1e-14)
    close(row[1:4], [0.0, -0.75, 0.0], 1e-14)
    close(row[4], 0.75, 1e-14)
    close(row[5], 0.75 * (1.0 + math.log(3.0)), 1e-14)


def test_identity_frames_reduce_to_plain_point_distances():
    inp = small(10)
    inp["rot"] = np.broadcast_to(np.eye(3), inp["rot"].shape).copy()
    inp["trans"] = np.zeros_like(inp["trans"])
    inp["q"] = np.zeros_like(inp["q"])
    inp["w_bias"] = np.zeros_like(inp["w_bias"])
    c = ipa_constants(4, 2)
    _, a = ipa_dense(inp, return_attn=True)
    qp, kp = inp["q_pts"].astype(float), inp["k_pts"].astype(float)
    for h in range(3):
        d2 = ((qp[0, :, None, h] - kp[0, None, :, h]) ** 2).sum((-1, -2))
        lg = -c["w_L"] * float(inp["gamma"][h]) * c["w_C"] / 2 * d2
        e = np.exp(lg - lg.max(-1, keepdims=True))
        close(a[0, h], e / e.sum(-1, keepdims=True), 1e-12)


def test_scalar_only_matches_library_attention():
    # gamma = 0 and w_bias = 0: textbook softmax(w_L/sqrt(C) q k^T) v, checked
    # against torch.nn.functional.scaled_dot_product_attention in float64.
    torch = pytest.importorskip("torch")
    inp = small(11, masked_tail_frac=0.25)
    inp["gamma"] = np.zeros_like(inp["gamma"])
    inp["w_bias"] = np.zeros_like(inp["w_bias"])
    out = ipa_dense(inp)
    c = ipa_constants(4, 2)
    q = torch.tensor(inp["q"], dtype=torch.float64).permute(0, 2, 1, 3)
    k = torch.tensor(inp["k"], dtype=torch.float64).permute(0, 2, 1, 3)
    v = torch.tensor(inp["v"], dtype=torch.float64).permute(0, 2, 1, 3)
    m = torch.tensor(inp["mask"])
    am = (m[:, None, :, None] & m[:, None, None, :])
    ref = torch.nn.functional.scaled_dot_product_attention(
        q, k, v, attn_mask=am, scale=c["w_L"] * c["scalar_scale"])
    ref = ref.permute(0, 2, 1, 3).numpy()
    live = inp["mask"]
    close(out[live][..., :4], ref[live], 1e-12)


# ---------------------------------------------------------- blocked driver
def test_blocked_rows_equal_full():
    inp = small(12, L=40)
    close(ipa_dense_blocked(inp, block=16), ipa_dense(inp), 1e-13)
    rows = np.array([3, 17, 39])
    close(ipa_dense(inp, rows=rows), ipa_dense(inp)[:, rows], 1e-13)
