"""Pins of the MEET distance-aware attention oracle (MEET §2.2, eq. (6)-(8))
against things other than itself: the augmented query/key identity of
eq. (7)-(8), torch's scaled_dot_product_attention with an explicit distance
bias, rigid-motion invariance, pure-Python loops, and closed-form limits."""
import math

import numpy as np
import pytest
import torch

from oracle import meet_dense, meet_logits
from rna_structure_models_b200.synth import MeetDims, meet_inputs, random_rotations


def small(seed=0, **kw):
    return meet_inputs(MeetDims(B=2, L=24, H=3, C=8), seed, **kw)


def test_logits_equal_augmented_dot_product_of_eq_7_8():
    # phi(x_i) = s (+)_k [x_k^2, 1, -2 x_k], psi(x_j) = s (+)_k [1, x_k^2, x_k];
    # A = rho <[q, -phi], [k, psi]>
    inp = small(1)
    q, k, x = (inp[n].astype(np.float64) for n in ("q", "k", "x"))
    rho, s = inp["rho"].astype(np.float64), inp["s"].astype(np.float64)
    B, L, H, C = q.shape
    A = meet_logits(inp)
    for h in range(H):
        phi = np.concatenate([np.stack([x[..., kk] ** 2, np.ones_like(x[..., kk]), -2 * x[..., kk]], -1)
                              for kk in range(3)], -1) * s[h]
        psi = np.concatenate([np.stack([np.ones_like(x[..., kk]), x[..., kk] ** 2, x[..., kk]], -1)
                              for kk in range(3)], -1) * s[h]
        Q = np.concatenate([q[:, :, h], -phi], -1)
        K = np.concatenate([k[:, :, h], psi], -1)
        ref = rho[h] * np.einsum("bid,bjd->bij", Q, K)
        assert np.allclose(A[:, h], ref, rtol=1e-10, atol=1e-8)


def test_matches_sdpa_with_explicit_distance_bias():
    inp = small(2, masked_tail_frac=0.25)
    q, k, v, x = (torch.from_numpy(inp[n]).double() for n in ("q", "k", "v", "x"))
    rho, s = torch.from_numpy(inp["rho"]).double(), torch.from_numpy(inp["s"]).double()
    mask = torch.from_numpy(inp["mask"])
    d2 = torch.cdist(x, x) ** 2                                           # [B, L, L]
    bias = -(rho * s ** 2)[None, :, None, None] * d2[:, None]             # [B, H, L, L]
    allowed = mask[:, None, :, None] & mask[:, None, None, :]
    bias = bias.masked_fill(~allowed, float("-inf"))
    qh = (q * rho[None, None, :, None]).permute(0, 2, 1, 3)
    o = torch.nn.functional.scaled_dot_product_attention(qh, k.permute(0, 2, 1, 3), v.permute(0, 2, 1, 3),
                                                         attn_mask=bias, scale=1.0).permute(0, 2, 1, 3)
    ref = meet_dense(inp)
    valid = inp["mask"]
    assert np.allclose(o.numpy()[valid], ref[valid], atol=1e-12)
    assert np.all(ref[~valid] == 0.0)


def test_invariant_under_rigid_motion_of_coordinates():
    inp = small(3)
    base = meet_dense(inp)
    rng = np.random.default_rng(7)
    G = random_rotations(rng, 1)[0]
    moved = dict(inp)
    moved["x"] = inp["x"].astype(np.float64) @ G.T + rng.normal(size=3) * 50.0
    assert np.allclose(meet_dense(moved), base, atol=1e-10)
    # control: moving one coordinate does change the output
    other = dict(inp)
    other["x"] = inp["x"].astype(np.float64).copy()
    other["x"][0, 5] += 3.0
    assert not np.allclose(meet_dense(other), base, atol=1e-6)


def test_pure_python_loops_tiny_case():
    inp = meet_inputs(MeetDims(B=1, L=5, H=2, C=3), 4, masked_tail_frac=0.2)
    q, k, v, x = (inp[n].astype(np.float64) for n in ("q", "k", "v", "x"))
    rho, s, mask = inp["rho"], inp["s"], inp["mask"]
    B, L, H, C = q.shape
    ref = meet_dense(inp)
    for i in range(L):
        for h in range(H):
            logits = []
            for j in range(L):
                if mask[0, i] and mask[0, j]:
                    dot = sum(q[0, i, h, c] * k[0, j, h, c] for c in range(C))
                    dist2 = sum((x[0, i, d] - x[0, j, d]) ** 2 for d in range(3))
                    logits.append((j, float(rho[h]) * (dot - float(s[h]) ** 2 * dist2)))
            want = [0.0] * C
            if logits:
                mx = max(a for _, a in logits)
                w = [(j, math.exp(a - mx)) for j, a in logits]
                tot = sum(e for _, e in w)
                for j, e in w:
                    for c in range(C):
                        want[c] += e / tot * v[0, j, h, c]
            assert np.allclose(ref[0, i, h], want, atol=1e-12)


def test_zero_distance_scale_is_plain_attention_and_rows_are_convex_combinations():
    inp = small(5)
    inp["s"] = np.zeros_like(inp["s"])
    o, a = meet_dense(inp, return_attn=True)
    q, k, v = (inp[n].astype(np.float64) for n in ("q", "k", "v"))
    logits = np.einsum("bihc,bjhc->bhij", q, k) * inp["rho"].astype(np.float64)[None, :, None, None]
    w = np.exp(logits - logits.max(-1, keepdims=True))
    w /= w.sum(-1, keepdims=True)
    assert np.allclose(a, w, atol=1e-12)
    assert np.allclose(a.sum(-1), 1.0)


def test_large_distance_scale_attends_to_itself():
    # with s large, ||x_i - x_j||^2 >= 3.8^2 * (something) for j != i dominates:
    # the only surviving key is i itself (distance 0)
    inp = small(6)
    inp["s"] = np.full_like(inp["s"], 20.0)
    o = meet_dense(inp)
    assert np.allclose(o, inp["v"].astype(np.float64), atol=1e-9)


def test_masks_all_masked_and_single_valid_key():
    inp = small(8)
    inp["mask"][0, :] = False
    inp["mask"][1, :] = False
    inp["mask"][1, 7] = True
    o = meet_dense(inp)
    assert np.all(o[0] == 0.0)
    assert np.allclose(o[1, 7], inp["v"][1, 7].astype(np.float64))
    assert np.all(o[1, :7] == 0.0) and np.all(o[1, 8:] == 0.0)


@pytest.mark.parametrize("rows", [[0], [3, 17, 23]])
def test_row_subsets_match_full(rows):
    inp = small(9, masked_tail_frac=0.1)
    assert np.allclose(meet_dense(inp, rows=rows), meet_dense(inp)[:, rows], atol=1e-14)
