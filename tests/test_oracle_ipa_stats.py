"""Pins of the training-forward statistics oracle (log-sum-exp of the logits
and the pair-value aggregate U): brute-force loops, closed forms, and
agreement with the separately pinned forward oracle's attention weights and
pair output."""
import math

import numpy as np

from oracle import ipa_dense
from oracle.ipa_stats import ipa_forward_stats
from rna_structure_models_b200.synth import IpaDims, ipa_inputs


def small(seed=0, L=6, **kw):
    inp = ipa_inputs(IpaDims(B=2, L=L, H=3, C=4, Pq=2, Pv=3, R=2, Cz=3), seed, jitter=0.5)
    inp["mask"] = inp["mask"].copy()
    for k, v in kw.items():
        inp[k] = v
    return inp


def test_lse_reproduces_the_forward_attention():
    inp = small(1)
    inp["mask"][1, 2] = False
    lse, _ = ipa_forward_stats(inp)
    out, a = ipa_dense(inp, return_attn=True)
    # exp(l - lse) must be the attention of the forward oracle: recover l from
    # the attention of allowed pairs: log a = l - lse, so every allowed a_ij
    # sums to 1 along j and lse is the log of the partition sum
    allowed = inp["mask"][:, None, :, None] & inp["mask"][:, None, None, :]
    allowed = np.broadcast_to(allowed, a.shape)
    assert np.allclose(a.sum(-1)[np.any(allowed, -1)], 1.0)
    # brute force partition sums from Python loops over the logit definition
    q, k = inp["q"].astype(float), inp["k"].astype(float)
    rot, tr = inp["rot"].astype(float), inp["trans"].astype(float)
    qp, kp = inp["q_pts"].astype(float), inp["k_pts"].astype(float)
    z1, z2 = inp["z1"].astype(float), inp["z2"].astype(float)
    wb, gm = inp["w_bias"].astype(float), inp["gamma"].astype(float)
    B, L, H, C = q.shape
    Pq, R, Cz = qp.shape[3], z1.shape[2], z1.shape[3]
    w_L, w_C, ss = math.sqrt(1 / 3), math.sqrt(2 / (9 * Pq)), 1 / math.sqrt(C)
    for b in range(B):
        for h in range(H):
            for i in range(L):
                tot = 0.0
                for j in range(L):
                    if not (inp["mask"][b, i] and inp["mask"][b, j]):
                        continue
                    s = ss * sum(q[b, i, h, c] * k[b, j, h, c] for c in range(C))
                    bias = sum(wb[c, h] * sum(z1[b, i, r, c] * z2[b, j, r, c] for r in range(R)) for c in range(Cz))
                    d2 = 0.0
                    for p in range(Pq):
                        gi = rot[b, i] @ qp[b, i, h, p] + tr[b, i]
                        gj = rot[b, j] @ kp[b, j, h, p] + tr[b, j]
                        d2 += float(np.sum((gi - gj) ** 2))
                    tot += math.exp(w_L * (s + bias - gm[h] * w_C / 2 * d2))
                if inp["mask"][b, i]:
                    assert abs(lse[b, h, i] - math.log(tot)) < 1e-9 * max(1.0, abs(math.log(tot)))
                else:
                    assert lse[b, h, i] == np.inf


def test_pair_aggregate_contracts_to_the_pair_output():
    inp = small(2, L=9)
    inp["mask"][0, 5:] = False
    _, U = ipa_forward_stats(inp)
    out = ipa_dense(inp)
    C, Pv, Cz = 4, 3, 3
    o_pair = out[..., C + 4 * Pv:]
    z1 = inp["z1"].astype(float)
    folded = np.einsum("birc,bihrc->bihc", z1, U)
    assert np.allclose(folded, o_pair, atol=1e-12, rtol=1e-10)
    # and by loops: U_ihrc = sum_j a_ij z2_jrc
    _, a = ipa_dense(inp, return_attn=True)
    z2 = inp["z2"].astype(float)
    b, i, h, r, c = 0, 3, 1, 1, 2
    ref = sum(a[b, h, i, j] * z2[b, j, r, c] for j in range(9))
    assert abs(U[b, i, h, r, c] - ref) < 1e-12


def test_single_residue_and_dead_rows():
    inp = small(3, L=1)
    lse, U = ipa_forward_stats(inp)
    # one residue: the only logit is the self term, so lse = l_ii and U = z2_i
    assert np.allclose(U[:, 0, :, :, :], inp["z2"][:, 0, None, :, :].astype(float))
    inp2 = small(4, L=4)
    inp2["mask"][1, :] = False
    lse2, U2 = ipa_forward_stats(inp2)
    assert np.all(lse2[1] == np.inf) and np.all(U2[1] == 0)
    assert np.all(np.isfinite(lse2[0]))


def test_two_residue_closed_form():
    # identity frames, no points, no pair bias: l_ij = w_L s <q_i, k_j>, so
    # lse_i = log(exp(l_i0) + exp(l_i1)) by hand
    inp = small(5, L=2)
    inp["rot"] = np.broadcast_to(np.eye(3), inp["rot"].shape).astype(np.float32).copy()
    inp["gamma"] = np.zeros_like(inp["gamma"])
    inp["w_bias"] = np.zeros_like(inp["w_bias"])
    lse, U = ipa_forward_stats(inp)
    q, k = inp["q"].astype(float), inp["k"].astype(float)
    w = math.sqrt(1 / 3) / 2.0          # w_L / sqrt(C), C = 4
    for b in range(2):
        for h in range(3):
            for i in range(2):
                l0 = w * float(q[b, i, h] @ k[b, 0, h])
                l1 = w * float(q[b, i, h] @ k[b, 1, h])
                assert abs(lse[b, h, i] - math.log(math.exp(l0) + math.exp(l1))) < 1e-12
                a1 = math.exp(l1) / (math.exp(l0) + math.exp(l1))
                ref = (1 - a1) * inp["z2"][b, 0].astype(float) + a1 * inp["z2"][b, 1].astype(float)
                assert np.allclose(U[b, i, h], ref, atol=1e-12)
