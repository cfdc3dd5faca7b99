"""Gradients of the Invariant Point Attention core: a plain float64 CPU
oracle.

TEST INFRASTRUCTURE ONLY: imported by tests/, never by the product path.
Shares no code with the CUDA library.

Flash Invariant Point Attention is used to train structure models (TL;DR:
drop-in replacement for IPA in training), so the core must also be
differentiated.  Given an upstream gradient g_out of the core's output
[B, L, H, C | 3 Pv | Pv | Cz] (the layout of `ipa_dense`), this module runs
the forward steps of `ipa_dense` again and then their adjoints in reverse
order, one step at a time:

  7'. rows without an allowed key pass nothing on.
  6'. n = |o_pt|: d o_pt += g_n o_pt / |o_pt| (the zero vector when
      o_pt = 0, the same convention the variant page fixes for a distance);
      o_pt = R_i^T (og - t_i): d og = R_i d o_pt, dR_i += (og - t_i) d o_pt^T,
      dt_i -= d og;
      o = sum_j a v_j, og = sum_j a gv_j, o_pair_c = sum_j a z_ijc:
      da_ij = <g_o, v_j> + <d og, gv_j> + sum_c g_pair_c z_ijc,
      dv_j = sum_i a g_o_i, d gv_j = sum_i a d og_i, dz_ijc = a g_pair_ic.
  5'. softmax: dl_ij = a_ij (da_ij - sum_k a_ik da_ik).
  4'. l = w_L (s <q, k> + b_ij - gamma w_C / 2 sum_p |gq_p - gk_p|^2):
      dq = w_L s sum_j dl k_j, dk = w_L s sum_i dl q_i,
      d gq_p = -w_L gamma w_C sum_j dl (gq_p - gk_p), d gk_p = the opposite
      sum over i, d gamma = -w_L w_C / 2 sum dl |gq - gk|^2.
  3'. b_ij = sum_c w_bias[c, h] z_ijc: d w_bias = w_L sum dl z,
      dz_ijc += w_L sum_h dl^h w_bias[c, h].
  2'. z_ijc = sum_r z1_irc z2_jrc: dz1 = sum_j dz z2_j, dz2 = sum_i dz z1_i.
  1'. gq = R q_pts + t etc.: d q_pts = R^T d gq, dR += d gq q_pts^T,
      dt += d gq (and the same for the key and value points).
The mask has no gradient.  Everything is materialised (small sizes only).
"""
from __future__ import annotations

import numpy as np

from .ipa_dense import ipa_constants

__all__ = ["ipa_grad", "ipa_grad_gamma_scale"]


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def ipa_grad(inp: dict, g_out, *, w_L=None, w_C=None, scalar_scale=None) -> dict:
    """Gradients of sum(g_out * ipa_dense(inp)) with respect to q, k, v,
    q_pts, k_pts, v_pts, rot, trans, z1, z2, w_bias and gamma (float64)."""
    q, k, v = _f64(inp["q"]), _f64(inp["k"]), _f64(inp["v"])
    q_pts, k_pts, v_pts = _f64(inp["q_pts"]), _f64(inp["k_pts"]), _f64(inp["v_pts"])
    rot, trans = _f64(inp["rot"]), _f64(inp["trans"])
    z1, z2 = _f64(inp["z1"]), _f64(inp["z2"])
    w_bias, gamma = _f64(inp["w_bias"]), _f64(inp["gamma"])
    mask = np.asarray(inp["mask"], dtype=bool)
    B, L, H, C = q.shape
    Pq, Pv = q_pts.shape[3], v_pts.shape[3]
    Cz = z1.shape[3]
    consts = ipa_constants(C, Pq)
    w_L = consts["w_L"] if w_L is None else w_L
    w_C = consts["w_C"] if w_C is None else w_C
    ss = consts["scalar_scale"] if scalar_scale is None else scalar_scale
    g = _f64(g_out)
    g_o = g[..., :C]
    g_pt = g[..., C:C + 3 * Pv].reshape(B, L, H, Pv, 3)
    g_n = g[..., C + 3 * Pv:C + 4 * Pv]
    g_pair = g[..., C + 4 * Pv:]

    # forward (as ipa_dense), keeping the intermediates
    gq = np.einsum("blxy,blhpy->blhpx", rot, q_pts) + trans[:, :, None, None, :]
    gk = np.einsum("blxy,blhpy->blhpx", rot, k_pts) + trans[:, :, None, None, :]
    gv = np.einsum("blxy,blhpy->blhpx", rot, v_pts) + trans[:, :, None, None, :]
    z = np.einsum("birc,bjrc->bijc", z1, z2)
    bias = np.einsum("bijc,ch->bhij", z, w_bias)
    diff = gq[:, :, None] - gk[:, None, :]                           # [B, i, j, H, Pq, 3]
    d2 = np.einsum("bijhpx,bijhpx->bhij", diff, diff)
    logits = w_L * (ss * np.einsum("bihc,bjhc->bhij", q, k) + bias
                    - (gamma * w_C / 2.0)[None, :, None, None] * d2)
    allowed = mask[:, :, None] & mask[:, None, :]
    allowed_h = np.broadcast_to(allowed[:, None], logits.shape)
    neg = np.where(allowed_h, logits, -np.inf)
    mx = neg.max(axis=-1, keepdims=True)
    mx = np.where(np.isfinite(mx), mx, 0.0)
    e = np.where(allowed_h, np.exp(neg - mx), 0.0)
    s = e.sum(axis=-1, keepdims=True)
    a = np.where(s > 0, e / np.where(s > 0, s, 1.0), 0.0)
    og = np.einsum("bhij,bjhpx->bihpx", a, gv)
    rel = og - trans[:, :, None, None, :]
    o_pt = np.einsum("bixy,bihpx->bihpy", rot, rel)
    nrm = np.sqrt(np.einsum("bihpx,bihpx->bihp", o_pt, o_pt))

    # 7'. dead rows pass nothing on
    live = allowed.any(axis=-1)[:, :, None, None]
    g_o, g_n, g_pair = (np.where(live, x, 0.0) for x in (g_o, g_n, g_pair))
    g_pt = np.where(live[..., None], g_pt, 0.0)

    # 6'. outputs
    unit = np.where((nrm > 0)[..., None], o_pt / np.where(nrm > 0, nrm, 1.0)[..., None], 0.0)
    d_opt = g_pt + g_n[..., None] * unit
    d_og = np.einsum("bixy,bihpy->bihpx", rot, d_opt)
    d_rot = np.einsum("bihpx,bihpy->bixy", rel, d_opt)
    d_trans = -d_og.sum(axis=(2, 3))
    da = (np.einsum("bihc,bjhc->bhij", g_o, v) + np.einsum("bihpx,bjhpx->bhij", d_og, gv)
          + np.einsum("bihc,bijc->bhij", g_pair, z))
    d_v = np.einsum("bhij,bihc->bjhc", a, g_o)
    d_gv = np.einsum("bhij,bihpx->bjhpx", a, d_og)
    d_z = np.einsum("bhij,bihc->bijc", a, g_pair)

    # 5'. softmax
    dl = a * (da - np.sum(a * da, axis=-1, keepdims=True))

    # 4'. logit terms
    d_q = w_L * ss * np.einsum("bhij,bjhc->bihc", dl, k)
    d_k = w_L * ss * np.einsum("bhij,bihc->bjhc", dl, q)
    coef = w_L * gamma * w_C                                          # [H]
    d_gq = -coef[None, None, :, None, None] * np.einsum("bhij,bijhpx->bihpx", dl, diff)
    d_gk = coef[None, None, :, None, None] * np.einsum("bhij,bijhpx->bjhpx", dl, diff)
    d_gamma = -w_L * w_C / 2.0 * np.einsum("bhij,bhij->h", dl, d2)

    # 3'. pair bias
    d_wb = w_L * np.einsum("bhij,bijc->ch", dl, z)
    d_z += w_L * np.einsum("bhij,ch->bijc", dl, w_bias)

    # 2'. factorised pair tensor
    d_z1 = np.einsum("bijc,bjrc->birc", d_z, z2)
    d_z2 = np.einsum("bijc,birc->bjrc", d_z, z1)

    # 1'. frames
    def back(d_glob, pts):
        d_loc = np.einsum("blxy,blhpx->blhpy", rot, d_glob)
        d_r = np.einsum("blhpx,blhpy->blxy", d_glob, pts)
        return d_loc, d_r, d_glob.sum(axis=(2, 3))

    d_qp, r1, t1 = back(d_gq, q_pts)
    d_kp, r2, t2 = back(d_gk, k_pts)
    d_vp, r3, t3 = back(d_gv, v_pts)
    d_rot = d_rot + r1 + r2 + r3
    d_trans = d_trans + t1 + t2 + t3
    return {"q": d_q, "k": d_k, "v": d_v, "q_pts": d_qp, "k_pts": d_kp, "v_pts": d_vp, "rot": d_rot,
            "trans": d_trans, "z1": d_z1, "z2": d_z2, "w_bias": d_wb, "gamma": d_gamma}


def ipa_grad_gamma_scale(inp: dict, g_out, *, w_L=None, w_C=None, scalar_scale=None) -> np.ndarray:
    """Per head, the root-sum-square of the magnitudes of the terms that
    d gamma sums (a tolerance scale, not a gradient).

    Steps 5' and 4' above give d gamma_h = -w_L w_C / 2 sum_{b,i,j} dl d2 with
    dl_ij = a_ij (da_ij - D_i), D_i = sum_k a_ik da_ik.  Each term is at most
    t_ij = w_L w_C / 2 a_ij (|da_ij| + |D_i|) d2_ij in magnitude, and a d gamma
    formed from rounded operands carries errors of about (unit roundoff) x t_ij
    per term; errors without a common sign add in quadrature, so their sum is
    of the size sqrt(sum t_ij^2), returned here [H].  The signed sum itself
    cancels: |d gamma_h| is typically 10^-3 .. 10^-1 of this scale at a few
    hundred residues.

    da is taken with the value points relative to the mean translation of the
    batch element's live residues: that shifts each row of da by a constant,
    which dl does not see, and makes the scale independent of where the
    structure sits (under a global rigid motion it is unchanged).

    One (b, h) slice at a time, [L, L] arrays only (the forward of ipa_dense:
    logits, masked softmax, outputs; then da and D as in ipa_grad)."""
    q, k, v = _f64(inp["q"]), _f64(inp["k"]), _f64(inp["v"])
    q_pts, k_pts, v_pts = _f64(inp["q_pts"]), _f64(inp["k_pts"]), _f64(inp["v_pts"])
    rot, trans = _f64(inp["rot"]), _f64(inp["trans"])
    z1, z2 = _f64(inp["z1"]), _f64(inp["z2"])
    w_bias, gamma = _f64(inp["w_bias"]), _f64(inp["gamma"])
    mask = np.asarray(inp["mask"], dtype=bool)
    B, L, H, C = q.shape
    Pq, Pv = q_pts.shape[3], v_pts.shape[3]
    R, Cz = z1.shape[2], z1.shape[3]
    consts = ipa_constants(C, Pq)
    w_L = consts["w_L"] if w_L is None else w_L
    w_C = consts["w_C"] if w_C is None else w_C
    ss = consts["scalar_scale"] if scalar_scale is None else scalar_scale
    g = _f64(g_out)
    sq = np.zeros(H)
    for b in range(B):
        allowed = mask[b][:, None] & mask[b][None, :]
        live = allowed.any(axis=1)
        gq = np.einsum("lxy,lhpy->lhpx", rot[b], q_pts[b]) + trans[b][:, None, None, :]
        gk = np.einsum("lxy,lhpy->lhpx", rot[b], k_pts[b]) + trans[b][:, None, None, :]
        gv = np.einsum("lxy,lhpy->lhpx", rot[b], v_pts[b]) + trans[b][:, None, None, :]
        cen = trans[b][mask[b]].mean(axis=0) if mask[b].any() else np.zeros(3)
        for h in range(H):
            d2 = np.zeros((L, L))
            for p in range(Pq):
                dd = gq[:, None, h, p, :] - gk[None, :, h, p, :]
                d2 += np.einsum("ijx,ijx->ij", dd, dd)
            wz1 = (z1[b] * w_bias[:, h][None, None, :]).reshape(L, R * Cz)
            bias = wz1 @ z2[b].reshape(L, R * Cz).T                   # sum_c w_bias[c, h] z_ijc
            logits = w_L * (ss * q[b, :, h] @ k[b, :, h].T + bias - gamma[h] * w_C / 2.0 * d2)
            neg = np.where(allowed, logits, -np.inf)
            mx = np.where(live, neg.max(axis=1), 0.0)
            e = np.where(allowed, np.exp(neg - mx[:, None]), 0.0)
            ssum = e.sum(axis=1)
            a = np.where(ssum[:, None] > 0, e / np.where(ssum > 0, ssum, 1.0)[:, None], 0.0)
            gh = np.where(live[:, None], g[b, :, h], 0.0)
            g_o = gh[:, :C]
            g_pt = gh[:, C:C + 3 * Pv].reshape(L, Pv, 3)
            g_n = gh[:, C + 3 * Pv:C + 4 * Pv]
            g_pair = gh[:, C + 4 * Pv:]
            og = np.einsum("ij,jpx->ipx", a, gv[:, h])
            o_pt = np.einsum("ixy,ipx->ipy", rot[b], og - trans[b][:, None, :])
            nrm = np.sqrt(np.einsum("ipx,ipx->ip", o_pt, o_pt))
            unit = np.where((nrm > 0)[..., None], o_pt / np.where(nrm > 0, nrm, 1.0)[..., None], 0.0)
            d_og = np.einsum("ixy,ipy->ipx", rot[b], g_pt + g_n[..., None] * unit)
            gz1 = (z1[b] * g_pair[:, None, :]).reshape(L, R * Cz)
            gv_c = gv[:, h] - cen[None, None, :]
            da = (g_o @ v[b, :, h].T + d_og.reshape(L, -1) @ gv_c.reshape(L, -1).T
                  + gz1 @ z2[b].reshape(L, R * Cz).T)
            D = np.sum(a * da, axis=1)
            t = w_L * w_C / 2.0 * a * (np.abs(da) + np.abs(D)[:, None]) * d2
            sq[h] += float(np.sum(t * t))
    return np.sqrt(sq)
