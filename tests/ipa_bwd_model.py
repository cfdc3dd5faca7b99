"""A NumPy model of the decomposition planned for the IPA backward kernels.

Test-only (never imported by the product).  It computes the gradients of the
IPA core the way the two flash-style kernels will -- augmented fp16 rows with
per-64-residue tile origins, a query-side pass (row sums of dS, dQ rows) and
a key-side pass (column sums, dK and dV rows), then a per-residue mapping --
so that the algebra of that plan (origin corrections, the ln 2 scaling, D_i
from the forward output, d gamma from row / column sums, the pair block) can
be checked against the float64 gradient oracle before any kernel exists.

Contractions are float64 products of the fp16-rounded operands, standing in
for the tensor cores' fp32 accumulation.
"""
from __future__ import annotations

import math

import numpy as np

L2E = 1.0 / math.log(2.0)
LN2 = math.log(2.0)
TILE = 64


def f16(x):
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def hi_lo(x):
    h = f16(x)
    return h, f16(np.asarray(x, dtype=np.float64) - h)


def ipa_bwd_model(inp: dict, g_out, fwd_out, *, w_L, w_C, scalar_scale, stages: dict | None = None) -> dict:
    """Gradients of sum(g_out * core(inp)); fwd_out is the core's output.

    If `stages` is a dict, it receives, per (b, h), the intermediate arrays of
    each planned kernel stage (operand rows, log2 logits, log-sum-exp, pair
    aggregate, dS, the two passes' accumulators and row / column sums), so a
    kernel can be compared stage by stage."""
    q, k, v = (np.asarray(inp[n], np.float64) for n in ("q", "k", "v"))
    qp, kp, vp = (np.asarray(inp[n], np.float64) for n in ("q_pts", "k_pts", "v_pts"))
    rot, trans = np.asarray(inp["rot"], np.float64), np.asarray(inp["trans"], np.float64)
    z1, z2 = np.asarray(inp["z1"], np.float64), np.asarray(inp["z2"], np.float64)
    wb, gamma = np.asarray(inp["w_bias"], np.float64), np.asarray(inp["gamma"], np.float64)
    mask = np.asarray(inp["mask"], bool)
    B, L, H, C = q.shape
    Pq, Pv = qp.shape[3], vp.shape[3]
    R, Cz = z1.shape[2], z1.shape[3]
    ss = scalar_scale
    g = np.asarray(g_out, np.float64)
    o_fwd = np.asarray(fwd_out, np.float64)
    nt = (L + TILE - 1) // TILE
    tile_of = np.arange(L) // TILE

    grads = {n: np.zeros_like(np.asarray(inp[n], np.float64)) for n in
             ("q", "k", "v", "q_pts", "k_pts", "v_pts", "rot", "trans", "z1", "z2", "w_bias", "gamma")}
    for b in range(B):
        valid = mask[b]
        t = trans[b]
        cen = t[valid].mean(axis=0) if valid.any() else np.zeros(3)
        tc = t - cen
        origin = np.zeros((nt, 3))
        for T in range(nt):
            sel = valid[T * TILE:(T + 1) * TILE]
            if sel.any():
                origin[T] = tc[T * TILE:(T + 1) * TILE][sel].mean(axis=0)
        o_res = origin[tile_of]                                         # [L, 3] origin of each residue's tile
        gq = np.einsum("lxy,lhpy->lhpx", rot[b], qp[b]) + tc[:, None, None]   # centroid-relative
        gk = np.einsum("lxy,lhpy->lhpx", rot[b], kp[b]) + tc[:, None, None]
        gv = np.einsum("lxy,lhpy->lhpx", rot[b], vp[b]) + tc[:, None, None]
        gq_l = gq - o_res[:, None, None]                                # tile-local
        gk_l = gk - o_res[:, None, None]
        gv_l = gv - o_res[:, None, None]
        allowed = valid[:, None] & valid[None, :]
        live = allowed.any(axis=1)
        Z2 = f16(z2[b].reshape(L, R * Cz))
        d_rot = np.zeros((L, 3, 3))
        d_tr = np.zeros((L, 3))
        d_z1 = np.zeros((L, R * Cz))
        d_z2 = np.zeros((L, R * Cz))
        for h in range(H):
            c = L2E * w_L * gamma[h] * w_C / 2.0
            # -- operands of the query-side pass: points scaled by 2c on the query side
            Qs = f16(L2E * w_L * ss * q[b, :, h])
            QH, QL = hi_lo(2 * c * gq_l[:, h].reshape(L, -1))
            KH, KL = hi_lo(gk_l[:, h].reshape(L, -1))
            Qrow = np.concatenate([Qs, QH, QH, QL], axis=1)
            Krow = np.concatenate([f16(k[b, :, h]), KH, KL, KH], axis=1)
            QP = f16(L2E * w_L * (z1[b] * wb[:, h][None, None, :]).reshape(L, R * Cz))
            sq = gq_l[:, h].sum(axis=1)                                 # [L, 3] sum over points
            sk = gk_l[:, h].sum(axis=1)
            nq = np.einsum("lpx,lpx->l", gq_l[:, h], gq_l[:, h])
            nk = np.einsum("lpx,lpx->l", gk_l[:, h], gk_l[:, h])
            d = o_res[None, :, :] - o_res[:, None, :]                   # o_J - o_I  [i, j, 3]
            # log2 logit = MMA + row term (per i, J) + column term (per j, I)
            x = (Qrow @ Krow.T + QP @ Z2.T
                 - c * nq[:, None] - c * Pq * np.einsum("ijx,ijx->ij", d, d) + 2 * c * np.einsum("ijx,ix->ij", d, sq)
                 - c * nk[None, :] - 2 * c * np.einsum("ijx,jx->ij", d, sk))
            x = np.where(allowed, x, -np.inf)
            # the forward's natural log-sum-exp and pair aggregate (training-mode outputs)
            lse2 = np.full(L, np.inf)
            mrow = np.where(live, x.max(axis=1), 0.0)
            e = np.where(allowed, np.exp2(x - mrow[:, None]), 0.0)
            lse2[live] = mrow[live] + np.log2(e[live].sum(axis=1))
            a = np.where(allowed, np.exp2(x - lse2[:, None]), 0.0)
            U = a @ z2[b].reshape(L, R * Cz)
            # -- upstream gradient rows (epilogue adjoint), from the forward output
            gh = np.where(live[:, None], g[b, :, h], 0.0)
            g_o, g_pt = gh[:, :C], gh[:, C:C + 3 * Pv].reshape(L, Pv, 3)
            g_n, g_pair = gh[:, C + 3 * Pv:C + 4 * Pv], gh[:, C + 4 * Pv:]
            o_pt = o_fwd[b, :, h, C:C + 3 * Pv].reshape(L, Pv, 3)
            nrm = np.linalg.norm(o_pt, axis=2)
            unit = np.where((nrm > 0)[..., None], o_pt / np.where(nrm > 0, nrm, 1.0)[..., None], 0.0)
            d_opt = g_pt + g_n[..., None] * unit
            dog = f16(np.einsum("lxy,lpy->lpx", rot[b], d_opt))        # global-frame, rounded once
            dU = f16(z1[b].reshape(L, R, Cz) * g_pair[:, None, :]).reshape(L, R * Cz)
            dO = np.concatenate([f16(g_o), dog.reshape(L, -1), dog.reshape(L, -1)], axis=1)
            VH, VL = hi_lo(gv_l[:, h].reshape(L, -1))
            Va = np.concatenate([f16(v[b, :, h]), VH, VL], axis=1)
            DG = dog.sum(axis=1)                                        # [L, 3]
            dP = dO @ Va.T + dU @ Z2.T + DG @ o_res.T                   # value points relative to their tile
            # D_i from the forward output (same rounded dO, dU)
            og_rel = np.einsum("lxy,lpy->lpx", rot[b], o_pt) + tc[:, None] + 0.0   # og - cen
            D = (dO[:, :C] * o_fwd[b, :, h, :C]).sum(1) + np.einsum("lpx,lpx->l", dog, og_rel) + (dU * U).sum(1)
            dS = np.where(allowed, LN2 * a * (dP - D[:, None]), 0.0)     # dL / d(log2 logit)
            # -- query-side pass
            dQrow = dS @ Krow
            dQP = dS @ Z2
            rs = dS.sum(axis=1)
            RSo = dS @ o_res                                            # sum_J o_J (row sum over tile J)
            # -- key-side pass: points scaled by 2c on the key side
            QH2, QL2 = hi_lo(gq_l[:, h].reshape(L, -1))                 # unscaled query points
            Qrow2 = np.concatenate([Qs, QH2, QH2, QL2], axis=1)
            dKrow = dS.T @ Qrow2
            dZ2 = dS.T @ QP + a.T @ dU
            dVa = a.T @ dO
            cs = dS.sum(axis=0)
            CSo = dS.T @ o_res
            if stages is not None:
                stages[(b, h)] = {
                    "Qrow": Qrow, "Krow": Krow, "QP": QP, "Z2": Z2, "Qrow_keyside": Qrow2, "Va": Va, "dO": dO,
                    "dU": dU, "origin": o_res, "x": x, "lse": lse2 * LN2, "U": U, "D": D, "dS": dS,
                    "dQrow": dQrow, "dQP": dQP, "rs": rs, "RSo": RSo, "dKrow": dKrow, "dZ2": dZ2, "dVa": dVa,
                    "cs": cs, "CSo": CSo}
            # -- mapping back
            grads["q"][b, :, h] = L2E * w_L * ss * dQrow[:, :C]
            grads["k"][b, :, h] = dKrow[:, :C]
            grads["v"][b, :, h] = dVa[:, :C]
            n3q, n3v = 3 * Pq, 3 * Pv
            Gq = (dQrow[:, C:C + n3q] + dQrow[:, C + n3q:C + 2 * n3q]).reshape(L, Pq, 3) + RSo[:, None, :]
            gq_c = gq_l[:, h] + o_res[:, None]
            dgq = 2 * c * (Gq - rs[:, None, None] * gq_c)               # dx/dgq_i = -2c (gq_i - gk_j)
            Gk = (dKrow[:, C:C + n3q] + dKrow[:, C + 2 * n3q:C + 3 * n3q]).reshape(L, Pq, 3) + CSo[:, None, :]
            gk_c = gk_l[:, h] + o_res[:, None]
            dgk = 2 * c * (Gk - cs[:, None, None] * gk_c)
            dgv = dVa[:, C:C + n3v].reshape(L, Pv, 3)
            # d gamma: x holds -c |gq - gk|^2 with c proportional to gamma
            d2sum = (np.sum(rs * np.einsum("lpx,lpx->l", gq_c, gq_c)) - 2 * np.sum(gq_c * Gq)
                     + np.sum(cs * np.einsum("lpx,lpx->l", gk_c, gk_c)))
            grads["gamma"][h] += -(L2E * w_L * w_C / 2.0) * d2sum
            for dg_, pts in ((dgq, qp[b, :, h]), (dgk, kp[b, :, h]), (dgv, vp[b, :, h])):
                d_rot += np.einsum("lpx,lpy->lxy", dg_, pts)
                d_tr += dg_.sum(axis=1)
            grads["q_pts"][b, :, h] = np.einsum("lxy,lpx->lpy", rot[b], dgq)
            grads["k_pts"][b, :, h] = np.einsum("lxy,lpx->lpy", rot[b], dgk)
            grads["v_pts"][b, :, h] = np.einsum("lxy,lpx->lpy", rot[b], dgv)
            # o_pt = R^T (og - t): d rot += (og - t) d_opt^T, dt -= R d_opt
            og_minus_t = np.einsum("lxy,lpy->lpx", rot[b], o_pt)
            d_rot += np.einsum("lpx,lpy->lxy", og_minus_t, d_opt)
            d_tr -= np.einsum("lxy,lpy->lx", rot[b], d_opt)
            # pair block
            wbs = np.tile(wb[:, h], R)                                  # column r*Cz + c -> w_bias[c, h]
            d_z1 += L2E * w_L * wbs[None, :] * dQP + (U.reshape(L, R, Cz) * g_pair[:, None, :]).reshape(L, -1)
            d_z2 += dZ2
            grads["w_bias"][:, h] += L2E * w_L * (z1[b].reshape(L, R * Cz) * dQP).reshape(L, R, Cz).sum(axis=(0, 1))
        grads["rot"][b] = d_rot
        grads["trans"][b] = d_tr
        grads["z1"][b] = d_z1.reshape(L, R, Cz)
        grads["z2"][b] = d_z2.reshape(L, R, Cz)
    return grads
