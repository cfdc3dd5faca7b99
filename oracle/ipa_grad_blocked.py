"""Gradients of the IPA core over blocks of query rows: the float64 oracle of
`ipa_grad` with bounded memory, for long sequences.

TEST INFRASTRUCTURE ONLY: imported by tests/, never by the product path.
Shares no code with the CUDA library.

Every step of the gradient in `ipa_grad` is either a per-query-row quantity
(softmax, the attention derivative, the query and output gradients) or a sum
over query rows (the key, value and pair-factor gradients, w_bias, gamma).
So the gradient is the sum, over blocks of query rows, of the contributions
of each block, where a block materialises only its [rows, L] slice of the
pair tensor and the logits.  The steps below are those of `ipa_grad`,
restricted to the rows of a block.
"""
from __future__ import annotations

import numpy as np

from .ipa_dense import ipa_constants

__all__ = ["ipa_grad_blocked"]


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def ipa_grad_blocked(inp: dict, g_out, *, block: int = 64, rows=None, w_L=None, w_C=None,
                     scalar_scale=None) -> dict:
    """Gradients of sum(g_out * ipa_dense(inp)) (same keys as ipa_grad).

    With `rows` given, only those query rows' contributions are summed: the
    query-side gradients (q, q_pts) at those rows are then exact, since they
    depend on their own row alone; every other entry is a partial sum."""
    q, k, v = _f64(inp["q"]), _f64(inp["k"]), _f64(inp["v"])
    q_pts, k_pts, v_pts = _f64(inp["q_pts"]), _f64(inp["k_pts"]), _f64(inp["v_pts"])
    rot, trans = _f64(inp["rot"]), _f64(inp["trans"])
    z1, z2 = _f64(inp["z1"]), _f64(inp["z2"])
    w_bias, gamma = _f64(inp["w_bias"]), _f64(inp["gamma"])
    mask = np.asarray(inp["mask"], dtype=bool)
    B, L, H, C = q.shape
    Pq, Pv = q_pts.shape[3], v_pts.shape[3]
    consts = ipa_constants(C, Pq)
    w_L = consts["w_L"] if w_L is None else w_L
    w_C = consts["w_C"] if w_C is None else w_C
    ss = consts["scalar_scale"] if scalar_scale is None else scalar_scale
    g = _f64(g_out)

    gq_all = np.einsum("blxy,blhpy->blhpx", rot, q_pts) + trans[:, :, None, None, :]
    gk = np.einsum("blxy,blhpy->blhpx", rot, k_pts) + trans[:, :, None, None, :]
    gv = np.einsum("blxy,blhpy->blhpx", rot, v_pts) + trans[:, :, None, None, :]

    d_q = np.zeros_like(q)
    d_k = np.zeros_like(k)
    d_v = np.zeros_like(v)
    d_gq = np.zeros_like(gq_all)
    d_gk = np.zeros_like(gk)
    d_gv = np.zeros_like(gv)
    d_rot = np.zeros_like(rot)
    d_trans = np.zeros_like(trans)
    d_z1 = np.zeros_like(z1)
    d_z2 = np.zeros_like(z2)
    d_wb = np.zeros_like(w_bias)
    d_gamma = np.zeros_like(gamma)
    coef = w_L * gamma * w_C

    all_rows = np.arange(L) if rows is None else np.asarray(rows)
    for s0 in range(0, len(all_rows), block):
        rows = all_rows[s0:s0 + block]
        gq = gq_all[:, rows]
        zr = np.einsum("birc,bjrc->bijc", z1[:, rows], z2)
        bias = np.einsum("bijc,ch->bhij", zr, w_bias)
        diff = gq[:, :, None] - gk[:, None, :]
        d2 = np.einsum("bijhpx,bijhpx->bhij", diff, diff)
        logits = w_L * (ss * np.einsum("bihc,bjhc->bhij", q[:, rows], k) + bias
                        - (gamma * w_C / 2.0)[None, :, None, None] * d2)
        allowed = mask[:, rows, None] & mask[:, None, :]
        allowed_h = np.broadcast_to(allowed[:, None], logits.shape)
        neg = np.where(allowed_h, logits, -np.inf)
        mx = neg.max(axis=-1, keepdims=True)
        mx = np.where(np.isfinite(mx), mx, 0.0)
        e = np.where(allowed_h, np.exp(neg - mx), 0.0)
        sm = e.sum(axis=-1, keepdims=True)
        a = np.where(sm > 0, e / np.where(sm > 0, sm, 1.0), 0.0)
        og = np.einsum("bhij,bjhpx->bihpx", a, gv)
        rel = og - trans[:, rows, None, None, :]
        o_pt = np.einsum("bixy,bihpx->bihpy", rot[:, rows], rel)
        nrm = np.sqrt(np.einsum("bihpx,bihpx->bihp", o_pt, o_pt))

        gr = g[:, rows]
        live = allowed.any(axis=-1)[:, :, None, None]
        g_o = np.where(live, gr[..., :C], 0.0)
        g_pt = np.where(live[..., None], gr[..., C:C + 3 * Pv].reshape(B, len(rows), H, Pv, 3), 0.0)
        g_n = np.where(live, gr[..., C + 3 * Pv:C + 4 * Pv], 0.0)
        g_pair = np.where(live, gr[..., C + 4 * Pv:], 0.0)

        unit = np.where((nrm > 0)[..., None], o_pt / np.where(nrm > 0, nrm, 1.0)[..., None], 0.0)
        d_opt = g_pt + g_n[..., None] * unit
        d_og = np.einsum("bixy,bihpy->bihpx", rot[:, rows], d_opt)
        d_rot[:, rows] += np.einsum("bihpx,bihpy->bixy", rel, d_opt)
        d_trans[:, rows] -= d_og.sum(axis=(2, 3))
        da = (np.einsum("bihc,bjhc->bhij", g_o, v) + np.einsum("bihpx,bjhpx->bhij", d_og, gv)
              + np.einsum("bihc,bijc->bhij", g_pair, zr))
        d_v += np.einsum("bhij,bihc->bjhc", a, g_o)
        d_gv += np.einsum("bhij,bihpx->bjhpx", a, d_og)
        d_z = np.einsum("bhij,bihc->bijc", a, g_pair)

        dl = a * (da - np.sum(a * da, axis=-1, keepdims=True))

        d_q[:, rows] += w_L * ss * np.einsum("bhij,bjhc->bihc", dl, k)
        d_k += w_L * ss * np.einsum("bhij,bihc->bjhc", dl, q[:, rows])
        d_gq[:, rows] += -coef[None, None, :, None, None] * np.einsum("bhij,bijhpx->bihpx", dl, diff)
        d_gk += coef[None, None, :, None, None] * np.einsum("bhij,bijhpx->bjhpx", dl, diff)
        d_gamma += -w_L * w_C / 2.0 * np.einsum("bhij,bhij->h", dl, d2)

        d_wb += w_L * np.einsum("bhij,bijc->ch", dl, zr)
        d_z += w_L * np.einsum("bhij,ch->bijc", dl, w_bias)

        d_z1[:, rows] += np.einsum("bijc,bjrc->birc", d_z, z2)
        d_z2 += np.einsum("bijc,birc->bjrc", d_z, z1[:, rows])

    def back(d_glob, pts):
        d_loc = np.einsum("blxy,blhpx->blhpy", rot, d_glob)
        d_r = np.einsum("blhpx,blhpy->blxy", d_glob, pts)
        return d_loc, d_r, d_glob.sum(axis=(2, 3))

    d_qp, r1, t1 = back(d_gq, q_pts)
    d_kp, r2, t2 = back(d_gk, k_pts)
    d_vp, r3, t3 = back(d_gv, v_pts)
    return {"q": d_q, "k": d_k, "v": d_v, "q_pts": d_qp, "k_pts": d_kp, "v_pts": d_vp,
            "rot": d_rot + r1 + r2 + r3, "trans": d_trans + t1 + t2 + t3, "z1": d_z1, "z2": d_z2,
            "w_bias": d_wb, "gamma": d_gamma}
