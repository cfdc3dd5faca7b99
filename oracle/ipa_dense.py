"""Dense float64 CPU oracle of the Invariant Point Attention core.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this file; only tests/, __graft_entry__.smoke() and bench.py's CPU
baseline / reference arm do.  It shares no code, constants or helpers with the
CUDA library.

What it computes (Flash Invariant Point Attention, TL;DR and Abstract: IPA over
residue frames with a factorised pair representation z_ij = z1_i^T z2_j; the
factorisation is exact, so the dense IPA below is the definition the fused
kernel must reproduce).  Everything is materialised: the pair tensor
z [B, nq, L, Cz] and the logits [B, H, nq, L].

For batch b, query residue i, key residue j, head h:
  1. global points  gq_ihp = R_i q_pts_ihp + t_i,  gk_jhp = R_j k_pts_jhp + t_j,
                    gv_jhp = R_j v_pts_jhp + t_j
     (R_i maps column vectors from residue i's local frame to the global one).
  2. pair tensor    z_ijc = sum_r z1_irc * z2_jrc
  3. pair bias      b^h_ij = sum_c w_bias[c, h] * z_ijc
  4. logit          l^h_ij = w_L * ( scalar_scale * <q_ih, k_jh> + b^h_ij
                                     - gamma_h * w_C / 2 * sum_p |gq_ihp - gk_jhp|^2 )
  5. allowed_ij = mask_i and mask_j; a^h_ij = softmax over the allowed j
     (a row without any allowed j gives a = 0).
  6. outputs        o_ih      = sum_j a v_jh
                    o_pt_ihp  = R_i^T (sum_j a gv_jhp - t_i)
                    n_ihp     = |o_pt_ihp|
                    o_pair_ihc = sum_j a z_ijc
  7. a row without any allowed key has every output feature equal to 0.
  Layout of the result: [B, L, H, C | Pv*3 (xyz inner) | Pv | Cz], float64.

Readings where the pages are silent (each listed with its reason in the
design notes): w_L = sqrt(1/3), w_C = sqrt(2 / (9 Pq)), scalar_scale = 1/sqrt(C)
(the AlphaFold-2 IPA constants, passed explicitly so they can be changed); the
pair bias sits inside w_L; no epsilon in the point norms; gamma arrives
already positive.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = ["ipa_constants", "ipa_dense", "ipa_dense_blocked"]


def ipa_constants(C: int, Pq: int) -> dict:
    """Default weights of the three logit terms (AlphaFold-2 IPA values)."""
    return {"w_L": math.sqrt(1.0 / 3.0), "w_C": math.sqrt(2.0 / (9.0 * Pq)),
            "scalar_scale": 1.0 / math.sqrt(C)}


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def ipa_dense(inp: dict, *, rows=None, w_L=None, w_C=None, scalar_scale=None,
              return_attn: bool = False):
    """Dense IPA for the query residues `rows` (default: all) of every batch.

    Returns out [B, nq, H, F] (and, if return_attn, a [B, H, nq, L]).
    """
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
    scalar_scale = consts["scalar_scale"] if scalar_scale is None else scalar_scale
    rows = np.arange(L) if rows is None else np.asarray(rows)

    # 1. frames applied to the local points
    gq = np.einsum("blxy,blhpy->blhpx", rot[:, rows], q_pts[:, rows]) + trans[:, rows, None, None, :]
    gk = np.einsum("blxy,blhpy->blhpx", rot, k_pts) + trans[:, :, None, None, :]
    gv = np.einsum("blxy,blhpy->blhpx", rot, v_pts) + trans[:, :, None, None, :]

    # 2.-3. materialised pair tensor and its per-head bias
    z = np.einsum("birc,bjrc->bijc", z1[:, rows], z2)
    bias = np.einsum("bijc,ch->bhij", z, w_bias)

    # 4. logits
    scal = np.einsum("bihc,bjhc->bhij", q[:, rows], k)
    diff = gq[:, :, None, :, :, :] - gk[:, None, :, :, :, :]      # [B, nq, L, H, Pq, 3]
    d2 = np.einsum("bijhpx,bijhpx->bhij", diff, diff)
    logits = w_L * (scalar_scale * scal + bias
                    - (gamma * w_C / 2.0)[None, :, None, None] * d2)

    # 5. masked softmax over keys
    allowed = mask[:, rows, None] & mask[:, None, :]                 # [B, nq, L]
    allowed_h = np.broadcast_to(allowed[:, None], logits.shape)
    neg = np.where(allowed_h, logits, -np.inf)
    mx = neg.max(axis=-1, keepdims=True)
    mx = np.where(np.isfinite(mx), mx, 0.0)
    e = np.where(allowed_h, np.exp(neg - mx), 0.0)
    s = e.sum(axis=-1, keepdims=True)
    a = np.where(s > 0, e / np.where(s > 0, s, 1.0), 0.0)

    # 6. aggregation
    o = np.einsum("bhij,bjhc->bihc", a, v)
    og = np.einsum("bhij,bjhpx->bihpx", a, gv)
    o_pt = np.einsum("bixy,bihpx->bihpy", rot[:, rows], og - trans[:, rows, None, None, :])
    nrm = np.sqrt(np.einsum("bihpx,bihpx->bihp", o_pt, o_pt))
    o_pair = np.einsum("bhij,bijc->bihc", a, z)

    # 7. rows without any allowed key are all-zero
    live = allowed.any(axis=-1)                                      # [B, nq]
    out = np.concatenate([o, o_pt.reshape(B, len(rows), H, 3 * Pv), nrm, o_pair], axis=-1)
    out = np.where(live[:, :, None, None], out, 0.0)
    if return_attn:
        return out, a
    return out


def ipa_dense_blocked(inp: dict, rows=None, block: int = 64, **kw):
    """Same arithmetic as ipa_dense, run over blocks of `block` query rows so
    that the materialised pair tensor stays bounded at long L."""
    L = inp["q"].shape[1]
    rows = np.arange(L) if rows is None else np.asarray(rows)
    parts = [ipa_dense(inp, rows=rows[s:s + block], **kw) for s in range(0, len(rows), block)]
    return np.concatenate(parts, axis=1)

