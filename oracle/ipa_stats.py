"""Softmax statistics of the Invariant Point Attention core kept by a training
forward pass: a plain float64 CPU oracle.

TEST INFRASTRUCTURE ONLY: imported by tests/, never by the product path.
Shares no code with the CUDA library.

Flash Invariant Point Attention trains the factorised IPA (TL;DR; Figure 3,
FoldFlow retrained with it), so a forward pass that is to be differentiated
keeps two per-row quantities besides its output:

  lse_bhi      = log sum_{allowed j} exp(l^h_ij)          [B, H, L]
                 (+inf for a row without any allowed key, so that
                 exp(l - lse) = 0 there)
  U_bihrc      = sum_j a^h_ij z2_jrc                      [B, L, H, R, Cz]
                 (the pair-value aggregate before the contraction with z1_i:
                 o_pair_ihc = sum_r z1_irc U_ihrc)

with the logits l and the attention a of `ipa_dense` (same definition, same
readings: all three logit terms inside w_L, masks on both residues, a = 0 on
rows without an allowed key).  Everything is materialised.
"""
from __future__ import annotations

import numpy as np

from .ipa_dense import ipa_constants

__all__ = ["ipa_forward_stats"]


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def ipa_forward_stats(inp: dict, *, rows=None, w_L=None, w_C=None, scalar_scale=None):
    """(lse [B, H, nq], U [B, nq, H, R, Cz]) for the query residues `rows`."""
    q, k = _f64(inp["q"]), _f64(inp["k"])
    q_pts, k_pts = _f64(inp["q_pts"]), _f64(inp["k_pts"])
    rot, trans = _f64(inp["rot"]), _f64(inp["trans"])
    z1, z2 = _f64(inp["z1"]), _f64(inp["z2"])
    w_bias, gamma = _f64(inp["w_bias"]), _f64(inp["gamma"])
    mask = np.asarray(inp["mask"], dtype=bool)
    B, L, H, C = q.shape
    Pq = q_pts.shape[3]
    consts = ipa_constants(C, Pq)
    w_L = consts["w_L"] if w_L is None else w_L
    w_C = consts["w_C"] if w_C is None else w_C
    scalar_scale = consts["scalar_scale"] if scalar_scale is None else scalar_scale
    rows = np.arange(L) if rows is None else np.asarray(rows)

    # logits (definition of the IPA core, step by step)
    gq = np.einsum("blxy,blhpy->blhpx", rot[:, rows], q_pts[:, rows]) + trans[:, rows, None, None, :]
    gk = np.einsum("blxy,blhpy->blhpx", rot, k_pts) + trans[:, :, None, None, :]
    z = np.einsum("birc,bjrc->bijc", z1[:, rows], z2)
    bias = np.einsum("bijc,ch->bhij", z, w_bias)
    scal = np.einsum("bihc,bjhc->bhij", q[:, rows], k)
    diff = gq[:, :, None] - gk[:, None, :]
    d2 = np.einsum("bijhpx,bijhpx->bhij", diff, diff)
    logits = w_L * (scalar_scale * scal + bias - (gamma * w_C / 2.0)[None, :, None, None] * d2)

    allowed = mask[:, rows, None] & mask[:, None, :]
    allowed_h = np.broadcast_to(allowed[:, None], logits.shape)
    neg = np.where(allowed_h, logits, -np.inf)
    mx = neg.max(axis=-1)                                            # [B, H, nq]
    live = np.isfinite(mx)
    m0 = np.where(live, mx, 0.0)
    e = np.where(allowed_h, np.exp(neg - m0[..., None]), 0.0)
    s = e.sum(axis=-1)
    lse = np.where(live, m0 + np.log(np.where(live, s, 1.0)), np.inf)
    a = np.where(allowed_h, np.exp(neg - np.where(live, lse, 0.0)[..., None]), 0.0)
    U = np.einsum("bhij,bjrc->bihrc", a, z2)
    return lse, U
