"""Distance-aware attention of MEET (§2.2 "distance-aware attention",
eq. (6)): a plain float64 CPU oracle.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and
bench.py's CPU-baseline / reference arm, never by the product path.

For head h, query i and key j (eq. (6)):

    A_ij^h = rho_h * ( <q_i^h, k_j^h> - s_h^2 * ||x_i - x_j||^2 )

with rho_h the attention scale and s_h the distance scale of the head.  The
passage defines these logits only; the rest is this build's reading of a
standard attention layer built on them:

* the softmax runs over the keys j allowed for query i (mask_i and mask_j);
* the output is o_i^h = sum_j softmax_j(A_i.^h) v_j^h;
* a row with no allowed key is 0.

The distance is the plain squared Euclidean distance, written out here
directly (eq. (7)-(8) fold it into augmented query and key vectors; the
tests check that identity separately).  Nothing is blocked or reordered.
"""
from __future__ import annotations

import numpy as np


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def meet_logits(inp: dict, rows=None) -> np.ndarray:
    """A[b, h, i, j] of eq. (6), float64, for the query rows `rows` (all by
    default); masks are not applied."""
    q, k, x = _f64(inp["q"]), _f64(inp["k"]), _f64(inp["x"])
    rho, s = _f64(inp["rho"]), _f64(inp["s"])
    if rows is not None:
        rows = np.asarray(rows)
        q, xq = q[:, rows], x[:, rows]
    else:
        xq = x
    qk = np.einsum("bihc,bjhc->bhij", q, k)
    diff = xq[:, :, None, :] - x[:, None, :, :]                   # [B, Lq, L, 3]
    d2 = np.einsum("bijk,bijk->bij", diff, diff)                  # ||x_i - x_j||^2
    return rho[None, :, None, None] * (qk - (s ** 2)[None, :, None, None] * d2[:, None])


def meet_dense(inp: dict, rows=None, return_attn: bool = False):
    """Output o[b, i, h, c] (float64) for the query rows `rows` (all by
    default); with return_attn also the attention weights [B, H, Lq, L]."""
    v = _f64(inp["v"])
    mask = np.asarray(inp["mask"], dtype=bool)
    A = meet_logits(inp, rows)
    mq = mask if rows is None else mask[:, np.asarray(rows)]
    allowed = mq[:, None, :, None] & mask[:, None, None, :]       # [B, 1, Lq, L]
    A = np.where(allowed, A, -np.inf)
    m = A.max(axis=-1, keepdims=True)
    live = np.isfinite(m)
    e = np.where(allowed, np.exp(A - np.where(live, m, 0.0)), 0.0)
    den = e.sum(axis=-1, keepdims=True)
    a = np.where(live, e / np.where(live, den, 1.0), 0.0)         # rows with no allowed key: 0
    o = np.einsum("bhij,bjhc->bihc", a, v)
    return (o, a) if return_attn else o
