"""Dense float64 CPU oracle of the geometric direction-and-distance attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this file; only tests/, __graft_entry__.smoke() and bench.py's CPU
baseline / reference arm do.  It shares no code with the CUDA library.

Follows "Geometric direction-and-distance attention" (BioTorch exercise,
section "Required behavior"), step by step:
  1. qd_i = R_i q_direction_i, kd_j = R_j k_direction_j,
     qp_i = R_i q_point_i + t_i, kp_j = R_j k_point_j + t_j   (per head)
  2. score s_ijh = (softplus(direction_scale_h) <qd_i, kd_j>
                    - softplus(distance_scale_h) |qp_i - kp_j|_2) / sqrt(3)
     softplus evaluated stably as max(x, 0) + log1p(exp(-|x|)); the distance
     is not squared and has no epsilon.
  3. allowed = frame_mask_i and frame_mask_j and pair_mask[b, h, i, j]
     (pair_mask optional, broadcast to [B, H, N, N]); stable masked softmax
     over j; a head row with no allowed key is exactly zero.
  4. values rotated with R_j only (no translation), aggregated with the
     attention, rotated back with R_i^T -> vectors [B, N, H, M, 3].
  5. output = flatten(vectors in H, M, xyz order) @ output_weight
     (+ output_bias); forced to zero for a query where no head has an
     allowed key.
Returns (vectors, attention [B, H, N, N], output [B, N, Cout]), float64.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = ["softplus_stable", "geo_dense", "geo_dense_blocked"]


def softplus_stable(x):
    """log(1 + exp(x)) without overflow for large |x|."""
    x = np.asarray(x, dtype=np.float64)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def _f64(a):
    return None if a is None else np.asarray(a, dtype=np.float64)


def geo_dense(inp: dict, rows=None):
    """Dense variant for query residues `rows` (default all).

    Returns vectors [B, nq, H, M, 3], attention [B, H, nq, N], output [B, nq, Cout].
    """
    qdir, kdir = _f64(inp["q_direction"]), _f64(inp["k_direction"])
    qpt, kpt = _f64(inp["q_point"]), _f64(inp["k_point"])
    values = _f64(inp["values"])
    rot, trans = _f64(inp["rotation"]), _f64(inp["translation"])
    w_out, b_out = _f64(inp["output_weight"]), _f64(inp.get("output_bias"))
    fmask = np.asarray(inp["frame_mask"], dtype=bool)
    pmask = inp.get("pair_mask")
    B, N, H, _ = qdir.shape
    M = values.shape[3]
    rows = np.arange(N) if rows is None else np.asarray(rows)
    nq = len(rows)

    # 1. rotate directions, transform points
    qd = np.einsum("bnxy,bnhy->bnhx", rot[:, rows], qdir[:, rows])
    kd = np.einsum("bnxy,bnhy->bnhx", rot, kdir)
    qp = np.einsum("bnxy,bnhy->bnhx", rot[:, rows], qpt[:, rows]) + trans[:, rows, None, :]
    kp = np.einsum("bnxy,bnhy->bnhx", rot, kpt) + trans[:, :, None, :]

    # 2. scores
    a_h = softplus_stable(inp["direction_scale"])
    b_h = softplus_stable(inp["distance_scale"])
    dot = np.einsum("bihx,bjhx->bhij", qd, kd)
    diff = qp[:, :, None, :, :] - kp[:, None, :, :, :]              # [B, nq, N, H, 3]
    dist = np.sqrt(np.einsum("bijhx,bijhx->bhij", diff, diff))
    s = (a_h[None, :, None, None] * dot - b_h[None, :, None, None] * dist) / math.sqrt(3.0)

    # 3. masked softmax
    allowed = np.broadcast_to((fmask[:, rows, None] & fmask[:, None, :])[:, None], s.shape)
    if pmask is not None:
        pm = np.broadcast_to(np.asarray(pmask, dtype=bool), (B, H, N, N))[:, :, rows, :]
        allowed = allowed & pm
    neg = np.where(allowed, s, -np.inf)
    mx = neg.max(axis=-1, keepdims=True)
    mx = np.where(np.isfinite(mx), mx, 0.0)
    e = np.where(allowed, np.exp(neg - mx), 0.0)
    tot = e.sum(axis=-1, keepdims=True)
    attn = np.where(tot > 0, e / np.where(tot > 0, tot, 1.0), 0.0)

    # 4. rotate values by R_j, aggregate, rotate back by R_i^T
    vr = np.einsum("bjxy,bjhmy->bjhmx", rot, values)
    agg = np.einsum("bhij,bjhmx->bihmx", attn, vr)
    vectors = np.einsum("bixy,bihmx->bihmy", rot[:, rows], agg)

    # 5. readout, empty queries forced to zero
    flat = vectors.reshape(B, nq, H * M * 3)
    out = flat @ w_out
    if b_out is not None:
        out = out + b_out
    live = allowed.any(axis=-1).any(axis=1)                          # [B, nq]
    out = np.where(live[:, :, None], out, 0.0)
    return vectors, attn, out


def geo_dense_blocked(inp: dict, rows=None, block: int = 128, with_attention: bool = True):
    """geo_dense over blocks of query rows (bounded memory at N = 2048)."""
    N = inp["q_direction"].shape[1]
    rows = np.arange(N) if rows is None else np.asarray(rows)
    vs, ats, outs = [], [], []
    for s in range(0, len(rows), block):
        v, a, o = geo_dense(inp, rows=rows[s:s + block])
        vs.append(v)
        outs.append(o)
        if with_attention:
            ats.append(a)
    att = np.concatenate(ats, axis=2) if with_attention else None
    return np.concatenate(vs, axis=1), att, np.concatenate(outs, axis=1)
