"""Gradients of the geometric direction-and-distance attention: a plain
float64 CPU oracle.

TEST INFRASTRUCTURE ONLY: imported by tests/ (and __graft_entry__.smoke()),
never by the product path.  Shares no code with the CUDA library.

"Geometric direction-and-distance attention" (Required behavior) asks for
the gradients of the operator, with the derivative of the unsquared distance
at a zero displacement defined as the zero vector.  Given the upstream
gradients g_output [B, N, Cout], g_attention [B, H, N, N] and g_vectors
[B, N, H, M, 3] (the last two optional, zero when absent), this module runs
the forward steps of `geo_dense` again and then their adjoints in reverse
order, written out one step at a time:

  5'. readout: only queries with an allowed key pass g_output on;
      dW = flat(vectors)^T g_output, db = sum of g_output over those queries,
      g_vectors += g_output W^T.
  4'. vectors_i = R_i^T agg_i: d agg_i = R_i g_vectors_i, dR_i += agg_i g^T.
      agg_i = sum_j a_ij vr_j: d vr_j = sum_i a_ij d agg_i,
      da_ij = <d agg_i, vr_j> + g_attention_ij.
      vr_j = R_j values_j: d values_j = R_j^T d vr_j, dR_j += d vr_j values_j^T.
  3'. softmax: ds_ij = a_ij (da_ij - sum_k a_ik da_ik).
  2'. s_ij = (A_h <qd_i, kd_j> - B_h |qp_i - kp_j|) / sqrt(3) with
      A_h = softplus(direction_scale_h), B_h = softplus(distance_scale_h):
      d qd_i = A/sqrt3 sum_j ds_ij kd_j,  d kd_j = A/sqrt3 sum_i ds_ij qd_i,
      d qp_i = -B/sqrt3 sum_j ds_ij u_ij, d kp_j = B/sqrt3 sum_i ds_ij u_ij,
      u_ij = (qp_i - kp_j) / |qp_i - kp_j| (the zero vector when qp_i = kp_j),
      dA_h = sum ds <qd, kd> / sqrt3, dB_h = -sum ds |qp - kp| / sqrt3,
      d scale = dA * sigmoid(scale) (softplus' = sigmoid).
  1'. qd_i = R_i q_direction_i etc.: d q_direction_i = R_i^T d qd_i,
      dR_i += d qd_i q_direction_i^T; points also give dt_i += d qp_i.

Gradients of the masks do not exist; all are returned in float64.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = ["geo_grad"]


def _f64(a):
    return None if a is None else np.asarray(a, dtype=np.float64)


def _sigmoid(x):
    return np.where(x >= 0, 1.0 / (1.0 + np.exp(-np.abs(x))), np.exp(-np.abs(x)) / (1.0 + np.exp(-np.abs(x))))


def _softplus(x):
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def geo_grad(inp: dict, g_output, g_attention=None, g_vectors=None) -> dict:
    """Gradients of sum(g_output * output) + sum(g_attention * attention)
    + sum(g_vectors * vectors) with respect to every floating input."""
    qdir, kdir = _f64(inp["q_direction"]), _f64(inp["k_direction"])
    qpt, kpt = _f64(inp["q_point"]), _f64(inp["k_point"])
    values = _f64(inp["values"])
    rot, trans = _f64(inp["rotation"]), _f64(inp["translation"])
    w_out = _f64(inp["output_weight"])
    has_bias = inp.get("output_bias") is not None
    dsc, xsc = _f64(inp["direction_scale"]), _f64(inp["distance_scale"])
    fmask = np.asarray(inp["frame_mask"], dtype=bool)
    pmask = inp.get("pair_mask")
    B, N, H, _ = qdir.shape
    M = values.shape[3]
    r3 = math.sqrt(3.0)
    g_output = _f64(g_output)
    g_attention = np.zeros((B, H, N, N)) if g_attention is None else _f64(g_attention)
    g_vectors = np.zeros((B, N, H, M, 3)) if g_vectors is None else _f64(g_vectors)

    # forward steps 1-5 (as in geo_dense), keeping the intermediates
    qd = np.einsum("bnxy,bnhy->bnhx", rot, qdir)
    kd = np.einsum("bnxy,bnhy->bnhx", rot, kdir)
    qp = np.einsum("bnxy,bnhy->bnhx", rot, qpt) + trans[:, :, None, :]
    kp = np.einsum("bnxy,bnhy->bnhx", rot, kpt) + trans[:, :, None, :]
    A, Bd = _softplus(dsc), _softplus(xsc)
    dot = np.einsum("bihx,bjhx->bhij", qd, kd)
    diff = qp[:, :, None, :, :] - kp[:, None, :, :, :]              # [B, N, N, H, 3]
    dist = np.sqrt(np.einsum("bijhx,bijhx->bhij", diff, diff))
    s = (A[None, :, None, None] * dot - Bd[None, :, None, None] * dist) / r3
    allowed = np.broadcast_to((fmask[:, :, None] & fmask[:, None, :])[:, None], s.shape)
    if pmask is not None:
        allowed = allowed & np.broadcast_to(np.asarray(pmask, dtype=bool), (B, H, N, N))
    neg = np.where(allowed, s, -np.inf)
    mx = neg.max(axis=-1, keepdims=True)
    mx = np.where(np.isfinite(mx), mx, 0.0)
    e = np.where(allowed, np.exp(neg - mx), 0.0)
    tot = e.sum(axis=-1, keepdims=True)
    a = np.where(tot > 0, e / np.where(tot > 0, tot, 1.0), 0.0)
    vr = np.einsum("bjxy,bjhmy->bjhmx", rot, values)
    agg = np.einsum("bhij,bjhmx->bihmx", a, vr)
    vectors = np.einsum("bixy,bihmx->bihmy", rot, agg)
    live = allowed.any(axis=-1).any(axis=1)                           # [B, N]

    # 5'. readout
    go = np.where(live[:, :, None], g_output, 0.0)                   # dead queries pass nothing on
    flat = vectors.reshape(B, N, H * M * 3)
    d_w = np.einsum("bnk,bnc->kc", flat, go)
    d_b = go.sum(axis=(0, 1)) if has_bias else None
    g_vec = g_vectors + np.einsum("bnc,kc->bnk", go, w_out).reshape(B, N, H, M, 3)

    # 4'. back-rotation, aggregation, value rotation
    d_rot = np.einsum("bihmx,bihmy->bixy", agg, g_vec)
    d_agg = np.einsum("bixy,bihmy->bihmx", rot, g_vec)
    d_vr = np.einsum("bhij,bihmx->bjhmx", a, d_agg)
    da = np.einsum("bihmx,bjhmx->bhij", d_agg, vr) + g_attention
    d_values = np.einsum("bjxy,bjhmx->bjhmy", rot, d_vr)
    d_rot += np.einsum("bjhmx,bjhmy->bjxy", d_vr, values)

    # 3'. softmax
    ds = a * (da - np.sum(a * da, axis=-1, keepdims=True))

    # 2'. score
    safe = np.where(dist > 0, dist, 1.0)
    u = np.where((dist > 0)[..., None], np.moveaxis(diff, 3, 1) / safe[..., None], 0.0)   # [B, H, N, N, 3]
    d_qd = (A[None, None, :, None] / r3) * np.einsum("bhij,bjhx->bihx", ds, kd)
    d_kd = (A[None, None, :, None] / r3) * np.einsum("bhij,bihx->bjhx", ds, qd)
    d_qp = -(Bd[None, None, :, None] / r3) * np.einsum("bhij,bhijx->bihx", ds, u)
    d_kp = (Bd[None, None, :, None] / r3) * np.einsum("bhij,bhijx->bjhx", ds, u)
    dA = np.einsum("bhij,bhij->h", ds, dot) / r3
    dB = -np.einsum("bhij,bhij->h", ds, dist) / r3

    # 1'. frames
    d_qdir = np.einsum("bnxy,bnhx->bnhy", rot, d_qd)
    d_kdir = np.einsum("bnxy,bnhx->bnhy", rot, d_kd)
    d_qpt = np.einsum("bnxy,bnhx->bnhy", rot, d_qp)
    d_kpt = np.einsum("bnxy,bnhx->bnhy", rot, d_kp)
    d_rot += (np.einsum("bnhx,bnhy->bnxy", d_qd, qdir) + np.einsum("bnhx,bnhy->bnxy", d_kd, kdir)
              + np.einsum("bnhx,bnhy->bnxy", d_qp, qpt) + np.einsum("bnhx,bnhy->bnxy", d_kp, kpt))
    d_trans = d_qp.sum(axis=2) + d_kp.sum(axis=2)

    return {"q_direction": d_qdir, "k_direction": d_kdir, "q_point": d_qpt, "k_point": d_kpt,
            "values": d_values, "direction_scale": dA * _sigmoid(dsc), "distance_scale": dB * _sigmoid(xsc),
            "output_weight": d_w, "output_bias": d_b, "rotation": d_rot, "translation": d_trans}
