"""The IPA layer around the factorised core: a plain float64 CPU oracle.

TEST INFRASTRUCTURE ONLY: imported by tests/ (and __graft_entry__.smoke()),
never by the product path.  Shares no code with the CUDA library.

Flash Invariant Point Attention replaces only the attention inside the IPA
layer of AlphaFold-2-style structure modules; the layer keeps its linear
projections.  This build reads the layer as (no layer norm, dropout or
residual, which sit outside it):

  1. Y_i = s_i W_in + b_in, s_i the single representation [c_s] of residue i;
     the columns of Y are, in order, q (H x C), k (H x C), v (H x C),
     q_pts (H x Pq x 3), k_pts (H x Pq x 3), v_pts (H x Pv x 3), each head-
     major with the channel (or the point, then xyz) innermost;
  2. o_i = the IPA core (ipa_dense) on those per-head inputs, the frames, the
     pair factors z1, z2 and w_bias, gamma, mask: [H, F], F = C + 4 Pv + Cz;
  3. out_i = flatten(o_i) W_out + b_out  [c_s].
Every step is a plain float64 product or the core oracle.
"""
from __future__ import annotations

import numpy as np

from .ipa_dense import ipa_dense

__all__ = ["ipa_module", "projection_width", "split_projection"]


def projection_width(H: int, C: int, Pq: int, Pv: int) -> int:
    return H * (3 * C + 3 * (2 * Pq + Pv))


def split_projection(Y, H: int, C: int, Pq: int, Pv: int) -> dict:
    """Views of Y [B, L, width] as the core's q, k, v, q_pts, k_pts, v_pts."""
    B, L, _ = Y.shape
    out, o = {}, 0
    for name, shape in (("q", (H, C)), ("k", (H, C)), ("v", (H, C)), ("q_pts", (H, Pq, 3)),
                        ("k_pts", (H, Pq, 3)), ("v_pts", (H, Pv, 3))):
        n = int(np.prod(shape))
        out[name] = Y[:, :, o:o + n].reshape(B, L, *shape)
        o += n
    return out


def ipa_module(inp: dict, *, return_core: bool = False, **consts):
    """out [B, L, c_s] (float64); with return_core also the core output
    [B, L, H, F]."""
    s = np.asarray(inp["s"], dtype=np.float64)
    W_in, W_out = np.asarray(inp["w_in"], np.float64), np.asarray(inp["w_out"], np.float64)
    b_in = 0.0 if inp.get("b_in") is None else np.asarray(inp["b_in"], np.float64)
    b_out = 0.0 if inp.get("b_out") is None else np.asarray(inp["b_out"], np.float64)
    H = np.asarray(inp["gamma"]).shape[0]
    Pq, Pv = inp["dims"].Pq, inp["dims"].Pv
    C = inp["dims"].C
    Y = s @ W_in + b_in                                                   # 1.
    core_inp = dict(split_projection(Y, H, C, Pq, Pv))
    for k in ("rot", "trans", "z1", "z2", "w_bias", "gamma", "mask"):
        core_inp[k] = inp[k]
    core = ipa_dense(core_inp, **consts)                                  # 2.
    B, L = s.shape[:2]
    out = core.reshape(B, L, -1) @ W_out + b_out                          # 3.
    return (out, core) if return_core else out
