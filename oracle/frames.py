"""Residue frames from backbone atoms: a plain float64 CPU oracle.

TEST INFRASTRUCTURE ONLY: imported by tests/ (and __graft_entry__.smoke()),
never by the product path.

Flash Invariant Point Attention, Figure 1 (the protein backbone frame): the
frame of residue i is centred on C_alpha, and the vectors C_alpha -> N and
C_alpha -> C span it by Gram-Schmidt; the third axis completes it.  The
pages do not fix which vector comes first or the handedness; this build
reads them as

    e1 = (C - CA) / |C - CA|
    u2 = (N - CA) - (e1 . (N - CA)) e1,   e2 = u2 / |u2|
    e3 = e1 x e2                           (right-handed, det R = +1)
    R  = [e1 | e2 | e3]  (columns),  t = CA

so that R maps local column vectors to global ones, as the IPA inputs
expect.  Written out step by step, no blocking.
"""
from __future__ import annotations

import numpy as np


def frames_from_backbone(n, ca, c):
    """n, ca, c: [..., 3] atom positions -> (R [..., 3, 3], t [..., 3]),
    float64."""
    n, ca, c = (np.asarray(a, dtype=np.float64) for a in (n, ca, c))
    v1 = c - ca
    v2 = n - ca
    e1 = v1 / np.linalg.norm(v1, axis=-1, keepdims=True)
    u2 = v2 - np.sum(e1 * v2, axis=-1, keepdims=True) * e1
    e2 = u2 / np.linalg.norm(u2, axis=-1, keepdims=True)
    e3 = np.cross(e1, e2)
    R = np.stack([e1, e2, e3], axis=-1)          # columns e1, e2, e3
    return R, ca.copy()
