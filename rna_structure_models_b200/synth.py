"""Seeded synthetic inputs for the IPA core and the geometric attention variant.

This module only draws random numbers in the shapes, distributions and
structure of the workloads; it computes none of the attention arithmetic.
Both the float64 oracle (tests only) and the CUDA path are fed from here.

Structure of the inputs (stand-ins for the protein / RNA backbones that the
Flash Invariant Point Attention paper trains on, Fig. 2-4, which are not
available here):
  * frames T_i = (R_i, t_i): R_i a proper rotation from the QR decomposition
    of a Gaussian 3x3 matrix (sign fixed by diag(R), first column flipped if
    det < 0); t_i a C-alpha-like random walk with 3.8 Angstrom steps in
    directions uniform on the sphere, starting at the origin;
  * q/k/v, query/key/value points and the pair factors z1/z2 ~ N(0, 1);
  * w_bias ~ N(0, 0.1^2) (std 0.1); gamma = softplus(N(0, 1)) (already > 0).

Draw order (fixed, one numpy PCG64 stream per call): rotations, walk,
(jitter), q, k, v, q_pts, k_pts, v_pts, z1, z2, w_bias, gamma, masks.
Arrays are drawn in float64 and returned as float32 (masks as bool); the
oracle up-casts the same float32 values, so parity never measures input
rounding.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "IpaDims", "GeoDims", "ipa_inputs", "geo_inputs", "ipa_preset", "geo_preset",
    "IPA_PRESETS", "random_rotations", "random_walk", "MeetDims", "meet_inputs", "backbone_inputs",
]


@dataclass(frozen=True)
class IpaDims:
    B: int
    L: int
    H: int
    C: int = 16
    Pq: int = 4
    Pv: int = 8
    R: int = 2
    Cz: int = 128

    @property
    def F(self) -> int:
        """Output features per (residue, head): scalar | points xyz | point norms | pair."""
        return self.C + 3 * self.Pv + self.Pv + self.Cz


@dataclass(frozen=True)
class GeoDims:
    B: int
    N: int
    H: int
    M: int
    Cout: int


@dataclass(frozen=True)
class MeetDims:
    """Distance-aware attention (MEET §2.2): B batch, L atoms, H heads, C
    query/key/value channels per head."""
    B: int = 1
    L: int = 512
    H: int = 8
    C: int = 16


def random_rotations(rng: np.random.Generator, n: int) -> np.ndarray:
    """n proper rotations: QR of Gaussian 3x3, sign-fixed, det forced to +1."""
    a = rng.standard_normal((n, 3, 3))
    q, r = np.linalg.qr(a)
    d = np.sign(np.diagonal(r, axis1=1, axis2=2))
    d[d == 0] = 1.0
    q = q * d[:, None, :]
    neg = np.linalg.det(q) < 0
    q[neg, :, 0] *= -1.0
    return q


def random_walk(rng: np.random.Generator, n: int, step: float = 3.8) -> np.ndarray:
    """Positions of an n-point walk with fixed step length and isotropic directions."""
    u = rng.standard_normal((max(n - 1, 0), 3))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    t = np.zeros((n, 3))
    if n > 1:
        t[1:] = np.cumsum(step * u, axis=0)
    return t


def _softplus_draw(x: np.ndarray) -> np.ndarray:
    # distribution of gamma in the workloads: softplus of a standard normal draw
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def ipa_inputs(dims: IpaDims, seed: int = 0, *, masked_tail_frac: float = 0.0,
               ragged: tuple[int, int] | None = None, jitter: float = 0.0) -> dict:
    """Seeded IPA-core inputs.

    masked_tail_frac: the last round(frac * L) residues of every batch element
      are masked out (mask False).
    ragged: (lo, hi) -> per batch element a length L_b uniform in [lo, hi]
      (inclusive); mask[b, i] = i < L_b.
    jitter: std (Angstrom) of isotropic Gaussian noise added to the walk.
    """
    B, L, H, C, Pq, Pv, R, Cz = (dims.B, dims.L, dims.H, dims.C, dims.Pq,
                                 dims.Pv, dims.R, dims.Cz)
    rng = np.random.Generator(np.random.PCG64(seed))
    rot = random_rotations(rng, B * L).reshape(B, L, 3, 3)
    trans = np.stack([random_walk(rng, L) for _ in range(B)])
    if jitter > 0.0:
        trans = trans + jitter * rng.standard_normal(trans.shape)
    q = rng.standard_normal((B, L, H, C))
    k = rng.standard_normal((B, L, H, C))
    v = rng.standard_normal((B, L, H, C))
    q_pts = rng.standard_normal((B, L, H, Pq, 3))
    k_pts = rng.standard_normal((B, L, H, Pq, 3))
    v_pts = rng.standard_normal((B, L, H, Pv, 3))
    z1 = rng.standard_normal((B, L, R, Cz))
    z2 = rng.standard_normal((B, L, R, Cz))
    w_bias = 0.1 * rng.standard_normal((Cz, H))
    gamma = _softplus_draw(rng.standard_normal(H))
    mask = np.ones((B, L), dtype=bool)
    lengths = np.full(B, L)
    if ragged is not None:
        lengths = rng.integers(ragged[0], ragged[1] + 1, size=B)
        mask = np.arange(L)[None, :] < lengths[:, None]
    if masked_tail_frac > 0.0:
        n_mask = int(round(masked_tail_frac * L))
        if n_mask > 0:
            mask[:, L - n_mask:] = False
            lengths = np.minimum(lengths, L - n_mask)
    f32 = lambda a: np.ascontiguousarray(a, dtype=np.float32)  # noqa: E731
    return {
        "dims": dims,
        "q": f32(q), "k": f32(k), "v": f32(v),
        "q_pts": f32(q_pts), "k_pts": f32(k_pts), "v_pts": f32(v_pts),
        "rot": f32(rot), "trans": f32(trans),
        "z1": f32(z1), "z2": f32(z2),
        "w_bias": f32(w_bias), "gamma": f32(gamma),
        "mask": np.ascontiguousarray(mask),
        "lengths": lengths,
    }


def geo_inputs(dims: GeoDims, seed: int = 0, *, pair_drop: float = 0.2,
               frame_drop: float = 0.05, with_pair_mask: bool = True,
               with_bias: bool = True) -> dict:
    """Seeded inputs of the direction/distance geometric attention variant.

    Draw order: rotations, walk, q_direction, k_direction, q_point, k_point,
    values, direction_scale, distance_scale, output_weight, output_bias,
    frame_mask, pair_mask.  output_weight ~ N(0, 1/(H*M*3)) and
    output_bias ~ N(0, 0.1^2) (the pages give no distribution for them).
    """
    B, N, H, M, Cout = dims.B, dims.N, dims.H, dims.M, dims.Cout
    rng = np.random.Generator(np.random.PCG64(seed))
    rot = random_rotations(rng, B * N).reshape(B, N, 3, 3)
    trans = np.stack([random_walk(rng, N) for _ in range(B)])
    qd = rng.standard_normal((B, N, H, 3))
    kd = rng.standard_normal((B, N, H, 3))
    qp = rng.standard_normal((B, N, H, 3))
    kp = rng.standard_normal((B, N, H, 3))
    values = rng.standard_normal((B, N, H, M, 3))
    dscale = rng.standard_normal(H)
    xscale = rng.standard_normal(H)
    w_out = rng.standard_normal((H * M * 3, Cout)) / math.sqrt(H * M * 3)
    b_out = 0.1 * rng.standard_normal(Cout)
    frame_mask = rng.random((B, N)) >= frame_drop
    pair_mask = None
    if with_pair_mask:
        pair_mask = rng.random((B, H, N, N)) >= pair_drop
    f32 = lambda a: np.ascontiguousarray(a, dtype=np.float32)  # noqa: E731
    return {
        "dims": dims,
        "q_direction": f32(qd), "k_direction": f32(kd),
        "q_point": f32(qp), "k_point": f32(kp), "values": f32(values),
        "direction_scale": f32(dscale), "distance_scale": f32(xscale),
        "output_weight": f32(w_out),
        "output_bias": f32(b_out) if with_bias else None,
        "rotation": f32(rot), "translation": f32(trans),
        "frame_mask": np.ascontiguousarray(frame_mask),
        "pair_mask": pair_mask,
    }


def geo_upstream(dims: GeoDims, seed: int = 0, *, with_attention: bool = True,
                 with_vectors: bool = True) -> dict:
    """Seeded upstream gradients of the variant's three results, N(0, 1):
    g_output [B, N, Cout], g_attention [B, H, N, N], g_vectors
    [B, N, H, M, 3] (the last two None when not requested).  Draw order as
    listed."""
    B, N, H, M, Cout = dims.B, dims.N, dims.H, dims.M, dims.Cout
    rng = np.random.Generator(np.random.PCG64(seed))
    f32 = lambda a: np.ascontiguousarray(a, dtype=np.float32)  # noqa: E731
    g_out = f32(rng.standard_normal((B, N, Cout)))
    g_att = f32(rng.standard_normal((B, H, N, N))) if with_attention else None
    g_vec = f32(rng.standard_normal((B, N, H, M, 3))) if with_vectors else None
    return {"g_output": g_out, "g_attention": g_att, "g_vectors": g_vec}


def meet_inputs(dims: MeetDims, seed: int = 0, *, masked_tail_frac: float = 0.0) -> dict:
    """Seeded inputs of the distance-aware attention of MEET §2.2.

    Draw order: walk (coordinates x, 3.8 A steps), q, k, v ~ N(0, 1),
    rho_h ~ U(0.5, 1.5) / sqrt(C) (attention scale), s_h ~ U(0.05, 0.3)
    (distance scale, per A), masks.  The pages give no distributions for
    rho and s; these keep the distance term and the dot product of similar
    size for neighbours a few residues apart.
    """
    B, L, H, C = dims.B, dims.L, dims.H, dims.C
    rng = np.random.Generator(np.random.PCG64(seed))
    x = np.stack([random_walk(rng, L) for _ in range(B)])
    q = rng.standard_normal((B, L, H, C))
    k = rng.standard_normal((B, L, H, C))
    v = rng.standard_normal((B, L, H, C))
    rho = rng.uniform(0.5, 1.5, H) / math.sqrt(C)
    s = rng.uniform(0.05, 0.3, H)
    mask = np.ones((B, L), dtype=bool)
    nmask = int(round(masked_tail_frac * L))
    if nmask:
        mask[:, L - nmask:] = False
    f32 = lambda a: np.ascontiguousarray(a, dtype=np.float32)  # noqa: E731
    return {"dims": dims, "q": f32(q), "k": f32(k), "v": f32(v), "x": f32(x),
            "rho": f32(rho), "s": f32(s), "mask": mask}


def backbone_inputs(B: int, L: int, seed: int = 0, *, jitter: float = 0.0) -> dict:
    """Seeded backbone atoms N, CA, C [B, L, 3] and the frames they were
    built from: CA on the 3.8 A walk, C at 1.52 A along the local x axis, N
    at 1.46 A in the local xy plane at 111 degrees from it (rounded textbook
    bond lengths and N-CA-C angle), then optional N(0, jitter) noise on N
    and C.  Draw order: rotations, walk, noise."""
    rng = np.random.Generator(np.random.PCG64(seed))
    R = random_rotations(rng, B * L).reshape(B, L, 3, 3)
    ca = np.stack([random_walk(rng, L) for _ in range(B)])
    ang = math.radians(111.0)
    c_loc = np.array([1.52, 0.0, 0.0])
    n_loc = 1.46 * np.array([math.cos(ang), math.sin(ang), 0.0])
    c = ca + np.einsum("blxy,y->blx", R, c_loc)
    n = ca + np.einsum("blxy,y->blx", R, n_loc)
    if jitter:
        n = n + jitter * rng.standard_normal(n.shape)
        c = c + jitter * rng.standard_normal(c.shape)
    f32 = lambda a: np.ascontiguousarray(a, dtype=np.float32)  # noqa: E731
    return {"n": f32(n), "ca": f32(ca), "c": f32(c), "rot": R, "trans": ca}


@dataclass(frozen=True)
class ModuleDims:
    """IPA layer around the core: the core's dims plus the width c_s of the
    single representation."""
    B: int = 1
    L: int = 512
    H: int = 12
    C: int = 16
    Pq: int = 4
    Pv: int = 8
    R: int = 2
    Cz: int = 128
    c_s: int = 384


def module_inputs(dims: ModuleDims, seed: int = 0, *, masked_tail_frac: float = 0.0, jitter: float = 0.0) -> dict:
    """Seeded inputs of the IPA layer: the core's frames, pair factors,
    w_bias, gamma and mask (as ipa_inputs draws them; its q / k / v / points
    are dropped), then s ~ N(0, 1) [B, L, c_s], W_in ~ N(0, 1 / c_s)
    [c_s, H (3 C + 3 (2 Pq + Pv))], b_in ~ N(0, 0.1^2), W_out ~ N(0, 1 / (H F))
    [H F, c_s] with F = C + 4 Pv + Cz, b_out ~ N(0, 0.1^2), in that order."""
    core = ipa_inputs(IpaDims(B=dims.B, L=dims.L, H=dims.H, C=dims.C, Pq=dims.Pq, Pv=dims.Pv, R=dims.R,
                              Cz=dims.Cz), seed, masked_tail_frac=masked_tail_frac, jitter=jitter)
    rng = np.random.Generator(np.random.PCG64(seed + 7919))
    width = dims.H * (3 * dims.C + 3 * (2 * dims.Pq + dims.Pv))
    F = dims.C + 4 * dims.Pv + dims.Cz
    f32 = lambda a: np.ascontiguousarray(a, dtype=np.float32)  # noqa: E731
    out = {k: core[k] for k in ("rot", "trans", "z1", "z2", "w_bias", "gamma", "mask")}
    out["s"] = f32(rng.standard_normal((dims.B, dims.L, dims.c_s)))
    out["w_in"] = f32(rng.standard_normal((dims.c_s, width)) / math.sqrt(dims.c_s))
    out["b_in"] = f32(0.1 * rng.standard_normal(width))
    out["w_out"] = f32(rng.standard_normal((dims.H * F, dims.c_s)) / math.sqrt(dims.H * F))
    out["b_out"] = f32(0.1 * rng.standard_normal(dims.c_s))
    out["dims"] = dims
    return out


# Named workloads.  Sizes follow the IPA module of AlphaFold-2-style models
# (12 heads, 16 scalar channels, 4 query / 8 value points) with a rank-2
# factorised pair representation of 128 channels.
IPA_PRESETS = {
    "tiny": (IpaDims(B=1, L=64, H=4, C=16, Pq=4, Pv=8, R=2, Cz=16), {}),
    "af2": (IpaDims(B=1, L=512, H=12, Cz=128), {"masked_tail_frac": 0.1}),
    "long2048": (IpaDims(B=1, L=2048, H=12, Cz=128), {}),
    "long4096": (IpaDims(B=1, L=4096, H=12, Cz=128), {}),
    "long8192": (IpaDims(B=1, L=8192, H=12, Cz=128), {}),
    "long16384": (IpaDims(B=1, L=16384, H=12, Cz=128), {}),
    "batched": (IpaDims(B=32, L=128, H=8, Cz=64), {"ragged": (64, 128), "jitter": 1.0}),
}


def ipa_preset(name: str, seed: int = 0) -> dict:
    dims, kw = IPA_PRESETS[name]
    return ipa_inputs(dims, seed, **kw)


GEO_PRESET = GeoDims(B=2, N=2048, H=8, M=4, Cout=256)


def geo_preset(seed: int = 0, **kw) -> dict:
    return geo_inputs(GEO_PRESET, seed, **kw)
