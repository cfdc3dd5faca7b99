"""Pins of the IPA-layer oracle (projections around the core, Flash Invariant
Point Attention): the core output equals the core oracle on explicitly
projected inputs, brute-force loops for the two projections, SE(3)
invariance, and the column order of the input projection."""
import numpy as np

from oracle import ipa_dense, ipa_module, projection_width, split_projection
from rna_structure_models_b200.synth import ModuleDims, module_inputs, random_rotations

TINY = ModuleDims(B=2, L=9, H=2, C=4, Pq=2, Pv=3, R=2, Cz=4, c_s=6)


def test_projection_loops_and_core_by_hand():
    inp = module_inputs(TINY, 0, masked_tail_frac=0.2)
    d = TINY
    out, core = ipa_module(inp, return_core=True)
    s, W, b = (inp[k].astype(np.float64) for k in ("s", "w_in", "b_in"))
    width = projection_width(d.H, d.C, d.Pq, d.Pv)
    Y = np.zeros((d.B, d.L, width))
    for bb in range(d.B):
        for i in range(d.L):
            for c in range(width):
                Y[bb, i, c] = b[c] + sum(s[bb, i, k] * W[k, c] for k in range(d.c_s))
    # q of head h, channel c sits at column h*C + c; q_pts of head h, point p, axis x at 3HC + (h*Pq + p)*3 + x
    sp = split_projection(Y, d.H, d.C, d.Pq, d.Pv)
    assert np.array_equal(sp["q"][0, 1, 1, 2], Y[0, 1, 1 * d.C + 2])
    assert np.array_equal(sp["q_pts"][1, 3, 1, 0, 2], Y[1, 3, 3 * d.H * d.C + (1 * d.Pq + 0) * 3 + 2])
    assert np.array_equal(sp["v_pts"][0, 0, 0, 2, 1],
                          Y[0, 0, 3 * d.H * d.C + 2 * d.H * d.Pq * 3 + 2 * 3 + 1])
    core_inp = dict(sp, **{k: inp[k] for k in ("rot", "trans", "z1", "z2", "w_bias", "gamma", "mask")})
    assert np.allclose(core, ipa_dense(core_inp), atol=1e-12)
    F = d.C + 4 * d.Pv + d.Cz
    Wo, bo = inp["w_out"].astype(np.float64), inp["b_out"].astype(np.float64)
    flat = core.reshape(d.B, d.L, d.H * F)
    for bb in range(d.B):
        for i in range(d.L):
            for c in range(d.c_s):
                ref = bo[c] + sum(flat[bb, i, k] * Wo[k, c] for k in range(d.H * F))
                assert abs(out[bb, i, c] - ref) <= 1e-12 * max(1.0, abs(ref))


def test_invariant_under_a_global_rigid_motion():
    inp = module_inputs(ModuleDims(B=1, L=24, H=3, C=8, Pq=2, Pv=2, R=2, Cz=8, c_s=16), 1)
    rng = np.random.default_rng(2)
    G = random_rotations(rng, 1)[0]
    t = rng.normal(size=3) * 30
    moved = dict(inp, rot=np.einsum("xy,blyz->blxz", G, inp["rot"]), trans=inp["trans"] @ G.T + t)
    assert np.allclose(ipa_module(moved), ipa_module(inp), atol=1e-9)


def test_single_representation_drives_the_output():
    inp = module_inputs(TINY, 3)
    other = dict(inp, s=inp["s"] + 1.0)
    assert not np.allclose(ipa_module(other), ipa_module(inp))
