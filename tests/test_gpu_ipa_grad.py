"""Gradients of the fused IPA core on the GPU (training forward + backward,
through the C ABI) against the float64 gradient oracle on the same seeded
inputs and upstream gradients.

Bounds (fixed before the first GPU run, from the arithmetic): every gradient
tensor within rel-Fro 2e-3 and max-abs 1e-2 * max(1, max|reference|) of the
oracle, the Frobenius norm of the reference floored at sqrt(size) (an RMS of
1).  (The floors were added after the first runs: with one residue the
softmax has a single key, so the exact gradients of q and of the
translations are identically zero, which no bound relative to them can hold;
the upstream gradients are N(0, 1), so 1 is their scale.  The variant's
gradient bound has the same form.)
The kernels' operands are the forward's fp16 rows (2^-11 relative rounding)
plus fp16 dS / P / dO / dU; a CPU model of exactly this decomposition reached
rel-Fro 2e-4 .. 5e-4, so 2e-3 leaves a 4x margin.
d gamma is the exception: one number per head, the signed sum over every
allowed pair of dl_ij |gq_i - gk_j|^2 (dl = a (da - D)), which cancels to
10^-4 .. 10^-1 of the size of its terms.  Every term carries the operands'
fp16 roundings, so no arithmetic on fp16 operands reaches 2e-3 of the sum
itself (the CPU model of the decomposition gives 3e-3 at L = 65 with dS
exact, 6e-3 with dS rounded to fp16).  Its bound is the usual relative-plus-absolute form for a sum,
|error_h| <= 2e-3 |d gamma_h| + 2^-11 R_h, where 2^-11 is the fp16 unit
roundoff and R_h the root-sum-square of the terms' magnitudes
(ipa_grad_gamma_scale: errors without a common sign add in quadrature); the
CPU model stays within 1.1e-4 R_h.  The training forward's
statistics (log-sum-exp, pair aggregate U) are held to the forward output's
bounds (max-abs 2e-2, rel-Fro 5e-3).
"""
import os

import numpy as np
import pytest
import torch

from oracle import ipa_dense, ipa_forward_stats, ipa_grad, ipa_grad_gamma_scale
from oracle.ipa_grad_blocked import ipa_grad_blocked
from rna_structure_models_b200 import api
from rna_structure_models_b200.synth import IpaDims, ipa_inputs, ipa_preset, random_rotations
from tests.gpu_util import assert_parity, errors, to_dev

pytestmark = pytest.mark.gpu

GRAD_REL_FRO = 2e-3
GRAD_MAX_REL = 1e-2
GAMMA_ABS = 2.0 ** -11        # fp16 unit roundoff, times the root-sum-square of d gamma's terms


def upstream(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape).astype(np.float32)


def run_gpu(inp, g):
    dev = to_dev({k: inp[k] for k in api.IPA_INPUTS})
    out, lse, U = api.ipa_attn_train(dev)
    grads = api.ipa_attn_backward(dev, out, lse, U, torch.from_numpy(g).cuda())
    torch.cuda.synchronize()
    return out, lse, U, {k: v.cpu().numpy() for k, v in grads.items()}


def assert_grads(got, ref, what, keys=None, gamma_scale=None):
    for key in (keys or api.IPA_GRADS):
        g, r = np.asarray(got[key], np.float64), np.asarray(ref[key], np.float64)
        assert np.all(np.isfinite(g)), f"{what} {key}: non-finite"
        if key == "gamma":
            assert gamma_scale is not None, "d gamma needs its scale (ipa_grad_gamma_scale)"
            bound = GRAD_REL_FRO * np.abs(r) + GAMMA_ABS * np.asarray(gamma_scale, np.float64)
            err = np.abs(g - r)
            log = os.environ.get("PARITY_LOG")
            if log:
                with open(log, "a") as f:
                    f.write(f"grad {what} gamma\terr/bound={float(np.max(err / bound)):.3e}\n")
            assert np.all(err <= bound), f"{what} gamma: error {err} above {bound} (ref {r})"
            continue
        m, _ = errors(g, r)
        rf = float(np.linalg.norm(g - r) / max(float(np.linalg.norm(r)), np.sqrt(r.size)))
        scale = max(float(np.max(np.abs(r))), 1.0)
        log = os.environ.get("PARITY_LOG")
        if log:
            with open(log, "a") as f:
                f.write(f"grad {what} {key}\tmax_abs/max|ref|={m / scale:.3e}\trel_fro={rf:.3e}\n")
        assert m <= GRAD_MAX_REL * scale and rf <= GRAD_REL_FRO, \
            f"{what} {key}: max-abs {m:.3e} (max|ref| {scale:.3e}), rel-Fro {rf:.3e}"


@pytest.mark.parametrize("name", ["tiny", "af2", "batched"])
def test_training_forward_statistics(cuda_device, name):
    inp = ipa_preset(name)
    dev = to_dev({k: inp[k] for k in api.IPA_INPUTS})
    out, lse, U = api.ipa_attn_train(dev)
    torch.cuda.synchronize()
    # the training forward runs every pair tile whole; the inference forward
    # may run the last, partial wave as key chunks whose P is rounded against
    # each chunk's own maximum, so the two agree within the rounding of P
    # (bit for bit where no tile is split, as in the tiny preset)
    inf = api.ipa_attn(dev)
    rel = float((out - inf).norm() / out.norm())
    assert rel < 1e-3, rel
    if name == "tiny":
        assert torch.equal(out, inf)
    lse_ref, U_ref = ipa_forward_stats(inp)
    lse_g = lse.cpu().numpy()
    live = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse_g), live)
    assert_parity(lse_g[live], lse_ref[live], what=f"lse {name}")
    assert_parity(U.cpu().numpy(), U_ref, what=f"U {name}")


@pytest.mark.parametrize("name", ["tiny", "af2", "batched"])
def test_gradients_presets(cuda_device, name):
    inp = ipa_preset(name)
    B, L, H = inp["q"].shape[:3]
    F = 16 + 32 + inp["z1"].shape[3]
    g = upstream((B, L, H, F), 21)
    _, _, _, got = run_gpu(inp, g)
    ref = ipa_grad(inp, g) if L <= 128 else ipa_grad_blocked(inp, g, block=32)
    assert_grads(got, ref, name, gamma_scale=ipa_grad_gamma_scale(inp, g))


@pytest.mark.parametrize("Cz", [16, 32, 64])    # pair widths 64 (3 stages), 64, 128
@pytest.mark.parametrize("L", [1, 2, 63, 65, 129, 200])
def test_gradients_ragged(cuda_device, L, Cz):
    inp = ipa_inputs(IpaDims(B=2, L=L, H=3, Cz=Cz), 31)
    if L > 3:
        inp["mask"][1, L // 2:] = False
        inp["mask"][0, 1] = False
    g = upstream((2, L, 3, 48 + Cz), 32)
    _, _, _, got = run_gpu(inp, g)
    assert_grads(got, ipa_grad(inp, g), f"L={L} Cz={Cz}", gamma_scale=ipa_grad_gamma_scale(inp, g))


def test_gradients_dead_rows_and_empty_batch(cuda_device):
    inp = ipa_inputs(IpaDims(B=3, L=70, H=2, Cz=32), 33)
    inp["mask"][0, :] = False
    inp["mask"][1, :] = False
    inp["mask"][1, 40] = True
    g = upstream((3, 70, 2, 80), 34)
    _, lse, _, got = run_gpu(inp, g)
    assert torch.isinf(lse[0]).all() and torch.isinf(lse[1, :, :40]).all()
    for key in ("q", "k", "v", "q_pts", "k_pts", "v_pts", "rot", "trans", "z1", "z2"):
        assert np.all(got[key][0] == 0), key
    assert_grads(got, ipa_grad(inp, g), "dead rows", gamma_scale=ipa_grad_gamma_scale(inp, g))


def test_gradient_of_a_zero_point_norm(cuda_device):
    # one residue with zero value points: o_pt = R^T (R 0 + t - t) = 0 exactly,
    # where the derivative of |o_pt| is taken as 0
    inp = ipa_inputs(IpaDims(B=1, L=1, H=2, Cz=16), 35)
    inp["v_pts"][:] = 0.0
    g = upstream((1, 1, 2, 64), 36)
    out, _, _, got = run_gpu(inp, g)
    assert np.all(out.cpu().numpy()[..., 16:48] == 0.0)
    assert_grads(got, ipa_grad(inp, g), "zero norm", gamma_scale=ipa_grad_gamma_scale(inp, g))


def test_gradients_strided_inputs_match_contiguous(cuda_device):
    inp = ipa_inputs(IpaDims(B=2, L=96, H=4, Cz=48), 37)
    g = upstream((2, 96, 4, 96), 38)
    dev = to_dev({k: inp[k] for k in api.IPA_INPUTS})
    out, lse, U = api.ipa_attn_train(dev)
    gt = torch.from_numpy(g).cuda()
    ref = api.ipa_attn_backward(dev, out, lse, U, gt)
    nc = {}
    for k_, t in dev.items():
        if t.dim() >= 2:
            perm = list(range(t.dim()))[::-1]
            nc[k_] = t.permute(perm).contiguous().permute(np.argsort(perm).tolist())
        else:
            nc[k_] = torch.stack([t, t], 1)[:, 0]
    gnc = gt.permute(3, 2, 1, 0).contiguous().permute(3, 2, 1, 0)
    got = api.ipa_attn_backward(nc, out, lse, U, gnc)
    torch.cuda.synchronize()
    for key in api.IPA_GRADS:
        assert torch.equal(got[key], ref[key]), key


def test_gradients_are_reproducible(cuda_device):
    inp = ipa_preset("af2")
    g = upstream((1, 512, 12, 176), 39)
    a = run_gpu(inp, g)[3]
    b = run_gpu(inp, g)[3]
    for key in api.IPA_GRADS:
        assert np.array_equal(a[key], b[key]), key


def test_gradients_with_the_key_pass_split(cuda_device):
    """B = 2, L = 512, H = 12: 96 query-pass and 96 key-pass CTAs, one per SM
    on 148 SMs, leave a last wave of 44 key-pass CTAs.  Each of those runs as
    two chunks of its 16 query tiles (the reserve holds 96 chunks); the chunk
    that finishes last adds the partial sums in chunk order.  Every gradient against the oracle, and the
    same bits on a second call whichever chunk finishes last."""
    inp = ipa_inputs(IpaDims(B=2, L=512, H=12, Cz=128), 47)
    inp["mask"][1, 400:] = False
    g = upstream((2, 512, 12, 176), 48)
    got = run_gpu(inp, g)[3]
    again = run_gpu(inp, g)[3]
    for key in api.IPA_GRADS:
        assert np.array_equal(got[key], again[key]), key
    ref = ipa_grad_blocked(inp, g, block=32)
    assert_grads(got, ref, "key-pass split", gamma_scale=ipa_grad_gamma_scale(inp, g))


def sampled_query_rows(inp, L, n):
    t = inp["trans"][0] - inp["trans"][0].mean(0)
    far = np.argsort(-np.linalg.norm(t, axis=1))[:8]
    edges = [0, 63, 64, 127, 128, L // 2, L - 65, L - 1]
    rnd = np.random.default_rng(5).choice(L, n, replace=False)
    return np.unique(np.concatenate([far, edges, rnd]))


def test_long_context_query_gradients_and_invariants(cuda_device):
    # L = 4096, H = 12, R Cz = 256 (the long-context workload).  The query-side
    # gradients of a residue (q, q_pts) depend on its own row alone, so the
    # oracle computes them exactly for sampled rows; the rest is held to
    # properties that hold at any size: the loss is invariant under a global
    # translation (sum_i d trans_i = 0) and every gradient transforms
    # covariantly under a global rigid motion.
    L = 4096
    inp = ipa_inputs(IpaDims(B=1, L=L, H=12), 0)
    g = upstream((1, L, 12, 176), 40)
    _, _, _, got = run_gpu(inp, g)
    rows = sampled_query_rows(inp, L, 24)
    ref = ipa_grad_blocked(inp, g, rows=rows, block=16)
    assert_grads({k: got[k][:, rows] for k in ("q", "q_pts")}, {k: ref[k][:, rows] for k in ("q", "q_pts")},
                 "L=4096 sampled rows", keys=("q", "q_pts"))
    dt = got["trans"].astype(np.float64)
    assert np.linalg.norm(dt.sum(axis=1)) <= 1e-3 * np.abs(dt).sum(axis=1).max()
    rng = np.random.default_rng(41)
    G = random_rotations(rng, 1)[0]
    moved = dict(inp)
    moved["rot"] = np.einsum("xy,blyz->blxz", G, inp["rot"].astype(np.float64)).astype(np.float32)
    moved["trans"] = (inp["trans"].astype(np.float64) @ G.T + rng.normal(size=3) * 20.0).astype(np.float32)
    _, _, _, mv = run_gpu(moved, g)
    for key in ("q", "k", "v", "q_pts", "k_pts", "v_pts", "z1", "z2", "w_bias", "gamma"):
        m, rf = errors(mv[key], got[key])
        log = os.environ.get("PARITY_LOG")
        if log:
            with open(log, "a") as f:
                f.write(f"grad L=4096 moved {key}\trel_fro={rf:.3e}\n")
        assert rf <= GRAD_REL_FRO, (key, rf)
    m, rf = errors(mv["trans"], got["trans"] @ G.T)
    assert rf <= GRAD_REL_FRO, ("trans", rf)
    m, rf = errors(mv["rot"], np.einsum("xy,blyz->blxz", G, got["rot"]))
    assert rf <= GRAD_REL_FRO, ("rot", rf)
