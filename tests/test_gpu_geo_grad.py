"""Parity of the variant's gradients ("Geometric direction-and-distance
attention", Required behavior: gradients, zero distance derivative at a zero
displacement) computed by the CUDA kernels through the C ABI, with the
float64 gradient oracle on the same seeded inputs and upstream gradients."""
import numpy as np
import pytest
import torch

from oracle import geo_grad
from rna_structure_models_b200 import api
from rna_structure_models_b200.synth import GeoDims, geo_inputs, geo_preset, geo_upstream, random_rotations
from tests.gpu_util import assert_parity, to_dev

pytestmark = pytest.mark.gpu

# fp32 kernels, sums of up to N pair terms: bounds relative to the largest
# gradient entry (max-abs) and to the gradient's norm (rel-Fro)
GRAD_MAX_ABS = 2e-4
GRAD_REL_FRO = 2e-5


def gpu_grads(inp, up, dtype=torch.float32):
    dev = to_dev({k: inp.get(k) for k in api.GEO_INPUTS}, dtype=dtype)
    for k in api.GEO_INPUTS:
        dev.setdefault(k, None)
    u = to_dev({k: v for k, v in up.items() if v is not None}, dtype=dtype)
    g = api.geo_attn_backward(dev, u["g_output"], u.get("g_attention"), u.get("g_vectors"))
    torch.cuda.synchronize()
    return {k: (v.cpu().numpy() if v is not None else None) for k, v in g.items()}


def check(gpu, ref, what):
    for k, r in ref.items():
        if r is None:
            assert gpu[k] is None, k
            continue
        scale = max(1.0, float(np.max(np.abs(r))))
        assert_parity(gpu[k], r, GRAD_MAX_ABS * scale, GRAD_REL_FRO, f"{what} d{k}")


@pytest.mark.parametrize("N,M", [(1, 1), (7, 2), (64, 4), (129, 3), (300, 8)])
def test_parity_small_and_ragged(cuda_device, N, M):
    dims = GeoDims(B=2, N=N, H=3, M=M, Cout=11)
    inp = geo_inputs(dims, N, frame_drop=0.1)
    up = geo_upstream(dims, N + 1)
    check(gpu_grads(inp, up), geo_grad(inp, **up), f"N={N} M={M}")


@pytest.mark.parametrize("with_att,with_vec", [(False, False), (True, False), (False, True)])
def test_optional_upstream_gradients(cuda_device, with_att, with_vec):
    dims = GeoDims(B=1, N=96, H=4, M=2, Cout=8)
    inp = geo_inputs(dims, 3)
    up = geo_upstream(dims, 4, with_attention=with_att, with_vectors=with_vec)
    check(gpu_grads(inp, up), geo_grad(inp, **up), f"att={with_att} vec={with_vec}")


def test_no_bias_no_pair_mask(cuda_device):
    dims = GeoDims(B=2, N=80, H=2, M=4, Cout=16)
    inp = geo_inputs(dims, 5, with_pair_mask=False, with_bias=False)
    up = geo_upstream(dims, 6)
    gpu = gpu_grads(inp, up)
    assert gpu["output_bias"] is None
    check(gpu, geo_grad(inp, **up), "no bias")


def test_broadcast_pair_mask_and_dead_queries(cuda_device):
    dims = GeoDims(B=2, N=70, H=3, M=2, Cout=5)
    inp = geo_inputs(dims, 7, with_pair_mask=False)
    pm = np.random.default_rng(8).random((1, 3, 1, 70)) > 0.3        # per-head key exclusion
    inp["pair_mask"] = np.ascontiguousarray(np.broadcast_to(pm, (1, 3, 70, 70)))
    inp["frame_mask"][1, :5] = False
    up = geo_upstream(dims, 9)
    ref = geo_grad(dict(inp, pair_mask=pm), **up)
    dev_inp = dict(inp)
    dev_inp["pair_mask"] = pm                                         # stride-0 broadcast on the device
    dev = to_dev({k: dev_inp.get(k) for k in api.GEO_INPUTS})
    dev["pair_mask"] = dev["pair_mask"].expand(2, 3, 70, 70)
    u = to_dev(up)
    g = api.geo_attn_backward(dev, u["g_output"], u["g_attention"], u["g_vectors"])
    gpu = {k: (v.cpu().numpy() if v is not None else None) for k, v in g.items()}
    check(gpu, ref, "broadcast mask")
    assert np.all(gpu["q_direction"][1, :5] == 0.0) and np.all(gpu["values"][1, :5] == 0.0)


def test_zero_displacement(cuda_device):
    dims = GeoDims(B=1, N=40, H=2, M=2, Cout=4)
    inp = geo_inputs(dims, 10, with_pair_mask=False, frame_drop=0.0)
    inp["rotation"][0, 3] = np.eye(3, dtype=np.float32)
    inp["rotation"][0, 8] = np.eye(3, dtype=np.float32)
    inp["translation"][0, 3] = 0.0
    inp["translation"][0, 8] = 0.0
    inp["k_point"][0, 8, 1] = inp["q_point"][0, 3, 1]        # qp_3 = kp_8 exactly in fp32 and fp64
    up = geo_upstream(dims, 11)
    gpu = gpu_grads(inp, up)
    assert all(np.all(np.isfinite(v)) for v in gpu.values() if v is not None)
    check(gpu, geo_grad(inp, **up), "zero displacement")


def test_float64_inputs_and_strided_views(cuda_device):
    dims = GeoDims(B=2, N=50, H=3, M=3, Cout=6)
    inp = geo_inputs(dims, 12)
    up = geo_upstream(dims, 13)
    ref = geo_grad(inp, **up)
    check(gpu_grads(inp, up, dtype=torch.float64), ref, "f64")
    dev = to_dev({k: inp.get(k) for k in api.GEO_INPUTS})
    # q_direction as a view with the head axis outermost
    qd = dev["q_direction"].permute(2, 0, 1, 3).contiguous().permute(1, 2, 0, 3)
    assert not qd.is_contiguous()
    dev["q_direction"] = qd
    u = to_dev(up)
    g = api.geo_attn_backward(dev, u["g_output"], u["g_attention"].transpose(2, 3).contiguous().transpose(2, 3),
                              u["g_vectors"])
    check({k: (v.cpu().numpy() if v is not None else None) for k, v in g.items()}, ref, "strided")


def test_medium_size_full_parity(cuda_device):
    dims = GeoDims(B=1, N=512, H=8, M=4, Cout=64)
    inp = geo_inputs(dims, 14)
    up = geo_upstream(dims, 15)
    check(gpu_grads(inp, up), geo_grad(inp, **up), "N=512")


def test_full_workload_covariance_under_rigid_motion(cuda_device):
    inp = geo_preset(0)
    dims = inp["dims"]
    up = geo_upstream(dims, 16)
    g = gpu_grads(inp, up)
    assert all(np.all(np.isfinite(v)) for v in g.values() if v is not None)
    rng = np.random.default_rng(17)
    G = random_rotations(rng, 1)[0]
    moved = dict(inp, rotation=np.einsum("xy,bnyz->bnxz", G, inp["rotation"]).astype(np.float32),
                 translation=(inp["translation"] @ G.T + rng.normal(size=3) * 5).astype(np.float32))
    gm = gpu_grads(moved, up)
    for k in ("q_direction", "k_direction", "q_point", "k_point", "values", "direction_scale",
              "distance_scale", "output_weight", "output_bias"):
        scale = max(1.0, float(np.max(np.abs(g[k]))))
        assert np.max(np.abs(gm[k] - g[k])) <= 2e-3 * scale, k
    scale = max(1.0, float(np.max(np.abs(g["rotation"]))))
    assert np.max(np.abs(gm["rotation"] - np.einsum("xy,bnyz->bnxz", G, g["rotation"]))) <= 2e-3 * scale
    scale = max(1.0, float(np.max(np.abs(g["translation"]))))
    assert np.max(np.abs(gm["translation"] - g["translation"] @ G.T)) <= 2e-3 * scale
