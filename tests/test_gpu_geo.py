"""Parity of the geometric direction/distance attention (CUDA, through the
C ABI) with the float64 oracle."""
import numpy as np
import pytest
import torch

from oracle import geo_dense, geo_dense_blocked
from rna_structure_models_b200 import api
from rna_structure_models_b200.synth import GeoDims, geo_inputs, geo_preset, random_rotations
from tests.gpu_util import GEO_MAX_ABS, GEO_REL_FRO, assert_parity, to_dev

pytestmark = pytest.mark.gpu


def run_gpu(inp, with_attention=True, dtype=torch.float32):
    dev = to_dev({k: inp.get(k) for k in api.GEO_INPUTS}, dtype=dtype)
    for k in api.GEO_INPUTS:
        dev.setdefault(k, None)
    res = api.geo_attn(dev, with_attention=with_attention)
    torch.cuda.synchronize()
    return {k: (v.cpu().numpy() if v is not None else None) for k, v in res.items()}


def check(gpu, ref, what, att=True):
    v, a, o = ref
    assert_parity(gpu["vectors"], v, GEO_MAX_ABS, GEO_REL_FRO, what + " vectors")
    assert_parity(gpu["output"], o, GEO_MAX_ABS, GEO_REL_FRO, what + " output")
    if att:
        assert_parity(gpu["attention"], a, GEO_MAX_ABS, GEO_REL_FRO, what + " attention")


@pytest.mark.parametrize("N,M", [(1, 1), (7, 2), (64, 4), (100, 3), (257, 8)])
def test_small_parity(cuda_device, N, M):
    inp = geo_inputs(GeoDims(B=2, N=N, H=3, M=M, Cout=11), N)
    check(run_gpu(inp), geo_dense(inp), f"N={N}")


def test_full_workload_sampled_rows(cuda_device):
    inp = geo_preset(0)
    gpu = run_gpu(inp)
    rows = np.unique(np.concatenate([[0, 1, 2047], np.random.default_rng(2).choice(2048, 125, replace=False)]))
    v, a, o = geo_dense_blocked(inp, rows=rows, block=64)
    check({"vectors": gpu["vectors"][:, rows], "output": gpu["output"][:, rows],
           "attention": gpu["attention"][:, :, rows]}, (v, a, o), "N=2048")
    # attention rows of valid queries sum to one
    s = gpu["attention"].sum(-1)
    live = s > 0
    assert np.abs(s[live] - 1).max() < 1e-4


def test_without_attention_map_and_without_mask_or_bias(cuda_device):
    inp = geo_inputs(GeoDims(B=1, N=300, H=4, M=2, Cout=9), 3, with_pair_mask=False, with_bias=False)
    gpu = run_gpu(inp, with_attention=False)
    assert gpu["attention"] is None
    check(gpu, geo_dense(inp), "no-mask", att=False)


def test_float64_inputs(cuda_device):
    inp = geo_inputs(GeoDims(B=1, N=90, H=2, M=2, Cout=5), 4)
    check(run_gpu(inp, dtype=torch.float64), geo_dense(inp), "fp64")


def test_broadcast_pair_mask(cuda_device):
    inp = geo_inputs(GeoDims(B=2, N=80, H=3, M=2, Cout=4), 5, with_pair_mask=False)
    pm = np.random.default_rng(5).random((1, 1, 80, 80)) > 0.3
    inp["pair_mask"] = pm
    ref = geo_dense(inp)
    dev = to_dev({k: inp.get(k) for k in api.GEO_INPUTS})
    dev["pair_mask"] = torch.from_numpy(pm).cuda().expand(2, 3, 80, 80)   # stride-0 broadcast
    res = api.geo_attn(dev)
    gpu = {k: v.cpu().numpy() for k, v in res.items()}
    check(gpu, ref, "broadcast")


def test_empty_rows_and_heads(cuda_device):
    inp = geo_inputs(GeoDims(B=1, N=70, H=3, M=2, Cout=6), 6)
    inp["frame_mask"][0, 10] = False
    inp["pair_mask"][0, :, 20, :] = False      # no head allowed: output must be 0, not the bias
    inp["pair_mask"][0, 1, 30, :] = False      # one head empty: exact zeros in that head
    gpu = run_gpu(inp)
    assert np.all(gpu["output"][0, 10] == 0) and np.all(gpu["output"][0, 20] == 0)
    assert np.all(gpu["vectors"][0, 30, 1] == 0) and np.all(gpu["attention"][0, 1, 30] == 0)
    check(gpu, geo_dense(inp), "empty")


def test_invariance(cuda_device):
    inp = geo_inputs(GeoDims(B=1, N=200, H=4, M=3, Cout=7), 7)
    base = run_gpu(inp)
    rng = np.random.default_rng(8)
    G = random_rotations(rng, 1)[0]
    mv = dict(inp)
    mv["rotation"] = np.einsum("xy,bnyz->bnxz", G, inp["rotation"].astype(float)).astype(np.float32)
    mv["translation"] = (inp["translation"].astype(float) @ G.T + rng.normal(size=3) * 20).astype(np.float32)
    out = run_gpu(mv)
    for k in ("vectors", "output", "attention"):
        rel = np.linalg.norm(out[k] - base[k]) / np.linalg.norm(base[k])
        assert rel < 1e-4, (k, rel)


def test_noncontiguous_inputs_and_untouched(cuda_device):
    inp = geo_inputs(GeoDims(B=1, N=50, H=2, M=2, Cout=5), 9)
    dev = to_dev({k: inp.get(k) for k in api.GEO_INPUTS})
    ref = {k: v.clone() for k, v in api.geo_attn(dev).items()}
    nc = {}
    for k, t in dev.items():
        if t is not None and t.dim() >= 2:
            perm = list(range(t.dim()))[::-1]
            nc[k] = t.permute(perm).contiguous().permute(np.argsort(perm).tolist())
        else:
            nc[k] = t
    before = {k: v.clone() for k, v in nc.items() if v is not None}
    out = api.geo_attn(nc)
    for k in ref:
        assert torch.equal(out[k], ref[k]), k
    for k, v in before.items():
        assert torch.equal(nc[k], v), k
