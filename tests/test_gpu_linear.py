"""Parity of the tensor-core projection y = x W + b (CUDA, through the C ABI)
with float64 matrix products.

The call multiplies fp32 operands on the tf32 path (rows of x and W 16-byte
aligned) and fp16 copies of them otherwise.  Tight check: y equals, to within
fp32 accumulation, the float64 product of the operands rounded as one of the
two paths rounds them (fp16 round-to-nearest; tf32, the tensor core reading
the top 19 bits: truncated or rounded to nearest).  Loose check: against the
unrounded fp32 operands to within that rounding (rel-Fro 2e-3)."""
import numpy as np
import pytest
import torch

from rna_structure_models_b200 import api

pytestmark = pytest.mark.gpu


def draw(M, K, N, seed, bias=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)).astype(np.float32)
    w = (rng.standard_normal((K, N)) / np.sqrt(K)).astype(np.float32)
    b = (0.1 * rng.standard_normal(N)).astype(np.float32) if bias else None
    return x, w, b


def tf32(a, nearest):
    """a (float32) with the low 13 mantissa bits dropped (truncated) or
    rounded to nearest even (finite values)."""
    u = a.astype(np.float32).view(np.uint32).astype(np.uint64)
    if nearest:
        u = u + 0xFFF + ((u >> 13) & 1)
    return (u & 0xFFFFE000).astype(np.uint32).view(np.float32)


def check(y, x, w, b):
    bias = 0.0 if b is None else b.astype(np.float64)
    candidates = {
        "fp16": (x.astype(np.float16), w.astype(np.float16)),
        "tf32 truncated": (tf32(x, False), tf32(w, False)),
        "tf32 nearest": (tf32(x, True), tf32(w, True)),
    }
    worst = {}
    for name, (xr, wr) in candidates.items():
        xr, wr = xr.astype(np.float64), wr.astype(np.float64)
        excess = np.abs(y - (xr @ wr + bias)) - (1e-4 * (np.abs(xr) @ np.abs(wr)) + 1e-6)
        worst[name] = float(np.max(excess))
    assert min(worst.values()) <= 0.0, worst
    ref = x.astype(np.float64) @ w.astype(np.float64) + bias
    rel = np.linalg.norm(y - ref) / max(np.linalg.norm(ref), 1e-30)
    assert rel <= 2e-3, rel


@pytest.mark.parametrize("M,K,N", [(1, 1, 1), (5, 17, 3), (128, 64, 128), (200, 96, 70), (300, 385, 257),
                                   (129, 640, 1000)])
def test_ragged_shapes(cuda_device, M, K, N):
    x, w, b = draw(M, K, N, M + K + N)
    y = api.linear(torch.from_numpy(x).cuda(), torch.from_numpy(w).cuda(), torch.from_numpy(b).cuda())
    check(y.cpu().numpy().astype(np.float64), x, w, b)


@pytest.mark.parametrize("M,K,N", [(4096, 384, 1152), (4096, 2112, 384)])
def test_module_projection_shapes(cuda_device, M, K, N):
    x, w, b = draw(M, K, N, 7)
    y = api.linear(torch.from_numpy(x).cuda(), torch.from_numpy(w).cuda(), torch.from_numpy(b).cuda())
    check(y.cpu().numpy().astype(np.float64), x, w, b)


def test_strided_operands_and_no_bias(cuda_device):
    x, w, _ = draw(150, 200, 90, 11, bias=False)
    xt = torch.from_numpy(np.ascontiguousarray(x.T)).cuda().t()          # column-major view of x
    wt = torch.from_numpy(np.ascontiguousarray(w.T)).cuda().t()
    assert not xt.is_contiguous() and not wt.is_contiguous()
    y = api.linear(xt, wt)
    check(y.cpu().numpy().astype(np.float64), x, w, None)


def test_plan_reuse_on_a_side_stream(cuda_device):
    x, w, b = draw(640, 256, 192, 12)
    plan = api.LinearPlan(640, 256, 192)
    s = torch.cuda.Stream()
    xd, wd, bd = (torch.from_numpy(a).cuda() for a in (x, w, b))
    s.wait_stream(torch.cuda.current_stream())
    out = torch.full((640, 192), float("nan"), device="cuda")
    for _ in range(3):
        plan(xd, wd, bd, out=out, stream=s)
    s.synchronize()
    plan.check()
    check(out.cpu().numpy().astype(np.float64), x, w, b)
