"""Parity of the tensor-core projection y = x W + b (CUDA, through the C ABI)
with float64 matrix products: against the fp16-rounded operands (the kernel's
own inputs) to within fp32 accumulation, and against the unrounded fp32
operands to within the fp16 rounding of x and W."""
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


def check(y, x, w, b):
    x16 = x.astype(np.float16).astype(np.float64)
    w16 = w.astype(np.float16).astype(np.float64)
    ref16 = x16 @ w16 + (0.0 if b is None else b.astype(np.float64))
    bound = np.abs(x16) @ np.abs(w16)
    assert np.all(np.abs(y - ref16) <= 1e-4 * bound + 1e-6), float(np.max(np.abs(y - ref16) - 1e-4 * bound))
    ref = x.astype(np.float64) @ w.astype(np.float64) + (0.0 if b is None else b)
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
