"""Guard bands around every buffer the library writes.

compute-sanitizer is not available to these tests, so out-of-bounds writes
are looked for directly: each output tensor and each workspace is carved out
of a larger device allocation whose 4 KB before and after the payload are
filled with the byte 0x7F.  After a call on ragged sizes (tile remainders of
1, 63, 65, 129 and 383 rows) the guard bytes must be untouched.  The payload
itself starts filled with 0x7F too, so a kernel that read workspace it had
not written first would also change its results, which are compared with a
call on ordinary (zero-initialised) buffers.

Every case runs twice: on the product library and on its bounds-checked
build, where each store index is checked against its buffer and an index
outside it raises IPA_ERR_BOUNDS from the plan's `check()`.
"""
import numpy as np
import pytest
import torch

from rna_structure_models_b200 import api
from rna_structure_models_b200.synth import (GeoDims, IpaDims, MeetDims, ModuleDims, backbone_inputs,
                                             geo_inputs, geo_upstream, ipa_inputs, meet_inputs, module_inputs)
from tests.gpu_util import checked_library, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(params=["product", "checked"], autouse=True)
def library_build(request):
    if request.param == "product":
        yield request.param
    else:
        with checked_library():
            yield request.param

GUARD = 4096
FILL = 0x7F
RAGGED = [1, 63, 65, 129, 383]


class Guarded:
    """Device buffers with guard bands; `check()` asserts they are intact."""

    def __init__(self, device="cuda"):
        self.device = device
        self.raws = []

    def bytes(self, nbytes):
        pad = (nbytes + 255) // 256 * 256
        raw = torch.full((GUARD + pad + GUARD,), FILL, dtype=torch.uint8, device=self.device)
        assert raw.data_ptr() % 256 == 0
        self.raws.append((raw, nbytes))
        return raw[GUARD:GUARD + nbytes]

    def f32(self, shape):
        n = int(np.prod(shape))
        return self.bytes(4 * n).view(torch.float32).view(*shape)

    def like(self, t):
        return None if t is None else self.f32(tuple(t.shape))

    def check(self):
        torch.cuda.synchronize()
        for raw, nbytes in self.raws:
            head = raw[:GUARD]
            tail = raw[GUARD + nbytes:]
            assert bool((head == FILL).all()), "write before the start of a buffer"
            assert bool((tail == FILL).all()), f"write past the end of a {nbytes}-byte buffer"


@pytest.mark.parametrize("L", RAGGED)
@pytest.mark.parametrize("Cz", [32, 64])      # R Cz = 64: single-CTA core; 128: CTA-pair core
def test_ipa_core_guard_bands(cuda_device, L, Cz):
    inp = ipa_inputs(IpaDims(B=2, L=L, H=3, Cz=Cz), 3)
    if L > 3:
        inp["mask"][1, L // 2:] = False
    dev = to_dev({k: inp[k] for k in api.IPA_INPUTS})
    ref = api.ipa_attn(dev)
    g = Guarded()
    plan = api.IpaPlan(2, L, 3, 16, 4, 8, 2, Cz, device="cuda")
    plan.workspace = g.bytes(plan.workspace.numel())
    out = g.f32(tuple(ref.shape))
    plan(*[dev[n] for n in api.IPA_INPUTS], out=out)
    g.check()
    plan.check()
    assert torch.equal(out, ref)


@pytest.mark.parametrize("N", RAGGED)
def test_variant_and_gradient_guard_bands(cuda_device, N):
    dims = GeoDims(B=2, N=N, H=3, M=4, Cout=40)
    raw = geo_inputs(dims, 5)
    inp = to_dev({k: v for k, v in raw.items() if k != "dims"})
    for k in api.GEO_INPUTS:
        inp.setdefault(k, None)
    ref = api.geo_attn(inp)
    g = Guarded()
    plan = api.GeoPlan(dims.B, dims.N, dims.H, dims.M, dims.Cout, device="cuda")
    plan.workspace = g.bytes(plan.workspace.numel())
    out = {k: g.like(v) for k, v in ref.items()}
    plan(inp, out=out)
    g.check()
    plan.check()
    for k in ref:
        assert torch.equal(out[k], ref[k]), k

    up = to_dev(geo_upstream(dims, 6))
    gref = api.geo_attn_backward(inp, up["g_output"], up.get("g_attention"), up.get("g_vectors"))
    g2 = Guarded()
    gplan = api.GeoGradPlan(dims.B, dims.N, dims.H, dims.M, dims.Cout, device="cuda")
    gplan.workspace = g2.bytes(gplan.workspace.numel())
    gout = {k: g2.like(v) for k, v in gref.items()}
    gplan(inp, up["g_output"], up.get("g_attention"), up.get("g_vectors"), out=gout)
    g2.check()
    gplan.check()
    for k in gref:
        if gref[k] is not None:
            assert torch.equal(gout[k], gref[k]), k


@pytest.mark.parametrize("L", RAGGED)
def test_meet_guard_bands(cuda_device, L):
    inp = to_dev({k: v for k, v in meet_inputs(MeetDims(B=2, L=L, H=4), 2).items() if k in api.MEET_INPUTS})
    ref = api.meet_attn(inp)
    g = Guarded()
    plan = api.MeetPlan(2, L, 4, device="cuda")
    plan.workspace = g.bytes(plan.workspace.numel())
    out = g.like(ref)
    plan(*[inp[n] for n in api.MEET_INPUTS], out=out)
    g.check()
    plan.check()
    assert torch.equal(out, ref)


@pytest.mark.parametrize("L", RAGGED)
def test_frames_guard_bands(cuda_device, L):
    bb = to_dev(backbone_inputs(2, L, 4, jitter=0.1))
    rot_ref, tr_ref = api.frames_from_backbone(bb["n"], bb["ca"], bb["c"])
    g = Guarded()
    rot, tr = g.like(rot_ref), g.like(tr_ref)
    api.frames_from_backbone(bb["n"], bb["ca"], bb["c"], rot=rot, trans=tr)
    g.check()
    assert torch.equal(rot, rot_ref) and torch.equal(tr, tr_ref)


@pytest.mark.parametrize("M,K,N", [(1, 7, 3), (63, 40, 65), (129, 96, 200), (383, 384, 131)])
def test_linear_guard_bands(cuda_device, M, K, N):
    gen = torch.Generator().manual_seed(M * 7 + N)
    x = torch.randn(M, K, generator=gen).cuda()
    w = torch.randn(K, N, generator=gen).cuda()
    b = torch.randn(N, generator=gen).cuda()
    ref = api.linear(x, w, b)
    g = Guarded()
    plan = api.LinearPlan(M, K, N, device="cuda")
    plan.workspace = g.bytes(plan.workspace.numel())
    y = g.f32((M, N))
    plan(x, w, b, out=y)
    g.check()
    plan.check()
    assert torch.equal(y, ref)


@pytest.mark.parametrize("L", [1, 65, 383])
def test_layer_guard_bands(cuda_device, L):
    dims = ModuleDims(B=2, L=L, H=3, Cz=32, c_s=48)
    inp = to_dev({k: v for k, v in module_inputs(dims, 8, masked_tail_frac=0.1).items() if k in api.MODULE_INPUTS})
    ref, ref_core = api.ipa_module(inp, with_core=True)
    g = Guarded()
    plan = api.ModulePlan(2, L, 3, 16, 4, 8, 2, 32, 48, device="cuda")
    plan.workspace = g.bytes(plan.workspace.numel())
    out, core = g.like(ref), g.like(ref_core)
    plan(inp, out=out, core_out=core)
    g.check()
    plan.check()
    assert torch.equal(out, ref) and torch.equal(core, ref_core)


@pytest.mark.parametrize("L", RAGGED)
@pytest.mark.parametrize("Cz", [32, 64])
def test_ipa_training_and_gradient_guard_bands(cuda_device, L, Cz):
    inp = ipa_inputs(IpaDims(B=2, L=L, H=3, Cz=Cz), 9)
    if L > 3:
        inp["mask"][1, L // 2:] = False
    dev = to_dev({k: inp[k] for k in api.IPA_INPUTS})
    ref_out, ref_lse, ref_u = api.ipa_attn_train(dev)
    gen = torch.Generator(device="cuda").manual_seed(L)
    g_out = torch.randn(ref_out.shape, device="cuda", generator=gen)
    ref = api.ipa_attn_backward(dev, ref_out, ref_lse, ref_u, g_out)
    g = Guarded()
    plan = api.IpaPlan(2, L, 3, 16, 4, 8, 2, Cz, device="cuda")
    plan.workspace = g.bytes(plan.workspace.numel())
    out, lse, u = g.like(ref_out), g.like(ref_lse), g.like(ref_u)
    plan.train(*[dev[n] for n in api.IPA_INPUTS], out=out, lse=lse, u_agg=u)
    g.check()
    plan.check()
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse) and torch.equal(u, ref_u)
    g2 = Guarded()
    gplan = api.IpaGradPlan(2, L, 3, 16, 4, 8, 2, Cz, device="cuda")
    gplan.workspace = g2.bytes(gplan.workspace.numel())
    grads = {k: g2.like(v) for k, v in ref.items()}
    gplan(dev, out, lse, u, g_out, grads=grads)
    g2.check()
    gplan.check()
    for k in ref:
        assert torch.equal(grads[k], ref[k]), k
