"""The bounds-checked build of the library (compiled with -DIPA_BOUNDS_CHECK).

In that build every pointer a kernel stores through to global memory comes
from a span checked against the extent of its buffer; a span outside it
records 0x10000 | (file tag << 12) | line in the error word and the store is
redirected to a scratch area.  Here:
  * a probe kernel shows the check itself: an index inside the buffer is
    stored, indices before and after it are reported with the site of the
    store and leave the buffer and its guard bands untouched;
  * every entry point, on ragged sizes, runs in the checked build without a
    report and with results equal bit for bit to the product build's (the
    checks change no arithmetic), which also covers the two calls that have
    no error word (frames, distogram): a redirected store would show up as a
    difference.
The guard-band tests run all their cases on the checked build as well.
"""
import ctypes
import os

import numpy as np
import pytest
import torch

from rna_structure_models_b200 import api, build
from rna_structure_models_b200.synth import (GeoDims, IpaDims, MeetDims, ModuleDims, backbone_inputs, geo_inputs,
                                             geo_upstream, ipa_inputs, meet_inputs, module_inputs, random_walk)
from tests.gpu_util import checked_library, to_dev

pytestmark = pytest.mark.gpu

GUARD = 4096


@pytest.fixture(scope="module")
def bounds_probe():
    if not os.path.exists(build.BOUNDS_PROBE_LIB):
        build.build_bounds_probe()
    lib = ctypes.CDLL(build.BOUNDS_PROBE_LIB)
    lib.probe_bounds_store.argtypes = [ctypes.c_void_p, ctypes.c_longlong, ctypes.c_longlong, ctypes.c_void_p,
                                       ctypes.c_void_p]
    lib.probe_bounds_store.restype = ctypes.c_int
    lib.probe_bounds_site.restype = ctypes.c_int
    return lib


@pytest.mark.parametrize("idx", [0, 5, 63, -1, 64, 65, 1 << 20, -(1 << 20)])
def test_store_check_reports_an_index_outside_the_buffer(cuda_device, bounds_probe, idx):
    n = 64
    raw = torch.full((GUARD + 4 * n + GUARD,), 0x7F, dtype=torch.uint8, device="cuda")
    buf = raw[GUARD:GUARD + 4 * n].view(torch.float32)
    before = raw.clone()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = bounds_probe.probe_bounds_store(buf.data_ptr(), n, idx, err.data_ptr(),
                                         torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rc == 0
    code = int(err.item())
    changed = (raw != before).nonzero().flatten().cpu().numpy()
    if 0 <= idx < n:
        assert code == 0
        assert float(buf[idx]) == 1.0
        assert list(changed) == list(range(GUARD + 4 * idx, GUARD + 4 * idx + 4))
    else:
        assert code == 0x10000 | bounds_probe.probe_bounds_site()
        assert (code >> 12) & 0xF == 15                     # the probe's file tag
        assert changed.size == 0, "a redirected store reached the buffer or its guard bands"
        lib = api.library()
        assert lib.ipa_device_error_status(code) == 9       # IPA_ERR_BOUNDS
        assert b"bounds" in lib.ipa_status_string(9)


def both_builds(fn):
    """fn() under the product library, then under the checked one; returns
    the two results (tensors copied to the host)."""
    def host(r):
        if isinstance(r, dict):
            return {k: host(v) for k, v in r.items()}
        if isinstance(r, (tuple, list)):
            return [host(v) for v in r]
        return None if r is None else r.detach().cpu()
    prod = host(fn())
    with checked_library():
        chk = host(fn())
    return prod, chk


def assert_same(a, b, what=""):
    if isinstance(a, dict):
        assert a.keys() == b.keys()
        for k in a:
            assert_same(a[k], b[k], f"{what}.{k}")
    elif isinstance(a, list):
        for i, (x, y) in enumerate(zip(a, b)):
            assert_same(x, y, f"{what}[{i}]")
    elif a is None:
        assert b is None, what
    else:
        assert torch.equal(a, b), f"{what}: the checked build differs from the product build"


@pytest.mark.parametrize("L", [1, 65, 383])
@pytest.mark.parametrize("Cz", [32, 64])
def test_ipa_forward_training_and_gradients(cuda_device, L, Cz):
    inp = ipa_inputs(IpaDims(B=2, L=L, H=3, Cz=Cz), 21)
    if L > 3:
        inp["mask"][1, L // 3:] = False
    dev = to_dev({k: inp[k] for k in api.IPA_INPUTS})

    def run():
        out = api.ipa_attn(dev)
        o, lse, u = api.ipa_attn_train(dev)
        g_out = torch.randn(o.shape, device="cuda", generator=torch.Generator(device="cuda").manual_seed(L))
        grads = api.ipa_attn_backward(dev, o, lse, u, g_out)
        return {"out": out, "train": [o, lse, u], "grads": grads}

    assert_same(*both_builds(run), "ipa")


def test_ipa_production_width_at_length_2048(cuda_device):
    """The pair kernel's production shape (R Cz = 256, TMA output pass), its
    key-split tail and the gradient passes at a length spanning many tiles,
    in both builds."""
    inp = ipa_inputs(IpaDims(B=1, L=2048, H=4, Cz=128), 31)
    inp["mask"][0, 2000:] = False
    dev = to_dev({k: inp[k] for k in api.IPA_INPUTS})

    def run():
        o, lse, u = api.ipa_attn_train(dev)
        g_out = torch.randn(o.shape, device="cuda", generator=torch.Generator(device="cuda").manual_seed(5))
        # the inference call splits its tiles' keys in two chunks (partial
        # accumulators, tickets, merge), the training call does not
        return {"infer": api.ipa_attn(dev), "train": [o, lse, u],
                "grads": api.ipa_attn_backward(dev, o, lse, u, g_out)}

    assert_same(*both_builds(run), "ipa L=2048")


@pytest.mark.parametrize("N", [1, 65, 383])
def test_variant_forward_and_gradients(cuda_device, N):
    dims = GeoDims(B=2, N=N, H=3, M=4, Cout=40)
    raw = geo_inputs(dims, 22)
    inp = to_dev({k: v for k, v in raw.items() if k != "dims"})
    for k in api.GEO_INPUTS:
        inp.setdefault(k, None)
    up = to_dev(geo_upstream(dims, 23))

    def run():
        out = api.geo_attn(inp)
        grads = api.geo_attn_backward(inp, up["g_output"], up.get("g_attention"), up.get("g_vectors"))
        return {"fwd": out, "grads": grads}

    assert_same(*both_builds(run), "geo")


@pytest.mark.parametrize("L", [1, 129])
def test_meet_layer_frames_linear_distogram(cuda_device, L):
    meet = to_dev({k: v for k, v in meet_inputs(MeetDims(B=2, L=L, H=4), 24).items() if k in api.MEET_INPUTS})
    mdims = ModuleDims(B=2, L=L, H=3, Cz=32, c_s=48)
    layer = to_dev({k: v for k, v in module_inputs(mdims, 25, masked_tail_frac=0.1).items()
                    if k in api.MODULE_INPUTS})
    bb = to_dev(backbone_inputs(2, L, 26, jitter=0.1))
    gen = torch.Generator().manual_seed(L)
    x = torch.randn(L + 2, 96, generator=gen).cuda()
    w = torch.randn(96, 131, generator=gen).cuda()
    b = torch.randn(131, generator=gen).cuda()
    rng = np.random.default_rng(L)
    pos = torch.from_numpy(np.stack([random_walk(rng, L) for _ in range(2)]).astype(np.float32)).cuda()
    pmask = torch.ones((2, L), dtype=torch.bool, device="cuda")
    pmask[1, L // 2:] = False

    def run():
        return {"meet": api.meet_attn(meet),
                "layer": list(api.ipa_module(layer, with_core=True)),
                "frames": list(api.frames_from_backbone(bb["n"], bb["ca"], bb["c"])),
                "linear": api.linear(x, w, b),
                "distogram": list(api.knn_distogram(pos, pmask, 8, [2.0, 3.5, 5.0, 8.0, 12.0]))}

    assert_same(*both_builds(run), "rest")
