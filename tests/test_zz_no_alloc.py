"""The allocation-free geometric-attention entry point (geo_attn_fwd_static).

It serves callers that may not allocate device memory where they run the
operator; its scratch is a fixed array inside the library.  Its results must
equal those of the regular entry point (geo_attn_fwd with a caller-provided
workspace).  This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

from rna_structure_models_b200 import api
from rna_structure_models_b200.synth import GeoDims, geo_inputs
from tests.gpu_util import GEO_MAX_ABS, to_dev

OUTS = ("vectors", "output", "attention")
SCRATCH_BYTES = 8 * 1024 * 1024   # GEO_STATIC_SCRATCH_BYTES in include/flashipa_b200.h


def _lib():
    lib = api.library()
    lib.geo_attn_fwd_static.argtypes = [ctypes.POINTER(api.GeoParams)] + \
        [ctypes.POINTER(api.IpaTensor)] * 16 + [ctypes.c_void_p, ctypes.c_void_p]
    lib.geo_attn_fwd_static.restype = ctypes.c_int
    return lib


def _call_static(p, descs, stream=None, err_ptr=None):
    return _lib().geo_attn_fwd_static(ctypes.byref(p), *[ctypes.byref(d) for d in descs],
                                      ctypes.c_void_p(stream), ctypes.c_void_p(err_ptr))


def test_sizes_beyond_the_fixed_scratch_are_rejected():
    # needs no GPU: the size check happens before anything touches the device
    lib = _lib()
    big = api.GeoParams(4, 8192, 8, 4, 256)
    assert lib.geo_attn_workspace_size(ctypes.byref(big)) > SCRATCH_BYTES
    fake = api.IpaTensor()
    fake.data = 1 << 20
    st = _call_static(big, [fake] * 16, None, 1 << 20)
    assert st == 5    # IPA_ERR_WORKSPACE


@pytest.mark.gpu
def test_matches_regular_entry_point_on_two_calls(cuda_device):
    # The larger call runs first, so the smaller one finds the array filled
    # with the larger call's leftovers: a read of any byte the call did not
    # write first would change its result.  Both entry points run the same
    # deterministic kernels (no atomics), so the outputs must be identical.
    for dims, seed in ((GeoDims(B=2, N=2048, H=8, M=4, Cout=256), 11), (GeoDims(B=2, N=700, H=6, M=4, Cout=64), 12)):
        p = api.GeoParams(dims.B, dims.N, dims.H, dims.M, dims.Cout)
        assert api.library().geo_attn_workspace_size(ctypes.byref(p)) <= SCRATCH_BYTES
        plan = api.GeoPlan(dims.B, dims.N, dims.H, dims.M, dims.Cout, device=cuda_device)
        inp = to_dev({k: v for k, v in geo_inputs(dims, seed).items() if k != "dims"})
        for k in api.GEO_INPUTS:
            inp.setdefault(k, None)
        ref = plan(inp)
        torch.cuda.synchronize()
        plan.check()
        outs = {k: torch.full_like(v, float("nan")) for k, v in ref.items()}
        descs = [api.tensor_desc(inp.get(n)) for n in api.GEO_INPUTS]
        descs += [api.tensor_desc(outs[k]) for k in OUTS]
        err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
        st = _call_static(p, descs, torch.cuda.current_stream().cuda_stream, err.data_ptr())
        torch.cuda.synchronize()
        assert st == 0, api.library().ipa_status_string(st)
        assert int(err.item()) == 0
        for k in OUTS:
            assert torch.isfinite(outs[k]).all(), k
            assert (outs[k] - ref[k]).abs().max().item() <= GEO_MAX_ABS, k
            assert torch.equal(outs[k], ref[k]), k
