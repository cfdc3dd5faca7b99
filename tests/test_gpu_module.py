"""Parity of the IPA layer around the fused core (input projection, core,
output projection; one C-ABI call) with the float64 layer oracle."""
import numpy as np
import pytest
import torch

from oracle import ipa_module
from rna_structure_models_b200 import api
from rna_structure_models_b200.synth import ModuleDims, module_inputs
from tests.gpu_util import assert_parity, to_dev

pytestmark = pytest.mark.gpu


def run(inp):
    dev = to_dev({k: inp[k] for k in api.MODULE_INPUTS})
    out, core = api.ipa_module(dev, with_core=True)
    torch.cuda.synchronize()
    return out.cpu().numpy(), core.cpu().numpy()


@pytest.mark.parametrize("dims,kw", [
    (ModuleDims(B=2, L=200, H=4, Cz=64, c_s=64), {"masked_tail_frac": 0.1}),
    (ModuleDims(B=1, L=131, H=3, Cz=16, c_s=40), {}),
    (ModuleDims(B=1, L=512, H=12, Cz=128, c_s=384), {"masked_tail_frac": 0.1}),
])
def test_layer_parity(cuda_device, dims, kw):
    inp = module_inputs(dims, 0, **kw)
    out, core = run(inp)
    ref_out, ref_core = ipa_module(inp, return_core=True)
    assert_parity(core, ref_core, what=f"layer core L={dims.L}")
    assert_parity(out, ref_out, what=f"layer out L={dims.L}")


def test_layer_without_biases_and_strided_s(cuda_device):
    dims = ModuleDims(B=2, L=96, H=2, Cz=32, c_s=48)
    inp = module_inputs(dims, 1)
    inp["b_in"], inp["b_out"] = None, None
    dev = to_dev({k: inp[k] for k in api.MODULE_INPUTS if inp[k] is not None})
    dev["b_in"] = dev["b_out"] = None
    # s as a column slice of a wider buffer: rows still flatten (stride(B) = L stride(L))
    wide = torch.zeros((2, 96, 64), device="cuda")
    wide[:, :, 8:56] = dev["s"]
    dev["s"] = wide[:, :, 8:56]
    out = api.ipa_module(dev)
    ref = ipa_module(inp)
    assert_parity(out.cpu().numpy(), ref, what="layer no bias")
