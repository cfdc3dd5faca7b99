"""Parity of the backbone-frame kernel (Flash Invariant Point Attention,
Figure 1: Gram-Schmidt frame on C_alpha; CUDA, through the C ABI) with the
float64 oracle, and of the IPA core fed with those frames."""
import numpy as np
import pytest
import torch

from oracle import frames_from_backbone, ipa_dense
from rna_structure_models_b200 import api
from rna_structure_models_b200.synth import IpaDims, backbone_inputs, ipa_inputs
from tests.gpu_util import assert_parity, to_dev

pytestmark = pytest.mark.gpu

# fp32 arithmetic on unit vectors: a few ulp of 1.0 after two normalisations
FRAME_ATOL = 1e-5


def gpu_frames(bb, **kw):
    d = to_dev({k: bb[k] for k in ("n", "ca", "c")})
    R, t = api.frames_from_backbone(d["n"], d["ca"], d["c"], **kw)
    torch.cuda.synchronize()
    return R.cpu().numpy(), t.cpu().numpy()


@pytest.mark.parametrize("B,L", [(1, 1), (1, 255), (3, 257), (2, 40000)])
def test_parity_ragged_sizes(cuda_device, B, L):
    bb = backbone_inputs(B, L, 3, jitter=0.3)
    R, t = gpu_frames(bb)
    Rr, tr = frames_from_backbone(bb["n"], bb["ca"], bb["c"])
    assert np.max(np.abs(R - Rr)) <= FRAME_ATOL
    assert np.array_equal(t, bb["ca"])                       # translation is C_alpha, bit for bit
    assert np.allclose(np.einsum("blxi,blxj->blij", R, R), np.eye(3), atol=3 * FRAME_ATOL)


def test_strided_atoms_from_one_backbone_tensor(cuda_device):
    bb = backbone_inputs(2, 500, 4, jitter=0.2)
    atoms = torch.from_numpy(np.stack([bb["n"], bb["ca"], bb["c"]], axis=2)).cuda()   # [B, L, 3 atoms, 3]
    n, ca, c = atoms[:, :, 0], atoms[:, :, 1], atoms[:, :, 2]                         # stride 9 along L
    assert not n.is_contiguous()
    R, t = api.frames_from_backbone(n, ca, c)
    Rr, _ = frames_from_backbone(bb["n"], bb["ca"], bb["c"])
    assert np.max(np.abs(R.cpu().numpy() - Rr)) <= FRAME_ATOL
    assert np.array_equal(t.cpu().numpy(), bb["ca"])


def test_writes_into_caller_buffers_on_a_side_stream(cuda_device):
    bb = backbone_inputs(1, 1000, 6, jitter=0.1)
    d = to_dev({k: bb[k] for k in ("n", "ca", "c")})
    rot = torch.full((1, 1000, 3, 3), float("nan"), device="cuda")
    trans = torch.full((1, 1000, 3), float("nan"), device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    R, t = api.frames_from_backbone(d["n"], d["ca"], d["c"], rot=rot, trans=trans, stream=s)
    s.synchronize()
    assert R.data_ptr() == rot.data_ptr() and t.data_ptr() == trans.data_ptr()
    Rr, _ = frames_from_backbone(bb["n"], bb["ca"], bb["c"])
    assert np.max(np.abs(rot.cpu().numpy() - Rr)) <= FRAME_ATOL


def test_recovers_generating_frames(cuda_device):
    bb = backbone_inputs(2, 300, 7)
    R, _ = gpu_frames(bb)
    assert np.max(np.abs(R - bb["rot"])) <= 3e-5                 # atoms are float32-rounded


def test_ipa_on_kernel_frames_matches_oracle_on_oracle_frames(cuda_device):
    B, L = 2, 300
    inp = ipa_inputs(IpaDims(B=B, L=L, H=4, Cz=64), 8, masked_tail_frac=0.1)
    bb = backbone_inputs(B, L, 9, jitter=0.3)
    Rr, tr = frames_from_backbone(bb["n"], bb["ca"], bb["c"])
    ref = ipa_dense(dict(inp, rot=Rr, trans=tr))
    dev = to_dev({k: inp[k] for k in api.IPA_INPUTS})
    bd = to_dev({k: bb[k] for k in ("n", "ca", "c")})
    dev["rot"], dev["trans"] = api.frames_from_backbone(bd["n"], bd["ca"], bd["c"])
    out = api.ipa_attn(dev)
    assert_parity(out.cpu().numpy(), ref, what="ipa on kernel frames")
