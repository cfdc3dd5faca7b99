"""Parity of the distance-aware attention of MEET (§2.2, eq. (6)) run on the
fused IPA core (CUDA, through the C ABI) with the float64 oracle: small and
ragged sizes, masks, long sampled rows, rigid-motion invariance, strides.
Operands are fp16 in the core, so the IPA tolerances apply."""
import numpy as np
import pytest
import torch

from oracle import meet_dense
from rna_structure_models_b200 import api
from rna_structure_models_b200.synth import MeetDims, meet_inputs, random_rotations
from tests.gpu_util import assert_parity, to_dev

pytestmark = pytest.mark.gpu


def run_gpu(inp):
    out = api.meet_attn(to_dev({k: inp[k] for k in api.MEET_INPUTS}))
    return out.cpu().numpy()


@pytest.mark.parametrize("L", [1, 2, 63, 64, 65, 129, 300])
def test_ragged_lengths(cuda_device, L):
    inp = meet_inputs(MeetDims(B=2, L=L, H=4), 11)
    if L > 3:
        inp["mask"][1, L // 2:] = False
    assert_parity(run_gpu(inp), meet_dense(inp), what=f"meet L={L}")


def test_masked_tail_and_dead_rows(cuda_device):
    inp = meet_inputs(MeetDims(B=3, L=200, H=8), 12, masked_tail_frac=0.1)
    inp["mask"][0, :] = False
    inp["mask"][2, :] = False
    inp["mask"][2, 31] = True
    gpu = run_gpu(inp)
    assert np.all(gpu[0] == 0.0)
    assert np.all(gpu[2, :31] == 0.0) and np.all(gpu[2, 32:] == 0.0)
    assert_parity(gpu, meet_dense(inp), what="meet masks")


def test_long_sequence_sampled_rows(cuda_device):
    inp = meet_inputs(MeetDims(B=1, L=4096, H=8), 13)
    gpu = run_gpu(inp)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 2047, 4094, 4095],
                                     np.random.default_rng(2).choice(4096, 48, replace=False)]))
    assert_parity(gpu[:, rows], meet_dense(inp, rows=rows), what="meet L=4096")


def test_invariant_under_rigid_motion(cuda_device):
    inp = meet_inputs(MeetDims(B=1, L=256, H=4), 14)
    base = run_gpu(inp)
    rng = np.random.default_rng(3)
    G = random_rotations(rng, 1)[0]
    moved = dict(inp)
    moved["x"] = (inp["x"].astype(np.float64) @ G.T + rng.normal(size=3) * 40.0).astype(np.float32)
    out = run_gpu(moved)
    assert np.linalg.norm(out - base) / np.linalg.norm(base) <= 1e-3


def test_noncontiguous_inputs_match_contiguous(cuda_device):
    inp = meet_inputs(MeetDims(B=2, L=96, H=4), 15)
    dev = to_dev({k: inp[k] for k in api.MEET_INPUTS})
    ref = api.meet_attn(dev).cpu()
    nc = {}
    for k, t in dev.items():
        if t.dim() >= 2:
            perm = list(range(t.dim()))[::-1]
            nc[k] = t.permute(perm).contiguous().permute(np.argsort(perm).tolist())
            assert not nc[k].is_contiguous()
        else:
            nc[k] = torch.stack([t, t], 1)[:, 0]
    assert torch.equal(api.meet_attn(nc).cpu(), ref)
