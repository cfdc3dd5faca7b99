"""Building blocks of the fused kernel, one at a time, on the GPU: TMA loads
with 128-byte swizzle, tcgen05 MMAs with K-major / MN-major shared-memory
operands and with the A operand in tensor memory, tcgen05 loads, and the
bounded mbarrier wait."""
import ctypes
import os

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROBE = os.path.join(ROOT, "tests", "libflashipa_probe.so")

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def probe(cuda_device):
    if not os.path.exists(PROBE):
        pytest.fail("probe library not built (python -m rna_structure_models_b200.build)")
    lib = ctypes.CDLL(PROBE)
    lib.probe_umma.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                               ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    lib.probe_umma.restype = ctypes.c_int
    lib.probe_bounded_wait.argtypes = [ctypes.c_void_p, ctypes.c_ulonglong, ctypes.c_void_p]
    lib.probe_bounded_wait.restype = ctypes.c_int
    lib.probe_umma_pair.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                    ctypes.c_void_p, ctypes.c_void_p]
    lib.probe_umma_pair.restype = ctypes.c_int
    return lib


def run(lib, mode, nn=64, seed=0):
    g = torch.Generator(device="cpu").manual_seed(seed)
    A = torch.randn(128, 64, generator=g).half().cuda()
    if mode == 2:
        B = torch.randn(64, nn, generator=g).half().cuda()     # [K, N], N contiguous
        ref = A.float() @ B.float()
    else:
        B = torch.randn(64, 64, generator=g).half().cuda()     # [N, K], K contiguous
        ref = A.float() @ B.float().t()
    D = torch.zeros(128, nn, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = lib.probe_umma(mode, nn, A.data_ptr(), B.data_ptr(), D.data_ptr(), err.data_ptr(),
                        torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rc == 0
    assert int(err.item()) == 0
    return D, ref


@pytest.mark.parametrize("mode,nn", [(0, 64), (1, 64), (2, 64), (2, 256), (3, 64)])
def test_umma_building_block(probe, mode, nn):
    D, ref = run(probe, mode, nn)
    # fp16 x fp16 products are exact in fp32; only the accumulation order differs
    assert torch.allclose(D, ref, rtol=1e-5, atol=1e-4), (D - ref).abs().max().item()


def test_bounded_wait_reports_instead_of_hanging(probe):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = probe.probe_bounded_wait(err.data_ptr(), 20_000_000, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rc == 0
    assert int(err.item()) == 5          # DEV_TIMEOUT_PROBE
    # the context is still usable afterwards
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum()) == 8.0


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_cta_pair_building_block(probe, mode):
    g = torch.Generator(device="cpu").manual_seed(10 + mode)
    A = torch.randn(256, 64, generator=g).half().cuda()
    if mode == 0:
        B = torch.randn(128, 64, generator=g).half().cuda()     # [N, K]
        ref = A.float() @ B.float().t()
    else:
        nn = 256 if mode == 1 else 64
        B = torch.randn(64, nn, generator=g).half().cuda()      # [K, N]
        ref = A.float() @ B.float()
    D = torch.zeros(ref.shape, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = probe.probe_umma_pair(mode, A.data_ptr(), B.data_ptr(), D.data_ptr(), err.data_ptr(),
                               torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rc == 0
    assert int(err.item()) == 0
    assert torch.allclose(D, ref, rtol=1e-5, atol=1e-4), (D - ref).abs().max().item()
