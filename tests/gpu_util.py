"""Helpers shared by the GPU tests: move seeded inputs to the device and
compare against the oracle with the tolerances the fused path is held to."""
import contextlib
import os

import numpy as np
import torch

# Fused IPA core (fp16 operands, fp32 accumulation) against the float64 oracle.
IPA_MAX_ABS = 2e-2
IPA_REL_FRO = 5e-3
# Geometric variant computes in fp32 throughout.
GEO_MAX_ABS = 5e-4
GEO_REL_FRO = 1e-5


def to_dev(inp: dict, device="cuda", dtype=torch.float32) -> dict:
    out = {}
    for k, v in inp.items():
        if isinstance(v, np.ndarray):
            t = torch.from_numpy(np.ascontiguousarray(v))
            if t.dtype != torch.bool:
                t = t.to(dtype)
            out[k] = t.to(device)
        elif v is None:
            out[k] = None
    return out


def errors(gpu, ref):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    d = gpu - ref
    maxabs = float(np.max(np.abs(d))) if d.size else 0.0
    nref = float(np.linalg.norm(ref))
    relf = float(np.linalg.norm(d) / nref) if nref > 0 else float(np.linalg.norm(d))
    return maxabs, relf


def assert_parity(gpu, ref, max_abs=IPA_MAX_ABS, rel_fro=IPA_REL_FRO, what=""):
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite values"
    m, r = errors(gpu, ref)
    log = os.environ.get("PARITY_LOG")
    if log:
        with open(log, "a") as f:
            f.write(f"{what}\tmax_abs={m:.3e}\trel_fro={r:.3e}\tbound=({max_abs}, {rel_fro})\n")
    assert m <= max_abs and r <= rel_fro, f"{what}: max-abs {m:.3e} (<= {max_abs}), rel-Fro {r:.3e} (<= {rel_fro})"
    return m, r


@contextlib.contextmanager
def checked_library():
    """Route the binding's calls to the bounds-checked build of the library
    (every global store index checked against its buffer; an index outside
    it is reported as IPA_ERR_BOUNDS through the plans' error words).  The
    build is compiled here when missing or older than a source."""
    from rna_structure_models_b200 import api, build
    if build.checked_is_stale():
        build.build_checked()
    saved = api._lib
    api._lib = None
    try:
        lib = api.library(build.CHECKED_LIB)
        assert lib.ipa_version().decode().endswith("bounds-checked")
        yield lib
    finally:
        api._lib = saved
