"""The decomposition planned for the IPA backward kernels (tests/ipa_bwd_model:
fp16 augmented rows with per-tile origins, query-side and key-side passes,
row / column sums, per-residue mapping) against the float64 gradient oracle,
at sizes that span several 64-residue origin tiles and a ragged tail."""
import numpy as np
import pytest

from oracle import ipa_constants, ipa_dense, ipa_grad
from rna_structure_models_b200.synth import IpaDims, ipa_inputs
from tests.ipa_bwd_model import ipa_bwd_model


@pytest.mark.parametrize("L,H,Cz,kw", [(150, 2, 16, {"masked_tail_frac": 0.1}), (200, 3, 64, {"jitter": 1.0}),
                                       (70, 2, 128, {})])
def test_planned_decomposition_matches_the_oracle(L, H, Cz, kw):
    inp = ipa_inputs(IpaDims(B=1, L=L, H=H, Cz=Cz), L, **kw)
    consts = ipa_constants(16, 4)
    out = ipa_dense(inp)
    g = np.random.default_rng(L).standard_normal(out.shape)
    ref = ipa_grad(inp, g)
    got = ipa_bwd_model(inp, g, out, **consts)
    for key, r in ref.items():
        err = np.linalg.norm(got[key] - r) / max(np.linalg.norm(r), 1e-30)
        assert err <= 2e-3, (key, err)
