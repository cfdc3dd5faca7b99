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


def test_stage_references_are_consistent():
    # the per-stage arrays a kernel will be compared with: softmax rows sum to 1,
    # the log-sum-exp is the oracle's, dS rows sum to ~0 on live rows
    inp = ipa_inputs(IpaDims(B=1, L=130, H=2, Cz=16), 3, masked_tail_frac=0.1)
    consts = ipa_constants(16, 4)
    out = ipa_dense(inp)
    g = np.random.default_rng(4).standard_normal(out.shape)
    stages = {}
    ipa_bwd_model(inp, g, out, stages=stages, **consts)
    assert set(stages) == {(0, 0), (0, 1)}
    st = stages[(0, 1)]
    live = np.isfinite(st["lse"]) & (inp["mask"][0])
    a = np.where(np.isfinite(st["x"]), np.exp2(st["x"] - (st["lse"] / np.log(2))[:, None]), 0.0)
    assert np.allclose(a[live].sum(axis=1), 1.0, atol=1e-9)
    # natural log-sum-exp of the true logits, from the oracle's own attention
    _, attn = ipa_dense(inp, return_attn=True)
    logits_nat = st["x"] * np.log(2)
    i = np.flatnonzero(live)[5]
    j = np.flatnonzero(attn[0, 1, i] > 0)[0]
    assert abs(np.exp(logits_nat[i, j] - st["lse"][i]) - attn[0, 1, i, j]) <= 2e-3 * attn[0, 1, i, j]
    assert np.max(np.abs(st["rs"][live])) <= 1e-3 * np.max(np.abs(st["dS"]))
