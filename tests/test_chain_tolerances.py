"""The chained tolerances of the GPU tests (tests/helpers.py) against the
oracle-only simulation that justifies them (tests/chain_tolerances.py): each
bound must keep at least a factor of two over the movement the simulated GPU
perturbation (bf16 storage plus 2^-9 relative attention error) causes."""
import pytest

import chain_tolerances as ct
from ar_video_diffusion_b200 import synth
from helpers import CHAIN_DW_REL, CHAIN_EPS_REL, CHAIN_W8A8_FRO, CHAIN_W8A8_MAX

MARGIN = 2.0


def test_absorb_chain_bounds_cover_the_simulated_perturbation():
    res = ct.absorb_chain_sensitivity(synth.WORKLOADS["rollout_small"], [0, 1, 2, 3])
    for r in res:
        assert r["rows"] == 1440
        assert 0 < r["dw_rel"] and MARGIN * r["dw_rel"] <= CHAIN_DW_REL, r
        assert 0 < r["eps_rel"] and MARGIN * r["eps_rel"] <= CHAIN_EPS_REL, r


@pytest.mark.parametrize("form", ["per-token", "mx"])
def test_w8a8_chain_bounds_cover_the_simulated_perturbation(form):
    from oracle import w8a8_oracle as w8
    res = ct.w8a8_chain_sensitivity(project=w8.project_w8a8 if form == "per-token" else w8.project_mx_rows)
    for r in res:
        assert 0 < r["fro"] and MARGIN * r["fro"] <= CHAIN_W8A8_FRO, r
        assert 0 < r["max"] and MARGIN * r["max"] <= CHAIN_W8A8_MAX, r


def test_perturbation_is_what_the_bounds_assume():
    """The simulated error is the stated one: at zero noise and with inputs
    already on the bf16 grid the perturbed chain equals the exact one."""
    import numpy as np
    rng = np.random.default_rng(0)
    a = synth.round_bf16(rng.standard_normal((64, 8)).astype(np.float32)).astype(np.float64)
    f = synth.round_bf16(rng.standard_normal((64, 8)).astype(np.float32)).astype(np.float64)
    old = ct.NOISE
    try:
        ct.NOISE = 0.0
        pl, pf = ct.perturb(a, f, rng)
    finally:
        ct.NOISE = old
    assert np.array_equal(pl, a)
    # delta is stored in bf16: the perturbed A_full is A_loc + bf16(A_full - A_loc)
    d = synth.round_bf16((f - a).astype(np.float32)).astype(np.float64)
    assert np.array_equal(pf, a + d)
    with pytest.raises(AssertionError):
        assert np.array_equal(ct.perturb(a, f, rng)[0], a)  # the noise is really applied
