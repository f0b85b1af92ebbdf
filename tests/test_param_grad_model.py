"""The tolerance model of the parameter-gradient parity checks (no GPU): the
closed-form gate and lambda gradients built from the oracle's forward
intermediates equal the oracle's autograd gradients, and the rounding scale
sigma predicts the drift of those gradients when the stored O_sp / O_race are
rounded to bf16 (one realization of the perturbation sigma models)."""

import pytest
import torch

from sparse_rank_hybrid_simhash_b200.workloads import WORKLOADS, make_inputs

from parity import ULP, oracle_unit, param_grads_closed_form


@pytest.mark.parametrize("causal,fixed,lookback", [(False, False, 1), (True, False, 1),
                                                   (False, True, 2)])
def test_closed_form_parameter_gradients_match_autograd(causal, fixed, lookback):
    w = WORKLOADS["iid-4k"].replace(B=1, H=2, N=256, chunk=32, causal=causal, lookback=lookback,
                                    gate_fixed=fixed, gate_s=0.7, gate_r=0.4, lam=1.3)
    inp = make_inputs(w, with_dy=True)
    refs = [oracle_unit(w, inp, 0, h, backward=True) for h in range(w.H)]
    closed, var = param_grads_closed_form(refs)
    names = ("dlambda",) if fixed else ("dgate_w", "dgate_b", "dlambda")
    for name in names:
        ref = torch.stack([r["grad_" + name].reshape(-1) for r in refs]).sum(0)
        got = closed[name].reshape(-1)
        assert (got - ref).norm() <= 1e-10 * max(ref.norm(), 1e-30), name
    # rounding the stored intermediates to bf16 moves the gradients by a
    # fraction of sigma (a rounding error is at most half an ulp)
    rounded = [dict(r, o_sp=r["o_sp"].bfloat16().double(), o_race=r["o_race"].bfloat16().double())
               for r in refs]
    moved, _ = param_grads_closed_form(rounded)
    for name in names:
        drift = (moved[name] - closed[name]).norm().item()
        sigma = ULP["bf16"] * var[name].sqrt().norm().item()
        assert 0 < drift <= 2.0 * sigma, (name, drift, sigma)
