"""Why the bf16 parity bound reads the way it does (CPU only).

The literal bound max|out - oracle| <= 2e-2 RMS(oracle) is below the rounding
error of the bf16 output format itself on the CCGQA workloads: the exact
float64 result, correctly rounded to bf16, already misses it.  The tests keep
2e-2 as an RMS-relative bound and bound the worst element by an exactly
rounded bf16 model of the computation (tests/bf16_model.py); this file checks
that both statements hold for that model, so the bound is achievable, and that
the literal one is not."""
import numpy as np
import pytest

import oracle.ccgqa as O
from bf16_model import bf, check_bf16, model_prefill
from compressed_latent_grouped_b200.workloads import WORKLOADS, make_inputs
from gpu_ref import f64, oracle_layer

CASES = {
    "d32": WORKLOADS["bf16_prefill_b4_s4096"].with_(B=1, S=600),
    "d64": WORKLOADS["bf16_prefill_b1_s32768"].with_(S=600),
    "d128": WORKLOADS["bf16_gqa_b2_s8192"].with_(B=1, S=600),
}


@pytest.mark.parametrize("name", list(CASES))
def test_literal_bound_fails_for_exact_result_rounded_to_bf16(name):
    w = CASES[name]
    inp = make_inputs(w, seed=0)
    ref, _ = O.prefill(oracle_layer(w, inp), f64(inp["x"][0]))
    rms = np.sqrt(np.mean(ref ** 2))
    err = np.max(np.abs(bf(ref) - ref))
    assert err > 2e-2 * rms          # the literal statement is not attainable in bf16
    assert np.max(np.abs(ref)) > 8 * rms


@pytest.mark.parametrize("name", list(CASES))
def test_model_meets_the_bound_it_sets(name):
    w = CASES[name]
    inp = make_inputs(w, seed=0)
    lay = oracle_layer(w, inp)
    x = f64(inp["x"][0])
    ref, _ = O.prefill(lay, x)
    model, mst = model_prefill(lay, x)
    l2, _ = check_bf16(model, ref, model, mst.extra["spread"], name)
    assert l2 < 1e-2


def test_elementwise_bound_catches_a_localised_error():
    """A kernel error confined to a few elements (one head at a run of
    positions, say a wrong diagonal tile) hides inside the global bounds (a)
    and (b) but not inside the per-element bound (c)."""
    import bf16_model as M
    w = CASES["d64"]
    inp = make_inputs(w, seed=0)
    lay = oracle_layer(w, inp)
    x = f64(inp["x"][0])
    ref, _ = O.prefill(lay, x)
    model, mst = model_prefill(lay, x)
    rms = np.sqrt(np.mean(ref ** 2))
    bad = model.copy()
    bad[300:310, 64:128] += 3e-2 * rms        # head 1, ten positions
    d = np.abs(bad - ref)
    assert np.linalg.norm(bad - ref) / np.linalg.norm(ref) <= M.L2_TOL                 # (a) passes
    assert d.max() <= M.ABS_TOL * rms + M.MODEL_SLACK * np.abs(model - ref).max()  # (b) passes
    with pytest.raises(AssertionError, match="element"):
        check_bf16(bad, ref, model, mst.extra["spread"], "planted")
