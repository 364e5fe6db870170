"""Failure detection without a GPU fault: a bounded in-kernel wait that runs out
reports CCGQA_DEVERR_TIMEOUT through the caller's status word and returns, and
the CUDA context stays usable for the next call."""
import pytest
import torch

from compressed_latent_grouped_b200 import binding as B
from compressed_latent_grouped_b200.device import DeviceLayer
from compressed_latent_grouped_b200.workloads import WORKLOADS, make_inputs
from gpu_ref import check_prefill

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_reports_timeout_and_context_survives():
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    # about 5 ms at the B200's clock: a barrier nothing arrives on
    assert B.ccgqa_selftest_wait_timeout(10_000_000, err) == 0
    torch.cuda.synchronize()
    assert int(err.item()) & B.DEVERR_TIMEOUT
    # the next call on the same context runs and is correct
    w = WORKLOADS["bf16_prefill_b4_s4096"].with_(name="after_timeout", B=1, S=150)
    inp = make_inputs(w, seed=3)
    lay = DeviceLayer(w, inp)
    lay.alloc_cache()
    out = lay.prefill(inp["x"].cuda())
    torch.cuda.synchronize()
    assert lay.error_bits() == 0
    check_prefill(w, inp, 0, out[0].float().cpu().numpy(), what="after a timed-out wait")


def test_wait_self_test_rejects_out_of_range_limits():
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert B.ccgqa_selftest_wait_timeout(0, err, check=False) == 1
    assert B.ccgqa_selftest_wait_timeout(3_000_000_000, err, check=False) == 1
    torch.cuda.synchronize()
    assert int(err.item()) == 0
