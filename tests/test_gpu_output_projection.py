"""Output up-projection (ccgqa_output_projection) against the float64 oracle.

The oracle gets the GPU's own latent attention output as its input (prefill
parity is checked elsewhere), so these tests isolate the up-projection: small
cases element by element, ragged and decode-sized row counts, and the full-size
bench workload on sampled rows."""
import numpy as np
import pytest
import torch

import oracle.ccgqa as O
from compressed_latent_grouped_b200.device import DeviceLayer
from compressed_latent_grouped_b200.workloads import WORKLOADS, make_inputs, make_output_weights

pytestmark = pytest.mark.gpu

W2 = WORKLOADS["bf16_prefill_b4_s4096"]
W3 = WORKLOADS["bf16_prefill_b1_s32768"]


def _check(y, ref, dtype, what):
    y = y.astype(np.float64)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    err = np.abs(y - ref)
    if dtype == "bf16":
        # one bf16 rounding of y (at most 2^-9 |y|) plus fp32 accumulation
        assert float(np.linalg.norm(y - ref) / np.linalg.norm(ref)) <= 2e-3, what
        assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 1e-3 * rms), what
    else:
        assert float(err.max()) <= 1e-4 * rms, what


def _latent_output(w, seed):
    inp = make_inputs(w, seed=seed)
    lay = DeviceLayer(w, inp)
    lay.alloc_cache()
    o = lay.prefill(inp["x"].cuda())
    return lay, o


@pytest.mark.parametrize("w", [W2.with_(name="op_d32", B=2, S=200),
                               W3.with_(name="op_d64", S=131),
                               WORKLOADS["f32_s128"].with_(name="op_f32", B=2, S=77)],
                         ids=lambda w: w.name)
def test_output_projection_small_elementwise(w):
    lay, o = _latent_output(w, seed=5)
    W_o = make_output_weights(w, seed=5).cuda()
    y = lay.output_projection(o, W_o)
    torch.cuda.synchronize()
    assert lay.error_bits() == 0
    M = w.B * w.S
    ref = O.output_projection(o.reshape(M, -1).double().cpu().numpy(),
                              W_o.double().cpu().numpy())
    _check(y.float().cpu().numpy(), ref, w.dtype, w.name)


@pytest.mark.parametrize("M", [1, 4, 130])
def test_output_projection_decode_and_ragged_rows(M):
    w = W2.with_(name="op_rows", B=1, S=M)
    lay, o = _latent_output(w, seed=6)
    W_o = make_output_weights(w, seed=6).cuda()
    y = lay.output_projection(o.reshape(M, -1), W_o)
    torch.cuda.synchronize()
    assert lay.error_bits() == 0
    ref = O.output_projection(o.reshape(M, -1).double().cpu().numpy(),
                              W_o.double().cpu().numpy())
    _check(y.float().cpu().numpy(), ref, "bf16", f"M={M}")


def test_output_projection_full_size_sampled_rows():
    w = W2                                            # M = 16384, E = 2048, Hq d = 512
    g = torch.Generator().manual_seed(7)
    o = (torch.randn(w.B * w.S, w.Hq * w.d, generator=g)).to(torch.bfloat16).cuda()
    inp = make_inputs(w.with_(B=1, S=8), seed=7)      # weights only; the layer needs a config
    lay = DeviceLayer(w, inp)
    W_o = make_output_weights(w, seed=7).cuda()
    y = lay.output_projection(o, W_o)
    torch.cuda.synchronize()
    assert lay.error_bits() == 0
    rows = np.unique(np.concatenate([np.arange(128), np.arange(w.B * w.S - 128, w.B * w.S),
                                     np.random.default_rng(8).integers(0, w.B * w.S, 256)]))
    ref = O.output_projection(o[rows].double().cpu().numpy(), W_o.double().cpu().numpy())
    _check(y[rows].float().cpu().numpy(), ref, "bf16", "full size")
