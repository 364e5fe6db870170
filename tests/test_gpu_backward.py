"""Backward-pass parity: ccgqa_prefill_backward through the C ABI against the
float64 oracle's backward on the same seeded inputs, every gradient element
by element.

fp32: max|gpu - oracle| <= 1e-4 RMS(oracle) for each gradient.  bf16: the
forward values the gradients go through (q~, k~, v~, q, k, v) are rounded to
bf16 as in the forward, so each gradient is checked as the forward's output
is: relative L2 <= 2e-2, and its worst element against an exactly rounded
bf16 model of the same backward (max|gpu - oracle| <= 2e-2 RMS + 1.5 x the
model's own worst error)."""
import numpy as np
import pytest
import torch

import oracle.ccgqa as O
from bf16_model import model_prefill_backward
from compressed_latent_grouped_b200 import binding as B
from compressed_latent_grouped_b200.device import DeviceLayer
from compressed_latent_grouped_b200.workloads import WORKLOADS, make_inputs
from gpu_ref import f64, oracle_layer

pytestmark = pytest.mark.gpu

W1 = WORKLOADS["f32_s128"]
W2 = WORKLOADS["bf16_prefill_b4_s4096"]
W3 = WORKLOADS["bf16_prefill_b1_s32768"]
W5 = WORKLOADS["bf16_gqa_b2_s8192"]

CASES = {
    "f32_d16": W1.with_(name="bwd_f32", S=70),
    "f32_variants": W1.with_(name="bwd_f32var", S=60, channel_conv=True, qk_mean=2, value_shift=2),
    "f32_d32_g3_noncausal": W1.with_(name="bwd_f32g3", E=768, C=4, Hq=6, Hkv=2, S=45, causal=False),
    "bf16_d32": W2.with_(name="bwd_d32", B=2, S=150),
    "bf16_d64": W3.with_(name="bwd_d64", S=133),
    "bf16_d128_packed": W5.with_(name="bwd_d128", B=1, S=100),
    "bf16_d64_variants": W3.with_(name="bwd_d64var", S=90, qk_mean=2, value_shift=2,
                                  channel_conv=True),
    "bf16_d32_conv2_nochan": W2.with_(name="bwd_k2", B=1, S=77, conv_width=2),
    # CUDA-core attention backward in bf16: a group of 3 heads, and d = 16
    "bf16_d32_g3_simt": W2.with_(name="bwd_g3", B=1, S=90, E=768, C=4, Hq=6, Hkv=2),
    "bf16_d16_simt": W1.with_(name="bwd_d16", dtype="bf16", S=80),
    # tensor-core attention backward over several tiles and a ragged tail:
    # two CTAs of query tiles and of key tiles, non-causal, a group of 1 and 8
    "bf16_d64_tiles": W3.with_(name="bwd_d64_tiles", S=700),
    "bf16_d32_noncausal": W2.with_(name="bwd_d32_nc", B=1, S=300, causal=False),
    "bf16_d64_g1": W3.with_(name="bwd_d64_g1", S=333, Hq=2, Hkv=2, E=1024),
    "bf16_d128_g8": W5.with_(name="bwd_d128_g8", B=1, S=260, Hq=32, Hkv=4),
}


def _check(name, gpu, ref, model, what):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite"
    rms = float(np.sqrt(np.mean(ref ** 2)))
    err = float(np.max(np.abs(gpu - ref)))
    if model is None:                       # fp32
        assert err <= 1e-4 * rms, f"{what}: max err {err:.3e} > 1e-4 RMS {rms:.3e}"
        print(f"[backward parity] {what}: max|gpu-oracle|/RMS {err / rms:.2e}")
        return
    l2 = float(np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-300))
    e_model = float(np.max(np.abs(np.asarray(model) - ref)))
    print(f"[backward parity] {what}: L2 {l2:.2e}, max|gpu-oracle|/RMS {err / rms:.2e}, "
          f"model {e_model / rms:.2e}")
    assert l2 <= 2e-2, f"{what}: relative L2 {l2:.3e} > 2e-2"
    assert err <= 2e-2 * rms + 1.5 * e_model, \
        f"{what}: max err {err:.3e} > 2e-2 RMS ({rms:.3e}) + 1.5 x model {e_model:.3e}"


@pytest.mark.parametrize("name", list(CASES))
def test_backward_matches_oracle(name):
    w = CASES[name]
    inp = make_inputs(w, seed=0)
    if name == "bf16_d32_conv2_nochan":
        inp["conv_q_chan"] = inp["conv_k_chan"] = None
    lay = DeviceLayer(w, inp)
    g = torch.Generator().manual_seed(9)
    width = w.Hq * w.d
    dout = torch.randn(w.B, w.S, width, generator=g).to(w.torch_dtype)
    x = inp["x"].cuda()
    dx, grads = lay.prefill_backward(x, dout.cuda())
    torch.cuda.synchronize()
    assert lay.error_bits() == 0
    olay = oracle_layer(w, inp)
    ref_w = {k: 0.0 for k in ("W_qkv", "conv_q_seq", "conv_q_chan", "conv_k_seq", "conv_k_chan")}
    mod_w = dict(ref_w)
    for b in range(w.B):
        xb, db = f64(inp["x"][b]), f64(dout[b])
        ref = O.prefill_backward(olay, xb, db)
        mod = model_prefill_backward(olay, xb, db) if w.dtype == "bf16" else None
        _check(name, dx[b].float().cpu().numpy(), ref["dx"], None if mod is None else mod["dx"],
               f"{name} dx b={b}")
        for k in ref_w:
            if ref[k] is not None:
                ref_w[k] = ref_w[k] + ref[k]
                if mod is not None:
                    mod_w[k] = mod_w[k] + mod[k]
    for k, r in ref_w.items():
        if isinstance(r, float):
            assert grads[k] is None or name == "bf16_d32_conv2_nochan"
            continue
        assert grads[k] is not None, k
        _check(name, grads[k].cpu().numpy(), r, None if w.dtype == "f32" else mod_w[k],
               f"{name} d{k}")


def test_backward_without_weight_gradients():
    """Weight gradients are optional: dx alone equals the full call's dx."""
    w = W3.with_(S=70)
    inp = make_inputs(w, seed=2)
    lay = DeviceLayer(w, inp)
    dout = torch.randn(w.B, w.S, w.Hq * w.d, generator=torch.Generator().manual_seed(1)
                       ).to(w.torch_dtype).cuda()
    x = inp["x"].cuda()
    a, _ = lay.prefill_backward(x, dout, with_weights=True)
    b, g = lay.prefill_backward(x, dout, with_weights=False)
    torch.cuda.synchronize()
    assert all(v is None for v in g.values())
    assert torch.equal(a, b)
