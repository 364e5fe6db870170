"""The allocation-free decode entry point, for callers that cannot allocate
device memory (their runtime owns all of it): ccgqa_decode_step_noalloc must
give the same results as ccgqa_decode_step with a caller-provided workspace,
on consecutive calls (the shared scratch array keeps the previous call's
contents, so the second call checks that nothing stale leaks through).  Both
entry points run the same kernels with the same plan on the same inputs, and
the split merge reads its partials in a fixed order, so the outputs must be
identical bit for bit.

Collected last on purpose: a failure here stops a -x run only after every
other test has run."""
import pytest
import torch

from compressed_latent_grouped_b200 import binding as B
from compressed_latent_grouped_b200.device import DeviceLayer
from compressed_latent_grouped_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

W4 = WORKLOADS["bf16_decode_b64_l16384"]

CASES = [
    # 6 sequences: the weight-streaming projection (no partials)
    W4.with_(name="noalloc_bf16_b6", B=6, S=900),
    # 64 sequences: the tensor-core projection, whose E-split partials are the
    # largest region of the shared scratch array
    W4.with_(name="noalloc_bf16_b64", B=64, S=256),
    W4.with_(name="noalloc_f32", B=3, S=200, dtype="f32"),
]


def _setup(w, inp):
    lay = DeviceLayer(w, inp, cap=w.S + 8)
    t = lay.alloc_cache()
    lay.append(inp["cache_k"].cuda(), inp["cache_v"].cuda())
    t["hist_q"].copy_(inp["hist_q"])
    t["hist_k"].copy_(inp["hist_k"])
    t["v_prev"].copy_(inp["v_prev"])
    return lay


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_noalloc_decode_matches_workspace_decode(w):
    assert B.ccgqa_decode_workspace_size(B.make_config(
        w.E, w.C, w.Hq, w.Hkv, rope_base=w.rope_base,
        dtype=B.F32 if w.dtype == "f32" else B.BF16), w.B, w.S + 8) <= \
        B.ccgqa_decode_noalloc_max_bytes()
    inp = make_inputs(w, seed=0)
    ref = _setup(w, inp)       # regular entry point, caller workspace
    na = _setup(w, inp)        # allocation-free entry point
    g = torch.Generator().manual_seed(3)
    for step in range(2):
        x_t = torch.randn(w.B, w.E, generator=g).to(w.torch_dtype).cuda()
        a = ref.decode_step(x_t)
        b = torch.empty_like(a)
        B.ccgqa_decode_step_noalloc(na.cfg, na.weights, x_t, na.cache, b, na.dev_err)
        torch.cuda.synchronize()
        assert ref.error_bits() == 0 and na.error_bits() == 0
        assert torch.equal(a, b), f"step {step}: outputs differ"
        for key in ("k", "v", "len", "hist_q", "hist_k", "v_prev"):
            assert torch.equal(ref.cache_tensors[key], na.cache_tensors[key]), (step, key)


def test_noalloc_takes_no_memory_after_the_first_call():
    """After one warm-up call on the device (which loads the library's module
    and with it the fixed scratch array), further calls leave the device's
    free memory unchanged."""
    w = CASES[1]
    inp = make_inputs(w, seed=1)
    na = _setup(w, inp)
    x_t = torch.randn(w.B, w.E, generator=torch.Generator().manual_seed(5)).to(w.torch_dtype).cuda()
    out = torch.empty(w.B, w.Hq * w.d, dtype=w.torch_dtype, device="cuda")
    B.ccgqa_decode_step_noalloc(na.cfg, na.weights, x_t, na.cache, out, na.dev_err)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        B.ccgqa_decode_step_noalloc(na.cfg, na.weights, x_t, na.cache, out, na.dev_err)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert na.error_bits() == 0
    assert free1 == free0, f"free device memory changed by {free0 - free1} bytes"


def test_noalloc_rejects_oversized_decode():
    w = W4.with_(B=64, S=16384)
    cfg = B.make_config(w.E, w.C, w.Hq, w.Hkv, rope_base=w.rope_base)
    need = B.ccgqa_decode_workspace_size(cfg, 4096, 1 << 20)
    assert need > B.ccgqa_decode_noalloc_max_bytes()
    inp = make_inputs(w.with_(B=2, S=16))
    lay = DeviceLayer(w.with_(B=2, S=16), inp, cap=16)
    lay.alloc_cache()
    big = B.ccgqa_kvcache(lay.cache.k, lay.cache.v, lay.cache.len, lay.cache.conv_hist_q,
                          lay.cache.conv_hist_k, lay.cache.v_prev, 4096, 1 << 20)
    x = torch.zeros(2, w.E, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(2, w.Hq * w.d, dtype=torch.bfloat16, device="cuda")
    st = B.ccgqa_decode_step_noalloc(lay.cfg, lay.weights, x, big, out, lay.dev_err, check=False)
    assert st == 4   # CCGQA_ERR_WORKSPACE, before any launch
