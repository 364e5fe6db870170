"""Prefill parity: the CUDA path through the C ABI against the float64 oracle.

Small cases are compared element by element (several 128-row tiles and a
ragged tail); the full-size workloads are run in the launch configuration the
benchmark times and compared on sampled query rows."""
import numpy as np
import pytest
import torch

from compressed_latent_grouped_b200 import binding as B
from compressed_latent_grouped_b200.device import DeviceLayer
from compressed_latent_grouped_b200.workloads import WORKLOADS, make_inputs, sample_rows
from gpu_ref import check_prefill

pytestmark = pytest.mark.gpu

W1 = WORKLOADS["f32_s128"]
W2 = WORKLOADS["bf16_prefill_b4_s4096"]
W3 = WORKLOADS["bf16_prefill_b1_s32768"]
W5 = WORKLOADS["bf16_gqa_b2_s8192"]

SMALL = {
    "f32_s128": W1,
    "f32_d64_s70": W3.with_(name="f32_d64", dtype="f32", B=2, S=70),
    "f32_d32_noncausal": W2.with_(name="f32_nc", dtype="f32", B=1, S=45, causal=False),
    "bf16_d32_s200": W2.with_(name="d32", B=2, S=200),
    "bf16_d64_s300": W3.with_(name="d64", S=300),
    "bf16_d128_s260_plain": W5.with_(name="d128", B=1, S=260),
    "bf16_d32_noncausal": W2.with_(name="d32nc", B=1, S=333, causal=False),
    "bf16_d64_mha": W3.with_(name="mha", E=1024, C=2, Hq=8, Hkv=8, S=150),
    "bf16_d64_g8": W3.with_(name="g8", E=2048, C=4, Hq=8, Hkv=1, S=140),
    "bf16_d128_conv": W5.with_(name="d128conv", B=1, S=190, conv_width=4, qk_mean=True,
                               value_shift=True, packed_input=False, E=2048, C=1, Hq=16, Hkv=4),
    "bf16_d64_s1": W3.with_(name="s1", S=1),
    "bf16_d64_s3": W3.with_(name="s3", S=3),
    "bf16_d32_conv2_nochan": W2.with_(name="k2", B=1, S=77, conv_width=2),
    "bf16_d64_norope": W3.with_(name="norope", S=129, rope_base=0.0),
    # tensor-core pre-attention: 3 and 1 conv taps (other bulk-copy sizes), and a
    # group of 16 query heads (17 staged heads, about 213 KB of shared memory)
    "bf16_d32_conv3": W2.with_(name="k3", B=1, S=259, conv_width=3),
    "bf16_d64_conv1": W3.with_(name="k1", S=131, conv_width=1),
    "bf16_d32_g16": W2.with_(name="g16", B=1, S=200, Hkv=1),
    # the whole C-ABI domain (any Hq % Hkv == 0; bf16 d = 16): d = 16 runs on the
    # CUDA-core attention, group sizes that do not divide 128 leave 128 mod G
    # rows of every query tile empty, and G > 128 runs on the CUDA cores
    "bf16_d16": W1.with_(name="bf16d16", dtype="bf16", B=2, S=200),
    "bf16_d64_g3": W3.with_(name="g3", E=1536, C=2, Hq=12, Hkv=4, S=300),
    "bf16_d32_g6": W2.with_(name="g6", B=1, E=1536, C=4, Hq=12, Hkv=2, S=250),
    "bf16_d128_g12": W5.with_(name="g12", B=1, S=200, E=3072, C=1, Hq=24, Hkv=2, conv_width=4,
                              qk_mean=True, value_shift=True, packed_input=False),
    "bf16_d64_g24_noncausal": W3.with_(name="g24", E=1536, C=1, Hq=24, Hkv=1, S=150,
                                       causal=False),
    "bf16_d16_g160": W1.with_(name="g160", dtype="bf16", E=2560, C=1, Hq=160, Hkv=1, S=40),
    "f32_d32_g3": W1.with_(name="f32g3", E=768, C=4, Hq=6, Hkv=2, S=100),
    # the readings' variants: QK-mean "self" and whole-head value-shift on the
    # tensor-core pre-attention, the temporal channel conv (per-tap matrices) on
    # the CUDA-core kernel, all three together in fp32
    "bf16_d32_qk_self": W2.with_(name="qkself", B=1, S=200, qk_mean=2),
    "bf16_d64_vs_heads": W3.with_(name="vsheads", S=150, value_shift=2),
    "bf16_d64_chanconv": W3.with_(name="chanconv", S=180, channel_conv=True),
    "bf16_d128_all_variants": W5.with_(name="allvar", B=1, S=140, conv_width=3, qk_mean=2,
                                       value_shift=2, packed_input=False, E=2048, C=1, Hq=16,
                                       Hkv=4, channel_conv=True),
    "f32_all_variants": W1.with_(name="f32allvar", S=100, channel_conv=True, qk_mean=2,
                                 value_shift=2),
}


def _run(w, inp, use_cache=True, cap=None):
    lay = DeviceLayer(w, inp, cap=cap)
    if use_cache:
        lay.alloc_cache()
    x = inp["x"].cuda()
    out = lay.prefill(x, use_cache=use_cache)
    torch.cuda.synchronize()
    assert lay.error_bits() == 0
    return lay, out


@pytest.mark.parametrize("name", list(SMALL))
def test_prefill_small_elementwise(name):
    w = SMALL[name]
    inp = make_inputs(w, seed=0)
    if name == "bf16_d32_conv2_nochan":
        inp["conv_q_chan"] = inp["conv_k_chan"] = None
    lay, out = _run(w, inp, use_cache=(name != "bf16_d64_norope"))
    got = out.float().cpu().numpy()
    for b in range(w.B):
        ck = cv = None
        if lay.cache is not None:
            ck = lay.cache_tensors["k"][b, :, : w.S].float().cpu().numpy().transpose(1, 0, 2)
            cv = lay.cache_tensors["v"][b, :, : w.S].float().cpu().numpy().transpose(1, 0, 2)
            assert int(lay.cache_tensors["len"][b]) == w.S
        check_prefill(w, inp, b, got[b], cache_k=ck, cache_v=cv, what=f"{name} b={b}")


@pytest.mark.parametrize("w", [W2, W3, W5], ids=lambda w: w.name)
def test_prefill_full_size_sampled_rows(w):
    inp = make_inputs(w, seed=0)
    _, out = _run(w, inp, use_cache=True)
    rows = sample_rows(w.S, 1024)
    for b in range(w.B):
        got = out[b, torch.from_numpy(rows).cuda()].float().cpu().numpy()
        check_prefill(w, inp, b, got, rows=rows, what=f"{w.name} b={b}")


def test_prefill_without_cache_matches_with_cache():
    w = W2.with_(B=1, S=257)
    inp = make_inputs(w, seed=3)
    _, a = _run(w, inp, use_cache=True)
    _, b = _run(w, inp, use_cache=False)
    assert torch.equal(a, b)


def test_prefill_is_deterministic():
    w = W3.with_(S=520)
    inp = make_inputs(w, seed=5)
    _, a = _run(w, inp)
    _, b = _run(w, inp)
    assert torch.equal(a, b)


def test_value_shift_gather_bit_exact():
    """With packed input the cache's values are a pure gather of v~ bits:
    lower half-channels from the same position, upper half from the previous
    one, zero at position 0."""
    w = W5.with_(B=2, S=300, value_shift=True)
    inp = make_inputs(w, seed=1)
    lay, _ = _run(w, inp)
    x = inp["x"]
    d, Hq, Hkv = w.d, w.Hq, w.Hkv
    vt = x[..., (Hq + Hkv) * d:].reshape(w.B, w.S, Hkv, d)
    v = lay.cache_tensors["v"][:, :, : w.S].cpu().permute(0, 2, 1, 3)
    h = d // 2
    assert torch.equal(v[..., :h].view(torch.int16), vt[..., :h].view(torch.int16))
    assert torch.equal(v[:, 1:, :, h:].view(torch.int16), vt[:, :-1, :, h:].view(torch.int16))
    assert torch.all(v[:, 0, :, h:].view(torch.int16) == 0)
    # decode state: the last v~ row and the last K-1 pre-conv rows, bit for bit
    assert torch.equal(lay.cache_tensors["v_prev"].cpu().view(torch.int16),
                       vt[:, -1].reshape(w.B, -1).view(torch.int16))


def test_whole_head_value_shift_gather_bit_exact():
    """Whole-head reading: the last floor(Hkv / 2) kv heads hold the previous
    position's v~ row bit for bit (zero at position 0), the others the
    current one."""
    w = W5.with_(B=1, S=200, value_shift=2)
    inp = make_inputs(w, seed=6)
    lay, _ = _run(w, inp)
    d, Hq, Hkv = w.d, w.Hq, w.Hkv
    vt = inp["x"][..., (Hq + Hkv) * d:].reshape(w.B, w.S, Hkv, d)
    v = lay.cache_tensors["v"][:, :, : w.S].cpu().permute(0, 2, 1, 3)
    g0 = Hkv - Hkv // 2
    assert torch.equal(v[:, :, :g0].view(torch.int16), vt[:, :, :g0].view(torch.int16))
    assert torch.equal(v[:, 1:, g0:].view(torch.int16), vt[:, :-1, g0:].view(torch.int16))
    assert torch.all(v[:, 0, g0:].view(torch.int16) == 0)


def test_decode_state_after_prefill_bit_exact():
    w = W2.with_(B=2, S=130, packed_input=True)
    inp = make_inputs(w, seed=2)
    lay, _ = _run(w, inp)
    x = inp["x"]
    d, Hq, Hkv = w.d, w.Hq, w.Hkv
    hq = lay.cache_tensors["hist_q"].cpu()
    hk = lay.cache_tensors["hist_k"].cpu()
    assert torch.equal(hq.view(torch.int16), x[:, -3:, : Hq * d].view(torch.int16))
    assert torch.equal(hk.view(torch.int16), x[:, -3:, Hq * d:(Hq + Hkv) * d].view(torch.int16))


def test_launches_are_counted():
    w = W2.with_(B=1, S=64)
    inp = make_inputs(w, seed=0)
    n0 = B.ccgqa_launch_count()
    _run(w, inp)
    # d = 32: the projection fused with the pre-attention, then attention
    assert B.ccgqa_launch_count() - n0 == 2
    B.ccgqa_set_fused_projection(False)
    try:
        n0 = B.ccgqa_launch_count()
        _run(w, inp)
        assert B.ccgqa_launch_count() - n0 == 3   # projection, pre-attention, attention
    finally:
        B.ccgqa_set_fused_projection(True)


def _growing_score_inputs(w, slope, seed=0):
    """Packed q|k|v with q along e_0 and key t along e_0 scaled by slope * t,
    so q.k / sqrt(d) = slope * t: every later 64-key half holds scores far
    above the running max, and the softmax must raise it (and rescale O)
    over and over.  Values are whole numbers, exact in bf16."""
    inp = make_inputs(w, seed=seed)
    d, Hq, Hkv = w.d, w.Hq, w.Hkv
    x = inp["x"].float()
    x[..., : (Hq + Hkv) * d] = 0.0
    q = x[..., : Hq * d].view(w.B, w.S, Hq, d)
    k = x[..., Hq * d: (Hq + Hkv) * d].view(w.B, w.S, Hkv, d)
    q[..., 0] = float(d) ** 0.5 if d in (64,) else 1.0
    scale_k = slope * float(d) ** 0.5 / float(q[0, 0, 0, 0])
    t = torch.arange(w.S, dtype=torch.float32)
    k[..., 0] = torch.round(scale_k * t)[None, :, None]
    inp["x"] = x.to(w.torch_dtype)
    return inp


@pytest.mark.parametrize("slope", [0.125, 2.0])
@pytest.mark.parametrize("w", [
    W2.with_(name="grow_d32", B=1, S=700, E=512, C=1, Hq=16, Hkv=4, conv_width=0, qk_mean=False,
             value_shift=False, rope_base=0.0, packed_input=True),
    W3.with_(name="grow_d64", B=1, S=520, E=512, C=1, Hq=8, Hkv=2, conv_width=0, qk_mean=False,
             value_shift=False, rope_base=0.0, packed_input=True),
    W5.with_(name="grow_d128", B=1, S=390, rope_base=0.0),
], ids=lambda w: w.name)
def test_prefill_growing_scores_raise_running_max(w, slope):
    # slope 1/8 nat per key: each half's sum overshoots (p up to 2^11);
    # slope 2: the first pass overflows to inf before the running max is raised
    inp = _growing_score_inputs(w, slope)
    lay, out = _run(w, inp, use_cache=False)
    got = out.float().cpu().numpy()
    assert np.all(np.isfinite(got))
    check_prefill(w, inp, 0, got[0], what=f"{w.name} slope={slope}")
