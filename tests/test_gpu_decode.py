"""KV-cache append and decode-step parity through the C ABI."""
import numpy as np
import pytest
import torch

import oracle.ccgqa as O
from compressed_latent_grouped_b200 import binding as B
from compressed_latent_grouped_b200.device import DeviceLayer
from compressed_latent_grouped_b200.workloads import WORKLOADS, make_inputs
from gpu_ref import check_prefill, check_rows, decode_references, f64, oracle_layer
from bf16_model import check_bf16, check_within_one_ulp, model_decode_step, model_prefill

pytestmark = pytest.mark.gpu

W2 = WORKLOADS["bf16_prefill_b4_s4096"]
W3 = WORKLOADS["bf16_prefill_b1_s32768"]
W4 = WORKLOADS["bf16_decode_b64_l16384"]
W5 = WORKLOADS["bf16_gqa_b2_s8192"]


def test_kvcache_append_bit_exact():
    w = W4.with_(B=3, S=100)
    lay = DeviceLayer(w, make_inputs(w), cap=256)
    t = lay.alloc_cache()
    g = torch.Generator().manual_seed(7)
    rows = []
    for n in (5, 1, 37):
        k = torch.randn(3, n, w.Hkv, w.d, generator=g).to(torch.bfloat16)
        v = torch.randn(3, n, w.Hkv, w.d, generator=g).to(torch.bfloat16)
        lay.append(k.cuda(), v.cuda())
        rows.append((k, v))
    torch.cuda.synchronize()
    assert lay.error_bits() == 0
    k_all = torch.cat([r[0] for r in rows], 1).permute(0, 2, 1, 3)
    v_all = torch.cat([r[1] for r in rows], 1).permute(0, 2, 1, 3)
    assert t["len"].cpu().tolist() == [43, 43, 43]
    assert torch.equal(t["k"][:, :, :43].cpu().view(torch.int16), k_all.view(torch.int16))
    assert torch.equal(t["v"][:, :, :43].cpu().view(torch.int16), v_all.view(torch.int16))
    assert torch.all(t["k"][:, :, 43:].cpu() == 0)


def test_kvcache_append_capacity_flag_leaves_cache_untouched():
    w = W4.with_(B=2, S=16)
    lay = DeviceLayer(w, make_inputs(w), cap=16)
    t = lay.alloc_cache()
    k = torch.ones(2, 10, w.Hkv, w.d, dtype=torch.bfloat16, device="cuda")
    lay.append(k, k)
    lay.append(k, k)          # 20 > 16: rejected on the device
    torch.cuda.synchronize()
    assert lay.error_bits() & B.DEVERR_CAPACITY
    assert t["len"].cpu().tolist() == [10, 10]
    assert torch.all(t["k"][:, :, 10:].cpu() == 0)


def _decode_setup(w, cap_extra=8, seed=0):
    inp = make_inputs(w, seed=seed)
    lay = DeviceLayer(w, inp, cap=w.S + cap_extra)
    t = lay.alloc_cache()
    lay.append(inp["cache_k"].cuda(), inp["cache_v"].cuda())
    if w.conv_width > 1:
        t["hist_q"].copy_(inp["hist_q"])
        t["hist_k"].copy_(inp["hist_k"])
    t["v_prev"].copy_(inp["v_prev"])
    return inp, lay


@pytest.mark.parametrize("w", [
    W4.with_(name="dec_small", B=5, S=700),
    W4.with_(name="dec_small_f32", B=3, S=130, dtype="f32"),
    W4.with_(name="dec_d32", B=3, S=333, E=2048, C=4, Hq=16, Hkv=4, rope_base=1e4),
    W4.with_(name="dec_d128_plain", B=2, S=300, E=4096, C=1, Hq=32, Hkv=8, conv_width=0,
             qk_mean=False, value_shift=False, packed_input=True),
    # d = 16 and group sizes beyond the tensor-core decode (G <= 16) or not
    # powers of two; G = 24, 40 and 160 take several CTAs per kv group (head chunks)
    W4.with_(name="dec_bf16_d16", B=3, S=300, E=256, C=4, Hq=4, Hkv=2, rope_base=1e4),
    W4.with_(name="dec_g3", B=3, S=400, E=1536, C=2, Hq=12, Hkv=4),
    W4.with_(name="dec_g24", B=2, S=260, E=1536, C=1, Hq=24, Hkv=1),
    W4.with_(name="dec_f32_g40", B=2, S=150, E=2560, C=1, Hq=40, Hkv=1, dtype="f32"),
    W4.with_(name="dec_d16_g160", B=2, S=90, E=2560, C=1, Hq=160, Hkv=1),
    # the readings' variants
    W4.with_(name="dec_qk_self", B=3, S=300, qk_mean=2),
    W4.with_(name="dec_vs_heads", B=3, S=250, E=2048, C=4, Hq=16, Hkv=4, value_shift=2,
             rope_base=1e4),
    W4.with_(name="dec_chanconv", B=3, S=200, channel_conv=True),
    W4.with_(name="dec_f32_all_variants", B=2, S=120, channel_conv=True, qk_mean=2,
             value_shift=2, dtype="f32"),
], ids=lambda w: w.name)
def test_decode_steps_match_oracle(w):
    inp, lay = _decode_setup(w)
    g = torch.Generator().manual_seed(11)
    width = w.n_qkv if w.packed_input else w.E
    xs, outs = [], []
    for step in range(3):
        x_t = torch.randn(w.B, width, generator=g).to(w.torch_dtype)
        outs.append(lay.decode_step(x_t.cuda()).float().cpu().numpy())
        torch.cuda.synchronize()
        assert lay.error_bits() == 0
        xs.append(x_t)
        assert lay.cache_tensors["len"].cpu().tolist() == [w.S + step + 1] * w.B
    k = lay.cache_tensors["k"][:, :, w.S: w.S + 3].float().cpu().numpy()
    for b in range(w.B):
        refs, models, st, mst = decode_references(w, inp, b, [f64(x[b]) for x in xs])
        for step in range(3):
            check_rows(w.dtype, outs[step][b], refs[step], models[step],
                       f"{w.name} step {step} b={b}")
        # the appended key rows
        if w.dtype == "f32":
            check_rows("f32", k[b].transpose(1, 0, 2), st.k[w.S: w.S + 3], None, "appended k")
        else:
            check_within_one_ulp(k[b].transpose(1, 0, 2), mst.k[w.S: w.S + 3], "appended k")


def test_decode_full_size():
    w = W4
    inp, lay = _decode_setup(w, cap_extra=64)
    x_t = inp["x_t"]
    out = lay.decode_step(x_t.cuda())
    torch.cuda.synchronize()
    assert lay.error_bits() == 0
    got = out.float().cpu().numpy()
    for b in range(w.B):
        refs, models, _, _ = decode_references(w, inp, b, [f64(x_t[b])])
        check_rows(w.dtype, got[b], refs[0], models[0], f"decode b={b}")
    assert lay.cache_tensors["len"].cpu().tolist() == [w.S + 1] * w.B


def test_decode_value_shift_bits():
    """The appended value row takes its upper half-channels bit for bit from
    the stored previous v~ row."""
    w = W4.with_(B=2, S=50)
    inp, lay = _decode_setup(w)
    vp = lay.cache_tensors["v_prev"].clone()
    lay.decode_step(inp["x_t"].cuda())
    torch.cuda.synchronize()
    d, h = w.d, w.d // 2
    row = lay.cache_tensors["v"][:, :, w.S]                 # [B, Hkv, d]
    assert torch.equal(row[..., h:].contiguous().view(torch.int16),
                       vp.view(w.B, w.Hkv, d)[..., h:].contiguous().view(torch.int16))


@pytest.mark.parametrize("w", [W2.with_(name="pd_d32", B=2, S=257),
                               W3.with_(name="pd_d64", S=200),
                               W5.with_(name="pd_d128", B=1, S=130),
                               W3.with_(name="pd_variants", S=150, qk_mean=2, value_shift=2,
                                        channel_conv=True)], ids=lambda w: w.name)
def test_prefill_then_decode_equals_longer_prefill(w):
    """prefill(S) row S-1 == prefill(S-1) followed by one decode step."""
    inp = make_inputs(w, seed=4)
    x = inp["x"].cuda()
    full = DeviceLayer(w, inp, cap=w.S)
    full.alloc_cache()
    full_out = full.prefill(x)
    part = DeviceLayer(w, inp, cap=w.S)
    part.alloc_cache()
    part.prefill(x[:, :-1].contiguous())
    o = part.decode_step(x[:, -1].contiguous())
    torch.cuda.synchronize()
    assert full.error_bits() == 0 and part.error_bits() == 0
    lo = oracle_layer(w, inp)
    for b in range(w.B):
        xb = f64(inp["x"][b])
        ref, _ = O.prefill(lo, xb, rows=np.array([w.S - 1]))
        # decode path: prefill model over S-1 tokens, then the decode-step model
        _, mst = model_prefill(lo, xb[:-1])
        m_dec, dst = model_decode_step(lo, mst, xb[-1])
        check_bf16(o[b].float().cpu().numpy(), ref[0], m_dec, dst.extra["spread"],
                   f"{w.name} decode b={b}")
        m_pf, pst = model_prefill(lo, xb, rows=np.array([w.S - 1]))
        check_bf16(full_out[b, -1].float().cpu().numpy(), ref[0], m_pf[0], pst.extra["spread"][0],
                   f"{w.name} prefill b={b}")
    # the caches agree except for the last row's bf16 rounding path
    for key in ("k", "v"):
        a = part.cache_tensors[key][:, :, : w.S - 1].float().cpu().numpy()
        b_ = full.cache_tensors[key][:, :, : w.S - 1].float().cpu().numpy()
        assert np.array_equal(a, b_), key
        # last row: projection summed in a different order before the same
        # bf16 rounding -> a few ulps at most
        a1 = part.cache_tensors[key][:, :, w.S - 1].float().cpu().numpy()
        b1 = full.cache_tensors[key][:, :, w.S - 1].float().cpu().numpy()
        assert np.max(np.abs(a1 - b1)) <= 2.0 ** -5 * np.max(np.abs(b1)), key
    assert part.cache_tensors["len"].cpu().tolist() == [w.S] * w.B


def test_decode_capacity_flag():
    w = W4.with_(B=2, S=40)
    inp, lay = _decode_setup(w, cap_extra=0)     # cache already full
    out = lay.decode_step(inp["x_t"].cuda())
    torch.cuda.synchronize()
    assert lay.error_bits() & B.DEVERR_CAPACITY
    assert lay.cache_tensors["len"].cpu().tolist() == [40, 40]
    assert torch.all(out.cpu() == 0)
