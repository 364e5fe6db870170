"""The latent projection fused with the pre-attention steps (bf16, d = 32).

ccgqa_prefill runs the projection GEMM and the conv / channel mix / QK-mean /
RoPE / value-shift as one kernel where it applies (the projected q~ | k~ | v~
never reach HBM).  Each CTA writes 125 positions and recomputes the 3 rows
before them that the conv reaches back to, so the cases below span several
CTAs with a ragged tail, every QK-mean and value-shift mode and conv widths
1 to 4.  Checked against the oracle (bf16 bounds), bit for bit against the
separate projection and pre-attention kernels on the same inputs, and for
the decode state it leaves."""
import numpy as np
import pytest
import torch

from compressed_latent_grouped_b200 import binding as B
from compressed_latent_grouped_b200.device import DeviceLayer
from compressed_latent_grouped_b200.workloads import WORKLOADS, make_inputs
from gpu_ref import check_prefill, f64

pytestmark = pytest.mark.gpu

W2 = WORKLOADS["bf16_prefill_b4_s4096"]      # d = 32, G = 4

CASES = [
    W2.with_(name="fu_d32", B=2, S=300),
    W2.with_(name="fu_short", B=1, S=7),
    W2.with_(name="fu_k1", B=1, S=260, conv_width=1),
    W2.with_(name="fu_k2_self", B=1, S=251, conv_width=2, qk_mean=2),
    W2.with_(name="fu_k3_heads", B=2, S=376, conv_width=3, value_shift=2),
    W2.with_(name="fu_plain", B=1, S=129, qk_mean=0, value_shift=0, rope_base=0.0),
    W2.with_(name="fu_g1", B=1, S=250, E=512, C=4, Hq=4, Hkv=4),
    W2.with_(name="fu_g2", B=1, S=250, E=1024, C=4, Hq=8, Hkv=4),
    W2.with_(name="fu_g6", B=1, S=250, E=1536, C=4, Hq=12, Hkv=2),
]


def _run(w, inp, fused):
    B.ccgqa_set_fused_projection(fused)
    try:
        lay = DeviceLayer(w, inp)
        t = lay.alloc_cache()
        n0 = B.ccgqa_launch_count()
        out = lay.prefill(inp["x"].cuda())
        torch.cuda.synchronize()
        launches = B.ccgqa_launch_count() - n0
        assert lay.error_bits() == 0
        return out, t, launches, lay
    finally:
        B.ccgqa_set_fused_projection(True)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_fused_prefill_matches_oracle_and_unfused(w):
    inp = make_inputs(w, seed=11)
    out_f, t_f, n_f, _ = _run(w, inp, True)
    out_u, t_u, n_u, _ = _run(w, inp, False)
    # the fused path is one kernel fewer (projection + pre-attention in one)
    assert n_f == n_u - 1, (n_f, n_u)
    for b in range(w.B):
        check_prefill(w, inp, b, out_f[b].float().cpu().numpy(),
                      cache_k=t_f["k"][b, :, : w.S].float().cpu().numpy().transpose(1, 0, 2),
                      cache_v=t_f["v"][b, :, : w.S].float().cpu().numpy().transpose(1, 0, 2),
                      what=f"{w.name} fused b={b}")
    # against the separate kernels: the projection is the same contraction over
    # the same K blocks, rounded to bf16 the same way, and every later step is
    # the same arithmetic on the same values, so the results are bit-identical
    # (the output, the cache rows and the decode state)
    bits = lambda t: t.contiguous().view(torch.int16) if t.dtype == torch.bfloat16 else t  # noqa: E731
    assert torch.equal(bits(out_f), bits(out_u)), "output"
    for key in ("k", "v", "hist_q", "hist_k", "v_prev", "len"):
        assert torch.equal(bits(t_f[key]), bits(t_u[key])), key


def test_fused_decode_state_continues_the_sequence():
    """A decode step after a fused prefill equals the oracle's continuation."""
    w = W2.with_(name="fu_state", B=2, S=252)
    inp = make_inputs(w, seed=5)
    lay = DeviceLayer(w, inp, cap=w.S + 8)
    lay.alloc_cache()
    lay.prefill(inp["x"].cuda())
    x_t = torch.randn(w.B, w.E, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16)
    out = lay.decode_step(x_t.cuda())
    torch.cuda.synchronize()
    assert lay.error_bits() == 0
    import oracle.ccgqa as O
    from bf16_model import model_decode_step, model_prefill, check_bf16
    from gpu_ref import oracle_layer
    lo = oracle_layer(w, inp)
    for b in range(w.B):
        xb = f64(inp["x"][b])
        full = np.concatenate([xb, f64(x_t[b])[None]], axis=0)
        ref, _ = O.prefill(lo, full, rows=np.array([w.S]))
        _, mst = model_prefill(lo, xb)
        m_dec, dst = model_decode_step(lo, mst, f64(x_t[b]))
        check_bf16(out[b].float().cpu().numpy(), ref[0], m_dec, dst.extra["spread"],
                   f"decode after fused prefill b={b}")


def test_fused_full_size_bit_identical_to_unfused():
    """The 4 x 4096 workload (E = 2048, 16 / 4 heads of dim 32): the fused
    kernel's output and cache equal the separate kernels' bit for bit."""
    w = W2
    inp = make_inputs(w, seed=0)
    out_f, t_f, n_f, _ = _run(w, inp, True)
    out_u, t_u, n_u, _ = _run(w, inp, False)
    assert (n_f, n_u) == (2, 3)
    bits = lambda t: t.contiguous().view(torch.int16) if t.dtype == torch.bfloat16 else t  # noqa: E731
    assert torch.equal(bits(out_f), bits(out_u))
    for key in ("k", "v", "hist_q", "hist_k", "v_prev", "len"):
        assert torch.equal(bits(t_f[key]), bits(t_u[key])), key


def test_fused_one_tile_multi_wave_bit_identical_to_unfused():
    """Six query heads per group (too many accumulators for the persistent
    form) over more CTAs than one wave: the one-tile kernel with the 2-stage
    ring, two CTAs per SM.  Bit-identical to the separate kernels."""
    w = W2.with_(name="fu_g6_waves", B=2, S=5000, E=1536, C=4, Hq=12, Hkv=2)
    assert -(-w.S // 125) * w.Hkv * w.B > torch.cuda.get_device_properties(0).multi_processor_count
    inp = make_inputs(w, seed=3)
    out_f, t_f, n_f, _ = _run(w, inp, True)
    out_u, t_u, n_u, _ = _run(w, inp, False)
    assert n_f == n_u - 1, (n_f, n_u)
    bits = lambda t: t.contiguous().view(torch.int16) if t.dtype == torch.bfloat16 else t  # noqa: E731
    assert torch.equal(bits(out_f), bits(out_u))
    for key in ("k", "v", "hist_q", "hist_k", "v_prev", "len"):
        assert torch.equal(bits(t_f[key]), bits(t_u[key])), key
