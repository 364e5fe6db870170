"""Helpers shared by the GPU tests: run the float64 oracle (and, for bf16, the
bf16 rounding model) on the same seeded inputs the CUDA path receives, and
compare within the parity bounds."""
from __future__ import annotations

import numpy as np
import torch

import oracle.ccgqa as O
from bf16_model import check_bf16, check_within_one_ulp, model_decode_step, model_prefill
from compressed_latent_grouped_b200.workloads import Workload

F32_TOL = 1e-4   # max |gpu - oracle| <= 1e-4 RMS(oracle) on the fp32 path


def f64(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def oracle_layer(w: Workload, inp: dict) -> O.Layer:
    return O.Layer(
        sh=O.Shape(w.E, w.C, w.Hq, w.Hkv), W_qkv=f64(inp.get("W_qkv")),
        conv_width=w.conv_width, conv_q_seq=f64(inp.get("conv_q_seq")),
        conv_q_chan=f64(inp.get("conv_q_chan")), conv_k_seq=f64(inp.get("conv_k_seq")),
        conv_k_chan=f64(inp.get("conv_k_chan")), qk_mean=int(w.qk_mean),
        value_shift=int(w.value_shift), rope_base=w.rope_base, causal=bool(w.causal),
        channel_conv=bool(w.channel_conv))


def assert_close_f32(gpu, ref, what=""):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite output"
    rms = float(np.sqrt(np.mean(ref ** 2)))
    err = float(np.max(np.abs(gpu - ref)))
    assert err <= F32_TOL * rms, f"{what}: max err {err:.3e} > {F32_TOL} RMS {rms:.3e}"
    return err / rms


def check_prefill(w: Workload, inp: dict, b: int, got, rows=None, cache_k=None, cache_v=None,
                  what=""):
    """got: GPU output rows [len(rows), Hq d]; cache_k/v: GPU cache rows [S, Hkv, d]."""
    lay = oracle_layer(w, inp)
    x = f64(inp["x"][b])
    ref, st = O.prefill(lay, x, rows=rows)
    if w.dtype == "f32":
        assert_close_f32(got, ref, what)
        if cache_k is not None:
            assert_close_f32(cache_k, st.k, what + " cache k")
            assert_close_f32(cache_v, st.v, what + " cache v")
        return
    model, mst = model_prefill(lay, x, rows=rows)
    check_bf16(got, ref, model, mst.extra["spread"], what)
    if cache_k is not None:
        check_within_one_ulp(cache_k, mst.k, what + " cache k")
        check_within_one_ulp(cache_v, mst.v, what + " cache v")


def decode_references(w: Workload, inp: dict, b: int, xs):
    """Oracle and bf16-model outputs of consecutive decode steps from the
    workload's synthetic state (xs: list of x_t rows as float64).  Each model
    entry is (output, a), a being the bound's weighted absolute value."""
    lay = oracle_layer(w, inp)
    st = O.State(k=f64(inp["cache_k"][b]), v=f64(inp["cache_v"][b]),
                 hist_q=f64(inp["hist_q"][b]), hist_k=f64(inp["hist_k"][b]),
                 v_prev=f64(inp["v_prev"][b]))
    mst = O.State(k=st.k.copy(), v=st.v.copy(), hist_q=st.hist_q.copy(),
                  hist_k=st.hist_k.copy(), v_prev=st.v_prev.copy())
    refs, models = [], []
    for x in xs:
        r, st = O.decode_step(lay, st, x)
        m, mst = model_decode_step(lay, mst, x)
        refs.append(r)
        models.append((m, mst.extra["spread"]))
    return refs, models, st, mst


def check_rows(dtype, got, ref, model, what=""):
    """model: (bf16-model output, a) from decode_references (unused for f32)."""
    if dtype == "f32":
        return assert_close_f32(got, ref, what)
    return check_bf16(got, ref, model[0], model[1], what)
