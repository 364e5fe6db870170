"""Planted mistakes in the oracle (CPU only): every plausible slip -- a dropped
term, a wrong sign or index, a transposed operand -- must make at least one pin
fail.  Each mutant replaces one oracle function for the duration of the test."""
import dataclasses
import math

import numpy as np
import pytest

import oracle.ccgqa as O
import oracle_pins

_orig = {name: getattr(O, name) for name in
         ("seq_conv", "channel_mix", "qk_mean", "rope", "value_shift", "attention",
          "down_project", "prefill", "decode_step", "_mix_qk", "qk_mean_self",
          "value_shift_heads", "channel_conv", "attention_backward", "_rope_backward",
          "_value_shift_backward", "_seq_conv_backward", "_channel_conv_backward",
          "prefill_backward")}


def _seq_conv_drop_last_tap(z, w, history=None):
    w = w.copy()
    w[:, -1] = 0
    return _orig["seq_conv"](z, w, history)


def _seq_conv_anticausal(z, w, history=None):
    return _orig["seq_conv"](z[::-1].copy(), w, None)[::-1].copy()


def _seq_conv_history_reversed(z, w, history=None):
    return _orig["seq_conv"](z, w, None if history is None else history[::-1].copy())


def _channel_mix_transposed(u, W):
    return _orig["channel_mix"](u, np.swapaxes(W, 1, 2))


def _qk_mean_self(q, k, G):
    return 0.5 * (q + q), 0.5 * (k + k)


def _qk_mean_no_half(q, k, G):
    a, b = _orig["qk_mean"](q, k, G)
    return 2 * a, 2 * b


def _qk_mean_head_mod(q, k, G):
    S, Hq, d = q.shape
    Hkv = k.shape[1]
    kk = k[:, np.arange(Hq) % Hkv]
    return 0.5 * (q + kk), _orig["qk_mean"](q, k, G)[1]


def _rope_sign(z, pos, base):
    return _orig["rope"](z, -np.asarray(pos, dtype=np.float64), base)


def _rope_interleaved(z, pos, base):
    d = z.shape[-1]
    perm = np.concatenate([np.arange(0, d, 2), np.arange(1, d, 2)])
    inv = np.argsort(perm)
    return _orig["rope"](z[..., perm], pos, base)[..., inv]


def _rope_theta(z, pos, base):
    # exponent -i/d instead of -2i/d: same as squaring the base's root
    return _orig["rope"](z, pos, math.sqrt(base) if base else base)


def _value_shift_lower(v, v_prev=None):
    out = _orig["value_shift"](v[..., ::-1].copy(), None if v_prev is None else v_prev[..., ::-1].copy())
    return out[..., ::-1].copy()


def _value_shift_two(v, v_prev=None):
    return _orig["value_shift"](_orig["value_shift"](v, v_prev), v_prev)


def _attention_no_scale(q, k, v, G, causal, q_pos=None):
    return _orig["attention"](q * math.sqrt(q.shape[-1]), k, v, G, causal, q_pos)


def _attention_strict_mask(q, k, v, G, causal, q_pos=None):
    T = q.shape[0]
    pos = np.arange(T) if q_pos is None else np.asarray(q_pos)
    if not causal:
        return _orig["attention"](q, k, v, G, causal, q_pos)
    out = np.zeros_like(q)
    for i, t in enumerate(pos):
        if t == 0:
            out[i] = 0
        else:
            out[i] = _orig["attention"](q[i:i + 1], k[:t], v[:t], G, True, np.array([t - 1]))[0]
    return out


def _attention_head_mod(q, k, v, G, causal, q_pos=None):
    Hq = q.shape[1]
    Hkv = k.shape[1]
    idx = np.arange(Hq) % Hkv
    return _orig["attention"](q, k[:, idx], v[:, idx], 1, causal, q_pos)


def _down_project_kv_swapped(x, W, sh):
    q, k, v = _orig["down_project"](x, W, sh)
    return q, v, k


def _prefill_hist_reversed(layer, x, rows=None):
    o, st = _orig["prefill"](layer, x, rows)
    st.hist_q = st.hist_q[::-1].copy()
    st.hist_k = st.hist_k[::-1].copy()
    return o, st


def _decode_keeps_old_vprev(layer, state, x_t):
    o, ns = _orig["decode_step"](layer, state, x_t)
    ns.v_prev = state.v_prev
    return o, ns


def _output_projection_transposed(o, W_o):
    return o @ W_o


def _output_projection_drop_last(o, W_o):
    return o[:, :-1] @ W_o[:, :-1].T


def _mix_qk_mean_of_post_conv(layer, q_pre, k_pre, hq=None, hk=None):
    # QK-mean fed the conv output instead of the pre-conv q~ and k~
    y_q, y_k = _orig["_mix_qk"](dataclasses.replace(layer, qk_mean=False), q_pre, k_pre, hq, hk)
    if layer.qk_mean:
        m_q, m_k = O.qk_mean(y_q, y_k, layer.sh.G)
        y_q, y_k = y_q + m_q, y_k + m_k
    return y_q, y_k


def _mix_qk_mix_before_conv(layer, q_pre, k_pre, hq=None, hk=None):
    # channel mix applied to the pre-conv rows (and history), then the conv
    if layer.conv_width == 0 or layer.conv_q_chan is None:
        return _orig["_mix_qk"](layer, q_pre, k_pre, hq, hk)
    sh = layer.sh

    def mixed(z, W, hist):
        zm = O.channel_mix(z, W)
        hm = None if hist is None else O.channel_mix(
            hist.reshape(hist.shape[0], -1, sh.d), W).reshape(hist.shape[0], -1)
        return zm, hm

    qm, hqm = mixed(q_pre, layer.conv_q_chan, hq)
    km, hkm = mixed(k_pre, layer.conv_k_chan, hk)
    nochan = dataclasses.replace(layer, conv_q_chan=None, conv_k_chan=None, qk_mean=False)
    y_q, y_k = _orig["_mix_qk"](nochan, qm, km, hqm, hkm)
    if layer.qk_mean:
        m_q, m_k = O.qk_mean(q_pre, k_pre, sh.G)
        y_q, y_k = y_q + m_q, y_k + m_k
    return y_q, y_k


def _prefill_rope_before_mean(layer, x, rows=None):
    # RoPE turns the conv output, and the QK-mean term is added unrotated
    o, st = _orig["prefill"](dataclasses.replace(layer, qk_mean=False), x, None)
    if not layer.qk_mean:
        return _orig["prefill"](layer, x, rows)
    sh = layer.sh
    m_q, m_k = O.qk_mean(st.extra["q_pre"], st.extra["k_pre"], sh.G)
    q = st.extra["q"] + m_q
    st.k = st.k + m_k
    st.extra["q"] = q
    pos = np.arange(x.shape[0])
    rows = pos if rows is None else np.asarray(rows)
    o = O.attention(q[rows], st.k, st.v, sh.G, layer.causal, q_pos=rows)
    return o.reshape(len(rows), -1), st


def _qk_mean_self_no_half(q_pre, y_q, k_pre, y_k):
    return q_pre + y_q, k_pre + y_k


def _qk_mean_self_k_unchanged(q_pre, y_q, k_pre, y_k):
    return 0.5 * (q_pre + y_q), y_k


def _value_shift_heads_first(v, v_prev=None):
    out = _orig["value_shift_heads"](v[:, ::-1].copy(), None if v_prev is None else v_prev[::-1].copy())
    return out[:, ::-1].copy()


def _value_shift_heads_ceil(v, v_prev=None):
    S, Hkv, d = v.shape
    prev = np.zeros((1, Hkv, d)) if v_prev is None else v_prev[None]
    sh = np.concatenate([prev, v[:-1]], axis=0)
    out = v.copy()
    g0 = Hkv // 2
    out[:, g0:] = sh[:, g0:]
    return out


def _channel_conv_transposed(z, W, history=None):
    return _orig["channel_conv"](z, np.swapaxes(W, 2, 3), history)


def _channel_conv_taps_reversed(z, W, history=None):
    return _orig["channel_conv"](z, W[:, ::-1].copy(), history)


def _attn_bwd_no_rowsum(q, k, v, G, causal, dout, q_pos=None):
    T, Hq, d = q.shape
    L = k.shape[0]
    pos = np.arange(T) if q_pos is None else np.asarray(q_pos)
    dq, dk, dv = _orig["attention_backward"](q, k, v, G, causal, dout, q_pos)
    scale = 1.0 / math.sqrt(d)
    for h in range(Hq):                       # ds = p * dp, the rowsum term dropped
        g = h // G
        sc = (q[:, h] @ k[:, g].T) * scale
        if causal:
            sc = np.where(np.arange(L)[None, :] <= pos[:, None], sc, -np.inf)
        p = np.exp(sc - sc.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        ds = p * (dout[:, h] @ v[:, g].T)
        dq[:, h] = ds @ k[:, g] * scale
    return dq, dk, dv


def _attn_bwd_dk_unscaled(q, k, v, G, causal, dout, q_pos=None):
    dq, dk, dv = _orig["attention_backward"](q, k, v, G, causal, dout, q_pos)
    return dq, dk * math.sqrt(q.shape[-1]), dv


def _rope_backward_same_angle(dz, positions, base):
    return _orig["rope"](dz, positions, base)


def _value_shift_backward_wrong_way(layer, dv):
    out = _orig["_value_shift_backward"](layer, dv[::-1].copy())
    return out[::-1].copy()


def _seq_conv_backward_causal(z, w, du):
    dz, dw = _orig["_seq_conv_backward"](z, w, du)
    S = z.shape[0]
    dz2 = np.zeros_like(z)
    for j in range(w.shape[1]):
        if j < S:
            dz2[j:] += w[:, j] * du[: S - j]
    return dz2, dw


def _channel_conv_backward_untransposed(z, W, dy):
    return _orig["_channel_conv_backward"](z, np.swapaxes(W, 2, 3), dy)


def _prefill_backward_qk_no_1_over_g(layer, x, dout):
    # the QK-mean's key gradient spread to every query head without 1/G
    lay = dataclasses.replace(layer)
    g = _orig["prefill_backward"](lay, x, dout)
    if not layer.qk_mean or int(layer.qk_mean) == O.QK_SELF or layer.sh.G == 1:
        return g
    g2 = _orig["prefill_backward"](dataclasses.replace(layer, qk_mean=0), x, dout)
    g["dx"] = g["dx"] + 0.3 * (g["dx"] - g2["dx"])
    return g


MUTANTS = {
    "seq_conv_drop_last_tap": ("seq_conv", _seq_conv_drop_last_tap),
    "seq_conv_anticausal": ("seq_conv", _seq_conv_anticausal),
    "seq_conv_history_reversed": ("seq_conv", _seq_conv_history_reversed),
    "channel_mix_transposed": ("channel_mix", _channel_mix_transposed),
    "qk_mean_self": ("qk_mean", _qk_mean_self),
    "qk_mean_no_half": ("qk_mean", _qk_mean_no_half),
    "qk_mean_head_mod": ("qk_mean", _qk_mean_head_mod),
    "rope_sign": ("rope", _rope_sign),
    "rope_interleaved": ("rope", _rope_interleaved),
    "rope_theta": ("rope", _rope_theta),
    "value_shift_lower_half": ("value_shift", _value_shift_lower),
    "value_shift_two_steps": ("value_shift", _value_shift_two),
    "attention_no_scale": ("attention", _attention_no_scale),
    "attention_strict_mask": ("attention", _attention_strict_mask),
    "attention_head_mod": ("attention", _attention_head_mod),
    "down_project_kv_swapped": ("down_project", _down_project_kv_swapped),
    "prefill_hist_reversed": ("prefill", _prefill_hist_reversed),
    "decode_keeps_old_vprev": ("decode_step", _decode_keeps_old_vprev),
    "output_projection_transposed": ("output_projection", _output_projection_transposed),
    "output_projection_drop_last": ("output_projection", _output_projection_drop_last),
    "qk_mean_of_post_conv": ("_mix_qk", _mix_qk_mean_of_post_conv),
    "channel_mix_before_conv": ("_mix_qk", _mix_qk_mix_before_conv),
    "rope_before_qk_mean": ("prefill", _prefill_rope_before_mean),
    "qk_mean_self_no_half": ("qk_mean_self", _qk_mean_self_no_half),
    "qk_mean_self_k_unchanged": ("qk_mean_self", _qk_mean_self_k_unchanged),
    "value_shift_heads_first": ("value_shift_heads", _value_shift_heads_first),
    "value_shift_heads_ceil": ("value_shift_heads", _value_shift_heads_ceil),
    "channel_conv_transposed": ("channel_conv", _channel_conv_transposed),
    "channel_conv_taps_reversed": ("channel_conv", _channel_conv_taps_reversed),
    "attention_backward_no_rowsum": ("attention_backward", _attn_bwd_no_rowsum),
    "attention_backward_dk_unscaled": ("attention_backward", _attn_bwd_dk_unscaled),
    "rope_backward_same_angle": ("_rope_backward", _rope_backward_same_angle),
    "value_shift_backward_wrong_way": ("_value_shift_backward", _value_shift_backward_wrong_way),
    "seq_conv_backward_causal": ("_seq_conv_backward", _seq_conv_backward_causal),
    "channel_conv_backward_untransposed": ("_channel_conv_backward",
                                           _channel_conv_backward_untransposed),
    "prefill_backward_qk_term_scaled": ("prefill_backward", _prefill_backward_qk_no_1_over_g),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    fn_name, mutant = MUTANTS[name]
    monkeypatch.setattr(O, fn_name, mutant)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches the planted mistake {name}"
