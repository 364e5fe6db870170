"""Pins for the float64 oracle: checks against facts that do not come from the
oracle itself (library special cases, closed forms, brute force, invariants and
the values printed on the GQA glossary page).

Each ``pin_*`` function raises AssertionError on failure.  They are collected
as tests by ``test_oracle_pins.py`` and re-run against deliberately broken
copies of the oracle by ``test_oracle_mutations.py``.
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch
import torch.nn.functional as F

import oracle.ccgqa as O

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_golden(name: str) -> dict:
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = (s.strip() for s in line.split("=", 1))
            vals[k] = v
    return vals


def _close(a, b, tol=1e-12, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} != {b.shape}"
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    assert err <= tol * scale, f"{what}: max abs err {err:.3e} > {tol:.1e}"


def _rng(seed=0):
    return np.random.default_rng(seed)


def _small_layer(E=64, C=2, Hq=4, Hkv=2, K=4, seed=3, qk=True, vs=True, base=100.0,
                 causal=True, chan=True, packed=False):
    sh = O.Shape(E, C, Hq, Hkv)
    r = _rng(seed)
    d = sh.d
    return O.Layer(
        sh=sh,
        W_qkv=None if packed else r.standard_normal((sh.n_qkv, E)) / math.sqrt(E),
        conv_width=K,
        conv_q_seq=r.standard_normal((Hq * d, K)) * 0.5 if K else None,
        conv_q_chan=(r.standard_normal((Hq, d, d)) / math.sqrt(d)) if (K and chan) else None,
        conv_k_seq=r.standard_normal((Hkv * d, K)) * 0.5 if K else None,
        conv_k_chan=(r.standard_normal((Hkv, d, d)) / math.sqrt(d)) if (K and chan) else None,
        qk_mean=qk, value_shift=vs, rope_base=base, causal=causal)


# --------------------------------------------------------------------------
# Attention core
# --------------------------------------------------------------------------
def brute_force_attention(q, k, v, G, causal, q_pos):
    """Pure-Python loops, written from the definition of softmax attention."""
    T, Hq, d = q.shape
    L = k.shape[0]
    out = np.zeros((T, Hq, d))
    for ti in range(T):
        for h in range(Hq):
            g = h // G
            scores = []
            for s in range(L):
                if causal and s > q_pos[ti]:
                    continue
                dot = 0.0
                for i in range(d):
                    dot += q[ti, h, i] * k[s, g, i]
                scores.append((s, dot / math.sqrt(d)))
            top = max(sc for _, sc in scores)
            w = [(s, math.exp(sc - top)) for s, sc in scores]
            tot = sum(x for _, x in w)
            for s, x in w:
                for i in range(d):
                    out[ti, h, i] += x / tot * v[s, g, i]
    return out


def pin_gqa_glossary_example():
    """The GQA page's example: grouped attention equals attention on copied
    key/value heads; shape and cached-value counts as printed."""
    g = read_golden("gqa_glossary_example.txt")
    B, Hq, Hkv, T, d = (int(g[k]) for k in ("batch", "query_heads", "kv_heads", "tokens", "head_dim"))
    gen = torch.Generator().manual_seed(0)
    q = torch.randn(B, Hq, T, d, generator=gen, dtype=torch.float64)
    k = torch.randn(B, Hkv, T, d, generator=gen, dtype=torch.float64)
    v = torch.randn(B, Hkv, T, d, generator=gen, dtype=torch.float64)
    grouped = F.scaled_dot_product_attention(q, k, v, is_causal=True, enable_gqa=True)
    copied = F.scaled_dot_product_attention(
        q, k.repeat_interleave(Hq // Hkv, dim=1), v.repeat_interleave(Hq // Hkv, dim=1),
        is_causal=True)
    assert tuple(grouped.shape) == tuple(int(s) for s in g["output_shape"].split())
    assert (bool(torch.allclose(grouped, copied, atol=1e-6)) == (g["matches_copied_heads"] == "True"))
    # the oracle on the same tensors ([T, H, d] layout)
    o = O.attention(q[0].permute(1, 0, 2).numpy(), k[0].permute(1, 0, 2).numpy(),
                    v[0].permute(1, 0, 2).numpy(), Hq // Hkv, True)
    _close(o, grouped[0].permute(1, 0, 2).numpy(), 1e-12, "oracle vs SDPA(enable_gqa)")
    _close(o, copied[0].permute(1, 0, 2).numpy(), 1e-12, "oracle vs SDPA(copied heads)")
    assert O.cache_values_per_token(Hkv, d) == int(g["cached_values_per_token_gqa"])
    assert O.cache_values_per_token(Hq, d) == int(g["cached_values_per_token_mha"])


def pin_mqa_and_mha_reductions():
    """One kv group is MQA; as many kv heads as query heads is MHA
    (GQA page, "Cómo funciona GQA")."""
    r = _rng(1)
    T, Hq, d = 7, 4, 8
    q = r.standard_normal((T, Hq, d))
    k1 = r.standard_normal((T, 1, d))
    v1 = r.standard_normal((T, 1, d))
    mqa = O.attention(q, k1, v1, Hq, True)
    for h in range(Hq):
        ref = F.scaled_dot_product_attention(
            torch.from_numpy(q[:, h][None]), torch.from_numpy(k1[:, 0][None]),
            torch.from_numpy(v1[:, 0][None]), is_causal=True)[0].numpy()
        _close(mqa[:, h], ref, 1e-12, f"MQA head {h}")
    kf = r.standard_normal((T, Hq, d))
    vf = r.standard_normal((T, Hq, d))
    mha = O.attention(q, kf, vf, 1, False)
    ref = F.scaled_dot_product_attention(
        torch.from_numpy(q.transpose(1, 0, 2)), torch.from_numpy(kf.transpose(1, 0, 2)),
        torch.from_numpy(vf.transpose(1, 0, 2)), is_causal=False).numpy().transpose(1, 0, 2)
    _close(mha, ref, 1e-12, "MHA")


def pin_attention_brute_force():
    """Tiny shapes against pure-Python loops, causal and not, with offset
    query positions and a group size of 3."""
    r = _rng(2)
    for causal in (True, False):
        T, L, Hq, Hkv, d = 5, 9, 6, 2, 4
        q = r.standard_normal((T, Hq, d))
        k = r.standard_normal((L, Hkv, d))
        v = r.standard_normal((L, Hkv, d))
        pos = np.array([0, 2, 3, 7, 8])
        _close(O.attention(q, k, v, 3, causal, q_pos=pos),
               brute_force_attention(q, k, v, 3, causal, pos), 1e-12, f"brute causal={causal}")


def pin_attention_closed_forms():
    """Single visible key returns its value; scores ln 3 apart give weights
    3/4 and 1/4; all-ones values give ones."""
    d = 4
    k = np.zeros((2, 1, d))
    k[0, 0, 0] = 1.0
    v = np.zeros((2, 1, d))
    v[0, 0, :] = [1, 2, 3, 4]
    v[1, 0, :] = [5, 6, 7, 8]
    q = np.zeros((2, 1, d))
    q[:, 0, 0] = math.sqrt(d) * math.log(3.0)   # score(key 0) - score(key 1) = ln 3
    o = O.attention(q, k, v, 1, True)
    _close(o[0, 0], v[0, 0], 1e-12, "first position sees only key 0")
    _close(o[1, 0], 0.75 * v[0, 0] + 0.25 * v[1, 0], 1e-12, "weights 3/4, 1/4")
    r = _rng(4)
    q = r.standard_normal((6, 4, 8)) * 3
    k = r.standard_normal((6, 2, 8)) * 3
    _close(O.attention(q, k, np.ones((6, 2, 8)), 2, True), np.ones((6, 4, 8)), 1e-12, "V = 1")


# --------------------------------------------------------------------------
# RoPE
# --------------------------------------------------------------------------
def pin_rope_closed_form():
    """d = 2: the single pair turns by t radians whatever the base.
    d = 4, base 100: pairs (0, 2) and (1, 3) turn by t and t / 10."""
    t = np.array([0.0, 1.0, 2.5, 40.0])
    z = np.zeros((4, 1, 2))
    z[:, 0, 0] = 1.0
    r = O.rope(z, t, 12345.0)
    _close(r[:, 0, 0], np.cos(t), 1e-14, "d=2 cos")
    _close(r[:, 0, 1], np.sin(t), 1e-14, "d=2 sin")
    z = np.zeros((4, 1, 4))
    z[:, 0, 1] = 1.0              # second pair, first component
    r = O.rope(z, t, 100.0)
    _close(r[:, 0, 1], np.cos(t / 10), 1e-14, "pair 1 cos")
    _close(r[:, 0, 3], np.sin(t / 10), 1e-14, "pair 1 sin")
    _close(r[:, 0, 0], 0 * t, 0, "pair 0 untouched")
    _close(r[:, 0, 2], 0 * t, 0, "pair 0 untouched")
    z = np.zeros((4, 1, 4))
    z[:, 0, 2] = 1.0              # first pair, second component: (0,1) -> (-sin, cos)
    r = O.rope(z, t, 100.0)
    _close(r[:, 0, 0], -np.sin(t), 1e-14, "rotate-half sign")
    _close(r[:, 0, 2], np.cos(t), 1e-14, "rotate-half cos")
    # position 0 is the identity; base 0 disables
    zz = _rng(5).standard_normal((3, 2, 8))
    _close(O.rope(zz, np.zeros(3), 1e4), zz, 0, "position 0")
    _close(O.rope(zz, np.arange(3), 0.0), zz, 0, "base 0")


def pin_rope_relative_offset():
    """Scores after RoPE depend only on the position difference."""
    r = _rng(6)
    q = r.standard_normal((1, 3, 16))
    k = r.standard_normal((1, 3, 16))
    for base in (1e4, 5e5):
        s0 = np.einsum("thd,thd->h", O.rope(q, np.array([9]), base), O.rope(k, np.array([4]), base))
        for p in (1, 37, 1000):
            s1 = np.einsum("thd,thd->h", O.rope(q, np.array([9 + p]), base),
                           O.rope(k, np.array([4 + p]), base))
            _close(s1, s0, 1e-9, f"shift {p}")
        # the norm is kept
        _close(np.linalg.norm(O.rope(q, np.array([123]), base)), np.linalg.norm(q), 1e-12, "norm")


# --------------------------------------------------------------------------
# Convolution, QK-mean, value-shift, projection
# --------------------------------------------------------------------------
def pin_seq_conv_closed_forms():
    r = _rng(7)
    S, Ch, K = 9, 5, 4
    z = r.standard_normal((S, Ch))
    w = np.zeros((Ch, K))
    w[:, 0] = 1.0
    _close(O.seq_conv(z, w), z, 0, "identity tap")
    for j in range(1, K):
        w = np.zeros((Ch, K))
        w[:, j] = 1.0
        exp = np.zeros_like(z)
        exp[j:] = z[:-j]
        _close(O.seq_conv(z, w), exp, 0, f"shift by {j}")
        hist = r.standard_normal((K - 1, Ch))
        exp_h = exp.copy()
        exp_h[:j] = hist[K - 1 - j: K - 1]   # rows -j .. -1 come from the history
        _close(O.seq_conv(z, w, hist), exp_h, 0, f"shift by {j} with history")
    # per-channel taps: channel c scaled by (c + 1), tap 0 only
    w = np.zeros((Ch, K))
    w[:, 0] = np.arange(1, Ch + 1)
    _close(O.seq_conv(z, w), z * np.arange(1, Ch + 1), 0, "depthwise scale")
    # sum of all taps = 1 on a constant sequence (away from the start)
    w = r.random((Ch, K))
    w /= w.sum(axis=1, keepdims=True)
    _close(O.seq_conv(np.ones((S, Ch)), w)[K - 1:], np.ones((S - K + 1, Ch)), 1e-14, "partition of unity")


def pin_channel_mix_permutation():
    """A cyclic permutation matrix moves channel i+1 to channel i; a transposed
    operand would move it the other way."""
    r = _rng(8)
    S, H, d = 3, 2, 5
    u = r.standard_normal((S, H, d))
    P = np.zeros((H, d, d))
    for i in range(d):
        P[:, i, (i + 1) % d] = 1.0
    _close(O.channel_mix(u, P), np.roll(u, -1, axis=2), 0, "cyclic permutation")
    D = np.zeros((H, d, d))
    D[0] = np.eye(d) * 2.0
    D[1] = np.eye(d) * -1.0
    exp = u.copy()
    exp[:, 0] *= 2.0
    exp[:, 1] *= -1.0
    _close(O.channel_mix(u, D), exp, 0, "per-head matrices")


def pin_qk_mean_closed_form():
    """Constant heads: q~ head h = h + 1, k~ head g = 10 (g + 1)."""
    S, Hq, Hkv, d = 2, 4, 2, 3
    G = Hq // Hkv
    q = np.zeros((S, Hq, d))
    k = np.zeros((S, Hkv, d))
    for h in range(Hq):
        q[:, h] = h + 1
    for g in range(Hkv):
        k[:, g] = 10 * (g + 1)
    m_q, m_k = O.qk_mean(q, k, G)
    exp_q = np.array([(1 + 10) / 2, (2 + 10) / 2, (3 + 20) / 2, (4 + 20) / 2])
    exp_k = np.array([((1 + 2) / 2 + 10) / 2, ((3 + 4) / 2 + 20) / 2])
    _close(m_q[0, :, 0], exp_q, 0, "m_q")
    _close(m_k[0, :, 0], exp_k, 0, "m_k")
    r = _rng(9)
    q1 = r.standard_normal((4, 3, 6))
    k1 = r.standard_normal((4, 3, 6))
    a, b = O.qk_mean(q1, k1, 1)
    _close(a, b, 0, "G = 1: one shared mean")


def pin_value_shift_gather():
    r = _rng(10)
    S, Hkv, d = 6, 3, 8
    v = r.standard_normal((S, Hkv, d))
    out = O.value_shift(v)
    assert np.array_equal(out[:, :, : d // 2], v[:, :, : d // 2])
    assert np.array_equal(out[1:, :, d // 2:], v[:-1, :, d // 2:])
    assert np.all(out[0, :, d // 2:] == 0)
    prev = r.standard_normal((Hkv, d))
    out = O.value_shift(v, prev)
    assert np.array_equal(out[0, :, d // 2:], prev[:, d // 2:])


def pin_down_project_blocks():
    """With W = I the projection returns the column blocks q | k | v in order."""
    sh = O.Shape(E=48, C=1, Hq=2, Hkv=1)     # d = 24, n_qkv = 96
    x = _rng(11).standard_normal((3, sh.n_qkv))
    q, k, v = O.down_project(x, None, sh)
    d = sh.d
    _close(q.reshape(3, -1), x[:, :2 * d], 0, "q block")
    _close(k.reshape(3, -1), x[:, 2 * d:3 * d], 0, "k block")
    _close(v.reshape(3, -1), x[:, 3 * d:], 0, "v block")
    sh2 = O.Shape(E=sh.n_qkv, C=2, Hq=1, Hkv=1)   # E = 96, d = 48, n_qkv = 144
    x2 = _rng(12).standard_normal((3, sh2.E))
    W2 = np.zeros((sh2.n_qkv, sh2.E))
    W2[:96, :96] = np.eye(96)                     # q = x[:, :48], k = x[:, 48:96], v = 0
    q2, k2, v2 = O.down_project(x2, W2, sh2)
    _close(q2.reshape(3, -1), x2[:, :48], 0, "q from W rows")
    _close(k2.reshape(3, -1), x2[:, 48:96], 0, "k from W rows")
    _close(v2, np.zeros_like(v2), 0, "v rows zero")


def pin_output_projection():
    """The up-projection against explicit loops, a permutation and linearity."""
    rng = _rng(21)
    M, J, E = 3, 5, 4                       # rectangular: a transposed W_o cannot apply
    o = rng.standard_normal((M, J))
    W = rng.standard_normal((E, J))
    y = O.output_projection(o, W)
    assert y.shape == (M, E)
    ref = np.zeros((M, E))
    for m in range(M):
        for e in range(E):
            acc = 0.0
            for j in range(J):
                acc += o[m, j] * W[e, j]
            ref[m, e] = acc
    _close(y, ref, 1e-12, "explicit loops")
    # W_o = a permutation matrix P (row e picks latent feature p[e]): y[:, e] = o[:, p[e]]
    p = np.array([2, 0, 3, 1])
    P = np.zeros((4, 4))
    P[np.arange(4), p] = 1.0
    o4 = rng.standard_normal((2, 4))
    _close(O.output_projection(o4, P), o4[:, p], 0, "permutation")
    # linear in o
    o2 = rng.standard_normal((M, J))
    _close(O.output_projection(2.5 * o + o2, W), 2.5 * y + O.output_projection(o2, W), 1e-12,
           "linearity")
    # after a prefill: the layer output of a tiny layer equals the loops on its rows
    sh = O.Shape(E=8, C=2, Hq=2, Hkv=1)     # latent width Hq d = 4
    layer = O.Layer(sh, rng.standard_normal((sh.n_qkv, sh.E)) / 3, conv_width=0,
                    qk_mean=False, value_shift=False)
    out, _ = O.prefill(layer, rng.standard_normal((3, sh.E)))
    Wo = rng.standard_normal((sh.E, sh.Hq * sh.d))
    y3 = O.output_projection(out, Wo)
    for m in range(3):
        for e in range(sh.E):
            assert abs(y3[m, e] - sum(out[m, j] * Wo[e, j] for j in range(4))) < 1e-12


# --------------------------------------------------------------------------
# Whole-layer invariants
# --------------------------------------------------------------------------
def _composition_layer(d, rope_base):
    """A packed-input layer (x rows are q~ | k~ | v~) with Hq = 2, Hkv = 1,
    conv width 2 and per-channel taps: even channels keep the current row
    (tap 0), odd channels take the previous row (tap 1).  The channel mix is
    the cyclic permutation y[i] = u[(i + 1) mod d] in both heads.  With lags
    that differ between neighbouring channels the conv and the mix do not
    commute, so their order is visible."""
    sh = O.Shape(E=2 * d, C=1, Hq=2, Hkv=1)
    P = np.zeros((d, d))
    for i in range(d):
        P[i, (i + 1) % d] = 1.0

    def taps(ch):
        w = np.zeros((ch, 2))
        w[np.arange(ch) % 2 == 0, 0] = 1.0
        w[np.arange(ch) % 2 == 1, 1] = 1.0
        return w

    return O.Layer(sh=sh, W_qkv=None, conv_width=2,
                   conv_q_seq=taps(2 * d), conv_q_chan=np.stack([P, P]),
                   conv_k_seq=taps(d), conv_k_chan=P[None].copy(),
                   qk_mean=True, value_shift=True, rope_base=rope_base, causal=True)


def _composition_by_hand(qt, kt, vt, d, rope_on):
    """q, k, v of the composition layer written out index by index from the
    spec's steps: sequence conv, then channel mix, then the QK-mean of the
    PRE-conv values added, then RoPE (d = 2: the pair turns by t radians),
    and the value-shift of the upper half-channels."""
    S = qt.shape[0]

    def pre(z, t, h, c):             # z[t - lag(c)], lag 0 on even and 1 on odd channels
        s = t - c % 2
        return z[s, h, c] if s >= 0 else 0.0

    q = np.zeros((S, 2, d))
    k = np.zeros((S, 1, d))
    v = np.zeros((S, 1, d))
    for t in range(S):
        for i in range(d):
            j = (i + 1) % d          # the mix reads conv channel i + 1
            for h in range(2):
                m_q = 0.5 * (qt[t, h, i] + kt[t, 0, i])
                q[t, h, i] = pre(qt, t, h, j) + m_q
            m_k = 0.5 * (0.5 * (qt[t, 0, i] + qt[t, 1, i]) + kt[t, 0, i])
            k[t, 0, i] = pre(kt, t, 0, j) + m_k
            if i < d // 2:
                v[t, 0, i] = vt[t, 0, i]
            else:
                v[t, 0, i] = vt[t - 1, 0, i] if t > 0 else 0.0
        if rope_on:                  # d = 2: (a, b) -> (a cos t - b sin t, a sin t + b cos t)
            c, s = math.cos(t), math.sin(t)
            for z in (q[t], k[t]):
                for h in range(z.shape[0]):
                    a, b = z[h, 0], z[h, 1]
                    z[h, 0], z[h, 1] = a * c - b * s, a * s + b * c
    return q, k, v


def pin_layer_composition():
    """The whole layer on a tiny case against values written out by hand:
    which tensors feed QK-mean (the pre-conv q~ and k~), the order of the
    sequence conv and the channel mix, and RoPE after the QK-mean add (CCA
    page, Methodologie items 2-4).  Checks the prefill's q, its cache k and v,
    every output row (brute-force attention on the hand values), and a decode
    step from the prefix state."""
    r = _rng(22)
    for d, base in ((4, 0.0), (2, 777.0)):
        lay = _composition_layer(d, base)
        S = 6
        x = r.standard_normal((S, 4 * d))
        qt = x[:, :2 * d].reshape(S, 2, d)
        kt = x[:, 2 * d:3 * d].reshape(S, 1, d)
        vt = x[:, 3 * d:].reshape(S, 1, d)
        q, k, v = _composition_by_hand(qt, kt, vt, d, base != 0.0)
        out, st = O.prefill(lay, x)
        _close(st.extra["q"], q, 1e-13, f"d={d} q")
        _close(st.k, k, 1e-13, f"d={d} cache k")
        _close(st.v, v, 0, f"d={d} cache v")
        o = brute_force_attention(q, k, v, 2, True, np.arange(S))
        _close(out, o.reshape(S, -1), 1e-12, f"d={d} output rows")
        # decode of the last token from the state after S - 1 tokens
        _, st5 = O.prefill(lay, x[:-1])
        od, nst = O.decode_step(lay, st5, x[-1])
        _close(nst.extra["q"][0], q[-1], 1e-13, f"d={d} decode q")
        _close(nst.k[-1], k[-1], 1e-13, f"d={d} decode k")
        _close(od, o[-1].reshape(-1), 1e-12, f"d={d} decode output")


def pin_qk_mean_self_composition():
    """The "self" QK-mean reading on the composition layer, written out by
    hand: each head's output is the mean of its own pre-conv value and its
    conv output, with no k term in q and no q term in k (CCA page,
    Methodologie item 2, the literal reading)."""
    r = _rng(23)
    d, S = 4, 6
    lay = _composition_layer(d, 0.0)
    lay.qk_mean = O.QK_SELF
    x = r.standard_normal((S, 4 * d))
    qt = x[:, :2 * d].reshape(S, 2, d)
    kt = x[:, 2 * d:3 * d].reshape(S, 1, d)

    def conv_mix(z, t, h, i):          # lag 0 on even, 1 on odd channels, then y[i] = u[i+1]
        j = (i + 1) % d
        s_ = t - j % 2
        return z[s_, h, j] if s_ >= 0 else 0.0

    q = np.zeros((S, 2, d))
    k = np.zeros((S, 1, d))
    for t in range(S):
        for i in range(d):
            for h in range(2):
                q[t, h, i] = 0.5 * (qt[t, h, i] + conv_mix(qt, t, h, i))
            k[t, 0, i] = 0.5 * (kt[t, 0, i] + conv_mix(kt, t, 0, i))
    _, st = O.prefill(lay, x)
    _close(st.extra["q"], q, 1e-14, "self q")
    _close(st.k, k, 1e-14, "self k")
    _, st5 = O.prefill(lay, x[:-1])
    _, nst = O.decode_step(lay, st5, x[-1])
    _close(nst.extra["q"][0], q[-1], 1e-14, "self decode q")
    _close(nst.k[-1], k[-1], 1e-14, "self decode k")


def pin_value_shift_heads_gather():
    """Whole-head value-shift: the last floor(Hkv/2) kv heads carry the
    previous token's values, bit for bit (CCA page, Methodologie item 3, read
    per head)."""
    r = _rng(24)
    for Hkv, shifted in ((4, {2, 3}), (3, {2}), (2, {1}), (1, set())):
        S, d = 5, 6
        v = r.standard_normal((S, Hkv, d))
        prev = r.standard_normal((Hkv, d))
        for vp in (None, prev):
            out = O.value_shift_heads(v, vp)
            for g in range(Hkv):
                for t in range(S):
                    if g in shifted:
                        want = (prev[g] if vp is not None else np.zeros(d)) if t == 0 else v[t - 1, g]
                    else:
                        want = v[t, g]
                    assert np.array_equal(out[t, g], want), (Hkv, g, t)


def pin_channel_conv_closed_forms():
    """The temporal channel conv: identity at tap 0, a cyclic channel
    permutation at tap 1 (which a transposed matrix or reversed taps would
    turn the other way), history rows, and a random two-tap case against
    explicit loops."""
    r = _rng(25)
    S, H, d, K = 5, 2, 4, 3
    z = r.standard_normal((S, H, d))
    W = np.zeros((H, K, d, d))
    W[:, 0] = np.eye(d)
    _close(O.channel_conv(z, W), z, 0, "identity tap")
    W = np.zeros((H, K, d, d))
    for i in range(d):
        W[:, 1, i, (i + 1) % d] = 1.0            # y[t, i] = z[t - 1, i + 1]
    exp = np.zeros_like(z)
    exp[1:] = np.roll(z[:-1], -1, axis=2)
    _close(O.channel_conv(z, W), exp, 0, "shifted permutation")
    hist = r.standard_normal((K - 1, H * d))
    exp_h = exp.copy()
    exp_h[0] = np.roll(hist[K - 2].reshape(H, d), -1, axis=1)   # row -1 is the newest history row
    _close(O.channel_conv(z, W, hist), exp_h, 0, "history")
    W = r.standard_normal((H, 2, d, d))
    y = O.channel_conv(z, W)
    for t in range(S):
        for h in range(H):
            for i in range(d):
                acc = 0.0
                for j in range(2):
                    if t - j >= 0:
                        for c in range(d):
                            acc += W[h, j, i, c] * z[t - j, h, c]
                assert abs(y[t, h, i] - acc) < 1e-12


def _variant_layers():
    """The reading variants: QK-mean "self", whole-head value-shift, and the
    temporal channel conv (per-tap d x d matrices)."""
    a = _small_layer()
    a.qk_mean = O.QK_SELF
    b = _small_layer(Hkv=2)
    b.value_shift = O.VS_WHOLE_HEADS
    c = _small_layer(seed=5)
    r = _rng(26)
    sh = c.sh
    c.channel_conv = True
    c.conv_q_chan = r.standard_normal((sh.Hq, 4, sh.d, sh.d)) / (2 * math.sqrt(sh.d))
    c.conv_k_chan = r.standard_normal((sh.Hkv, 4, sh.d, sh.d)) / (2 * math.sqrt(sh.d))
    c.conv_q_seq = c.conv_k_seq = None
    return a, b, c


def pin_causality():
    """Changing tokens after position t leaves outputs up to t unchanged
    (covers the convolution, the value-shift and the mask), for the default
    readings and the variants."""
    for lay in (_small_layer(), *_variant_layers()):
        r = _rng(13)
        S = 12
        x = r.standard_normal((S, lay.sh.E))
        o1, _ = O.prefill(lay, x)
        x2 = x.copy()
        x2[7:] = r.standard_normal((S - 7, lay.sh.E))
        o2, _ = O.prefill(lay, x2)
        _close(o2[:7], o1[:7], 1e-13, "prefix unchanged")
        assert np.max(np.abs(o2[7:] - o1[7:])) > 1e-3, "later rows must change"


def pin_decode_matches_prefill():
    """prefill over S tokens, row S-1 == prefill over S-1 tokens followed by one
    decode step; the decode state equals the longer prefill's state."""
    for lay in (_small_layer(), _small_layer(K=2, chan=False, qk=False),
                _small_layer(K=0, qk=False, vs=False, base=0.0), *_variant_layers()):
        r = _rng(14)
        S = 10
        x = r.standard_normal((S, lay.sh.E))
        full, st_full = O.prefill(lay, x)
        part, st = O.prefill(lay, x[:-1])
        o, st2 = O.decode_step(lay, st, x[-1])
        _close(o, full[-1], 1e-12, "decode row")
        _close(st2.k, st_full.k, 1e-12, "cache k")
        _close(st2.v, st_full.v, 1e-12, "cache v")
        _close(st2.hist_q, st_full.hist_q, 1e-13, "hist q")
        _close(st2.hist_k, st_full.hist_k, 1e-13, "hist k")
        _close(st2.v_prev, st_full.v_prev, 1e-13, "v_prev")
        # two more steps from the end of the full prefill stay consistent
        x3 = r.standard_normal((2, lay.sh.E))
        ref, _ = O.prefill(lay, np.concatenate([x, x3]))
        o1, s1 = O.decode_step(lay, st_full, x3[0])
        o2, _ = O.decode_step(lay, s1, x3[1])
        _close(np.stack([o1, o2]), ref[-2:], 1e-12, "two steps")


def pin_prefill_rows_subset():
    lay = _small_layer()
    x = _rng(15).standard_normal((11, lay.sh.E))
    full, _ = O.prefill(lay, x)
    rows = np.array([0, 3, 10])
    part, _ = O.prefill(lay, x, rows=rows)
    _close(part, full[rows], 0, "sampled rows")


def pin_features_off_is_plain_gqa():
    """With no conv, QK-mean, value-shift or RoPE the layer is plain GQA on the
    projected heads (library special case: SDPA with grouped heads)."""
    lay = _small_layer(K=0, qk=False, vs=False, base=0.0, packed=True)
    sh = lay.sh
    x = _rng(16).standard_normal((9, sh.n_qkv))
    o, _ = O.prefill(lay, x)
    d = sh.d
    q = torch.from_numpy(x[:, :sh.Hq * d].reshape(9, sh.Hq, d).transpose(1, 0, 2).copy())
    k = torch.from_numpy(x[:, sh.Hq * d:(sh.Hq + sh.Hkv) * d].reshape(9, sh.Hkv, d).transpose(1, 0, 2).copy())
    v = torch.from_numpy(x[:, (sh.Hq + sh.Hkv) * d:].reshape(9, sh.Hkv, d).transpose(1, 0, 2).copy())
    ref = F.scaled_dot_product_attention(q[None], k[None], v[None], is_causal=True, enable_gqa=True)
    _close(o, ref[0].permute(1, 0, 2).reshape(9, -1).numpy(), 1e-12, "plain GQA")


def pin_cache_sizing():
    """The GQA page's Llama 3.1 8B cache arithmetic."""
    g = read_golden("gqa_cache_sizing.txt")
    L, H, d, b, ctx, Hm = (int(g[k]) for k in ("layers", "kv_heads", "head_dim", "bytes_per_value",
                                               "context_tokens", "mha_kv_heads"))
    per_tok = L * O.cache_values_per_token(H, d) * b
    assert per_tok == int(g["kib_per_token_gqa"]) * 1024
    assert per_tok * ctx == int(g["gib_full_context_gqa"]) * 2 ** 30
    per_tok_m = L * O.cache_values_per_token(Hm, d) * b
    assert per_tok_m == int(g["kib_per_token_mha"]) * 1024
    assert per_tok_m * ctx == int(g["gib_full_context_mha"]) * 2 ** 30


def pin_compression_factor():
    """Attention work and cache shrink by the compression factor C at a fixed
    head count (CCA page, "Belangrijkste Bijdragen" and "Resultaten" 3)."""
    E, Hq, S = 4096, 32, 1000
    for C in (1, 2, 4, 8):
        sh = O.Shape(E, C, Hq, Hq)
        mha = O.Shape(E, 1, Hq, Hq)
        assert O.attention_flops(S, Hq, sh.d) * C == O.attention_flops(S, Hq, mha.d)
        assert O.cache_values_per_token(Hq, sh.d) * C == O.cache_values_per_token(Hq, mha.d)
    # counted flops equal the visible score pairs times 4 d
    assert O.attention_flops(4, 1, 8, causal=False) == 4 * 8 * 16


# --------------------------------------------------------------------------
# Backward pass
# --------------------------------------------------------------------------
def _fd_check(lay, x, dout, names, n_samples, rng, tol, what):
    """Central finite differences of L = sum(dout * prefill(x)) against the
    oracle's gradients, on sampled entries of x and of each named weight."""
    g = O.prefill_backward(lay, x, dout)
    eps = 1e-6

    def loss():
        o, _ = O.prefill(lay, x)
        return float(np.sum(o * dout))

    for name in names:
        arr = x if name == "dx" else getattr(lay, name)
        grad = g[name]
        assert grad is not None and grad.shape == arr.shape, (what, name)
        flat = arr.reshape(-1)
        picks = rng.choice(flat.size, size=min(n_samples, flat.size), replace=False)
        scale = max(1.0, float(np.max(np.abs(grad))))
        for i in picks:
            old = flat[i]
            flat[i] = old + eps
            lp = loss()
            flat[i] = old - eps
            lm = loss()
            flat[i] = old
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - grad.reshape(-1)[i]) <= tol * scale, \
                f"{what} d{name}[{i}]: finite difference {fd:.8e} vs {grad.reshape(-1)[i]:.8e}"


def pin_backward_finite_differences():
    """The layer's backward against central finite differences of its
    forward (float64, step 1e-6), for the default readings, each variant,
    plain GQA, a non-causal layer and one without RoPE, on sampled entries
    of the input and of every weight."""
    r = _rng(31)
    layers = [
        ("default", _small_layer(seed=7), True),
        ("noncausal", _small_layer(seed=8, causal=False), True),
        ("norope_k2_nochan", _small_layer(seed=9, K=2, chan=False, base=0.0), True),
        ("plain_gqa", _small_layer(seed=10, K=0, qk=False, vs=False, base=0.0), True),
        *[(f"variant{i}", lay, True) for i, lay in enumerate(_variant_layers())],
    ]
    for what, lay, _ in layers:
        S = 7
        x = r.standard_normal((S, lay.sh.E))
        dout = r.standard_normal((S, lay.sh.Hq * lay.sh.d))
        names = ["dx", "W_qkv"]
        for w in ("conv_q_seq", "conv_q_chan", "conv_k_seq", "conv_k_chan"):
            if getattr(lay, w) is not None and lay.conv_width > 0:
                names.append(w)
        _fd_check(lay, x, dout, names, 12, r, 1e-6, what)


def pin_attention_backward_closed_forms():
    """All-ones values make the output independent of the scores, so dq and
    dk vanish and dv holds the probability-weighted sums of dout (which
    add up to dout's total per head); a query that sees one key passes its
    gradient to that key's value unchanged."""
    r = _rng(32)
    T, Hq, Hkv, d = 6, 4, 2, 8
    q = r.standard_normal((T, Hq, d)) * 2
    k = r.standard_normal((T, Hkv, d)) * 2
    dout = r.standard_normal((T, Hq, d))
    dq, dk, dv = O.attention_backward(q, k, np.ones((T, Hkv, d)), 2, True, dout)
    _close(dq, np.zeros_like(dq), 1e-12, "V = 1: dq")
    _close(dk, np.zeros_like(dk), 1e-12, "V = 1: dk")
    _close(dv.sum(axis=0), dout.reshape(T, Hkv, 2, d).sum(axis=(0, 2)), 1e-12, "V = 1: dv total")
    v = r.standard_normal((T, Hkv, d))
    dq, dk, dv = O.attention_backward(q[:1], k, v, 2, True, dout[:1])   # position 0: key 0 only
    _close(dq, np.zeros_like(dq), 1e-12, "one key: dq")
    _close(dv[0], dout[0].reshape(Hkv, 2, d).sum(axis=1), 1e-12, "one key: dv")
    _close(dv[1:], np.zeros_like(dv[1:]), 0, "one key: other values")


def pin_attention_backward_sdpa():
    """The attention backward against torch's float64 autograd through
    scaled_dot_product_attention on copied kv heads (a library special case)."""
    r = _rng(33)
    for causal in (True, False):
        T, Hq, Hkv, d = 9, 6, 2, 8
        G = Hq // Hkv
        q = r.standard_normal((T, Hq, d))
        k = r.standard_normal((T, Hkv, d))
        v = r.standard_normal((T, Hkv, d))
        dout = r.standard_normal((T, Hq, d))
        tq = torch.from_numpy(q.transpose(1, 0, 2).copy()).requires_grad_()
        tk = torch.from_numpy(k.transpose(1, 0, 2).copy()).requires_grad_()
        tv = torch.from_numpy(v.transpose(1, 0, 2).copy()).requires_grad_()
        o = F.scaled_dot_product_attention(tq[None], tk.repeat_interleave(G, 0)[None],
                                           tv.repeat_interleave(G, 0)[None], is_causal=causal)
        o.backward(torch.from_numpy(dout.transpose(1, 0, 2).copy())[None])
        dq, dk, dv = O.attention_backward(q, k, v, G, causal, dout)
        _close(dq, tq.grad.numpy().transpose(1, 0, 2), 1e-12, f"dq causal={causal}")
        _close(dk, tk.grad.numpy().transpose(1, 0, 2), 1e-12, f"dk causal={causal}")
        _close(dv, tv.grad.numpy().transpose(1, 0, 2), 1e-12, f"dv causal={causal}")


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_") and callable(v)]
