"""Float64 CPU oracle for the CCGQA forward pass.

TEST INFRASTRUCTURE ONLY.  This module is the plain, slow statement of what the
CUDA path computes.  Only the test suite, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it; the
product package never does, and this module imports nothing from the product.

Sources (web pages; section names as printed on them):

* "Compressed Convolutional Attention: Efficient Attention in a Compressed
  Latent Space" (gist.science summary of arXiv 2510.04476), section
  "Methodologie", items 1-4, and section "Compressed Convolutional Grouped
  Query Attention (CCGQA)".  Abbreviated below as [CCA <section>].
* "Grouped Query Attention (GQA)" (Ultralytics glossary), sections
  "Cómo funciona GQA" and "Por qué GQA reduce la caché KV".  Abbreviated [GQA
  <section>].

The CCA page is a lay summary without formulas.  Where it leaves a step open
this oracle takes one fixed reading (each function says which); the CUDA
kernels follow the same reading.

Notation: S sequence length, E model width, C compression factor, Hq query
heads, Hkv kv heads, G = Hq / Hkv group size, d = E / (C * Hq) head dim,
K conv width.  All arrays are float64; the caller passes inputs already rounded
to the working dtype (bf16 or fp32) so both sides see identical values.

Parity pins: every function here is pinned by a test under ``tests/`` that
checks it against something other than itself (closed forms, a library special
case, brute force, invariants).  The semantics of the convolution, QK-mean and
value-shift readings themselves cannot be pinned against the pages (the pages
print no example): for those three readings the parity is "parity unpinned"
with respect to the paper, while the arithmetic of each reading is pinned, and
so is the order in which ``_mix_qk``, ``prefill`` and ``decode_step`` compose
them (a whole-layer case written out by hand).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "Shape", "down_project", "seq_conv", "channel_mix", "channel_conv", "qk_mean",
    "qk_mean_self", "rope", "value_shift", "value_shift_heads", "attention", "prefill",
    "decode_step", "kvcache_append", "output_projection", "cache_values_per_token",
    "attention_flops", "QK_OFF", "QK_CROSS", "QK_SELF", "VS_OFF", "VS_HALF_CHANNELS",
    "VS_WHOLE_HEADS", "attention_backward", "prefill_backward",
]

# Switches of the readings a layer can take (the CCA page's wording admits
# more than one; see the functions below).
QK_OFF, QK_CROSS, QK_SELF = 0, 1, 2
VS_OFF, VS_HALF_CHANNELS, VS_WHOLE_HEADS = 0, 1, 2


@dataclass(frozen=True)
class Shape:
    """Head geometry of one CCGQA layer [CCA Methodologie 1; CCGQA]."""

    E: int
    C: int
    Hq: int
    Hkv: int

    @property
    def d(self) -> int:
        # latent width e~ = E / C is split evenly over the query heads
        return self.E // (self.C * self.Hq)

    @property
    def G(self) -> int:
        # query heads that share one kv head [GQA Cómo funciona GQA]
        return self.Hq // self.Hkv

    @property
    def n_qkv(self) -> int:
        return (self.Hq + 2 * self.Hkv) * self.d


# --------------------------------------------------------------------------
# a1: latent down-projection  [CCA Methodologie 1 "Compressie in Latente Ruimte"]
# --------------------------------------------------------------------------
def down_project(x: np.ndarray, W_qkv: np.ndarray | None, sh: Shape):
    """Project tokens straight into the latent space of width E/C.

    x: [S, E] (or, when ``W_qkv is None``, already the projected rows
    [S, (Hq + 2 Hkv) d]).  W_qkv: [(Hq + 2 Hkv) d, E], output-feature major;
    rows [0, Hq d) give q~, the next Hkv d give k~, the last Hkv d give v~.
    Reading: no bias terms.
    Returns q_pre [S, Hq, d], k_pre [S, Hkv, d], v_lat [S, Hkv, d].
    """
    y = x if W_qkv is None else x @ W_qkv.T
    S = y.shape[0]
    d, Hq, Hkv = sh.d, sh.Hq, sh.Hkv
    q = y[:, : Hq * d].reshape(S, Hq, d)
    k = y[:, Hq * d: (Hq + Hkv) * d].reshape(S, Hkv, d)
    v = y[:, (Hq + Hkv) * d:].reshape(S, Hkv, d)
    return q, k, v


# --------------------------------------------------------------------------
# a2: causal sequence convolution  [CCA Methodologie 2 "Convolutionele Mixing"]
# --------------------------------------------------------------------------
def seq_conv(z: np.ndarray, w_seq: np.ndarray, history: np.ndarray | None = None):
    """Depthwise causal convolution along the sequence.

    z: [S, Ch]; w_seq: [Ch, K]; tap j multiplies the row j steps back:
        u[t, c] = sum_{j=0}^{K-1} w_seq[c, j] * z[t - j, c].
    Rows before the start come from ``history`` ([K-1, Ch], oldest first, so
    history[K-1-j] is row -j) or are zero when no history is given.
    Reading: depthwise, causal, left zero padding, no bias.
    """
    S, Ch = z.shape
    K = w_seq.shape[1]
    if history is None:
        history = np.zeros((K - 1, Ch))
    full = np.concatenate([history, z], axis=0)  # row t of z is row t+K-1 here
    u = np.zeros((S, Ch))
    for t in range(S):
        for j in range(K):
            u[t] += w_seq[:, j] * full[t + K - 1 - j]
    return u


# --------------------------------------------------------------------------
# a3: per-head channel mix  [CCA Methodologie 2, "binnen de kanalen van een head"]
# --------------------------------------------------------------------------
def channel_mix(u: np.ndarray, W_chan: np.ndarray):
    """Mix the channels inside each head: y[t, h, i] = sum_i' W[h, i, i'] u[t, h, i'].

    u: [S, H, d]; W_chan: [H, d, d].  Reading: a width-1 (per position) dense
    map inside every head, applied after the sequence convolution.
    """
    return np.einsum("hij,thj->thi", W_chan, u)


def channel_conv(z: np.ndarray, W: np.ndarray, history: np.ndarray | None = None):
    """Temporal channel convolution inside each head (a reading variant of
    [CCA Methodologie 2]: the conv mixes the channels of a head with its own
    d x d matrix at every tap, instead of a depthwise sequence conv followed
    by one per-position mix):
        y[t, h, :] = sum_{j=0}^{K-1} W[h, j] @ z[t - j, h, :].

    z: [S, H, d] pre-convolution rows; W: [H, K, d, d]; history: [K-1, H d]
    (oldest first, as for seq_conv) or None for zeros before the start.  The
    depthwise-plus-mix reading is the special case W[h, j] = W_c[h] diag(w_seq[h, :, j]).
    """
    S, H, d = z.shape
    K = W.shape[1]
    hist = np.zeros((K - 1, H, d)) if history is None else history.reshape(K - 1, H, d)
    full = np.concatenate([hist, z], axis=0)      # row t of z is row t+K-1 here
    y = np.zeros((S, H, d))
    for t in range(S):
        for j in range(K):
            y[t] += np.einsum("hij,hj->hi", W[:, j], full[t + K - 1 - j])
    return y


# --------------------------------------------------------------------------
# a4: QK-mean  [CCA Methodologie 2 "QK-Mean"]
# --------------------------------------------------------------------------
def qk_mean(q_pre: np.ndarray, k_pre: np.ndarray, G: int):
    """Shared pre-convolution mean added back to q and k (skip connection).

    Reading ("cross"): the mean of the pre-convolution query and key of the
    same position is added to both, with GQA head counts reconciled:
        m_q[t, h] = (q_pre[t, h] + k_pre[t, h // G]) / 2
        m_k[t, g] = (mean_{h in group g} q_pre[t, h] + k_pre[t, g]) / 2
    Returns (m_q [S, Hq, d], m_k [S, Hkv, d]).
    """
    S, Hq, d = q_pre.shape
    Hkv = k_pre.shape[1]
    k_rep = np.repeat(k_pre, G, axis=1)
    m_q = 0.5 * (q_pre + k_rep)
    q_grp = q_pre.reshape(S, Hkv, G, d).mean(axis=2)
    m_k = 0.5 * (q_grp + k_pre)
    return m_q, m_k


def qk_mean_self(q_pre, y_q, k_pre, y_k):
    """Reading variant "self" of [CCA Methodologie 2 "QK-Mean"]: each head's
    output is the mean of its own pre- and post-convolution values,
        q = (q_pre + y_q) / 2,   k = (k_pre + y_k) / 2,
    the literal reading of the garbled sentence (no mixing between q and k)."""
    return 0.5 * (q_pre + y_q), 0.5 * (k_pre + y_k)


# --------------------------------------------------------------------------
# a5: RoPE inside the latent heads  [CCA Methodologie 4 "Integratie van RoPE"]
# --------------------------------------------------------------------------
def rope(z: np.ndarray, positions: np.ndarray, base: float):
    """Rotary position embedding on every latent head, full head width.

    z: [S, H, d] at absolute positions ``positions`` [S] (0-based).  Pairs are
    (i, i + d/2) for i < d/2 ("rotate-half"); pair i turns by angle
    t * base ** (-2 i / d):
        (a, b) -> (a cos - b sin, a sin + b cos).
    base == 0 disables it.
    """
    if base == 0:
        return z.copy()
    d = z.shape[-1]
    half = d // 2
    i = np.arange(half, dtype=np.float64)
    theta = base ** (-2.0 * i / d)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * theta[None, :]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    a, b = z[..., :half], z[..., half:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


# --------------------------------------------------------------------------
# a6: value-shift  [CCA Methodologie 3 "Value-Shift"]
# --------------------------------------------------------------------------
def value_shift(v_lat: np.ndarray, v_prev: np.ndarray | None = None):
    """Each kv head gets values of the current token and of the previous one.

    Reading: channels [0, d/2) of a head keep the current row, channels
    [d/2, d) take the previous row's channels; the row before the first is
    ``v_prev`` ([Hkv, d]) or zero.  v_lat: [S, Hkv, d].
    """
    S, Hkv, d = v_lat.shape
    prev = np.zeros((1, Hkv, d)) if v_prev is None else v_prev[None]
    shifted = np.concatenate([prev, v_lat[:-1]], axis=0)
    out = v_lat.copy()
    out[..., d // 2:] = shifted[..., d // 2:]
    return out


def value_shift_heads(v_lat: np.ndarray, v_prev: np.ndarray | None = None):
    """Whole-head reading variant of [CCA Methodologie 3 "Value-Shift"]: half
    of the kv heads take the previous token's values.  The last floor(Hkv/2)
    heads are shifted (heads g >= Hkv - floor(Hkv/2)), the others keep the
    current row; the row before the first is ``v_prev`` ([Hkv, d]) or zero.
    With one kv head nothing is shifted."""
    S, Hkv, d = v_lat.shape
    prev = np.zeros((1, Hkv, d)) if v_prev is None else v_prev[None]
    shifted = np.concatenate([prev, v_lat[:-1]], axis=0)
    out = v_lat.copy()
    g0 = Hkv - Hkv // 2
    out[:, g0:] = shifted[:, g0:]
    return out


# --------------------------------------------------------------------------
# a8: grouped-query softmax attention  [CCA CCGQA; GQA Cómo funciona GQA]
# --------------------------------------------------------------------------
def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, G: int, causal: bool,
              q_pos: np.ndarray | None = None):
    """Scaled dot-product attention where query head h reads kv head h // G.

    q: [T, Hq, d] at positions ``q_pos`` (default 0..T-1); k, v: [L, Hkv, d]
    at positions 0..L-1.  With ``causal`` a query at position t sees keys
    s <= t.  Scale 1/sqrt(d); the softmax subtracts the row maximum.
    Returns o [T, Hq, d].
    """
    T, Hq, d = q.shape
    L = k.shape[0]
    if q_pos is None:
        q_pos = np.arange(T)
    q_pos = np.asarray(q_pos)
    o = np.zeros((T, Hq, d))
    scale = 1.0 / math.sqrt(d)
    keys = np.arange(L)
    for h in range(Hq):
        g = h // G
        sc = (q[:, h, :] @ k[:, g, :].T) * scale
        if causal:
            sc = np.where(keys[None, :] <= q_pos[:, None], sc, -np.inf)
        sc = sc - sc.max(axis=1, keepdims=True)
        p = np.exp(sc)
        p = p / p.sum(axis=1, keepdims=True)
        o[:, h, :] = p @ v[:, g, :]
    return o


# --------------------------------------------------------------------------
# The whole layer
# --------------------------------------------------------------------------
@dataclass
class Layer:
    """Switches and weights of one CCGQA layer (float64 copies)."""

    sh: Shape
    W_qkv: np.ndarray | None
    conv_width: int = 4
    conv_q_seq: np.ndarray | None = None     # [Hq d, K]
    conv_q_chan: np.ndarray | None = None    # [Hq, d, d] or None = no channel mix
    conv_k_seq: np.ndarray | None = None     # [Hkv d, K]
    conv_k_chan: np.ndarray | None = None    # [Hkv, d, d]
    qk_mean: int = QK_CROSS                  # QK_OFF / QK_CROSS / QK_SELF (bools: off / cross)
    value_shift: int = VS_HALF_CHANNELS      # VS_OFF / VS_HALF_CHANNELS / VS_WHOLE_HEADS
    rope_base: float = 10000.0
    causal: bool = True
    # True: the temporal channel conv (channel_conv); conv_*_chan are then
    # [H, K, d, d] per-tap matrices and conv_*_seq are unused
    channel_conv: bool = False


@dataclass
class State:
    """Decode state of one sequence: latent KV cache plus the short histories
    the causal convolution and the value-shift need."""

    k: np.ndarray                       # [len, Hkv, d]  post-RoPE keys
    v: np.ndarray                       # [len, Hkv, d]  shifted values
    hist_q: np.ndarray                  # [K-1, Hq d]  pre-conv q~ rows, oldest first
    hist_k: np.ndarray                  # [K-1, Hkv d]
    v_prev: np.ndarray                  # [Hkv d]  last v~ row (before the shift)
    extra: dict = field(default_factory=dict)

    @property
    def length(self) -> int:
        return self.k.shape[0]


def _mix_qk(layer: Layer, q_pre, k_pre, hq=None, hk=None):
    """Steps a2-a4 on q~ and k~ (pre-conv [T, H, d]) with optional histories."""
    sh = layer.sh
    T = q_pre.shape[0]
    d = sh.d
    if layer.conv_width > 0 and layer.channel_conv:
        y_q = channel_conv(q_pre, layer.conv_q_chan, hq)
        y_k = channel_conv(k_pre, layer.conv_k_chan, hk)
    elif layer.conv_width > 0:
        u_q = seq_conv(q_pre.reshape(T, -1), layer.conv_q_seq, hq).reshape(T, sh.Hq, d)
        u_k = seq_conv(k_pre.reshape(T, -1), layer.conv_k_seq, hk).reshape(T, sh.Hkv, d)
        y_q = u_q if layer.conv_q_chan is None else channel_mix(u_q, layer.conv_q_chan)
        y_k = u_k if layer.conv_k_chan is None else channel_mix(u_k, layer.conv_k_chan)
    else:
        y_q, y_k = q_pre.copy(), k_pre.copy()
    if int(layer.qk_mean) == QK_SELF:
        y_q, y_k = qk_mean_self(q_pre, y_q, k_pre, y_k)
    elif layer.qk_mean:
        m_q, m_k = qk_mean(q_pre, k_pre, sh.G)
        y_q = y_q + m_q
        y_k = y_k + m_k
    return y_q, y_k


def _shift_values(layer: Layer, v_lat, v_prev=None):
    """Step a6 under the layer's value-shift reading."""
    mode = int(layer.value_shift)
    if mode == VS_WHOLE_HEADS:
        return value_shift_heads(v_lat, v_prev)
    if mode:
        return value_shift(v_lat, v_prev)
    return v_lat.copy()


def prefill(layer: Layer, x: np.ndarray, rows: np.ndarray | None = None):
    """CCGQA forward of one sequence from an empty state.

    x: [S, E] (or packed q~|k~|v~ rows when W_qkv is None).
    rows: optional query positions to evaluate (all by default); keys and
    values are always built for every position.
    Returns (out [len(rows), Hq d], state) where ``state`` holds the cache
    (post-RoPE k, shifted v), the conv histories and the last v~ row, and
    ``state.extra`` holds q (post-RoPE, all rows) and the pre-conv tensors.
    """
    sh = layer.sh
    S = x.shape[0]
    q_pre, k_pre, v_lat = down_project(x, layer.W_qkv, sh)
    y_q, y_k = _mix_qk(layer, q_pre, k_pre)
    pos = np.arange(S)
    q = rope(y_q, pos, layer.rope_base)
    k = rope(y_k, pos, layer.rope_base)
    v = _shift_values(layer, v_lat)
    if rows is None:
        rows = pos
    rows = np.asarray(rows)
    o = attention(q[rows], k, v, sh.G, layer.causal, q_pos=rows)
    K = max(layer.conv_width, 1)
    hq = np.zeros((K - 1, sh.Hq * sh.d))
    hk = np.zeros((K - 1, sh.Hkv * sh.d))
    for j in range(1, K):            # history row K-1-j holds row S-j
        if S - j >= 0:
            hq[K - 1 - j] = q_pre[S - j].reshape(-1)
            hk[K - 1 - j] = k_pre[S - j].reshape(-1)
    st = State(k=k, v=v, hist_q=hq, hist_k=hk,
               v_prev=v_lat[S - 1].reshape(-1) if S > 0 else np.zeros(sh.Hkv * sh.d))
    st.extra.update(q=q, q_pre=q_pre, k_pre=k_pre, v_lat=v_lat)
    return o.reshape(len(rows), -1), st


def decode_step(layer: Layer, state: State, x_t: np.ndarray):
    """One new token per sequence against the latent KV cache.

    Equals row t = state.length of a prefill over all tokens so far: the
    conv reads its K-1 previous pre-conv rows from the state, RoPE uses
    position t, value-shift takes its upper half-channels from the stored
    previous v~ row, the new k/v row is appended, and the query attends over
    t + 1 keys.  Returns (out [Hq d], new state).
    """
    sh = layer.sh
    t = state.length
    q_pre, k_pre, v_lat = down_project(x_t[None, :], layer.W_qkv, sh)
    K = max(layer.conv_width, 1)
    hq = state.hist_q if K > 1 else None
    hk = state.hist_k if K > 1 else None
    y_q, y_k = _mix_qk(layer, q_pre, k_pre, hq, hk)
    pos = np.array([t])
    q = rope(y_q, pos, layer.rope_base)
    k = rope(y_k, pos, layer.rope_base)
    v = _shift_values(layer, v_lat, state.v_prev.reshape(sh.Hkv, sh.d))
    k_all = np.concatenate([state.k, k], axis=0)
    v_all = np.concatenate([state.v, v], axis=0)
    o = attention(q, k_all, v_all, sh.G, layer.causal, q_pos=pos)
    if K > 1:
        new_hq = np.concatenate([state.hist_q[1:], q_pre.reshape(1, -1)], axis=0)
        new_hk = np.concatenate([state.hist_k[1:], k_pre.reshape(1, -1)], axis=0)
    else:
        new_hq, new_hk = state.hist_q, state.hist_k
    ns = State(k=k_all, v=v_all, hist_q=new_hq, hist_k=new_hk,
               v_prev=v_lat.reshape(-1))
    ns.extra.update(q=q, k_new=k, v_new=v)
    return o.reshape(-1), ns


def kvcache_append(cache_k: np.ndarray, cache_v: np.ndarray, length: int,
                   k_new: np.ndarray, v_new: np.ndarray):
    """Write n new rows at positions [length, length + n) of a fixed-capacity
    cache [cap, Hkv, d]; returns the new length.  Raises when the rows do not
    fit (the cache keeps every token it has seen [CCA Probleemstelling 2])."""
    n = k_new.shape[0]
    if length + n > cache_k.shape[0]:
        raise ValueError("capacity")
    cache_k[length:length + n] = k_new
    cache_v[length:length + n] = v_new
    return length + n


# --------------------------------------------------------------------------
# Output up-projection  [CCA Methodologie 1 "Compressie in Latente Ruimte"]
# --------------------------------------------------------------------------
def output_projection(o: np.ndarray, W_o: np.ndarray):
    """Map the latent attention output back to the model width.

    The page runs the whole attention inside the latent space of width E/C and
    says nothing of how its result returns to width E.  Reading: one bias-free
    linear map W_o [E, Hq d] (output-feature major, like W_qkv) applied to the
    concatenated head outputs, y[m, e] = sum_j o[m, j] W_o[e, j].

    o: [M, Hq d] (rows of one or more prefill outputs, or decode outputs).
    Returns y: [M, E].
    """
    return o @ W_o.T


# --------------------------------------------------------------------------
# Closed-form bookkeeping  [GQA Por qué GQA reduce la caché KV; CCA Bijdragen]
# --------------------------------------------------------------------------
def cache_values_per_token(n_kv_heads: int, head_dim: int) -> int:
    """Values one layer keeps per token: a key and a value per kv head."""
    return 2 * n_kv_heads * head_dim


def attention_flops(S: int, Hq: int, d: int, causal: bool = True) -> float:
    """Multiply-add flops of QK^T plus PV for one sequence (2 flops per MAC);
    causal counts the S^2/2 visible scores."""
    pairs = S * S / 2 if causal else S * S
    return 2.0 * 2.0 * Hq * d * pairs


# --------------------------------------------------------------------------
# Backward pass  [CCA Resultaten 2: the layer is trained; its backward pass is
# the chain rule through the forward steps above, in reverse order]
# --------------------------------------------------------------------------
def attention_backward(q, k, v, G, causal, dout, q_pos=None):
    """Gradients of o = attention(q, k, v) for an upstream gradient dout
    [T, Hq, d]: returns (dq [T, Hq, d], dk [L, Hkv, d], dv [L, Hkv, d]).

    Per query head h with kv head g = h // G and scale 1/sqrt(d):
        p = softmax(q k^T / sqrt(d) + mask),   o = p v
        dv_g += p^T dout_h,   dp = dout_h v_g^T,
        ds = p * (dp - rowsum(dp * p)),
        dq_h = ds k_g / sqrt(d),   dk_g += ds^T q_h / sqrt(d).
    A kv head's gradients sum over the G query heads that read it.
    """
    T, Hq, d = q.shape
    L, Hkv, _ = k.shape
    if q_pos is None:
        q_pos = np.arange(T)
    q_pos = np.asarray(q_pos)
    scale = 1.0 / math.sqrt(d)
    keys = np.arange(L)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for h in range(Hq):
        g = h // G
        sc = (q[:, h, :] @ k[:, g, :].T) * scale
        if causal:
            sc = np.where(keys[None, :] <= q_pos[:, None], sc, -np.inf)
        sc = sc - sc.max(axis=1, keepdims=True)
        p = np.exp(sc)
        p = p / p.sum(axis=1, keepdims=True)
        do = dout[:, h, :]
        dv[:, g, :] += p.T @ do
        dp = do @ v[:, g, :].T
        ds = p * (dp - (dp * p).sum(axis=1, keepdims=True))
        dq[:, h, :] = (ds @ k[:, g, :]) * scale
        dk[:, g, :] += (ds.T @ q[:, h, :]) * scale
    return dq, dk, dv


def _rope_backward(dz, positions, base):
    """RoPE is a rotation per pair: its transpose turns by the opposite angle."""
    if base == 0:
        return dz.copy()
    return rope(dz, -np.asarray(positions, dtype=np.float64), base)


def _value_shift_backward(layer, dv):
    """Transpose of the value-shift gather: a shifted channel of row t came
    from row t - 1, so its gradient flows back one row (nothing flows to
    the row before the start)."""
    mode = int(layer.value_shift)
    dvt = dv.copy()
    if mode == VS_OFF:
        return dvt
    S, Hkv, d = dv.shape
    shifted = np.zeros_like(dv)
    shifted[:-1] = dv[1:]              # row t receives row t+1's gradient
    if mode == VS_WHOLE_HEADS:
        g0 = Hkv - Hkv // 2
        dvt[:, g0:] = shifted[:, g0:]
    else:
        dvt[..., d // 2:] = shifted[..., d // 2:]
    return dvt


def _seq_conv_backward(z, w_seq, du):
    """u[t, c] = sum_j w[c, j] z[t - j, c]  (zero before the start):
    dz[t, c] = sum_j w[c, j] du[t + j, c],  dw[c, j] = sum_t du[t, c] z[t - j, c]."""
    S, Ch = z.shape
    K = w_seq.shape[1]
    dz = np.zeros_like(z)
    dw = np.zeros_like(w_seq)
    for j in range(K):
        if j >= S:
            break
        dz[: S - j] += w_seq[:, j] * du[j:]
        dw[:, j] = (du[j:] * z[: S - j]).sum(axis=0)
    return dz, dw


def _channel_conv_backward(z, W, dy):
    """y[t, h] = sum_j W[h, j] z[t - j, h]:  dz[t, h] = sum_j W[h, j]^T dy[t + j, h],
    dW[h, j] = sum_t dy[t, h] (outer) z[t - j, h]."""
    S, H, d = z.shape
    K = W.shape[1]
    dz = np.zeros_like(z)
    dW = np.zeros_like(W)
    for j in range(K):
        if j >= S:
            break
        dz[: S - j] += np.einsum("hij,thi->thj", W[:, j], dy[j:])
        dW[:, j] = np.einsum("thi,thj->hij", dy[j:], z[: S - j])
    return dz, dW


def prefill_backward(layer: Layer, x: np.ndarray, dout: np.ndarray):
    """Gradients of the prefill of one sequence (from an empty state) for an
    upstream gradient dout [S, Hq d] of its output.

    Returns a dict: dx [S, E] (or [S, N_qkv] for packed input), dW_qkv
    [N_qkv, E] (None for packed input), and the conv weights' gradients under
    the names of the weights (None where the weight is unused).  The forward
    steps run in the pages' order; their transposes run in reverse.
    """
    sh = layer.sh
    S = x.shape[0]
    d, Hq, Hkv, G = sh.d, sh.Hq, sh.Hkv, sh.G
    # ---- forward, keeping what the backward needs
    q_pre, k_pre, v_lat = down_project(x, layer.W_qkv, sh)
    conv = layer.conv_width > 0
    if conv and layer.channel_conv:
        y_q = channel_conv(q_pre, layer.conv_q_chan)
        y_k = channel_conv(k_pre, layer.conv_k_chan)
        u_q = u_k = None
    elif conv:
        u_q = seq_conv(q_pre.reshape(S, -1), layer.conv_q_seq).reshape(S, Hq, d)
        u_k = seq_conv(k_pre.reshape(S, -1), layer.conv_k_seq).reshape(S, Hkv, d)
        y_q = u_q if layer.conv_q_chan is None else channel_mix(u_q, layer.conv_q_chan)
        y_k = u_k if layer.conv_k_chan is None else channel_mix(u_k, layer.conv_k_chan)
    else:
        y_q, y_k = q_pre.copy(), k_pre.copy()
    mode = int(layer.qk_mean)
    if mode == QK_SELF:
        qm, km = qk_mean_self(q_pre, y_q, k_pre, y_k)
    elif mode:
        m_q, m_k = qk_mean(q_pre, k_pre, G)
        qm, km = y_q + m_q, y_k + m_k
    else:
        qm, km = y_q, y_k
    pos = np.arange(S)
    q = rope(qm, pos, layer.rope_base)
    k = rope(km, pos, layer.rope_base)
    v = _shift_values(layer, v_lat)
    # ---- backward
    dq, dk, dv = attention_backward(q, k, v, G, layer.causal, dout.reshape(S, Hq, d))
    dv_lat = _value_shift_backward(layer, dv)
    dqm = _rope_backward(dq, pos, layer.rope_base)
    dkm = _rope_backward(dk, pos, layer.rope_base)
    if mode == QK_SELF:
        dy_q, dy_k = 0.5 * dqm, 0.5 * dkm
        dq_pre, dk_pre = 0.5 * dqm, 0.5 * dkm
    elif mode:
        dy_q, dy_k = dqm, dkm
        # m_q[h] = (q~[h] + k~[g]) / 2,  m_k[g] = (mean_h q~[h] + k~[g]) / 2
        dq_pre = 0.5 * dqm + (0.5 / G) * np.repeat(dkm, G, axis=1)
        dk_pre = 0.5 * dqm.reshape(S, Hkv, G, d).sum(axis=2) + 0.5 * dkm
    else:
        dy_q, dy_k = dqm, dkm
        dq_pre, dk_pre = np.zeros_like(q_pre), np.zeros_like(k_pre)
    grads = {"conv_q_seq": None, "conv_q_chan": None, "conv_k_seq": None, "conv_k_chan": None}
    if conv and layer.channel_conv:
        dz, grads["conv_q_chan"] = _channel_conv_backward(q_pre, layer.conv_q_chan, dy_q)
        dq_pre = dq_pre + dz
        dz, grads["conv_k_chan"] = _channel_conv_backward(k_pre, layer.conv_k_chan, dy_k)
        dk_pre = dk_pre + dz
    elif conv:
        for side, z, u, dy, Wc, ws, Hs in (("q", q_pre, u_q, dy_q, layer.conv_q_chan, layer.conv_q_seq, Hq),
                                           ("k", k_pre, u_k, dy_k, layer.conv_k_chan, layer.conv_k_seq, Hkv)):
            if Wc is None:
                du = dy
            else:
                du = np.einsum("hij,thi->thj", Wc, dy)          # W^T dy
                grads[f"conv_{side}_chan"] = np.einsum("thi,thj->hij", dy, u)
            dz, grads[f"conv_{side}_seq"] = _seq_conv_backward(z.reshape(S, -1), ws, du.reshape(S, -1))
            if side == "q":
                dq_pre = dq_pre + dz.reshape(S, Hs, d)
            else:
                dk_pre = dk_pre + dz.reshape(S, Hs, d)
    else:
        dq_pre = dq_pre + dy_q
        dk_pre = dk_pre + dy_k
    dzq = np.concatenate([dq_pre.reshape(S, -1), dk_pre.reshape(S, -1), dv_lat.reshape(S, -1)], axis=1)
    if layer.W_qkv is None:
        return {"dx": dzq, "W_qkv": None, **grads}
    return {"dx": dzq @ layer.W_qkv, "W_qkv": dzq.T @ x, **grads}
