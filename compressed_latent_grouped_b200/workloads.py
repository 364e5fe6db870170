"""Seeded synthetic workloads for CCGQA.

This module only draws random numbers and names shapes: it holds none of the
method's arithmetic.  The oracle (tests) and the CUDA path (tests, bench) both
consume the tensors it returns, already rounded to the working dtype.

Recipe (same for every workload): ``numpy.random.default_rng(seed)`` (PCG64),
standard normals drawn in float32, multiplied by the stated standard deviation,
then rounded to the workload's dtype with round-to-nearest-even.  Draw order is
fixed: x, W_qkv, conv_q_seq, conv_q_chan, conv_k_seq, conv_k_chan, then the
decode extras (cache k, cache v, hist_q, hist_k, v_prev, x_t).
Weights follow N(0, 1/fan_in): W_qkv fan_in = E, sequence-conv taps fan_in = K,
channel mix fan_in = d.  With the temporal channel conv (``channel_conv``) the
channel weights are per-tap matrices [H, K, d, d] with fan_in = K d, drawn in
the slots of the channel mix, and no sequence-conv taps are drawn.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str            # "f32" or "bf16"
    B: int
    S: int                # prefill length, or cache length L for decode workloads
    E: int
    C: int
    Hq: int
    Hkv: int
    conv_width: int = 4
    qk_mean: int = 1             # 0 off, 1 cross, 2 self
    value_shift: int = 1         # 0 off, 1 half channels, 2 whole kv heads
    rope_base: float = 10000.0
    causal: bool = True
    packed_input: bool = False   # x already holds q~|k~|v~ (no projection)
    decode: bool = False
    channel_conv: bool = False   # per-tap d x d channel matrices instead of taps + mix

    @property
    def d(self) -> int:
        return self.E // (self.C * self.Hq)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def n_qkv(self) -> int:
        return (self.Hq + 2 * self.Hkv) * self.d

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads the hot path is measured and checked on.
WORKLOADS = {
    # fp32 forward, S=128, E=256, C=4, 4 q heads / 2 kv heads of dim 16
    "f32_s128": Workload("f32_s128", "f32", B=1, S=128, E=256, C=4, Hq=4, Hkv=2),
    # bf16 prefill, B=4, S=4096, E=2048, C=4, 16/4 heads of dim 32
    "bf16_prefill_b4_s4096": Workload("bf16_prefill_b4_s4096", "bf16", B=4, S=4096,
                                      E=2048, C=4, Hq=16, Hkv=4),
    # bf16 long-context prefill, S=32768, E=4096, C=8, 8/2 heads of dim 64, RoPE 5e5
    "bf16_prefill_b1_s32768": Workload("bf16_prefill_b1_s32768", "bf16", B=1, S=32768,
                                       E=4096, C=8, Hq=8, Hkv=2, rope_base=500000.0),
    # bf16 decode: B=64, one token each, cache of 16384 tokens, E=4096, C=8, 8/2 heads
    "bf16_decode_b64_l16384": Workload("bf16_decode_b64_l16384", "bf16", B=64, S=16384,
                                       E=4096, C=8, Hq=8, Hkv=2, rope_base=500000.0,
                                       decode=True),
    # bf16 uncompressed GQA (C=1), no conv / QK-mean / shift, 32/8 heads of dim 128
    "bf16_gqa_b2_s8192": Workload("bf16_gqa_b2_s8192", "bf16", B=2, S=8192, E=4096, C=1,
                                  Hq=32, Hkv=8, conv_width=0, qk_mean=False,
                                  value_shift=False, rope_base=500000.0,
                                  packed_input=True),
}
WORKLOAD_ORDER = list(WORKLOADS)


def _round(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.to(torch.float32 if dtype == "f32" else torch.bfloat16)


def _normal(rng, shape, std, dtype):
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return _round(a, dtype)


def make_inputs(w: Workload, seed: int = 0, batch: int | None = None) -> dict:
    """Draw every input of workload ``w`` (CPU tensors in the working dtype).

    ``batch`` overrides w.B (used to draw a shard or a smaller sample with the
    same recipe).
    """
    B = w.B if batch is None else batch
    rng = np.random.default_rng(seed)
    dt = w.dtype
    d, K = w.d, w.conv_width
    out: dict = {}
    if w.decode:
        out["x"] = None
    elif w.packed_input:
        out["x"] = _normal(rng, (B, w.S, w.n_qkv), 1.0, dt)
    else:
        out["x"] = _normal(rng, (B, w.S, w.E), 1.0, dt)
    out["W_qkv"] = None if w.packed_input else _normal(rng, (w.n_qkv, w.E), (1.0 / w.E) ** 0.5, dt)
    if K > 0 and w.channel_conv:
        out["conv_q_seq"] = out["conv_k_seq"] = None
        out["conv_q_chan"] = _normal(rng, (w.Hq, K, d, d), (1.0 / (K * d)) ** 0.5, dt)
        out["conv_k_chan"] = _normal(rng, (w.Hkv, K, d, d), (1.0 / (K * d)) ** 0.5, dt)
    elif K > 0:
        out["conv_q_seq"] = _normal(rng, (w.Hq * d, K), (1.0 / K) ** 0.5, dt)
        out["conv_q_chan"] = _normal(rng, (w.Hq, d, d), (1.0 / d) ** 0.5, dt)
        out["conv_k_seq"] = _normal(rng, (w.Hkv * d, K), (1.0 / K) ** 0.5, dt)
        out["conv_k_chan"] = _normal(rng, (w.Hkv, d, d), (1.0 / d) ** 0.5, dt)
    else:
        out["conv_q_seq"] = out["conv_q_chan"] = out["conv_k_seq"] = out["conv_k_chan"] = None
    if w.decode:
        L = w.S
        out["cache_k"] = _normal(rng, (B, L, w.Hkv, d), 1.0, dt)
        out["cache_v"] = _normal(rng, (B, L, w.Hkv, d), 1.0, dt)
        km1 = max(K - 1, 0)
        out["hist_q"] = _normal(rng, (B, km1, w.Hq * d), 1.0, dt)
        out["hist_k"] = _normal(rng, (B, km1, w.Hkv * d), 1.0, dt)
        out["v_prev"] = _normal(rng, (B, w.Hkv * d), 1.0, dt)
        out["x_t"] = _normal(rng, (B, w.n_qkv if w.packed_input else w.E), 1.0, dt)
    return out


def make_output_weights(w: Workload, seed: int = 0) -> torch.Tensor:
    """W_o [E, Hq d] of the output up-projection, N(0, 1 / (Hq d)) in the working
    dtype, from a generator of its own (the draws of make_inputs are unchanged)."""
    rng = np.random.default_rng(seed + 7919)
    return _normal(rng, (w.E, w.Hq * w.d), (1.0 / (w.Hq * w.d)) ** 0.5, w.dtype)


def make_block_table(batch: int, pages_per_seq: int, n_pages: int, seed: int = 0) -> torch.Tensor:
    """Block table of a paged cache: [batch, pages_per_seq] int32 page ids,
    all distinct, drawn as the first batch * pages_per_seq entries of a seeded
    permutation of the pool's n_pages pages (so a sequence's pages are
    scattered over the pool in no order)."""
    assert n_pages >= batch * pages_per_seq
    rng = np.random.default_rng(seed + 104729)
    ids = rng.permutation(n_pages)[: batch * pages_per_seq].astype(np.int32)
    return torch.from_numpy(ids.reshape(batch, pages_per_seq))


def sample_rows(S: int, n: int = 1024, tile: int = 128, seed: int = 1) -> np.ndarray:
    """Query positions checked one by one on full-size workloads: the first and
    last ``tile`` positions, positions on both sides of every ``tile`` boundary
    (up to the budget), and seeded random positions, sorted and unique."""
    if S <= n:
        return np.arange(S)
    rng = np.random.default_rng(seed)
    base = set(range(min(tile, S))) | set(range(max(S - tile, 0), S))
    step = max(tile, (S // (n // 4)) // tile * tile)
    for b in range(tile, S, step):
        base.update((b - 1, b))
    rest = n - len(base)
    if rest > 0:
        base.update(rng.choice(S, size=rest, replace=False).tolist())
    return np.array(sorted(base), dtype=np.int64)
