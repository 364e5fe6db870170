"""Device-side plumbing around the C ABI: torch owns the memory (weights, KV
cache, decode state, workspaces, the device error word) and this module hands
pointers to the library.  No arithmetic of the method happens here."""
from __future__ import annotations

import torch

from . import binding as B
from .workloads import Workload


def config_of(w: Workload) -> B.ccgqa_config:
    return B.make_config(w.E, w.C, w.Hq, w.Hkv, conv_width=w.conv_width, qk_mean=w.qk_mean,
                         value_shift=w.value_shift, causal=w.causal, rope_base=w.rope_base,
                         dtype=B.F32 if w.dtype == "f32" else B.BF16,
                         channel_conv=w.channel_conv)


class DeviceLayer:
    """Weights of one CCGQA layer resident on the GPU plus the buffers the
    entry points need.  ``inputs`` is the dict produced by
    ``workloads.make_inputs`` (CPU tensors in the working dtype)."""

    def __init__(self, w: Workload, inputs: dict, device="cuda", batch: int | None = None,
                 cap: int | None = None):
        if not torch.cuda.is_available():
            raise RuntimeError("CCGQA needs a CUDA device")
        self.w = w
        self.device = torch.device(device)
        self.cfg = config_of(w)
        dev = lambda t: None if t is None else t.to(self.device).contiguous()  # noqa: E731
        self.W_qkv = dev(inputs.get("W_qkv"))
        self.conv = {k: dev(inputs.get(k)) for k in ("conv_q_seq", "conv_q_chan", "conv_k_seq",
                                                    "conv_k_chan")}
        self.weights = B.make_weights(self.W_qkv, self.conv["conv_q_seq"], self.conv["conv_q_chan"],
                                      self.conv["conv_k_seq"], self.conv["conv_k_chan"])
        self.batch = batch if batch is not None else w.B
        self.cap = cap if cap is not None else w.S
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.cache_tensors = None
        self.cache = None
        self._pf_ws = None
        self._dec_ws = None

    # -------------------------------------------------------------- buffers
    def alloc_cache(self, batch: int | None = None, cap: int | None = None,
                    block_table: torch.Tensor | None = None, page_size: int = 0,
                    n_pages: int = 0):
        """Contiguous cache [batch, Hkv, cap, d], or with ``block_table``
        ([batch, cap / page_size] int32) a pool of ``n_pages`` pages
        [n_pages, Hkv, page_size, d]."""
        w = self.w
        batch = self.batch if batch is None else batch
        cap = self.cap if cap is None else cap
        dt = w.torch_dtype
        km1 = max(w.conv_width - 1, 0)
        if block_table is not None:
            assert block_table.shape == (batch, cap // page_size) and cap % page_size == 0
            kv_shape = (n_pages, w.Hkv, page_size, w.d)
        else:
            kv_shape = (batch, w.Hkv, cap, w.d)
        t = dict(
            k=torch.zeros(kv_shape, dtype=dt, device=self.device),
            v=torch.zeros(kv_shape, dtype=dt, device=self.device),
            len=torch.zeros(batch, dtype=torch.int32, device=self.device),
            hist_q=torch.zeros(batch, max(km1, 1), w.Hq * w.d, dtype=dt, device=self.device),
            hist_k=torch.zeros(batch, max(km1, 1), w.Hkv * w.d, dtype=dt, device=self.device),
            v_prev=torch.zeros(batch, w.Hkv * w.d, dtype=dt, device=self.device),
        )
        if block_table is not None:
            t["block_table"] = block_table.to(self.device, torch.int32).contiguous()
        self.cache_tensors = t
        self.cache = B.make_kvcache(t["k"], t["v"], t["len"], t["hist_q"], t["hist_k"], t["v_prev"],
                                    t.get("block_table"))
        self.cache_batch, self.cache_cap = batch, cap
        return t

    def prefill_workspace(self, batch: int, seq_len: int):
        n = B.ccgqa_prefill_workspace_size(self.cfg, batch, seq_len)
        if n == 0:
            raise B.CCGQAError(1, "ccgqa_prefill_workspace_size")
        if self._pf_ws is None or self._pf_ws.numel() < n:
            self._pf_ws = torch.zeros(n, dtype=torch.uint8, device=self.device)
        return self._pf_ws

    def decode_workspace(self):
        n = B.ccgqa_decode_workspace_size(self.cfg, self.cache_batch, self.cache_cap)
        if self._dec_ws is None or self._dec_ws.numel() < n:
            self._dec_ws = torch.zeros(n, dtype=torch.uint8, device=self.device)
        return self._dec_ws

    # -------------------------------------------------------------- calls
    def prefill(self, x: torch.Tensor, out: torch.Tensor | None = None, use_cache: bool = True,
                stream=None):
        batch, seq_len = x.shape[0], x.shape[1]
        w = self.w
        if out is None:
            out = torch.empty(batch, seq_len, w.Hq * w.d, dtype=w.torch_dtype, device=self.device)
        ws = self.prefill_workspace(batch, seq_len)
        B.ccgqa_prefill(self.cfg, self.weights, x, batch, seq_len, out,
                        self.cache if use_cache else None, ws, self.dev_err, stream)
        return out

    def decode_step(self, x_t: torch.Tensor, out: torch.Tensor | None = None, stream=None):
        w = self.w
        batch = x_t.shape[0]
        if out is None:
            out = torch.empty(batch, w.Hq * w.d, dtype=w.torch_dtype, device=self.device)
        B.ccgqa_decode_step(self.cfg, self.weights, x_t, self.cache, out, self.decode_workspace(),
                            self.dev_err, stream)
        return out

    def append(self, k_new: torch.Tensor, v_new: torch.Tensor, stream=None):
        B.ccgqa_kvcache_append(self.cfg, self.cache, k_new, v_new, k_new.shape[1], self.dev_err,
                               stream)

    def output_projection(self, o: torch.Tensor, W_o: torch.Tensor,
                          y: torch.Tensor | None = None, stream=None):
        """y [M, E] = o [M, Hq d] W_o^T (W_o [E, Hq d] on this device)."""
        w = self.w
        M = o.numel() // (w.Hq * w.d)
        if y is None:
            y = torch.empty(M, w.E, dtype=w.torch_dtype, device=self.device)
        B.ccgqa_output_projection(self.cfg, W_o, o, M, y, self.dev_err, stream)
        return y

    def prefill_backward(self, x: torch.Tensor, dout: torch.Tensor, with_weights: bool = True,
                         stream=None):
        """Gradients of a prefill (from an empty state) for the output gradient
        dout [B, S, Hq d]: returns (dx, {weight name: fp32 gradient or None})."""
        batch, seq_len = x.shape[0], x.shape[1]
        n = B.ccgqa_prefill_backward_workspace_size(self.cfg, batch, seq_len)
        if n == 0:
            raise B.CCGQAError(1, "ccgqa_prefill_backward_workspace_size")
        ws = torch.empty(n, dtype=torch.uint8, device=self.device)
        dx = torch.empty_like(x)
        grads = {"W_qkv": self.W_qkv, **self.conv}
        g = {k: (torch.empty(v.shape, dtype=torch.float32, device=self.device)
                 if (with_weights and v is not None) else None) for k, v in grads.items()}
        if self.w.channel_conv:
            g["conv_q_seq"] = g["conv_k_seq"] = None
        wg = B.make_weight_grads(g["W_qkv"], g["conv_q_seq"], g["conv_q_chan"], g["conv_k_seq"],
                                 g["conv_k_chan"])
        B.ccgqa_prefill_backward(self.cfg, self.weights, x, batch, seq_len, dout, dx, wg, ws,
                                 self.dev_err, stream)
        return dx, g

    def error_bits(self) -> int:
        return int(self.dev_err.item())


class Graph:
    """Library calls recorded once into a CUDA graph (ccgqa_graph_*) and
    launched again with the same arguments: ``Graph(fn, stream)`` records what
    ``fn()`` enqueues on ``stream`` (a created torch stream, not the default
    stream); ``launch()`` replays it on that stream; ``close()`` frees it."""

    def __init__(self, fn, stream):
        self.stream = stream
        self.handle = None
        B.ccgqa_graph_begin(stream)
        try:
            with torch.cuda.stream(stream):
                fn()
        except BaseException:
            try:
                B.ccgqa_graph_destroy(B.ccgqa_graph_end(stream))
            except B.CCGQAError:
                pass
            raise
        self.handle = B.ccgqa_graph_end(stream)
        self.kernels = B.ccgqa_graph_kernel_count(self.handle)

    def launch(self):
        B.ccgqa_graph_launch(self.handle, self.stream)

    def close(self):
        if self.handle is not None:
            B.ccgqa_graph_destroy(self.handle)
            self.handle = None
