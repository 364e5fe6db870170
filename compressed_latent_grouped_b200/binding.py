"""ctypes binding of ``include/ccgqa.h`` (argument marshalling only).

Every function here keeps the C name, turns torch tensors into device pointers
and the current torch stream into a ``cudaStream_t``, calls the library, and
raises :class:`CCGQAError` on a non-OK status.  All arithmetic happens in the
library's CUDA kernels; there is no other code path.  When the compiled
library is missing the first call fails loudly.
"""
from __future__ import annotations

import ctypes
import os
import re
from ctypes import POINTER, c_char_p, c_double, c_int, c_int32, c_size_t, c_uint64, c_void_p

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libccgqa.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "ccgqa.h")

F32, BF16 = 0, 1
DEVERR_INDEX, DEVERR_TIMEOUT, DEVERR_CAPACITY = 1, 2, 4
STATUS = {0: "OK", 1: "ERR_INVALID_ARG", 2: "ERR_UNSUPPORTED", 3: "ERR_CAPACITY",
          4: "ERR_WORKSPACE", 5: "ERR_CUDA"}


class ccgqa_config(ctypes.Structure):
    _fields_ = [("E", c_int32), ("C", c_int32), ("n_q_heads", c_int32), ("n_kv_heads", c_int32),
                ("conv_width", c_int32), ("qk_mean", c_int32), ("value_shift", c_int32),
                ("causal", c_int32), ("rope_base", c_double), ("dtype", c_int32),
                ("channel_conv", c_int32)]


class ccgqa_weights(ctypes.Structure):
    _fields_ = [("W_qkv", c_void_p), ("conv_q_seq", c_void_p), ("conv_q_chan", c_void_p),
                ("conv_k_seq", c_void_p), ("conv_k_chan", c_void_p)]


class ccgqa_weight_grads(ctypes.Structure):
    _fields_ = [("W_qkv", c_void_p), ("conv_q_seq", c_void_p), ("conv_q_chan", c_void_p),
                ("conv_k_seq", c_void_p), ("conv_k_chan", c_void_p)]


class ccgqa_kvcache(ctypes.Structure):
    _fields_ = [("k", c_void_p), ("v", c_void_p), ("len", c_void_p), ("conv_hist_q", c_void_p),
                ("conv_hist_k", c_void_p), ("v_prev", c_void_p), ("batch", c_int32),
                ("cap", c_int32), ("block_table", c_void_p), ("page_size", c_int32),
                ("n_pages", c_int32)]


class CCGQAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {STATUS.get(status, status)} ({_status_string(status)})"
        if status == 5:
            msg += f" [{ccgqa_last_error_string()}]"
        super().__init__(msg)


_lib = None


def load() -> ctypes.CDLL:
    """Load ``libccgqa.so`` (built in-tree by ``build.py``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"CCGQA CUDA library not built: {LIB_PATH} is missing "
                           "(run `python -m compressed_latent_grouped_b200.build`)")
    lib = ctypes.CDLL(LIB_PATH)
    P = POINTER
    lib.ccgqa_prefill_workspace_size.argtypes = [P(ccgqa_config), c_int32, c_int32]
    lib.ccgqa_prefill_workspace_size.restype = c_size_t
    lib.ccgqa_decode_workspace_size.argtypes = [P(ccgqa_config), c_int32, c_int32]
    lib.ccgqa_decode_workspace_size.restype = c_size_t
    lib.ccgqa_prefill.argtypes = [P(ccgqa_config), P(ccgqa_weights), c_void_p, c_int32, c_int32,
                                  c_void_p, P(ccgqa_kvcache), c_void_p, c_size_t, c_void_p,
                                  c_void_p]
    lib.ccgqa_prefill.restype = c_int
    lib.ccgqa_decode_step.argtypes = [P(ccgqa_config), P(ccgqa_weights), c_void_p,
                                      P(ccgqa_kvcache), c_void_p, c_void_p, c_size_t, c_void_p,
                                      c_void_p]
    lib.ccgqa_decode_step.restype = c_int
    lib.ccgqa_decode_step_noalloc.argtypes = [P(ccgqa_config), P(ccgqa_weights), c_void_p,
                                              P(ccgqa_kvcache), c_void_p, c_void_p, c_void_p]
    lib.ccgqa_decode_step_noalloc.restype = c_int
    lib.ccgqa_decode_noalloc_max_bytes.argtypes = []
    lib.ccgqa_decode_noalloc_max_bytes.restype = c_size_t
    lib.ccgqa_kvcache_append.argtypes = [P(ccgqa_config), P(ccgqa_kvcache), c_void_p, c_void_p,
                                         c_int32, c_void_p, c_void_p]
    lib.ccgqa_kvcache_append.restype = c_int
    lib.ccgqa_output_projection.argtypes = [P(ccgqa_config), c_void_p, c_void_p, ctypes.c_int64,
                                            c_void_p, c_void_p, c_void_p]
    lib.ccgqa_output_projection.restype = c_int
    lib.ccgqa_prefill_backward_workspace_size.argtypes = [P(ccgqa_config), c_int32, c_int32]
    lib.ccgqa_prefill_backward_workspace_size.restype = c_size_t
    lib.ccgqa_prefill_backward.argtypes = [P(ccgqa_config), P(ccgqa_weights), c_void_p, c_int32,
                                           c_int32, c_void_p, c_void_p, P(ccgqa_weight_grads),
                                           c_void_p, c_size_t, c_void_p, c_void_p]
    lib.ccgqa_prefill_backward.restype = c_int
    lib.ccgqa_status_string.argtypes = [c_int]
    lib.ccgqa_status_string.restype = c_char_p
    lib.ccgqa_launch_count.argtypes = []
    lib.ccgqa_launch_count.restype = c_uint64
    lib.ccgqa_last_error_string.argtypes = []
    lib.ccgqa_last_error_string.restype = c_char_p
    lib.ccgqa_set_phase_events.argtypes = [c_void_p, c_int32]
    lib.ccgqa_set_phase_events.restype = None
    lib.ccgqa_set_fused_projection.argtypes = [c_int32]
    lib.ccgqa_set_fused_projection.restype = None
    lib.ccgqa_selftest_wait_timeout.argtypes = [ctypes.c_int64, c_void_p, c_void_p]
    lib.ccgqa_selftest_wait_timeout.restype = c_int
    lib.ccgqa_graph_begin.argtypes = [c_void_p]
    lib.ccgqa_graph_begin.restype = c_int
    lib.ccgqa_graph_end.argtypes = [c_void_p, POINTER(c_void_p)]
    lib.ccgqa_graph_end.restype = c_int
    lib.ccgqa_graph_launch.argtypes = [c_void_p, c_void_p]
    lib.ccgqa_graph_launch.restype = c_int
    lib.ccgqa_graph_kernel_count.argtypes = [c_void_p]
    lib.ccgqa_graph_kernel_count.restype = ctypes.c_int64
    lib.ccgqa_graph_destroy.argtypes = [c_void_p]
    lib.ccgqa_graph_destroy.restype = c_int
    _lib = lib
    return lib


def header_symbols() -> list[str]:
    """Entry points declared in include/ccgqa.h."""
    with open(HEADER) as f:
        text = f.read()
    return re.findall(r"CCGQA_API\s+[\w\s\*]+?\b(ccgqa_\w+)\s*\(", text)


def _status_string(status: int) -> str:
    try:
        return load().ccgqa_status_string(status).decode()
    except Exception:  # noqa: BLE001 - message only
        return "?"


# ------------------------------------------------------------------ marshalling
def _ptr(t):
    return None if t is None else c_void_p(t.data_ptr())


def _stream(stream=None):
    """torch stream (default: the current one) or a raw cudaStream_t integer."""
    if isinstance(stream, int):
        return c_void_p(stream or None)
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return c_void_p(stream.cuda_stream)


def make_config(E, C, n_q_heads, n_kv_heads, conv_width=4, qk_mean=1, value_shift=1, causal=1,
                rope_base=10000.0, dtype=BF16, channel_conv=0) -> ccgqa_config:
    """qk_mean: 0 off, 1 cross, 2 self; value_shift: 0 off, 1 half channels,
    2 whole heads; channel_conv: 1 for per-tap d x d matrices."""
    return ccgqa_config(E, C, n_q_heads, n_kv_heads, conv_width, int(qk_mean), int(value_shift),
                        int(causal), float(rope_base), dtype, int(channel_conv))


def make_weights(W_qkv=None, conv_q_seq=None, conv_q_chan=None, conv_k_seq=None,
                 conv_k_chan=None) -> ccgqa_weights:
    return ccgqa_weights(*(None if t is None else t.data_ptr()
                           for t in (W_qkv, conv_q_seq, conv_q_chan, conv_k_seq, conv_k_chan)))


def make_kvcache(k, v, len_, conv_hist_q=None, conv_hist_k=None, v_prev=None,
                 block_table=None) -> ccgqa_kvcache:
    """Contiguous cache: k, v [batch, Hkv, cap, d].  Paged cache: k, v are the
    pool [n_pages, Hkv, page_size, d] and block_table [batch, cap / page_size]
    (int32) names each sequence's pages."""
    ptr = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    if block_table is None:
        batch, _, cap, _ = k.shape
        return ccgqa_kvcache(k.data_ptr(), v.data_ptr(), len_.data_ptr(), ptr(conv_hist_q),
                             ptr(conv_hist_k), ptr(v_prev), batch, cap, None, 0, 0)
    n_pages, _, page_size, _ = k.shape
    batch, per_seq = block_table.shape
    return ccgqa_kvcache(k.data_ptr(), v.data_ptr(), len_.data_ptr(), ptr(conv_hist_q),
                         ptr(conv_hist_k), ptr(v_prev), batch, per_seq * page_size,
                         block_table.data_ptr(), page_size, n_pages)


# ------------------------------------------------------------------ entry points
def ccgqa_prefill_workspace_size(cfg: ccgqa_config, batch: int, seq_len: int) -> int:
    return int(load().ccgqa_prefill_workspace_size(ctypes.byref(cfg), batch, seq_len))


def ccgqa_decode_workspace_size(cfg: ccgqa_config, batch: int, cap: int) -> int:
    return int(load().ccgqa_decode_workspace_size(ctypes.byref(cfg), batch, cap))


def ccgqa_prefill(cfg, weights, x, batch, seq_len, out, cache, workspace, dev_err=None,
                  stream=None, check=True) -> int:
    lib = load()
    st = lib.ccgqa_prefill(ctypes.byref(cfg), ctypes.byref(weights), _ptr(x), batch, seq_len,
                           _ptr(out), None if cache is None else ctypes.byref(cache),
                           _ptr(workspace), workspace.numel() * workspace.element_size(),
                           _ptr(dev_err), _stream(stream))
    if check and st != 0:
        raise CCGQAError(st, "ccgqa_prefill")
    return st


def ccgqa_decode_step(cfg, weights, x_t, cache, out, workspace, dev_err=None, stream=None,
                      check=True) -> int:
    lib = load()
    st = lib.ccgqa_decode_step(ctypes.byref(cfg), ctypes.byref(weights), _ptr(x_t),
                               ctypes.byref(cache), _ptr(out), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _ptr(dev_err),
                               _stream(stream))
    if check and st != 0:
        raise CCGQAError(st, "ccgqa_decode_step")
    return st


def ccgqa_decode_step_noalloc(cfg, weights, x_t, cache, out, dev_err=None, stream=None,
                              check=True) -> int:
    lib = load()
    st = lib.ccgqa_decode_step_noalloc(ctypes.byref(cfg), ctypes.byref(weights), _ptr(x_t),
                                       ctypes.byref(cache), _ptr(out), _ptr(dev_err),
                                       _stream(stream))
    if check and st != 0:
        raise CCGQAError(st, "ccgqa_decode_step_noalloc")
    return st


def ccgqa_decode_noalloc_max_bytes() -> int:
    return int(load().ccgqa_decode_noalloc_max_bytes())


def ccgqa_kvcache_append(cfg, cache, k_new, v_new, n_new, dev_err=None, stream=None,
                         check=True) -> int:
    lib = load()
    st = lib.ccgqa_kvcache_append(ctypes.byref(cfg), ctypes.byref(cache), _ptr(k_new),
                                  _ptr(v_new), n_new, _ptr(dev_err), _stream(stream))
    if check and st != 0:
        raise CCGQAError(st, "ccgqa_kvcache_append")
    return st


def ccgqa_output_projection(cfg, W_o, o, M, y, dev_err=None, stream=None, check=True) -> int:
    st = load().ccgqa_output_projection(ctypes.byref(cfg), _ptr(W_o), _ptr(o), int(M), _ptr(y),
                                        _ptr(dev_err), _stream(stream))
    if check and st != 0:
        raise CCGQAError(st, "ccgqa_output_projection")
    return st


def make_weight_grads(W_qkv=None, conv_q_seq=None, conv_q_chan=None, conv_k_seq=None,
                      conv_k_chan=None) -> ccgqa_weight_grads:
    return ccgqa_weight_grads(*(None if t is None else t.data_ptr()
                                for t in (W_qkv, conv_q_seq, conv_q_chan, conv_k_seq, conv_k_chan)))


def ccgqa_prefill_backward_workspace_size(cfg: ccgqa_config, batch: int, seq_len: int) -> int:
    return load().ccgqa_prefill_backward_workspace_size(ctypes.byref(cfg), batch, seq_len)


def ccgqa_prefill_backward(cfg, weights, x, batch, seq_len, dout, dx, grads, workspace,
                           dev_err=None, stream=None, check=True) -> int:
    lib = load()
    st = lib.ccgqa_prefill_backward(ctypes.byref(cfg), ctypes.byref(weights), _ptr(x), batch,
                                    seq_len, _ptr(dout), _ptr(dx),
                                    None if grads is None else ctypes.byref(grads),
                                    _ptr(workspace),
                                    0 if workspace is None else workspace.numel(),
                                    _ptr(dev_err), _stream(stream))
    if check and st != 0:
        raise CCGQAError(st, "ccgqa_prefill_backward")
    return st


def ccgqa_status_string(status: int) -> str:
    return load().ccgqa_status_string(status).decode()


def ccgqa_last_error_string() -> str:
    return load().ccgqa_last_error_string().decode()


def ccgqa_launch_count() -> int:
    return int(load().ccgqa_launch_count())


def ccgqa_selftest_wait_timeout(limit_cycles: int, dev_err=None, stream=None, check=True) -> int:
    st = load().ccgqa_selftest_wait_timeout(int(limit_cycles), _ptr(dev_err), _stream(stream))
    if check and st != 0:
        raise CCGQAError(st, "ccgqa_selftest_wait_timeout")
    return st


def ccgqa_graph_begin(stream=None, check=True) -> int:
    st = load().ccgqa_graph_begin(_stream(stream))
    if check and st != 0:
        raise CCGQAError(st, "ccgqa_graph_begin")
    return st


def ccgqa_graph_end(stream=None) -> int:
    """Stop recording on `stream`; returns the graph handle (an integer)."""
    h = c_void_p()
    st = load().ccgqa_graph_end(_stream(stream), ctypes.byref(h))
    if st != 0:
        raise CCGQAError(st, "ccgqa_graph_end")
    return h.value


def ccgqa_graph_launch(graph: int, stream=None, check=True) -> int:
    st = load().ccgqa_graph_launch(c_void_p(graph), _stream(stream))
    if check and st != 0:
        raise CCGQAError(st, "ccgqa_graph_launch")
    return st


def ccgqa_graph_kernel_count(graph) -> int:
    return int(load().ccgqa_graph_kernel_count(c_void_p(graph)))


def ccgqa_graph_destroy(graph) -> None:
    st = load().ccgqa_graph_destroy(c_void_p(graph))
    if st != 0:
        raise CCGQAError(st, "ccgqa_graph_destroy")


_phase_keep = None


def ccgqa_set_fused_projection(enable: bool) -> None:
    """Process-wide: let ccgqa_prefill fuse the projection with the
    pre-attention where that kernel applies (default on)."""
    load().ccgqa_set_fused_projection(1 if enable else 0)


def ccgqa_set_phase_events(events) -> None:
    """Record four torch.cuda.Event (enable_timing=True) between the kernels of
    each following prefill / decode call on this thread; None turns it off."""
    global _phase_keep
    if events is None:
        _phase_keep = None
        load().ccgqa_set_phase_events(None, 0)
        return
    for e in events:
        if not e.cuda_event:      # torch creates the CUDA event on first record
            e.record()
    arr = (c_void_p * len(events))(*[e.cuda_event for e in events])
    _phase_keep = (arr, events)
    load().ccgqa_set_phase_events(ctypes.cast(arr, c_void_p), len(events))
