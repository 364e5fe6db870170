"""The C ABI on the host (no GPU needed): the library loads, exports every
entry point the header declares, its struct layouts match the C compiler's,
and argument validation rejects bad calls before any launch."""
import ctypes
import os
import subprocess
import tempfile

import pytest

from compressed_latent_grouped_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(B.LIB_PATH):
        from compressed_latent_grouped_b200 import build
        build.build()
    return B.load()


def test_exports_every_header_symbol(lib):
    names = B.header_symbols()
    assert set(names) >= {"ccgqa_prefill", "ccgqa_decode_step", "ccgqa_kvcache_append",
                          "ccgqa_prefill_workspace_size", "ccgqa_decode_workspace_size",
                          "ccgqa_status_string", "ccgqa_launch_count"}
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ccgqa.h but not exported"


def test_struct_layout_matches_c():
    src = r"""
#include <stdio.h>
#include <stddef.h>
#include "ccgqa.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu\n", sizeof(ccgqa_config), offsetof(ccgqa_config, rope_base),
         offsetof(ccgqa_config, dtype), sizeof(ccgqa_weights), sizeof(ccgqa_kvcache));
  printf("%zu %zu\n", offsetof(ccgqa_kvcache, batch), offsetof(ccgqa_kvcache, cap));
  printf("%zu %zu %zu\n", offsetof(ccgqa_kvcache, block_table), offsetof(ccgqa_kvcache, page_size),
         offsetof(ccgqa_kvcache, n_pages));
  return 0;
}
"""
    with tempfile.TemporaryDirectory() as td:
        c = os.path.join(td, "l.c")
        exe = os.path.join(td, "l")
        open(c, "w").write(src)
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe], check=True)
        out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split()
    vals = [int(v) for v in out]
    assert vals[0] == ctypes.sizeof(B.ccgqa_config)
    assert vals[1] == B.ccgqa_config.rope_base.offset
    assert vals[2] == B.ccgqa_config.dtype.offset
    assert vals[3] == ctypes.sizeof(B.ccgqa_weights)
    assert vals[4] == ctypes.sizeof(B.ccgqa_kvcache)
    assert vals[5] == B.ccgqa_kvcache.batch.offset
    assert vals[6] == B.ccgqa_kvcache.cap.offset
    assert vals[7] == B.ccgqa_kvcache.block_table.offset
    assert vals[8] == B.ccgqa_kvcache.page_size.offset
    assert vals[9] == B.ccgqa_kvcache.n_pages.offset


def test_status_strings(lib):
    for s in range(6):
        assert B.ccgqa_status_string(s)
    assert B.ccgqa_status_string(0) == "ok"


def _cfg(**kw):
    base = dict(E=2048, C=4, n_q_heads=16, n_kv_heads=4, conv_width=4, qk_mean=1, value_shift=1,
                causal=1, rope_base=1e4, dtype=B.BF16)
    base.update(kw)
    return B.make_config(**base)


def test_workspace_sizes(lib):
    cfg = _cfg()
    n = B.ccgqa_prefill_workspace_size(cfg, 4, 4096)
    d = 32
    N = (16 + 8) * d
    expect = 4 * 4096 * (N + 16 * d + 2 * 4 * d) * 2
    assert expect <= n <= expect + 4 * 256
    assert B.ccgqa_decode_workspace_size(cfg, 64, 16384) > 0
    # invalid geometry -> 0
    assert B.ccgqa_prefill_workspace_size(_cfg(n_kv_heads=3), 1, 16) == 0
    assert B.ccgqa_prefill_workspace_size(cfg, 0, 16) == 0


class _FakeTensor:
    """Stands in for a device tensor: the calls below are rejected by host
    validation before anything reaches the GPU."""

    def __init__(self, addr, nbytes=1 << 30):
        self.addr, self.nbytes = addr, nbytes

    def data_ptr(self):
        return self.addr

    def numel(self):
        return self.nbytes

    def element_size(self):
        return 1


@pytest.mark.parametrize("bad,status", [
    (dict(n_kv_heads=3), 1),           # Hq % Hkv != 0
    (dict(E=2050), 1),                 # E % (C Hq) != 0
    (dict(conv_width=5), 1),
    (dict(dtype=7), 1),
    (dict(rope_base=-1.0), 1),
    (dict(E=1024, C=8), 2),            # d = 8 unsupported
    # a group so large that the decode pre-step's (G + 2) d staged channels do
    # not fit in shared memory
    (dict(E=131072, C=1, n_q_heads=1024, n_kv_heads=1), 2),
])
def test_invalid_config_rejected(lib, bad, status):
    cfg = _cfg(**bad)
    w = B.make_weights()
    st = lib.ccgqa_prefill(ctypes.byref(cfg), ctypes.byref(w), ctypes.c_void_p(4096), 1, 16,
                           ctypes.c_void_p(8192), None, ctypes.c_void_p(1 << 20), 1 << 30, None,
                           None)
    assert st == status


@pytest.mark.parametrize("geo", [
    dict(E=256, C=1, n_q_heads=16, n_kv_heads=16),       # bf16 d = 16
    dict(E=1536, C=2, n_q_heads=12, n_kv_heads=4),       # G = 3
    dict(E=1536, C=4, n_q_heads=12, n_kv_heads=2),       # G = 6
    dict(E=3072, C=1, n_q_heads=24, n_kv_heads=2),       # G = 12, d = 128
    dict(E=1536, C=1, n_q_heads=24, n_kv_heads=1),       # G = 24
    dict(E=2560, C=1, n_q_heads=160, n_kv_heads=1),      # G = 160, d = 16
])
def test_whole_domain_accepted(lib, geo):
    """Every d in {16, 32, 64, 128} and every Hq % Hkv == 0 is a valid layer
    (the GQA page's grouping, with MQA and MHA as its ends)."""
    cfg = _cfg(**geo)
    assert B.ccgqa_prefill_workspace_size(cfg, 1, 64) > 0
    assert B.ccgqa_decode_workspace_size(cfg, 2, 64) > 0


def test_invalid_pointers_and_workspace_rejected(lib):
    cfg = _cfg(conv_width=0, qk_mean=0, value_shift=0)
    w = B.make_weights()
    ok_ws = _FakeTensor(1 << 20)
    assert B.ccgqa_prefill(cfg, w, _FakeTensor(4096), 1, 16, None, None, ok_ws, stream=0, check=False) == 1
    assert B.ccgqa_prefill(cfg, w, _FakeTensor(4097), 1, 16, _FakeTensor(8192), None, ok_ws,
                           stream=0, check=False) == 1                    # misaligned x
    assert B.ccgqa_prefill(cfg, w, _FakeTensor(4096), 1, 16, _FakeTensor(8192), None,
                           _FakeTensor(1 << 20, 16), stream=0, check=False) == 4   # workspace too small
    assert B.ccgqa_prefill(cfg, w, _FakeTensor(4096), 1, 16, _FakeTensor(8192), None,
                           _FakeTensor((1 << 20) + 16), stream=0, check=False) == 4  # misaligned workspace
    assert B.ccgqa_prefill(cfg, w, _FakeTensor(4096), 0, 16, _FakeTensor(8192), None, ok_ws,
                           stream=0, check=False) == 1
    # conv on but no conv weights
    cfg2 = _cfg()
    assert B.ccgqa_prefill(cfg2, w, _FakeTensor(4096), 1, 16, _FakeTensor(8192), None, ok_ws,
                           stream=0, check=False) == 1


def test_capacity_checked_on_host(lib):
    cfg = _cfg(conv_width=0, qk_mean=0, value_shift=0)
    cache = B.ccgqa_kvcache(4096, 8192, 12288, None, None, None, 1, 8)
    w = B.make_weights()
    st = lib.ccgqa_prefill(ctypes.byref(cfg), ctypes.byref(w), ctypes.c_void_p(4096), 1, 16,
                           ctypes.c_void_p(8192), ctypes.byref(cache), ctypes.c_void_p(1 << 20),
                           1 << 30, None, None)
    assert st == 3   # 16 tokens > cap 8
    st = lib.ccgqa_kvcache_append(ctypes.byref(cfg), ctypes.byref(cache), ctypes.c_void_p(4096),
                                  ctypes.c_void_p(8192), 9, None, None)
    assert st == 3
    cache.batch = 2
    st = lib.ccgqa_prefill(ctypes.byref(cfg), ctypes.byref(w), ctypes.c_void_p(4096), 1, 4,
                           ctypes.c_void_p(8192), ctypes.byref(cache), ctypes.c_void_p(1 << 20),
                           1 << 30, None, None)
    assert st == 1   # cache batch mismatch


@pytest.mark.parametrize("page_size,cap,n_pages,table,why", [
    (8, 64, 16, 1 << 16, "page below 16 tokens"),
    (48, 96, 16, 1 << 16, "page size not a power of two"),
    (8192, 8192, 16, 1 << 16, "page above 4096 tokens"),
    (32, 80, 16, 1 << 16, "page size does not divide cap"),
    (32, 64, 0, 1 << 16, "empty pool"),
    (32, 64, 1 << 30, 1 << 16, "n_pages * Hkv past int32"),
    (32, 64, 16, (1 << 16) + 2, "misaligned block table"),
])
def test_paged_cache_checked_on_host(lib, page_size, cap, n_pages, table, why):
    """A paged cache's geometry is validated before any launch (append and
    prefill both return CCGQA_ERR_INVALID_ARG)."""
    cfg = _cfg(conv_width=0, qk_mean=0, value_shift=0)
    cache = B.ccgqa_kvcache(4096, 8192, 12288, None, None, None, 1, cap, table, page_size,
                            n_pages)
    st = lib.ccgqa_kvcache_append(ctypes.byref(cfg), ctypes.byref(cache), ctypes.c_void_p(4096),
                                  ctypes.c_void_p(8192), 1, None, None)
    assert st == 1, why
    w = B.make_weights()
    st = lib.ccgqa_prefill(ctypes.byref(cfg), ctypes.byref(w), ctypes.c_void_p(4096), 1, 4,
                           ctypes.c_void_p(8192), ctypes.byref(cache), ctypes.c_void_p(1 << 20),
                           1 << 30, None, None)
    assert st == 1, why
    # the same cache with a valid geometry passes validation as far as capacity
    good = B.ccgqa_kvcache(4096, 8192, 12288, None, None, None, 1, 64, 1 << 16, 32, 16)
    st = lib.ccgqa_kvcache_append(ctypes.byref(cfg), ctypes.byref(good), ctypes.c_void_p(4096),
                                  ctypes.c_void_p(8192), 65, None, None)
    assert st == 3   # 65 tokens > cap 64: capacity, not geometry


def test_launch_count_starts_at_zero(lib):
    assert B.ccgqa_launch_count() == 0


def test_graph_calls_checked_on_host(lib):
    # the legacy default stream cannot be recorded; end/launch need a recording
    # or a graph; no CUDA call is reached by any of these
    assert lib.ccgqa_graph_begin(None) == 1
    h = ctypes.c_void_p()
    assert lib.ccgqa_graph_end(None, ctypes.byref(h)) == 1
    assert lib.ccgqa_graph_end(ctypes.c_void_p(4096), None) == 1
    assert lib.ccgqa_graph_launch(None, None) == 1
    assert lib.ccgqa_graph_kernel_count(None) == -1
    assert lib.ccgqa_graph_destroy(None) == 0
    assert B.ccgqa_launch_count() == 0


def test_output_projection_checked_on_host(lib):
    cfg = B.make_config(E=512, C=4, n_q_heads=4, n_kv_heads=2)      # d = 32
    fake = ctypes.c_void_p(4096)          # aligned, never dereferenced on these paths
    f = lib.ccgqa_output_projection
    assert f(ctypes.byref(cfg), fake, fake, 0, fake, None, None) == 1          # M <= 0
    assert f(ctypes.byref(cfg), None, fake, 4, fake, None, None) == 1          # NULL W_o
    assert f(ctypes.byref(cfg), fake, ctypes.c_void_p(4098), 4, fake, None, None) == 1
    assert f(ctypes.byref(cfg), fake, fake, (1 << 30) + 1, fake, None, None) == 2
    odd = B.make_config(E=20, C=1, n_q_heads=4, n_kv_heads=2)   # head dim 5: unsupported
    assert f(ctypes.byref(odd), fake, fake, 4, fake, None, None) == 2
    bad = B.make_config(E=500, C=4, n_q_heads=4, n_kv_heads=2)  # E not a multiple of C Hq
    assert f(ctypes.byref(bad), fake, fake, 4, fake, None, None) == 1
    assert B.ccgqa_launch_count() == 0


def test_backward_checked_on_host(lib):
    """ccgqa_prefill_backward validates before any launch (no GPU needed)."""
    cfg = _cfg()
    assert B.ccgqa_prefill_backward_workspace_size(cfg, 2, 128) > 0
    assert B.ccgqa_prefill_backward_workspace_size(_cfg(n_kv_heads=3), 2, 128) == 0
    w = B.make_weights()           # conv taps missing for conv_width 4
    fake = ctypes.c_void_p(1 << 20)
    f = lib.ccgqa_prefill_backward
    assert f(ctypes.byref(cfg), ctypes.byref(w), fake, 1, 16, fake, fake, None, fake,
             1 << 30, None, None) == 1
    w0 = B.make_weights()
    cfg0 = _cfg(conv_width=0, qk_mean=0, value_shift=0)
    assert f(ctypes.byref(cfg0), ctypes.byref(w0), None, 1, 16, fake, fake, None, fake,
             1 << 30, None, None) == 1                                   # no input
    assert f(ctypes.byref(cfg0), ctypes.byref(w0), fake, 0, 16, fake, fake, None, fake,
             1 << 30, None, None) == 1                                   # empty batch
    assert f(ctypes.byref(cfg0), ctypes.byref(w0), fake, 1, 16, fake, fake, None, None,
             0, None, None) == 4                                         # no workspace
