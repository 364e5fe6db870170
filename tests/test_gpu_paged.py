"""Paged latent KV cache through the C ABI.

The cache is allocated in fixed-size pages, each holding a run of
consecutive tokens of one sequence for all kv heads, named per sequence by a
block table ("Grouped Query Attention (GQA)", section "GQA y tecnicas
relacionadas": PagedAttention).  The page layout changes where rows live, not
what is computed: every kernel visits the same keys in the same order, so a
paged prefill / append / decode step must give BIT-IDENTICAL outputs, caches
and decode state to the contiguous cache (whose parity with the oracle the
other GPU tests check), and the oracle is checked here as well.  Block tables
are seeded permutations of a pool with spare pages, so a sequence's pages are
scattered and out of order."""
import numpy as np
import pytest
import torch

import oracle.ccgqa as O
from compressed_latent_grouped_b200 import binding as B
from compressed_latent_grouped_b200.device import DeviceLayer
from compressed_latent_grouped_b200.workloads import WORKLOADS, make_block_table, make_inputs
from gpu_ref import check_prefill, check_rows, decode_references, f64

pytestmark = pytest.mark.gpu

W2 = WORKLOADS["bf16_prefill_b4_s4096"]
W3 = WORKLOADS["bf16_prefill_b1_s32768"]
W4 = WORKLOADS["bf16_decode_b64_l16384"]
W5 = WORKLOADS["bf16_gqa_b2_s8192"]
SPARE_PAGES = 5


def _round_up(n, m):
    return (n + m - 1) // m * m


def paged_layer(w, inp, batch, cap, page, seed=0):
    """A DeviceLayer whose cache is a pool of pages with a seeded block table."""
    per_seq = cap // page
    n_pages = batch * per_seq + SPARE_PAGES
    lay = DeviceLayer(w, inp, batch=batch, cap=cap)
    table = make_block_table(batch, per_seq, n_pages, seed=seed)
    t = lay.alloc_cache(block_table=table, page_size=page, n_pages=n_pages)
    return lay, t


def gather(pool, table, page, L):
    """Logical rows [B, Hkv, L, d] of a paged pool (pure indexing)."""
    pages = pool[table.long()]                          # [B, per_seq, Hkv, page, d]
    Bn, per_seq, Hkv, P, d = pages.shape
    return pages.permute(0, 2, 1, 3, 4).reshape(Bn, Hkv, per_seq * P, d)[:, :, :L]


def bits(t):
    return t.contiguous().view(torch.int16 if t.dtype == torch.bfloat16 else torch.int32)


def assert_bit_equal(a, b, what):
    assert a.shape == b.shape, (what, a.shape, b.shape)
    assert torch.equal(bits(a), bits(b)), what


def _load_state(lay, t, w, inp):
    """Synthetic cache rows through ccgqa_kvcache_append, plus the decode state."""
    lay.append(inp["cache_k"].cuda(), inp["cache_v"].cuda())
    if w.conv_width > 1:
        t["hist_q"].copy_(inp["hist_q"])
        t["hist_k"].copy_(inp["hist_k"])
    t["v_prev"].copy_(inp["v_prev"])


DECODE_CASES = [
    # tensor-core decode attention (bf16, G <= 16): pages below, at and above
    # the 128-key chunk of the TMA producer
    (W4.with_(name="pg_dec_d64", B=5, S=700), 16),
    (W4.with_(name="pg_dec_d64", B=5, S=700), 256),
    (W4.with_(name="pg_dec_d32", B=3, S=333, E=2048, C=4, Hq=16, Hkv=4, rope_base=1e4), 64),
    (W4.with_(name="pg_dec_d128", B=2, S=300, E=4096, C=1, Hq=32, Hkv=8, conv_width=0,
              qk_mean=False, value_shift=False, packed_input=True), 128),
    # CUDA-core decode attention: fp32, bf16 d = 16, G beyond the tensor-core kernel
    (W4.with_(name="pg_dec_f32", B=3, S=130, dtype="f32"), 32),
    (W4.with_(name="pg_dec_bf16_d16", B=3, S=300, E=256, C=4, Hq=4, Hkv=2, rope_base=1e4), 16),
    (W4.with_(name="pg_dec_g24", B=2, S=260, E=1536, C=1, Hq=24, Hkv=1), 64),
    # the readings' variants
    (W4.with_(name="pg_dec_variants", B=3, S=200, channel_conv=True, qk_mean=2, value_shift=2), 32),
]


@pytest.mark.parametrize("w,page", DECODE_CASES, ids=lambda v: getattr(v, "name", str(v)))
def test_paged_decode_equals_contiguous_and_oracle(w, page):
    inp = make_inputs(w, seed=3)
    cap = _round_up(w.S + 8, page)
    con = DeviceLayer(w, inp, cap=cap)
    tc = con.alloc_cache()
    _load_state(con, tc, w, inp)
    pag, tp = paged_layer(w, inp, w.B, cap, page, seed=1)
    _load_state(pag, tp, w, inp)
    torch.cuda.synchronize()
    assert pag.error_bits() == 0
    # the append put every row at its page
    assert_bit_equal(gather(tp["k"], tp["block_table"], page, w.S), tc["k"][:, :, : w.S],
                     "appended k")
    assert_bit_equal(gather(tp["v"], tp["block_table"], page, w.S), tc["v"][:, :, : w.S],
                     "appended v")
    g = torch.Generator().manual_seed(12)
    width = w.n_qkv if w.packed_input else w.E
    xs, outs = [], []
    for step in range(3):
        x_t = torch.randn(w.B, width, generator=g).to(w.torch_dtype).cuda()
        oc = con.decode_step(x_t)
        op = pag.decode_step(x_t)
        torch.cuda.synchronize()
        assert con.error_bits() == 0 and pag.error_bits() == 0
        assert_bit_equal(op, oc, f"{w.name} page {page} step {step} output")
        xs.append(x_t.cpu())
        outs.append(op.float().cpu().numpy())
    L = w.S + 3
    assert tp["len"].cpu().tolist() == [L] * w.B
    for key in ("k", "v"):
        assert_bit_equal(gather(tp[key], tp["block_table"], page, L), tc[key][:, :, :L], key)
    for key in ("hist_q", "hist_k", "v_prev"):
        assert_bit_equal(tp[key], tc[key], key)
    # and the oracle, on the first and last sequence
    for b in (0, w.B - 1):
        refs, models, _, _ = decode_references(w, inp, b, [f64(x[b]) for x in xs])
        for step in range(3):
            check_rows(w.dtype, outs[step][b], refs[step], models[step],
                       f"{w.name} page {page} step {step} b={b}")


PREFILL_CASES = [
    (W2.with_(name="pg_pf_d32", B=2, S=300), 16),
    (W2.with_(name="pg_pf_d32", B=2, S=300), 512),
    (W3.with_(name="pg_pf_d64", S=260), 128),
    (W5.with_(name="pg_pf_d128", B=1, S=200), 64),
    (WORKLOADS["f32_s128"].with_(name="pg_pf_f32", B=2), 32),
    (W3.with_(name="pg_pf_variants", S=150, qk_mean=2, value_shift=2, channel_conv=True), 16),
]


@pytest.mark.parametrize("w,page", PREFILL_CASES, ids=lambda v: getattr(v, "name", str(v)))
def test_paged_prefill_equals_contiguous_and_oracle(w, page):
    """Prefill into a paged cache (the page-scatter kernel after the attention),
    then one decode step on each cache."""
    inp = make_inputs(w, seed=5)
    cap = _round_up(w.S + 16, page)
    x = inp["x"].cuda()
    con = DeviceLayer(w, inp, cap=cap)
    tc = con.alloc_cache()
    pag, tp = paged_layer(w, inp, w.B, cap, page, seed=2)
    oc = con.prefill(x)
    op = pag.prefill(x)
    torch.cuda.synchronize()
    assert con.error_bits() == 0 and pag.error_bits() == 0
    assert_bit_equal(op, oc, "prefill output")
    for key in ("k", "v"):
        assert_bit_equal(gather(tp[key], tp["block_table"], page, w.S), tc[key][:, :, : w.S], key)
    for key in ("hist_q", "hist_k", "v_prev", "len"):
        assert torch.equal(tp[key], tc[key]), key
    # the spare pages were not written
    used = torch.zeros(tp["k"].shape[0], dtype=torch.bool)
    used[tp["block_table"].cpu().long().flatten()] = True
    assert torch.all(tp["k"][~used.cuda()] == 0) and torch.all(tp["v"][~used.cuda()] == 0)
    check_prefill(w, inp, 0, op[0].float().cpu().numpy(), what=f"{w.name} page {page}")
    width = w.n_qkv if w.packed_input else w.E
    x_t = torch.randn(w.B, width, generator=torch.Generator().manual_seed(3)).to(w.torch_dtype)
    dc = con.decode_step(x_t.cuda())
    dp = pag.decode_step(x_t.cuda())
    torch.cuda.synchronize()
    assert pag.error_bits() == 0
    assert_bit_equal(dp, dc, "decode after paged prefill")


def test_paged_decode_full_size():
    """64 sequences x 16384 cached tokens in pages of 64 tokens: the step equals
    the contiguous cache's bit for bit; sampled sequences against the oracle."""
    w, page = W4, 64
    inp = make_inputs(w)
    cap = _round_up(w.S + 64, page)
    con = DeviceLayer(w, inp, cap=cap)
    tc = con.alloc_cache()
    _load_state(con, tc, w, inp)
    pag, tp = paged_layer(w, inp, w.B, cap, page, seed=9)
    _load_state(pag, tp, w, inp)
    x_t = inp["x_t"].cuda()
    oc = con.decode_step(x_t)
    op = pag.decode_step(x_t)
    torch.cuda.synchronize()
    assert con.error_bits() == 0 and pag.error_bits() == 0
    assert_bit_equal(op, oc, "full-size paged decode")
    got = op.float().cpu().numpy()
    for b in (0, 17, w.B - 1):
        refs, models, _, _ = decode_references(w, inp, b, [f64(inp["x_t"][b])])
        check_rows(w.dtype, got[b], refs[0], models[0], f"paged decode b={b}")


def test_paged_noalloc_equals_workspace_decode():
    w, page = W4.with_(B=4, S=500), 32
    inp = make_inputs(w, seed=8)
    cap = _round_up(w.S + 8, page)
    a, ta = paged_layer(w, inp, w.B, cap, page, seed=4)
    _load_state(a, ta, w, inp)
    b, tb = paged_layer(w, inp, w.B, cap, page, seed=4)
    _load_state(b, tb, w, inp)
    x_t = inp["x_t"].cuda()
    oa = a.decode_step(x_t)
    ob = torch.empty_like(oa)
    B.ccgqa_decode_step_noalloc(b.cfg, b.weights, x_t, b.cache, ob, b.dev_err)
    torch.cuda.synchronize()
    assert a.error_bits() == 0 and b.error_bits() == 0
    assert_bit_equal(ob, oa, "noalloc paged decode")
    assert_bit_equal(tb["k"], ta["k"], "pool k")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_paged_entry_outside_pool_sets_index_bit(dtype):
    """A block-table entry outside the pool, for a page the step reads and
    writes, sets CCGQA_DEVERR_INDEX.  The kernels check every id before use:
    the tensor-core producer turns it into a coordinate past the pool (TMA
    fills zeros there), the CUDA-core one skips that copy, the pre-step skips
    the row write.  The pool is not written outside the sequences' own pages and the
    other sequences' outputs are unaffected."""
    w, page = W4.with_(B=3, S=300, dtype=dtype), 64
    inp = make_inputs(w, seed=6)
    cap = _round_up(w.S + 8, page)
    good, tg = paged_layer(w, inp, w.B, cap, page, seed=7)
    _load_state(good, tg, w, inp)
    bad, tb = paged_layer(w, inp, w.B, cap, page, seed=7)
    _load_state(bad, tb, w, inp)
    torch.cuda.synchronize()
    pool_before = tb["k"].clone()
    # sequence 1: its page of token 100 and the page of the new token (300)
    # name ids past the pool / negative
    n_pages = tb["k"].shape[0]
    tb["block_table"][1, 100 // page] = n_pages + 3
    tb["block_table"][1, 300 // page] = -1
    x_t = inp["x_t"].cuda()
    og = good.decode_step(x_t)
    ob = bad.decode_step(x_t)
    torch.cuda.synchronize()
    assert good.error_bits() == 0
    assert bad.error_bits() & B.DEVERR_INDEX
    for s in (0, 2):
        assert_bit_equal(ob[s], og[s], f"sequence {s}")
    # nothing was written into a page that sequence 1's bad entries would have named
    changed = (tb["k"] != pool_before).flatten(1).any(1).cpu()
    own = set(tb["block_table"][[0, 2]].cpu().flatten().tolist())
    own |= {int(p) for p in tb["block_table"][1].cpu().tolist() if 0 <= p < n_pages}
    assert all(int(i) in own for i in torch.nonzero(changed).flatten().tolist())


def test_paged_append_entry_outside_pool_sets_index_bit():
    w, page = W4.with_(B=2, S=64), 16
    inp = make_inputs(w, seed=2)
    lay, t = paged_layer(w, inp, w.B, 64, page, seed=3)
    t["block_table"][0, 2] = -5
    k = torch.randn(2, 40, w.Hkv, w.d, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    lay.append(k.cuda(), k.cuda())
    torch.cuda.synchronize()
    assert lay.error_bits() & B.DEVERR_INDEX
    # rows of the other pages are written as usual
    tab = t["block_table"].cpu()
    for (b, p) in [(0, 0), (0, 1), (1, 0), (1, 1), (1, 2)]:
        lo, hi = p * page, min((p + 1) * page, 40)
        assert_bit_equal(t["k"][int(tab[b, p]), :, : hi - lo].cpu(),
                         k[b, lo:hi].permute(1, 0, 2), f"seq {b} page {p}")
