"""CUDA graphs of library calls (ccgqa_graph_*): a recorded prefill + decode
step replays bit for bit like the eager calls, on new inputs written into the
recorded buffers too; recording runs nothing and counts nothing; a call on
another stream while recording is refused."""
import pytest
import torch

from compressed_latent_grouped_b200 import binding as B
from compressed_latent_grouped_b200.device import DeviceLayer, Graph
from compressed_latent_grouped_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,batch,seq", [("bf16_prefill_b4_s4096", 2, 300),
                                            ("bf16_prefill_b1_s32768", 1, 700),
                                            ("f32_s128", 2, 130)])
def test_graph_replay_matches_eager(name, batch, seq):
    w = WORKLOADS[name].with_(name=f"graph_{name}", B=batch, S=seq)
    inp = make_inputs(w, seed=11)
    lay = DeviceLayer(w, inp, cap=seq + 2)
    lay.alloc_cache()
    x = inp["x"].cuda()
    g = torch.Generator().manual_seed(12)
    x_t = torch.randn(batch, w.E, generator=g).to(w.torch_dtype).cuda()
    out = torch.empty(batch, seq, w.Hq * w.d, dtype=w.torch_dtype, device="cuda")
    out_t = torch.empty(batch, w.Hq * w.d, dtype=w.torch_dtype, device="cuda")
    s = torch.cuda.Stream()

    def step():
        lay.prefill(x, out, stream=s)
        lay.decode_step(x_t, out_t, stream=s)

    with torch.cuda.stream(s):
        n0 = B.ccgqa_launch_count()
        step()                      # eager (also allocates the workspaces)
        s.synchronize()
        per_step = B.ccgqa_launch_count() - n0
        ref = (out.clone(), out_t.clone(), lay.cache_tensors["k"].clone(),
               lay.cache_tensors["v"].clone(), lay.cache_tensors["len"].clone())
        out.zero_()
        out_t.zero_()
        s.synchronize()

    n1 = B.ccgqa_launch_count()
    gr = Graph(step, s)
    try:
        assert B.ccgqa_launch_count() == n1          # recording launches nothing
        assert gr.kernels == per_step
        s.synchronize()
        assert not out.any() and not out_t.any()     # and ran nothing
        gr.launch()
        s.synchronize()
        assert B.ccgqa_launch_count() == n1 + per_step
        assert lay.error_bits() == 0
        c = lay.cache_tensors
        assert torch.equal(out, ref[0]) and torch.equal(out_t, ref[1])
        assert torch.equal(c["k"], ref[2]) and torch.equal(c["v"], ref[3])
        assert torch.equal(c["len"], ref[4])
        # new inputs in the recorded buffers: the replay follows them
        x2 = torch.randn(x.shape, generator=g).to(w.torch_dtype).cuda()
        xt2 = torch.randn(x_t.shape, generator=g).to(w.torch_dtype).cuda()
        with torch.cuda.stream(s):
            x.copy_(x2)
            x_t.copy_(xt2)
            gr.launch()
            o_g, ot_g = out.clone(), out_t.clone()
            step()                  # eager on the same new inputs
        s.synchronize()
        assert torch.equal(o_g, out) and torch.equal(ot_g, out_t)
        assert not torch.equal(o_g, ref[0])
    finally:
        gr.close()


def test_graph_refuses_other_stream_while_recording():
    w = WORKLOADS["bf16_prefill_b4_s4096"].with_(name="graph_refuse", B=1, S=64)
    inp = make_inputs(w, seed=5)
    lay = DeviceLayer(w, inp, cap=70)
    lay.alloc_cache()
    x = inp["x"].cuda()
    out = torch.empty(1, 64, w.Hq * w.d, dtype=w.torch_dtype, device="cuda")
    s, other = torch.cuda.Stream(), torch.cuda.Stream()
    lay.prefill(x, out, stream=s)    # workspaces exist before recording
    s.synchronize()
    B.ccgqa_graph_begin(s)
    try:
        st = B.ccgqa_prefill(lay.cfg, lay.weights, x, 1, 64, out, lay.cache,
                             lay.prefill_workspace(1, 64), lay.dev_err, other, check=False)
        assert st == 1
        assert B.ccgqa_graph_begin(s, check=False) == 1   # no nested recording
    finally:
        h = B.ccgqa_graph_end(s)
    assert B.ccgqa_graph_kernel_count(h) == 0
    B.ccgqa_graph_destroy(h)
