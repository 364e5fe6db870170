"""Benchmark of the CCGQA hot path on B200.

One step = one pass of the whole path on the largest single-GPU workloads: the
bf16 prefill of one S=32768 sequence (E=4096, C=8, 8 query / 2 kv heads of dim
64, RoPE base 5e5: latent projection on tcgen05, fused conv / QK-mean / RoPE /
value-shift, tcgen05 flash attention, cache write) followed by one decode step
of 64 sequences against latent caches of 16384 tokens each (projection,
one-token pre-step with cache append, split-K attention over 16385 keys).

Prints one JSON line (rank 0).  Timing: W untimed warm-up steps, then K steps,
each preceded by an untimed write of a buffer larger than L2 (and a reset of the
decode caches' lengths to 16384) and timed with CUDA events on the launching
stream; the job is bracketed by a barrier and torch.cuda.synchronize() on both
sides and the time is the max over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PREFILL_WL = "bf16_prefill_b1_s32768"
DECODE_WL = "bf16_decode_b64_l16384"
WORKLOAD = f"{PREFILL_WL} prefill + {DECODE_WL} decode step"
METRIC = "CCGQA prefill TFLOP/s & tokens/s; decode latent-KV GB/s vs B200 peak"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
ATTN_SRC = os.path.join(ROOT, "compressed_latent_grouped_b200", "csrc", "attn_prefill_tc.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_prefill_tc_traffic.txt")
# pairs c2 = 0, k, 2k, ... (k = SOFT_EVERY[d]) of the 32 exponential pairs in a
# 64-key half run on the FMA pipe (a polynomial) in attn_prefill_tc, the rest
# on the exp unit
SOFT_EVERY = {32: 5, 64: 3, 128: 4}


def attention_flops(B: int, S: int, Hq: int, d: int, causal: bool = True) -> float:
    """Algorithmic FLOPs of one prefill attention launch: 2 d for QK^T plus 2 d
    for PV per visible (query, key) pair; causal counts S^2/2 pairs."""
    pairs = S * S / 2 if causal else S * S
    return 4.0 * d * Hq * pairs * B


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def attn_traffic_per_launch():
    """DRAM bytes of one attention launch from the committed ncu capture, or
    None when the kernel source changed since the capture."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    vals = {}
    with open(TRAFFIC_FILE) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#") and "=" in line:
                k, v = (s.strip() for s in line.split("=", 1))
                vals[k] = v
    with open(ATTN_SRC, "rb") as f:
        h = hashlib.sha256(f.read()).hexdigest()[:16]
    if vals.get("source_sha256_16") != h or vals.get("workload") != PREFILL_WL:
        return None
    return float(vals["dram_bytes_per_launch"])


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x1: "gpu_idle", 0x2: "applications_clocks_setting",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int):
        self.samples, self.reasons, self.ok = [], set(), False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # noqa: BLE001 - report null clocks instead
            self.max_mhz = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.ok:
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def dist_setup(n_gpus):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl" if torch.cuda.is_available() else "gloo",
                                timeout=timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(value: float, world: int, device):
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------------- oracle
def _oracle_layer(w, inp):
    import oracle.ccgqa as O
    f = lambda t: None if t is None else t.double().numpy()  # noqa: E731
    return O.Layer(sh=O.Shape(w.E, w.C, w.Hq, w.Hkv), W_qkv=f(inp["W_qkv"]),
                   conv_width=w.conv_width, conv_q_seq=f(inp["conv_q_seq"]),
                   conv_q_chan=f(inp["conv_q_chan"]), conv_k_seq=f(inp["conv_k_seq"]),
                   conv_k_chan=f(inp["conv_k_chan"]), qk_mean=w.qk_mean,
                   value_shift=w.value_shift, rope_base=w.rope_base, causal=w.causal)


def oracle_prefill_time(w, inp, lay, b: int = 0, s_len: int | None = None, rows=None):
    """Host seconds of the float64 oracle's prefill of sequence b (its first
    s_len tokens, default all S; query rows ``rows``, default all)."""
    import oracle.ccgqa as O
    x = (inp["x"][b] if s_len is None else inp["x"][b, :s_len]).double().numpy()
    t0 = time.perf_counter()
    O.prefill(lay, x, rows=rows)
    return time.perf_counter() - t0


class OracleDecode:
    """Decode steps of the float64 oracle against the decode workload's caches
    (one sequence at a time; the state is built outside the timed call)."""

    def __init__(self, w, inp):
        self.w, self.inp = w, inp
        self.lay = _oracle_layer(w, inp)

    def state(self, b):
        import oracle.ccgqa as O
        inp = self.inp
        return O.State(k=inp["cache_k"][b].double().numpy(), v=inp["cache_v"][b].double().numpy(),
                       hist_q=inp["hist_q"][b].double().numpy(),
                       hist_k=inp["hist_k"][b].double().numpy(),
                       v_prev=inp["v_prev"][b].double().numpy())

    def time(self, b):
        import oracle.ccgqa as O
        st = self.state(b)
        x_t = self.inp["x_t"][b].double().numpy()
        t0 = time.perf_counter()
        O.decode_step(self.lay, st, x_t)
        return time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def cpu_baseline_headline(wp, inp_p, wd, inp_d):
    """The float64 oracle on the headline step, on a bounded sample.

    Prefill: the oracle's prefill of the S-token sequence with n query rows
    evaluated (keys and values always built for all S positions), timed at two
    row counts; a straight line through the two times extrapolates to all S rows
    (the oracle computes every score row in full, so its cost per row does not
    depend on the position).  Decode: the oracle's decode step of each of the
    B sequences against its full cache, timed one by one."""
    from compressed_latent_grouped_b200.workloads import sample_rows
    lay = _oracle_layer(wp, inp_p)
    n1, n2 = 64, 576
    rows = sample_rows(wp.S, n=n2, seed=11)
    t1 = oracle_prefill_time(wp, inp_p, lay, rows=rows[:: n2 // n1][:n1])
    t2 = oracle_prefill_time(wp, inp_p, lay, rows=rows)
    per_row = max(t2 - t1, 0.0) / (n2 - n1)
    t_prefill = t1 - per_row * n1 + per_row * wp.S
    dec = OracleDecode(wd, inp_d)
    t_dec = sum(dec.time(b) for b in range(wd.B))
    tokens = wp.B * wp.S + wd.B
    return {"value": tokens / (t_prefill + t_dec), "unit": "tokens/s", "cores": blas_threads(),
            "nproc": os.cpu_count(), "kind": "oracle",
            "sample": (f"prefill: float64 oracle over all {wp.S} tokens with {n1} and {n2} query "
                       f"rows evaluated ({t1:.1f} s, {t2:.1f} s), extrapolated linearly to "
                       f"{wp.S} rows = {t_prefill:.1f} s; decode: all {wd.B} sequences against "
                       f"their {wd.S}-token caches, timed ({t_dec:.1f} s); cores = BLAS "
                       f"threads (the rest of the oracle runs on one thread)"),
            "extrapolated": True, "host_seconds": t1 + t2 + t_dec}


def reference_sample_len(wp, inp_p, lay, n_calls, budget_s):
    """Prefix length S' (a multiple of 128, at most S) whose oracle prefill fits
    budget_s / n_calls, from a 512-token probe scaled by (S'/512)^2 (the
    attention's share grows quadratically, so the estimate errs long)."""
    probe = min(512, wp.S)
    t_probe = oracle_prefill_time(wp, inp_p, lay, s_len=probe)
    per_call = budget_s / max(n_calls, 1)
    s_len = int(probe * (per_call / max(t_probe, 1e-6)) ** 0.5) // 128 * 128
    return max(128, min(wp.S, s_len))


def run_reference(args, world, rank):
    """The reference arm: the float64 oracle on the host cores, on this arm's
    workload, each step a bounded sample of it."""
    from compressed_latent_grouped_b200.workloads import WORKLOADS, make_inputs
    if rank != 0:
        return
    wp, wd = WORKLOADS[PREFILL_WL], WORKLOADS[DECODE_WL]
    inp_p = make_inputs(wp, seed=0)
    inp_d = make_inputs(wd, seed=0, batch=8)
    lay = _oracle_layer(wp, inp_p)
    dec = OracleDecode(wd, inp_d)
    n = args.steps + args.warmup
    s_len = reference_sample_len(wp, inp_p, lay, n, 0.8 * args.ref_seconds)

    def one(i):
        return oracle_prefill_time(wp, inp_p, lay, s_len=s_len) + dec.time(i % 8)

    for i in range(args.warmup):
        one(i)
    t = sum(one(i) for i in range(args.steps))
    value = (s_len + 1) * args.steps / t
    sample = (f"per step: float64 prefill of the first {s_len} of {wp.S} tokens of the "
              f"{PREFILL_WL} sequence + 1 decode step of one of the {wd.B} sequences against "
              f"its {wd.S}-token cache")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * t / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded PCG64 normals)",
        "config": {"workload": WORKLOAD, "S": wp.S, "E": wp.E, "C": wp.C, "Hq": wp.Hq,
                   "Hkv": wp.Hkv, "d": wp.d, "decode_B": wd.B, "decode_L": wd.S,
                   "sample": sample},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(),
                         "nproc": os.cpu_count(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def exp_roofline(w, attn_ms, peaks):
    """The exponentials the exp unit executes against its peak: 16 ex2 per
    clock per SM (the B200 SFU rate, measured 15.8 on this part) x 148 SMs x the
    maximum SM clock.  A causal launch has B Hq S (S + 1) / 2 exponentials; the
    pairs SOFT_EVERY[d] apart run on the FMA pipe instead, so the exp unit's
    share is the rest, and frac is that share's rate over the unit's peak."""
    n_exp = w.B * w.Hq * w.S * (w.S + 1) / 2 if w.causal else w.B * w.Hq * w.S * w.S
    k = SOFT_EVERY.get(w.d, 4)
    mufu_share = 1.0 - ((32 + k - 1) // k) / 32.0
    mhz = peaks.get("sm_max_mhz", 1965.0)
    peak = 16 * 148 * mhz * 1e6 / 1e12
    achieved = n_exp * mufu_share / (attn_ms / 1e3) / 1e12
    return {"bound": "alu", "unit": "Texp/s", "achieved": achieved, "peak": peak,
            "frac": achieved / peak, "exp_per_launch": n_exp, "exp_unit_share": mufu_share,
            "peak_kind": f"exp unit (ex2): 16/clk/SM x 148 SMs x {mhz:.0f} MHz, derived "
                         f"(15.8/clk/SM measured with a throughput probe)"}


# ----------------------------------------------------------------------- per-workload kernels
def measure_prefill_workload(w, steps, dev):
    """Attention / projection / pre-attention device times of one prefill
    workload (events around each kernel; L2 flushed before every step)."""
    import torch
    from compressed_latent_grouped_b200 import binding as B
    from compressed_latent_grouped_b200.device import DeviceLayer
    from compressed_latent_grouped_b200.workloads import make_inputs
    inp = make_inputs(w, seed=0)
    lay = DeviceLayer(w, inp, device=dev, cap=w.S)
    lay.alloc_cache()
    x = inp["x"].to(dev)
    out = torch.empty(w.B, w.S, w.Hq * w.d, dtype=w.torch_dtype, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(3):
        lay.prefill(x, out)
    # two kernels per call: the projection ran fused with the pre-attention
    n0 = B.ccgqa_launch_count()
    lay.prefill(x, out)
    fused = B.ccgqa_launch_count() - n0 == 2 and not w.packed_input
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for e in evs:
        flush.zero_()
        B.ccgqa_set_phase_events(e)
        lay.prefill(x, out)
        B.ccgqa_set_phase_events(None)
    torch.cuda.synchronize()
    if lay.error_bits():
        raise RuntimeError(f"device error bits {lay.error_bits()}")
    ms = [sum(e[i].elapsed_time(e[i + 1]) for e in evs) / steps for i in range(3)]
    fl = attention_flops(w.B, w.S, w.Hq, w.d, w.causal)
    peaks, _ = load_peaks()
    res = {"attn_ms": ms[2], "attn_tflops": fl / (ms[2] / 1e3) / 1e12,
           "attn_tensor_frac": fl / (ms[2] / 1e3) / 1e12 / peaks["bf16_tflops"],
           "attn_exp_unit_frac": exp_roofline(w, ms[2], peaks)["frac"],
           "pre_attn_ms": ms[1], "prefill_ms": sum(ms),
           "tokens_per_s": w.B * w.S / (sum(ms) / 1e3)}
    if fused:
        # one kernel: the projection GEMM's FLOPs over its time
        res.pop("pre_attn_ms")
        res["proj_pre_fused_ms"] = ms[0] + ms[1]
        res["proj_pre_tflops"] = 2.0 * w.B * w.S * w.E * w.n_qkv / ((ms[0] + ms[1]) / 1e3) / 1e12
    elif not w.packed_input:
        res["proj_ms"] = ms[0]
        res["proj_tflops"] = 2.0 * w.B * w.S * w.E * w.n_qkv / (ms[0] / 1e3) / 1e12
        pre_bytes = 2 * w.B * w.S * w.n_qkv * 2
        res["pre_attn_hbm_frac"] = pre_bytes / (ms[1] / 1e3) / 1e9 / peaks["hbm_gbs"]
    return res


def setup_decode(w, dev, seed=0, extra_cap=64, page=0):
    """A decode layer whose caches hold w.S tokens per sequence, plus the
    device tensor that resets the lengths to w.S between timed steps.  With
    ``page`` > 0 the cache is a pool of pages of that many tokens named by a
    seeded block table (a sequence's pages scattered over the pool)."""
    import torch
    from compressed_latent_grouped_b200.device import DeviceLayer
    from compressed_latent_grouped_b200.workloads import make_block_table, make_inputs
    inp = make_inputs(w, seed=seed)
    cap = w.S + extra_cap
    lay = DeviceLayer(w, inp, device=dev, cap=cap)
    if page > 0:
        cap = (cap + page - 1) // page * page
        per_seq = cap // page
        n_pages = w.B * per_seq + 16
        lay.cap = cap
        t = lay.alloc_cache(cap=cap, block_table=make_block_table(w.B, per_seq, n_pages, seed),
                            page_size=page, n_pages=n_pages)
    else:
        t = lay.alloc_cache()
    lay.append(inp["cache_k"].to(dev), inp["cache_v"].to(dev))
    t["hist_q"].copy_(inp["hist_q"])
    t["hist_k"].copy_(inp["hist_k"])
    t["v_prev"].copy_(inp["v_prev"])
    len0 = torch.full((w.B,), w.S, dtype=torch.int32, device=dev)
    return lay, inp, len0


def decode_numbers(w, proj_ms, pre_ms, attn_ms, step_ms, peaks):
    """Decode-step figures: the kernels' times from events between them, the
    step's from events around the whole step only (an event between two
    kernels serialises them, so the kernel times add up to more than the step)."""
    kv = 2 * w.B * w.Hkv * (w.S + 1) * w.d * 2
    step = step_ms
    return {"kv_bytes": kv, "proj_ms": proj_ms, "pre_ms": pre_ms, "attn_ms": attn_ms,
            "step_ms": step, "sum_of_kernels_ms": proj_ms + pre_ms + attn_ms,
            "attn_gbs": kv / (attn_ms / 1e3) / 1e9,
            "attn_hbm_frac": kv / (attn_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
            "step_gbs": kv / (step / 1e3) / 1e9,
            "step_hbm_frac": kv / (step / 1e3) / 1e9 / peaks["hbm_gbs"],
            "tokens_per_s": w.B / (step / 1e3)}


def measure_decode_workload(w, steps, dev, page=0):
    """Decode step on a full latent cache (contiguous, or paged with ``page``
    tokens per page): device times of the projection, the one-token pre-step
    and the split-K attention over len + 1 keys."""
    import torch
    from compressed_latent_grouped_b200 import binding as B
    lay, inp, len0 = setup_decode(w, dev, page=page)
    x_t = inp["x_t"].to(dev)
    out = torch.empty(w.B, w.Hq * w.d, dtype=w.torch_dtype, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    lens = lay.cache_tensors["len"]
    for _ in range(3):
        lens.copy_(len0)
        lay.decode_step(x_t, out)
    # the whole step: events only around it
    whole = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(steps)]
    for e0, e1 in whole:
        lens.copy_(len0)
        flush.zero_()
        e0.record()
        lay.decode_step(x_t, out)
        e1.record()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for e in evs:
        lens.copy_(len0)
        flush.zero_()
        B.ccgqa_set_phase_events(e)
        lay.decode_step(x_t, out)
        B.ccgqa_set_phase_events(None)
    torch.cuda.synchronize()
    if lay.error_bits():
        raise RuntimeError(f"device error bits {lay.error_bits()}")
    ms = [sum(e[i].elapsed_time(e[i + 1]) for e in evs) / steps for i in range(3)]
    step_ms = sum(e0.elapsed_time(e1) for e0, e1 in whole) / steps
    peaks, _ = load_peaks()
    return decode_numbers(w, ms[0], ms[1], ms[2], step_ms, peaks)


def measure_output_projection(w, steps, dev):
    """The output up-projection alone on the workload's B S rows of latent
    output (y [B S, E] = o W_o^T): 4 warm-up launches, then ``steps`` timed one
    by one with CUDA events, L2 flushed before each."""
    import torch
    from compressed_latent_grouped_b200.device import DeviceLayer
    from compressed_latent_grouped_b200.workloads import make_inputs, make_output_weights
    lay = DeviceLayer(w, make_inputs(w.with_(B=1, S=8), seed=0), device=dev)
    g = torch.Generator().manual_seed(0)
    o = torch.randn(w.B * w.S, w.Hq * w.d, generator=g).to(w.torch_dtype).to(dev)
    W_o = make_output_weights(w).to(dev)
    y = torch.empty(w.B * w.S, w.E, dtype=w.torch_dtype, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(4):
        lay.output_projection(o, W_o, y)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for a, b in evs:
        flush.zero_()
        a.record()
        lay.output_projection(o, W_o, y)
        b.record()
    torch.cuda.synchronize()
    if lay.error_bits():
        raise RuntimeError(f"device error bits {lay.error_bits()}")
    ms = sum(a.elapsed_time(b) for a, b in evs) / steps
    flop = 2.0 * w.B * w.S * w.E * w.Hq * w.d
    peaks, _ = load_peaks()
    return {"ms": ms, "tflops": flop / (ms / 1e3) / 1e12,
            "tensor_frac": flop / (ms / 1e3) / 1e12 / peaks["bf16_tflops"]}


def measure_backward(w, steps, dev):
    """The backward pass of one prefill workload (ccgqa_prefill_backward: the
    forward recompute, attention backward, pre-attention transposes, weight
    gradients and dx), timed with events around each call."""
    import torch
    from compressed_latent_grouped_b200.device import DeviceLayer
    from compressed_latent_grouped_b200.workloads import make_inputs
    inp = make_inputs(w, seed=0)
    lay = DeviceLayer(w, inp, device=dev)
    x = inp["x"].to(dev)
    dout = torch.randn(w.B, w.S, w.Hq * w.d, generator=torch.Generator().manual_seed(3)
                       ).to(w.torch_dtype).to(dev)
    for _ in range(2):
        lay.prefill_backward(x, dout)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for a, b in evs:
        a.record()
        lay.prefill_backward(x, dout)
        b.record()
    torch.cuda.synchronize()
    if lay.error_bits():
        raise RuntimeError(f"device error bits {lay.error_bits()}")
    ms = sum(a.elapsed_time(b) for a, b in evs) / steps
    # attention backward: 2 d FLOP per visible pair for each of QK^T (recomputed
    # twice), PV (recomputed), dO V^T (twice), dV, dK and dQ
    pairs = w.B * w.Hq * (w.S * w.S / 2 if w.causal else w.S * w.S)
    attn_flop = 2.0 * w.d * pairs * 9
    gemm_flop = 0 if w.packed_input else 2 * 2.0 * w.B * w.S * w.E * w.n_qkv
    peaks, _ = load_peaks()
    return {"backward_ms": ms, "tokens_per_s": w.B * w.S / (ms / 1e3),
            "flop": attn_flop + gemm_flop,
            "tflops": (attn_flop + gemm_flop) / (ms / 1e3) / 1e12,
            "tensor_frac": (attn_flop + gemm_flop) / (ms / 1e3) / 1e12 / peaks["bf16_tflops"]}


def run_workload_only(args, local):
    """--workload: time one named workload's kernels (profiling runs)."""
    import torch
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from compressed_latent_grouped_b200.workloads import WORKLOADS
    w = WORKLOADS[args.workload]
    if args.batch:
        w = w.with_(B=args.batch)
    if args.seq:
        w = w.with_(S=args.seq)
    if args.decode:
        w = w.with_(decode=True)
    if args.unfused:
        from compressed_latent_grouped_b200 import binding as B
        B.ccgqa_set_fused_projection(False)
    if args.output_projection:
        res = measure_output_projection(w, args.steps, dev)
    elif args.backward:
        res = measure_backward(w, args.steps, dev)
    elif w.decode:
        res = measure_decode_workload(w, args.steps, dev, page=args.paged)
    else:
        res = measure_prefill_workload(w, args.steps, dev)
    print(json.dumps({"workload": args.workload, "B": w.B, "S": w.S, **res}), flush=True)


# ----------------------------------------------------------------------- ours
def run_ours(args, world, rank, local):
    import torch
    from compressed_latent_grouped_b200 import binding as B
    from compressed_latent_grouped_b200.device import DeviceLayer, Graph
    from compressed_latent_grouped_b200.workloads import WORKLOADS, make_inputs

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wp, wd = WORKLOADS[PREFILL_WL], WORKLOADS[DECODE_WL]
    inp_p = make_inputs(wp, seed=rank)
    pf = DeviceLayer(wp, inp_p, device=dev, cap=wp.S)
    pf.alloc_cache()
    x = inp_p["x"].to(dev)
    out = torch.empty(wp.B, wp.S, wp.Hq * wp.d, dtype=wp.torch_dtype, device=dev)
    dc, inp_d, len0 = setup_decode(wd, dev, seed=1000 + rank)
    x_t = inp_d["x_t"].to(dev)
    out_t = torch.empty(wd.B, wd.Hq * wd.d, dtype=wd.torch_dtype, device=dev)
    lens = dc.cache_tensors["len"]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    # a created stream (graphs cannot record the legacy default stream), made
    # current so the flush, the length reset and the events go on it too
    stream = torch.cuda.Stream(dev)
    torch.cuda.set_stream(stream)

    def step():
        pf.prefill(x, out)
        dc.decode_step(x_t, out_t)

    def between_steps():
        # untimed: evict L2 and put the decode caches back at wd.S tokens
        flush.zero_()
        lens.copy_(len0)

    for _ in range(max(args.warmup, 3)):
        between_steps()
        step()
    torch.cuda.synchronize()
    if pf.error_bits() or dc.error_bits():
        raise RuntimeError(f"device error bits {pf.error_bits()} {dc.error_bits()}")

    K = args.steps
    mk = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    st_ev = [(mk(), mk()) for _ in range(K)]
    pf_ev = [[mk() for _ in range(4)] for _ in range(K)]
    dc_ev = [[mk() for _ in range(4)] for _ in range(K)]
    for e_ in [e_ for l_ in pf_ev + dc_ev for e_ in l_]:
        e_.record(stream)          # create the CUDA events outside the timed passes
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    # the step recorded once as a CUDA graph of library calls (ccgqa_graph_*):
    # each timed step is one graph launch, the serving loop's form
    graph = Graph(step, stream)
    for _ in range(3):
        between_steps()
        graph.launch()
    torch.cuda.synchronize()
    eager_ev = [(mk(), mk()) for _ in range(K)]
    dstep_ev = [(mk(), mk()) for _ in range(K)]
    with sampler:
        # pass 1, the step time: events only around whole steps.  An event
        # recorded between two kernels serialises them (about 3 us a record on
        # B200), so the per-kernel events live in pass 3.
        n0 = B.ccgqa_launch_count()
        for i in range(K):
            between_steps()
            st_ev[i][0].record(stream)
            graph.launch()
            st_ev[i][1].record(stream)
        torch.cuda.synchronize()
        launches = B.ccgqa_launch_count() - n0
        # pass 2, the same K steps as eager library calls (no graph)
        for i in range(K):
            between_steps()
            eager_ev[i][0].record(stream)
            step()
            eager_ev[i][1].record(stream)
        # pass 3, the same K steps with events between the kernels (phase times)
        for i in range(K):
            between_steps()
            B.ccgqa_set_phase_events(pf_ev[i])
            pf.prefill(x, out)
            B.ccgqa_set_phase_events(dc_ev[i])
            dc.decode_step(x_t, out_t)
            B.ccgqa_set_phase_events(None)
        # pass 4, the decode step alone with events only around it
        for i in range(K):
            between_steps()
            dstep_ev[i][0].record(stream)
            dc.decode_step(x_t, out_t)
            dstep_ev[i][1].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    if pf.error_bits() or dc.error_bits():
        raise RuntimeError(f"device error bits {pf.error_bits()} {dc.error_bits()}")

    step_ms = [a.elapsed_time(b) for a, b in st_ev]
    t_ms = max_over_ranks(sum(step_ms), world, dev)
    eager_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in eager_ev), world, dev) / K
    graph.close()
    phase = lambda evs, i, j: sum(e[i].elapsed_time(e[j]) for e in evs) / K  # noqa: E731
    proj_ms, pre_ms, attn_ms = phase(pf_ev, 0, 1), phase(pf_ev, 1, 2), phase(pf_ev, 2, 3)
    dproj_ms, dpre_ms, dattn_ms = phase(dc_ev, 0, 1), phase(dc_ev, 1, 2), phase(dc_ev, 2, 3)
    prefill_ms = phase(pf_ev, 0, 3)

    tokens_per_step = wp.B * wp.S + wd.B
    value = tokens_per_step * K * world / (t_ms / 1e3)
    attn_flop = attention_flops(wp.B, wp.S, wp.Hq, wp.d, wp.causal)
    proj_flop = 2.0 * wp.B * wp.S * wp.E * wp.n_qkv
    # pre-attention: q~|k~|v~ read once, q, k, v written once (bf16)
    pre_bytes = 2 * wp.B * wp.S * wp.n_qkv * 2
    peaks, peak_kind = load_peaks()
    achieved = attn_flop / (attn_ms / 1e3) / 1e12
    traffic = attn_traffic_per_launch()
    dstep_ms = sum(a.elapsed_time(b) for a, b in dstep_ev) / K
    dec = decode_numbers(wd, dproj_ms, dpre_ms, dattn_ms, dstep_ms, peaks)

    # end to end through the public API: pinned host buffers in, results out.
    # Three streams, as a serving loop would run it: step i+1's inputs are copied
    # in and step i-1's results copied out while step i computes; device inputs
    # and outputs are double-buffered, and events order each buffer's reuse.
    x_h = inp_p["x"].pin_memory()
    xt_h = inp_d["x_t"].pin_memory()
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    outt_h = torch.empty(out_t.shape, dtype=out_t.dtype).pin_memory()
    x_d = [torch.empty_like(x) for _ in range(2)]
    xt_d = [torch.empty_like(x_t) for _ in range(2)]
    o_d = [torch.empty_like(out) for _ in range(2)]
    ot_d = [torch.empty_like(out_t) for _ in range(2)]
    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_ready = [ev() for _ in range(2)]
    in_free = [ev() for _ in range(2)]
    out_ready = [ev() for _ in range(2)]
    out_free = [ev() for _ in range(2)]
    for e_ in in_free + out_free:
        e_.record(stream)
    torch.cuda.synchronize()

    def e2e_steps(n):
        for i in range(n):
            k = i & 1
            s_in.wait_event(in_free[k])
            with torch.cuda.stream(s_in):
                x_d[k].copy_(x_h, non_blocking=True)
                xt_d[k].copy_(xt_h, non_blocking=True)
            in_ready[k].record(s_in)
            s_cmp.wait_event(in_ready[k])
            s_cmp.wait_event(out_free[k])
            with torch.cuda.stream(s_cmp):
                lens.copy_(len0)       # device-to-device, 256 bytes
            graphs[k].launch()
            in_free[k].record(s_cmp)
            out_ready[k].record(s_cmp)
            s_out.wait_event(out_ready[k])
            with torch.cuda.stream(s_out):
                out_h.copy_(o_d[k], non_blocking=True)
                outt_h.copy_(ot_d[k], non_blocking=True)
            out_free[k].record(s_out)

    graphs = [Graph(lambda k=k: (pf.prefill(x_d[k], o_d[k], stream=s_cmp),
                                 dc.decode_step(xt_d[k], ot_d[k], stream=s_cmp)), s_cmp)
              for k in range(2)]
    e2e_steps(2)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = mk(), mk()
    e0.record(s_in)
    e2e_steps(K)
    s_out.wait_stream(s_cmp)
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    for g_ in graphs:
        g_.close()
    barrier(world)
    if pf.error_bits() or dc.error_bits():
        raise RuntimeError(f"device error bits {pf.error_bits()} {dc.error_bits()}")
    h2d = x.numel() * x.element_size() + x_t.numel() * x_t.element_size()
    d2h = out.numel() * out.element_size() + out_t.numel() * out_t.element_size()
    del x_d, o_d, x_h, out_h
    torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_headline(wp, make_inputs(wp, seed=0), wd, make_inputs(wd, seed=1000))

    by_workload, oproj = None, None
    if rank == 0 and not args.no_extra:
        # the output up-projection of the prefill's rows (outside the step)
        oproj = measure_output_projection(wp, 20, dev)
        oproj["note"] = "not part of the step: y = out W_o^T, timed on its own"
        by_workload = {}
        for name in ("bf16_prefill_b4_s4096", "bf16_gqa_b2_s8192"):
            by_workload[name] = measure_prefill_workload(WORKLOADS[name], 20, dev)
        by_workload["bf16_prefill_b4_s4096"]["decode_b4_l4096"] = measure_decode_workload(
            WORKLOADS["bf16_prefill_b4_s4096"].with_(decode=True), 20, dev)
        # the headline decode step against a paged cache (pages of 64 and 16
        # tokens, scattered over the pool by a seeded block table)
        for page in (64, 16):
            by_workload[f"{DECODE_WL}_paged{page}"] = measure_decode_workload(wd, 20, dev,
                                                                              page=page)
        torch.cuda.empty_cache()

    if rank != 0:
        return
    timing = "CUDA events around each launch, third pass of the K steps"
    # The kernel is timed inside the step loop (K steps back to back, seconds of
    # load under the 1 kW cap; the clock record shows sw_power_cap): its peak is
    # the sustained cuBLAS figure, with the burst fraction beside it.
    sustained = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    roof_tensor = {"bound": "tensor", "kernel": f"attn_prefill_tc (d = {wp.d})",
                   "achieved": achieved, "peak": sustained, "unit": "TFLOP/s",
                   "frac": achieved / sustained, "traffic": traffic,
                   "peak_kind": f"{peak_kind} bf16 dense sustained (the kernel is timed inside "
                                f"the step loop)",
                   "frac_of_burst": achieved / peaks["bf16_tflops"],
                   "burst_peak": peaks["bf16_tflops"],
                   "flop_per_launch": attn_flop, "ms_per_launch": attn_ms, "timing": timing}
    roof_exp = {**exp_roofline(wp, attn_ms, peaks), "kernel": "attn_prefill_tc",
                "ms_per_launch": attn_ms, "timing": timing}
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": max(args.warmup, 3), "ms_per_step": t_ms / K,
        "eager_ms_per_step": eager_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded PCG64 normals, weights N(0, 1/fan_in))",
        "config": {"workload": WORKLOAD,
                   "prefill": {"B": wp.B, "S": wp.S, "E": wp.E, "C": wp.C, "Hq": wp.Hq,
                               "Hkv": wp.Hkv, "d": wp.d, "conv_width": wp.conv_width,
                               "rope_base": wp.rope_base},
                   "decode": {"B": wd.B, "L": wd.S, "E": wd.E, "C": wd.C, "Hq": wd.Hq,
                              "Hkv": wd.Hkv, "d": wd.d},
                   "parallelism": f"replicas x{world} (independent sequences per GPU)",
                   "l2": "flushed (256 MiB write) before every timed step; inputs larger "
                         "than L2 as well",
                   "launch": "each step one CUDA graph launch of the recorded library calls "
                             "(ccgqa_graph_launch); eager_ms_per_step: the same calls made "
                             "one by one"},
        "roofline": roof_tensor,
        "roofline_exp_unit": roof_exp,
        "kernels": {
            "proj_gemm": {"ms": proj_ms, "tflops": proj_flop / (proj_ms / 1e3) / 1e12,
                          "tensor_frac": proj_flop / (proj_ms / 1e3) / 1e12 / peaks["bf16_tflops"]},
            "pre_attn": {"ms": pre_ms, "bytes": pre_bytes,
                         "gbs": pre_bytes / (pre_ms / 1e3) / 1e9,
                         "hbm_frac": pre_bytes / (pre_ms / 1e3) / 1e9 / peaks["hbm_gbs"]},
            "attn_prefill_tc": {"ms": attn_ms, "tflops": achieved,
                                "tensor_frac": achieved / peaks["bf16_tflops"]},
            "decode_attn": {"ms": dattn_ms, "gbs": dec["attn_gbs"],
                            "hbm_frac": dec["attn_hbm_frac"]},
            "output_projection": oproj,
        },
        "phases_ms": {"proj_gemm": proj_ms, "pre_attn": pre_ms, "attn_prefill_tc": attn_ms,
                      "prefill_total": prefill_ms, "decode_proj": dproj_ms,
                      "decode_pre": dpre_ms, "decode_attn": dattn_ms},
        "prefill": {"tokens_per_s": wp.B * wp.S / (prefill_ms / 1e3) * world,
                    "tflops_attn_plus_proj": (attn_flop + proj_flop) / (prefill_ms / 1e3) / 1e12,
                    "tensor_frac_attn_plus_proj": (attn_flop + proj_flop) / (prefill_ms / 1e3)
                    / 1e12 / peaks["bf16_tflops"]},
        "decode": dec,
        "clocks": sampler.summary(),
        "e2e": {"value": tokens_per_step * K * world / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "cpu_baseline": cpu,
        "by_workload": by_workload,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-seconds", type=float, default=150.0,
                    help="--impl reference: host-time budget of the whole run")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other workloads' kernel measurements")
    ap.add_argument("--workload", default=None,
                    help="time only this workload's kernels (profiling)")
    ap.add_argument("--batch", type=int, default=0, help="with --workload: override B")
    ap.add_argument("--seq", type=int, default=0, help="with --workload: override S (or L)")
    ap.add_argument("--decode", action="store_true",
                    help="with --workload: time a decode step against a cache of S tokens")
    ap.add_argument("--unfused", action="store_true",
                    help="with --workload: run the projection and pre-attention as separate kernels")
    ap.add_argument("--paged", type=int, default=0,
                    help="with --workload and a decode: a paged cache of this many tokens per page")
    ap.add_argument("--output-projection", action="store_true",
                    help="with --workload: time the output up-projection of its B S rows")
    ap.add_argument("--backward", action="store_true",
                    help="with --workload: time the backward pass of its prefill")
    args = ap.parse_args()
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        elif args.workload:
            run_workload_only(args, local)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
