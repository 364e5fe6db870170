"""The benchmark's multi-process path on CPU: two ranks over gloo, launched the
way the multi-GPU runs are (torch.distributed.run, one process per rank,
127.0.0.1 rendezvous).  Covers the rank setup, the max-over-ranks timing
reduction, the barrier, per-rank input shards (independent sequences, weak
scaling) and the reference arm running on rank 0 alone."""
import json
import os
import socket
import subprocess
import sys
import textwrap

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _torchrun(args, timeout=240):
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port())] + args
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="2")
    return subprocess.run(cmd, capture_output=True, text=True, timeout=timeout, cwd=ROOT, env=env)


def _json_lines(text):
    out = []
    for line in text.splitlines():
        line = line.strip()
        if line.startswith("{"):
            out.append(json.loads(line))
    return out


def test_rank_helpers_two_ranks_gloo(tmp_path):
    script = tmp_path / "ranks.py"
    script.write_text(textwrap.dedent(f"""
        import json, sys
        sys.path.insert(0, {ROOT!r})
        import torch
        import torch.distributed as dist
        import bench
        from compressed_latent_grouped_b200.workloads import WORKLOADS, make_inputs
        world, rank, local = bench.dist_setup(2)
        assert dist.get_backend() == "gloo"
        # each rank times its own work; the job time is the slowest rank's
        t = bench.max_over_ranks(1.5 * (rank + 1), world, torch.device("cpu"))
        bench.barrier(world)
        # shards: rank r draws its own batch of sequences (seed = r)
        x = make_inputs(WORKLOADS["f32_s128"], seed=rank)["x"]
        mine = torch.tensor([float(x.double().sum())])
        every = [torch.zeros(1) for _ in range(world)]
        dist.all_gather(every, mine)
        # one file per rank: the ranks' stdout lines may interleave
        with open(sys.argv[1] + f"/rank{{rank}}.json", "w") as f:
            json.dump({{"rank": rank, "world": world, "local": local, "t": t,
                       "sums": [float(v) for v in every]}}, f)
        dist.destroy_process_group()
    """))
    r = _torchrun([str(script), str(tmp_path)])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads((tmp_path / f"rank{k}.json").read_text()) for k in range(2)]
    assert sorted(d["rank"] for d in lines) == [0, 1]
    for d in lines:
        assert d["world"] == 2 and d["local"] == d["rank"]
        assert d["t"] == 3.0                      # max over ranks, on every rank
        assert d["sums"][0] != d["sums"][1]       # the two shards are different sequences
    assert lines[0]["sums"] == lines[1]["sums"]


def test_reference_arm_runs_on_rank_zero_only():
    r = _torchrun(["bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1",
                   "--warmup", "0", "--ref-seconds", "2"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1, r.stdout
    d = lines[0]
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["unit"] == "tokens/s"
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert "float64 prefill of the first" in d["config"]["sample"]
