"""Host-side logic of bench.py on the CPU: the reference (CPU oracle) arm's JSON line, and the
multi-rank plumbing -- per-rank batches and max-over-ranks timing -- with world_size 2 over gloo."""
from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run_bench(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                          env=env, timeout=600, cwd=ROOT)


def test_reference_arm_prints_one_line():
    r = _run_bench(["--impl", "reference", "--steps", "2", "--warmup", "1", "--workload", "sweep_N2_B512_D128"])
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == "GB/s" and line["value"] > 0
    assert line["higher_is_better"] is True
    assert line["config"]["workload"] == "sweep_N2_B512_D128"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] == bench.host_cores() and cb["value"] == line["value"]
    assert cb["single_thread"]["cores"] == 1 and cb["single_thread"]["value"] > 0
    assert f"{bench.cpu_sample_tokens(bench_workload('sweep_N2_B512_D128'))}-token" in cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def bench_workload(name):
    from decode_context_attention_dcp_b200 import workloads as wl
    return wl.by_name(name)


def test_cpu_baseline_all_cores_and_one():
    """The CPU baseline times the same sample on all host cores and on one, and states both."""
    w = bench_workload("sweep_N2_B512_D128")
    cb = bench.cpu_baseline(w, budget_s=1.0)
    assert cb["kind"] == "oracle" and cb["cores"] == bench.host_cores() and cb["value"] > 0
    assert cb["single_thread"]["cores"] == 1 and cb["single_thread"]["value"] > 0
    assert cb["host_cores"] == os.cpu_count()
    assert f"{bench.cpu_sample_tokens(w)}-token" in cb["sample"]


def test_oracle_step_on_threads_moves_the_same_bytes():
    w = bench_workload("tiny")
    t1, b1 = bench.oracle_step_sample(w, 4, 1)
    t2, b2 = bench.oracle_step_sample(w, 4, 3)
    assert b1 == b2 == w.pack_bytes() + w.combine_bytes()


def test_reference_arm_other_ranks_exit_silently():
    r = _run_bench(["--impl", "reference", "--steps", "1", "--warmup", "0"], {"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_rank_seeds_are_distinct():
    seeds = {bench.rank_seed(100, r) for r in range(8)}
    assert len(seeds) == 8


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # per-rank inputs differ (weak scaling: each rank its own batch of the same shape)
        from decode_context_attention_dcp_b200 import workloads as wl
        w = wl.TINY.with_(seed=bench.rank_seed(wl.TINY.seed, rank))
        cp_out, _ = wl.pack_inputs(w)
        gathered = [torch.zeros_like(cp_out.float()) for _ in range(world)]
        dist.all_gather(gathered, cp_out.float())
        distinct = not torch.equal(gathered[0], gathered[1])
        bench.barrier()
        m = bench.max_over_ranks(float(rank + 1) * 1.5)
        out[rank] = (m, distinct, tuple(cp_out.shape))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    assert out[0][0] == 3.0 and out[1][0] == 3.0
    assert out[0][1] and out[1][1]
    assert out[0][2] == out[1][2] == (4, 16, 128)


def test_kernel_digest_tracks_code_not_comments(tmp_path, monkeypatch):
    """The digest that gates reported DRAM traffic changes with the kernel code and only with
    it: comments and whitespace do not count, a changed token does."""
    import shutil
    for sub in ("decode_context_attention_dcp_b200/csrc", "include"):
        shutil.copytree(os.path.join(ROOT, sub), tmp_path / sub)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    base = bench.kernel_digest()
    k = tmp_path / "decode_context_attention_dcp_b200/csrc/dcp_kernels.cuh"
    text = k.read_text()
    k.write_text("// an added comment\n/* and a block\n   comment */\n" + text.replace("\n", "\n\n", 5))
    assert bench.kernel_digest() == base
    k.write_text(text.replace("kPackStages = 3", "kPackStages = 4", 1))
    assert bench.kernel_digest() != base


def test_traffic_is_reported_only_for_the_current_code(tmp_path, monkeypatch):
    """load_traffic returns the committed counters while their digest matches the sources and
    None once the code differs."""
    import shutil
    for sub in ("decode_context_attention_dcp_b200/csrc", "include", "profiles"):
        shutil.copytree(os.path.join(ROOT, sub), tmp_path / sub)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    have = bench.load_traffic("dcp_pack", "sweep_N16_B16384_D512")
    k = tmp_path / "decode_context_attention_dcp_b200/csrc/dcp_kernels.cuh"
    k.write_text(k.read_text().replace("kPackStages = 3", "kPackStages = 4", 1))
    assert bench.load_traffic("dcp_pack", "sweep_N16_B16384_D512") is None
    assert have is None or have > 0


def test_workload_inputs_are_reproducible():
    """The same workload draws the same bits every time (the seeded generators are the only
    source of the inputs both sides see)."""
    from decode_context_attention_dcp_b200 import workloads as wl
    w = wl.CombineWorkload("repro", N=3, B=40, Hr=4, D=64, p_neginf=0.1, p_nan=0.05, empty_every=7, seed=11)
    a, b = wl.split_inputs(w), wl.split_inputs(w)
    assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16))
    assert torch.equal(a[1].view(torch.int32), b[1].view(torch.int32))
    c, d = wl.pack_inputs(w), wl.pack_inputs(w)
    assert torch.equal(c[0].view(torch.int16), d[0].view(torch.int16))
    assert torch.equal(c[1].view(torch.int32), d[1].view(torch.int32))
    s1, q1 = wl.decode_batch(wl.DecodeBatch(B=50, max_q=3, pad=4, seed=3))
    s2, q2 = wl.decode_batch(wl.DecodeBatch(B=50, max_q=3, pad=4, seed=3))
    assert torch.equal(s1, s2) and torch.equal(q1, q2) and int(q1[-1]) == 46 and int(q1[0]) == 0
    assert bool((q1[1:] > q1[:-1]).all()) and bool(((q1[1:] - q1[:-1]) <= 3).all())
