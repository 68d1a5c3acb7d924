#!/usr/bin/env python3
"""Bench of the DCP combine hot path on B200: one step = dcp_pack + dcp_unpack_combine.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole path over one batch: the pack of one rank's partial
attention output cp_attn_out [B, N*Hr, D] (+ LSE [B, N*Hr]) into the packed buffer
[N, B, Hr, D+2], then the fused unpack+combine of that buffer (every shard taken from it)
into [B, Hr, D].  Default workload: the largest bandwidth-sweep point (N=16, B=16384,
Hr=16, D=512, bf16).  Inputs are resident in HBM before timing and larger than L2.

Metric: effective HBM GB/s = algorithmic bytes / device time (CUDA events on the launching
stream), max over ranks; also (token*head)/s and the fraction of the measured HBM peak.
With N > 1 (torchrun, one process per GPU) every rank combines its own batch: weak scaling,
no data-path collective.  Rank 0 prints one JSON line.

The line also carries: per-kernel times and shares; "roofline" (the dominant kernel's
achieved GB/s against the measured copy peak, with ncu DRAM traffic when the committed
summary was taken on the current kernel code); "e2e" (the same step through the public API
with pinned host inputs copied in and the result copied out every step); "cpu_baseline"
(the oracle on a bounded token sample, on all host cores and on one, N = 1 only); "gpu_launches"; and the SM
clocks sampled during the timed region.

--impl reference times the fp64 CPU oracle on all host cores (token slices, one thread each) on
the same bounded sample of the workload as the CPU baseline (rank 0 only), for the same metric.  --sweep times every entry point on every
workload (median of launches with L2 flushed before each) and prints a markdown table.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "combine effective HBM GB/s and fraction of B200 peak; (token·head)/s"
DEFAULT_WORKLOAD = "sweep_N16_B16384_D512"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--e2e-chunks", type=int, default=8, help="token chunks pipelined over three streams")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--sweep", action="store_true",
                    help="instead of the JSON line: per-kernel GB/s on every workload, as a markdown table")
    ap.add_argument("--sweep-reps", type=int, default=50)
    ap.add_argument("--points", default="",
                    help="--sweep: comma-separated workload names to run (default: every workload)")
    ap.add_argument("--kernels", default="",
                    help="--sweep: comma-separated kernel rows to run, by exact name (default: all)")
    return ap.parse_args(argv)


# ---- multi-process plumbing (testable on CPU with gloo) -----------------------------------
def dist_env() -> tuple[int, int, int]:
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def rank_seed(base_seed: int, rank: int) -> int:
    """Weak scaling: every rank combines its own batch of the same shape, drawn with its own seed."""
    return base_seed + 7919 * rank


def max_over_ranks(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None) -> None:
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---- measurement side data -----------------------------------------------------------------
def kernel_digest() -> str:
    """Hash of the kernel sources' code (comments and whitespace removed): ncu counters are
    reported only for the code they were taken on."""
    h = hashlib.sha256()
    for sub in ("decode_context_attention_dcp_b200/csrc", "include"):
        d = os.path.join(ROOT, sub)
        for name in sorted(os.listdir(d)):
            with open(os.path.join(d, name), encoding="utf-8") as fh:
                text = fh.read()
            text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
            text = re.sub(r"//[^\n]*", " ", text)
            h.update(name.encode() + b"\0" + " ".join(text.split()).encode())
    return h.hexdigest()[:16]


def load_peak() -> tuple[float, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            v = float(json.load(fh)["hbm_gbs"])
        return v, "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def load_traffic(kernel: str, workload: str) -> float | None:
    """DRAM bytes per launch (read + write) from the committed ncu summary, if it was taken on the
    current kernel sources.  Table rows: | kernel | workload | digest | dram_read | dram_write | ..."""
    path = os.path.join(ROOT, "profiles", "dram_traffic_pack_unpack_combine_sweep_N16_B16384_D512.md")
    if not os.path.exists(path):
        return None
    digest = kernel_digest()
    for line in open(path):
        cells = [c.strip() for c in line.strip().strip("|").split("|")]
        if len(cells) >= 5 and cells[0] == kernel and cells[1] == workload and cells[2] == digest:
            try:
                return float(cells[3]) + float(cells[4])
            except ValueError:
                return None
    return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the GPU works."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        cmd = ["nvidia-smi", f"--query-gpu=timestamp,{self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            c = [x.strip() for x in line.split(",")]
            if len(c) < 9:
                continue
            try:
                rows.append((float(c[1]), float(c[2]), c[4:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        max_mhz = max(r[1] for r in rows)
        loaded = [r for r in rows if r[0] >= 0.5 * max_mhz] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[2][1:]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max_mhz, "reasons": reasons,
                "samples": len(rows)}


# ---- the CPU oracle (reference arm and CPU baseline) -----------------------------------------
def host_cores() -> int:
    """Host cores this process may run on."""
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)


def cpu_sample_tokens(w) -> int:
    """Tokens of the oracle's sample: one eighth of the batch, at most 2048 (both the CPU baseline
    and the reference arm use this sample)."""
    return max(1, min(2048, w.B // 8 or w.B))


_SAMPLES: dict = {}


def oracle_sample(w, tokens: int):
    """The sample's inputs as the oracle reads them: a ``tokens``-token batch drawn with the
    workload's recipe and seed (cp_attn_out [tokens, H, D] raw elements, cp_attn_lse fp32)."""
    key = (w, tokens)
    if key not in _SAMPLES:
        import numpy as np
        import torch

        from decode_context_attention_dcp_b200 import workloads as wl

        cp_out, cp_lse = wl.pack_inputs(w.with_(B=tokens))
        ro = cp_out.view(torch.int16).numpy().view(np.uint16) if cp_out.element_size() == 2 else cp_out.numpy()
        _SAMPLES.clear()
        _SAMPLES[key] = (ro, cp_lse.numpy())
    return _SAMPLES[key]


def oracle_step_sample(w, tokens: int, threads: int = 1):
    """One oracle step (pack, then unpack+combine, plain fp64 C) over the sample.  With
    ``threads`` > 1 the tokens are split into that many slices and each host thread runs both
    steps of the unchanged oracle on its own slice (ctypes releases the GIL).  Returns
    (seconds, algorithmic bytes)."""
    import concurrent.futures

    import oracle

    ro, rl = oracle_sample(w, tokens)
    o = oracle.load()
    code = {"bf16": oracle.BF16, "fp16": oracle.FP16, "fp32": oracle.FP32}[w.dtype]

    def run(t0: int, t1: int) -> None:
        send = o.pack(ro[t0:t1], rl[t0:t1], w.N, code)
        o.unpack_combine(send, code, w.D, return_lse=w.return_lse, is_lse_base_on_e=w.is_lse_base_on_e)

    threads = max(1, min(threads, tokens))
    step = (tokens + threads - 1) // threads
    bounds = [(t, min(tokens, t + step)) for t in range(0, tokens, step)]
    t0 = time.perf_counter()
    if len(bounds) == 1:
        run(*bounds[0])
    else:
        with concurrent.futures.ThreadPoolExecutor(max_workers=len(bounds)) as ex:
            for f in [ex.submit(run, a, b) for a, b in bounds]:
                f.result()
    dt = time.perf_counter() - t0
    ws = w.with_(B=tokens)
    return dt, ws.pack_bytes() + ws.combine_bytes()


def time_oracle(w, tokens: int, threads: int, budget_s: float, max_reps: int) -> tuple[float, int, float]:
    """(GB/s, repetitions, seconds) of oracle steps over the sample until the budget is spent."""
    total_t, total_b, reps = 0.0, 0, 0
    while reps < 1 or (total_t < budget_s and reps < max_reps):
        dt, nb = oracle_step_sample(w, tokens, threads)
        total_t += dt
        total_b += nb
        reps += 1
    return total_b / total_t / 1e9, reps, total_t


def sample_text(w, tokens: int) -> str:
    return (f"pack + unpack_combine of a {tokens}-token batch drawn with the workload's recipe "
            f"({tokens} of {w.B} tokens, all {w.N} shards, Hr={w.Hr}, D={w.D}); plain fp64 C")


def cpu_baseline(w, budget_s: float = 12.0) -> dict:
    """The oracle on the host's cores (all of them, token slices), and on one core, over the
    same sample."""
    tokens = cpu_sample_tokens(w)
    cores = host_cores()
    oracle_step_sample(w, tokens, cores)  # inputs drawn, pages touched
    v_all, r_all, t_all = time_oracle(w, tokens, cores, budget_s / 2, 32)
    v_one, r_one, t_one = time_oracle(w, tokens, 1, budget_s / 2, 8)
    return {"value": v_all, "unit": "GB/s", "cores": cores, "kind": "oracle", "host_cores": os.cpu_count(),
            "sample": f"{sample_text(w, tokens)}; {r_all} steps on {cores} threads ({t_all:.1f} s)",
            "single_thread": {"value": v_one, "unit": "GB/s", "cores": 1,
                              "sample": f"the same sample, {r_one} steps on one thread ({t_one:.1f} s)"}}


def run_reference(args) -> int:
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from decode_context_attention_dcp_b200 import workloads as wl

    w = wl.by_name(args.workload)
    tokens = cpu_sample_tokens(w)
    cores = host_cores()
    for _ in range(args.warmup):
        oracle_step_sample(w, tokens, cores)
    secs, nbytes = 0.0, 0
    for _ in range(args.steps):
        dt, nb = oracle_step_sample(w, tokens, cores)
        secs += dt
        nbytes += nb
    gbs = nbytes / secs / 1e9
    v_one, r_one, t_one = time_oracle(w, tokens, 1, 4.0, 4)
    sample = f"each step: {sample_text(w, tokens)}, token slices on {cores} threads"
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample,
                         "host_cores": os.cpu_count(),
                         "single_thread": {"value": v_one, "unit": "GB/s", "cores": 1,
                                           "sample": f"the same sample, {r_one} steps on one thread ({t_one:.1f} s)"}},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w) -> dict:
    return {"workload": w.name, "step": "dcp_pack + dcp_unpack_combine", "shards": w.N, "tokens": w.B,
            "heads_in": w.H, "heads_out": w.Hr, "head_dim": w.D, "io_dtype": w.dtype,
            "is_lse_base_on_e": w.is_lse_base_on_e, "return_lse": w.return_lse,
            "lse": f"U[{w.lse_lo},{w.lse_hi}], {w.p_neginf:.0%} -inf",
            "l2": "inputs larger than L2 (no flush between steps)"}


# ---- per-kernel sweep ------------------------------------------------------------------------
def run_sweep(args) -> int:
    """Median device time of each entry point on every workload (L2 flushed before each timed
    launch); prints a markdown table.  --points and --kernels restrict the table; only the
    buffers the selected rows use are allocated."""
    import torch

    import decode_context_attention_dcp_b200 as dcp
    from decode_context_attention_dcp_b200 import workloads as wl

    torch.cuda.set_device(0)
    peak, peak_src = load_peak()
    # L2 is emptied before each timed launch by READING 512 MB (4x L2): the lines it leaves are
    # clean, so nothing is written back to DRAM during the timed launch (a write-flush leaves up
    # to an L2's worth of dirty lines whose write-back the timed launch would pay for)
    flush = torch.zeros(128 << 20, dtype=torch.float32, device="cuda")
    points = [wl.TINY, wl.GQA, wl.MLA, wl.ROUNDTRIP, *wl.sweep()]
    if args.points:
        points = [wl.by_name(n) for n in args.points.split(",")]
    wanted = [k for k in args.kernels.split(",") if k]
    S = 4  # KV splits of the producer in the fused-pack rows
    print(f"| workload | N | B | Hr | D | dtype | kernel | bytes | us | GB/s | frac of {peak:.0f} ({peak_src}) |")
    print("|---|---|---|---|---|---|---|---|---|---|---|")
    for w in points:
        big = w.B >= 4096 or w is wl.MLA
        names = ["dcp_lse_combine", "dcp_unpack_combine", "dcp_pack"]
        if big:
            names += ["dcp_lse_combine_strided[head-major]", "dcp_lse_combine_varlen", f"dcp_combine_pack[S={S}]",
                      f"dcp_lse_combine+dcp_pack[S={S}]"]
        names = [n for n in names if not wanted or n in wanted]
        if not names:
            continue
        buf: dict = {}

        def get(key):
            """The point's buffers, made on first use."""
            if key in buf:
                return buf[key]
            if key in ("out", "lse"):
                outputs, lses = wl.split_inputs(w)
                buf["out"], buf["lse"] = outputs.cuda(), lses.cuda()
            elif key == "recv":
                d_out, d_lse = get("out"), get("lse")
                slot = d_lse.unsqueeze(-1).view(d_out.dtype) if w.elem_bytes == 2 else d_lse.unsqueeze(-1)
                buf[key] = torch.cat([d_out, slot], dim=-1)
            elif key == "cp":
                buf[key] = (get("out").permute(1, 0, 2, 3).reshape(w.B, w.H, w.D).contiguous(),
                            get("lse").permute(1, 0, 2).reshape(w.B, w.H).contiguous())
            elif key == "res":
                buf[key] = (torch.empty((w.B, w.Hr, w.D), dtype=wl.torch_dtype(w.dtype), device="cuda"),
                            torch.empty((w.B, w.Hr), dtype=torch.float32, device="cuda"))
            elif key == "send":
                buf[key] = torch.empty((w.N, w.B, w.Hr, w.W), dtype=wl.torch_dtype(w.dtype), device="cuda")
            elif key == "hm":
                # the same shards received head-scattered, [N, Hr, B, D] (dcp_lse_combine_strided)
                buf[key] = (get("out").permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3),
                            get("lse").permute(0, 2, 1).contiguous().permute(0, 2, 1))
            elif key == "varlen":
                # a decode batch in which about 30% of the requests are too short to reach every
                # shard (dcp_lse_combine_varlen reads only the shards that hold KV)
                seq_lens, qsl = wl.decode_batch(wl.DecodeBatch(B=w.B, p_short=0.3, short_max=w.N, seed=w.seed))
                req_of = torch.repeat_interleave(torch.arange(len(seq_lens)), qsl[1:] - qsl[:-1])
                held = torch.clamp(seq_lens.long(), 0, w.N)  # token interleave: min(N, seq) shards hold KV
                buf[key] = (seq_lens.cuda(), qsl.cuda(), int(held[req_of].sum()), len(seq_lens))
            elif key == "parts":
                # a producer with S KV splits per rank (its partials drawn on the device)
                gen = torch.Generator(device="cuda").manual_seed(w.seed)
                dt = wl.torch_dtype(w.dtype)
                buf[key] = (torch.randn((S, w.B, w.H, w.D), generator=gen, device="cuda").to(dt),
                            torch.rand((S, w.B, w.H), generator=gen, device="cuda") * 20.0)
            elif key == "merged":
                buf[key] = (torch.empty((w.B, w.H, w.D), dtype=wl.torch_dtype(w.dtype), device="cuda"),
                            torch.empty((w.B, w.H), dtype=torch.float32, device="cuda"))
            return buf[key]

        row = w.D * w.elem_bytes + 4
        fused_bytes = w.B * w.H * (S * row + row)

        def make(name):
            """(algorithmic bytes, launch) of one kernel row."""
            kw = dict(is_lse_base_on_e=w.is_lse_base_on_e, return_lse=w.return_lse)
            if name == "dcp_lse_combine":
                d_out, d_lse, (res, gl) = get("out"), get("lse"), get("res")
                return w.combine_bytes(), lambda: dcp.dcp_lse_combine(d_out, d_lse, res, gl, **kw)
            if name == "dcp_unpack_combine":
                recv, (res, gl) = get("recv"), get("res")
                return w.combine_bytes(), lambda: dcp.dcp_unpack_combine(recv, res, gl, **kw)
            if name == "dcp_pack":
                (cp_out, cp_lse), send = get("cp"), get("send")
                return w.pack_bytes(), lambda: dcp.dcp_pack(cp_out, cp_lse, send, w.N)
            if name.startswith("dcp_lse_combine_strided"):
                (hm_out, hm_lse), (res, gl) = get("hm"), get("res")
                return w.combine_bytes(), lambda: dcp.dcp_lse_combine(hm_out, hm_lse, res, gl, **kw)
            if name == "dcp_lse_combine_varlen":
                d_out, d_lse, (res, gl) = get("out"), get("lse"), get("res")
                d_seq, d_qsl, shards_read, reqs = get("varlen")
                return (w.varlen_combine_bytes(shards_read, reqs),
                        lambda: dcp.dcp_lse_combine_varlen(d_out, d_lse, res, d_seq, d_qsl, gl, **kw))
            (parts, part_lse), send = get("parts"), get("send")
            if name.startswith("dcp_combine_pack"):
                return fused_bytes, lambda: dcp.dcp_combine_pack(parts, part_lse, send, w.N)
            merged, merged_lse = get("merged")

            def two_step():
                dcp.dcp_lse_combine(parts, part_lse, merged, merged_lse, return_lse=True)
                dcp.dcp_pack(merged, merged_lse, send, w.N)
            return fused_bytes + 2 * w.B * w.H * row, two_step

        for name in names:
            nbytes, fn = make(name)
            for _ in range(3):
                fn()
            times = []
            for _ in range(args.sweep_reps):
                # the flush empties L2 and keeps the GPU busy while the host enqueues the timed
                # launch, so host-side call overhead never lands between the two events
                flush.sum()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                fn()
                b.record()
                torch.cuda.synchronize()
                times.append(a.elapsed_time(b))
            t = statistics.median(times)
            gbs = nbytes / (t * 1e-3) / 1e9
            print(f"| {w.name} | {w.N} | {w.B} | {w.Hr} | {w.D} | {w.dtype} | {name} | {nbytes} | {t * 1e3:.1f} | "
                  f"{gbs:.0f} | {gbs / peak:.3f} |", flush=True)
        buf.clear()
        torch.cuda.empty_cache()
    return 0


# ---- our arm ---------------------------------------------------------------------------------
def run_ours(args) -> int:
    import torch
    import torch.distributed as dist

    import decode_context_attention_dcp_b200 as dcp
    from decode_context_attention_dcp_b200 import workloads as wl

    rank, world, local_rank = dist_env()
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)
    lib = dcp.library()

    w = wl.by_name(args.workload)
    wr = w.with_(seed=rank_seed(w.seed, rank))
    cp_out_h, cp_lse_h = wl.pack_inputs(wr, pin_memory=True)
    cp_out = cp_out_h.to(device)
    cp_lse = cp_lse_h.to(device)
    P = dcp.dcp_lse_pack_dim(cp_out.dtype)
    send = torch.empty((w.N, w.B, w.Hr, w.D + P), dtype=cp_out.dtype, device=device)
    result = torch.empty((w.B, w.Hr, w.D), dtype=cp_out.dtype, device=device)
    glse = torch.empty((w.B, w.Hr), dtype=torch.float32, device=device) if w.return_lse else None
    stream = torch.cuda.Stream(device)
    sh = stream.cuda_stream
    code = dcp.DTYPE_CODES[cp_out.dtype]
    glse_ptr = glse.data_ptr() if glse is not None else None

    def pack(src, lse):
        st = lib.dcp_pack(src.data_ptr(), lse.data_ptr(), send.data_ptr(), w.B, w.H, w.D, w.N, code,
                          src.stride(0), src.stride(1), lse.stride(0), sh)
        if st:
            raise dcp.DCPError(st, dcp.dcp_last_error())

    def combine():
        st = lib.dcp_unpack_combine(send.data_ptr(), result.data_ptr(), glse_ptr, w.N, w.B, w.Hr, w.D,
                                    send.stride(0), code, int(w.is_lse_base_on_e), int(w.return_lse), sh)
        if st:
            raise dcp.DCPError(st, dcp.dcp_last_error())

    K, W = args.steps, args.warmup
    torch.cuda.synchronize(device)
    clocks = None
    sampler = None
    if not args.no_clocks:
        props = torch.cuda.get_device_properties(device)
        pci = (f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
               if hasattr(props, "pci_bus_id") else None)
        sampler = ClockSampler(pci)
        sampler.start()
    with torch.cuda.stream(stream):
        for _ in range(W):
            pack(cp_out, cp_lse)
            combine()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3 * K + 1)]
        stream.synchronize()
        barrier(device)
        torch.cuda.synchronize(device)
        ev[0].record(stream)
        for k in range(K):
            pack(cp_out, cp_lse)
            ev[3 * k + 1].record(stream)
            combine()
            ev[3 * k + 2].record(stream)
            if k + 1 < K:
                ev[3 * k + 3].record(stream)
        ev[3 * K].record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    if sampler is not None:
        clocks = sampler.stop()
    # per-kernel device time over the timed region: pack = [start of step, after pack],
    # combine = [after pack, after combine]
    t_pack = sum((ev[0] if k == 0 else ev[3 * k]).elapsed_time(ev[3 * k + 1]) for k in range(K))
    t_comb = sum(ev[3 * k + 1].elapsed_time(ev[3 * k + 2]) for k in range(K))
    t_total = ev[0].elapsed_time(ev[3 * K])
    t_total_max = max_over_ranks(t_total, device)
    t_pack_max = max_over_ranks(t_pack, device)
    t_comb_max = max_over_ranks(t_comb, device)

    bytes_pack, bytes_comb = w.pack_bytes(), w.combine_bytes()
    step_bytes = bytes_pack + bytes_comb
    ms_per_step = t_total_max / K
    value = world * step_bytes * K / (t_total_max * 1e-3) / 1e9
    peak, peak_src = load_peak()
    kernels = {
        "dcp_pack": {"ms_per_launch": t_pack_max / K, "bytes_per_launch": bytes_pack,
                     "gbs": bytes_pack / (t_pack_max / K * 1e-3) / 1e9},
        "dcp_unpack_combine": {"ms_per_launch": t_comb_max / K, "bytes_per_launch": bytes_comb,
                               "gbs": bytes_comb / (t_comb_max / K * 1e-3) / 1e9},
    }
    for v in kernels.values():
        v["frac_of_peak"] = v["gbs"] / peak
        v["share_of_step"] = v["ms_per_launch"] / ms_per_step
    dom = max(kernels, key=lambda k: kernels[k]["ms_per_launch"])
    dk = kernels[dom]
    roofline = {"bound": "hbm", "kernel": dom, "achieved": dk["gbs"], "peak": peak, "unit": "GB/s",
                "frac": dk["gbs"] / peak, "peak_source": f"{peak_src} ({'MEASURED_PEAKS.json hbm_gbs' if peak_src == 'measured' else 'profiling recipe fallback'})",
                "traffic": load_traffic(dom, w.name), "algorithmic_bytes_per_launch": dk["bytes_per_launch"]}

    # end to end through the public API: pinned host inputs in, host result out, every step.
    # The step's tokens go in chunks over three streams (host-to-device copies, the two kernels,
    # device-to-host copies), so that the copies in both directions and the kernels overlap,
    # as a caller streaming a batch through the library would run it.
    e2e = None
    if not args.no_e2e:
        res_h = torch.empty(result.shape, dtype=result.dtype, pin_memory=True)
        glse_h = torch.empty(glse.shape, dtype=glse.dtype, pin_memory=True) if glse is not None else None
        d_out = torch.empty_like(cp_out)
        d_lse = torch.empty_like(cp_lse)
        nc = max(1, min(args.e2e_chunks, w.B))
        bounds = [(w.B * c // nc, w.B * (c + 1) // nc) for c in range(nc)]
        sends = [torch.empty((w.N, b1 - b0, w.Hr, w.D + P), dtype=cp_out.dtype, device=device) for b0, b1 in bounds]
        s_in, s_run, s_out = (torch.cuda.Stream(device=device) for _ in range(3))
        ev = lambda: torch.cuda.Event()
        in_done, run_done, out_done = [ev() for _ in bounds], [ev() for _ in bounds], [ev() for _ in bounds]
        first = [True]

        def e2e_step():
            for c, (b0, b1) in enumerate(bounds):
                with torch.cuda.stream(s_in):
                    if not first[0]:
                        s_in.wait_event(run_done[c])      # the last step's kernels have read this chunk
                    d_out[b0:b1].copy_(cp_out_h[b0:b1], non_blocking=True)
                    d_lse[b0:b1].copy_(cp_lse_h[b0:b1], non_blocking=True)
                    in_done[c].record(s_in)
                with torch.cuda.stream(s_run):
                    s_run.wait_event(in_done[c])
                    if not first[0]:
                        s_run.wait_event(out_done[c])     # the last step's result chunk has left
                    dcp.dcp_pack(d_out[b0:b1], d_lse[b0:b1], sends[c], w.N)
                    dcp.dcp_unpack_combine(sends[c], result[b0:b1], None if glse is None else glse[b0:b1],
                                           is_lse_base_on_e=w.is_lse_base_on_e, return_lse=w.return_lse)
                    run_done[c].record(s_run)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(run_done[c])
                    res_h[b0:b1].copy_(result[b0:b1], non_blocking=True)
                    if glse_h is not None:
                        glse_h[b0:b1].copy_(glse[b0:b1], non_blocking=True)
                    out_done[c].record(s_out)
            first[0] = False

        e2e_step()
        torch.cuda.synchronize(device)
        barrier(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for st in (s_in, s_run, s_out):
            st.wait_event(e0)
        for _ in range(args.e2e_steps):
            e2e_step()
        for st in (s_in, s_run, s_out):
            stream.wait_stream(st)
        e1.record(stream)
        torch.cuda.synchronize(device)
        t_e2e = max_over_ranks(e0.elapsed_time(e1), device)
        h2d = cp_out.numel() * cp_out.element_size() + cp_lse.numel() * 4
        d2h = result.numel() * result.element_size() + (glse.numel() * 4 if glse is not None else 0)
        e2e = {"value": world * step_bytes * args.e2e_steps / (t_e2e * 1e-3) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
               "ms_per_step": t_e2e / args.e2e_steps, "token_chunks": nc,
               "streams": "host-to-device copies, dcp_pack + dcp_unpack_combine, device-to-host copies"}
        del d_out, d_lse, sends

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K, "warmup": W,
            "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic", "config": workload_config(w),
            "token_heads_per_s": world * w.B * w.Hr * K / (t_total_max * 1e-3),
            "frac_of_measured_peak": value / peak, "frac_of_nominal_8tbs": value / NOMINAL_HBM_GBS,
            "kernels": kernels, "roofline": roofline, "e2e": e2e, "cpu_baseline": cpu,
            "gpu_launches": 2 * K, "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        barrier(device)
        dist.destroy_process_group()
    return 0


def main(argv=None) -> int:
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.sweep:
        return run_sweep(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
