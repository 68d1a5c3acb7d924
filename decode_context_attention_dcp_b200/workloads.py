"""Seeded synthetic inputs for the DCP combine, shared by the tests and the bench.

This module draws random numbers and arranges them in the shapes of DCP decode
workloads.  It holds none of the method's arithmetic (no max, no exp, no
weighting, no packing): both the CUDA path and the CPU oracle receive exactly
the tensors built here, bit for bit.

Recipe (one ``torch.Generator`` per workload, seeded with the workload's seed,
draws taken in this order):
  1. attention outputs: normal(0, std), drawn in fp32 and rounded (RN-even) to
     the output dtype;
  2. LSEs: uniform(lo, hi) in fp32;
  3. special values: one more uniform u per LSE entry; u < p_neginf gives -inf,
     p_neginf <= u < p_neginf + p_nan gives the quiet NaN 0x7FC00000;
  4. structured holes: for ``empty_every = k``, every token b with b % k == 0
     has -inf at every shard (an empty KV context).
Large tensors are drawn in token slices, in token order, so memory stays bounded.
The slice size is a fixed function of the workload's shape (about 2^24 elements per
slice), so a workload's bits are reproducible; a different slicing would draw different
bits.
"""
from __future__ import annotations

import dataclasses
from typing import Iterator

import torch

_DTYPES = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}


def torch_dtype(name: str) -> torch.dtype:
    return _DTYPES[name]


@dataclasses.dataclass(frozen=True)
class CombineWorkload:
    """N shards of partial attention, each [B, Hr, D] plus a [B, Hr] fp32 LSE."""

    name: str
    N: int
    B: int
    Hr: int
    D: int
    dtype: str = "bf16"
    std: float = 1.0
    lse_lo: float = -5.0
    lse_hi: float = 15.0
    p_neginf: float = 0.0
    p_nan: float = 0.0
    empty_every: int = 0
    is_lse_base_on_e: bool = True
    return_lse: bool = False
    seed: int = 0

    @property
    def H(self) -> int:
        """All heads before the head scatter (the pack step's input has H = N * Hr)."""
        return self.N * self.Hr

    @property
    def pack_dim(self) -> int:
        return 1 if self.dtype == "fp32" else 2

    @property
    def W(self) -> int:
        return self.D + self.pack_dim

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "fp32" else 2

    def combine_bytes(self) -> int:
        """Algorithmic HBM bytes of one combine (either layout): read N rows of D elements plus
        an fp32 LSE per (token, head); write one row (+ the fp32 global LSE)."""
        units = self.B * self.Hr
        rd = units * self.N * (self.D * self.elem_bytes + 4)
        wr = units * (self.D * self.elem_bytes + (4 if self.return_lse else 0))
        return rd + wr

    def varlen_combine_bytes(self, shards_read: int, num_reqs: int) -> int:
        """Algorithmic HBM bytes of one variable-length combine in which `shards_read` (token,
        shard) pairs hold KV: those rows and LSEs (Hr heads each) are read, every result row is
        written (+ the global LSE), and the request metadata (seq_lens, query_start_loc) read."""
        rd = shards_read * self.Hr * (self.D * self.elem_bytes + 4) + 4 * (2 * num_reqs + 1)
        wr = self.B * self.Hr * (self.D * self.elem_bytes + (4 if self.return_lse else 0))
        return rd + wr

    def pack_bytes(self) -> int:
        """Algorithmic HBM bytes of one pack: each of the B*H rows (D elements + fp32 LSE) read once
        and written once."""
        rows = self.B * self.H
        return 2 * rows * (self.D * self.elem_bytes + 4)

    def with_(self, **kw) -> "CombineWorkload":
        return dataclasses.replace(self, **kw)


# The five DCP decode workloads.
TINY = CombineWorkload("tiny", N=2, B=4, Hr=8, D=128, lse_lo=-5.0, lse_hi=15.0, return_lse=True, seed=0)
GQA = CombineWorkload("gqa_packed", N=4, B=256, Hr=8, D=128, lse_lo=0.0, lse_hi=12.0, p_neginf=0.05, p_nan=0.01,
                      seed=1)
MLA = CombineWorkload("mla", N=8, B=1024, Hr=16, D=512, std=0.5, lse_lo=-2.0, lse_hi=20.0, empty_every=64,
                      is_lse_base_on_e=False, return_lse=True, seed=2)
ROUNDTRIP = CombineWorkload("roundtrip_fp16", N=8, B=2048, Hr=8, D=128, dtype="fp16", lse_lo=-10.0, lse_hi=30.0,
                            seed=3)


def sweep() -> list[CombineWorkload]:
    """Bandwidth sweep: N in {2,4,8,16} x B in {512,4096,16384} x D in {128,512}, Hr = 16."""
    pts = []
    i = 0
    for D in (128, 512):
        for N in (2, 4, 8, 16):
            for B in (512, 4096, 16384):
                pts.append(CombineWorkload(f"sweep_N{N}_B{B}_D{D}", N=N, B=B, Hr=16, D=D, lse_lo=-5.0, lse_hi=25.0,
                                           p_neginf=0.02, seed=100 + i))
                i += 1
    return pts


def by_name(name: str) -> CombineWorkload:
    for w in (TINY, GQA, MLA, ROUNDTRIP, *sweep()):
        if w.name == name:
            return w
    raise KeyError(name)


# ---------------------------------------------------------------------------------------
def _token_slices(B: int, per_slice: int) -> Iterator[tuple[int, int]]:
    b = 0
    while b < B:
        e = min(B, b + per_slice)
        yield b, e
        b = e


def _draw_lse(gen: torch.Generator, shape, w: CombineWorkload) -> torch.Tensor:
    lse = torch.empty(shape, dtype=torch.float32).uniform_(w.lse_lo, w.lse_hi, generator=gen)
    if w.p_neginf > 0 or w.p_nan > 0:
        u = torch.empty(shape, dtype=torch.float32).uniform_(0.0, 1.0, generator=gen)
        lse[u < w.p_neginf] = float("-inf")
        lse[(u >= w.p_neginf) & (u < w.p_neginf + w.p_nan)] = float("nan")
    return lse


def _slice_rows(w: CombineWorkload) -> int:
    per_token = max(1, w.N * w.Hr * w.D)
    return max(1, (1 << 24) // per_token)


def split_inputs(w: CombineWorkload, pin_memory: bool = False) -> tuple[torch.Tensor, torch.Tensor]:
    """Inputs in the split receive layout: outputs [N, B, Hr, D] (output dtype) and
    lses [N, B, Hr] (fp32), on the CPU."""
    gen = torch.Generator().manual_seed(w.seed)
    dt = torch_dtype(w.dtype)
    outputs = torch.empty((w.N, w.B, w.Hr, w.D), dtype=dt, pin_memory=pin_memory)
    lses = torch.empty((w.N, w.B, w.Hr), dtype=torch.float32, pin_memory=pin_memory)
    for b0, b1 in _token_slices(w.B, _slice_rows(w)):
        x = torch.empty((w.N, b1 - b0, w.Hr, w.D), dtype=torch.float32).normal_(0.0, w.std, generator=gen)
        outputs[:, b0:b1].copy_(x.to(dt))
    for b0, b1 in _token_slices(w.B, _slice_rows(w)):
        lses[:, b0:b1].copy_(_draw_lse(gen, (w.N, b1 - b0, w.Hr), w))
    if w.empty_every:
        lses[:, :: w.empty_every, :] = float("-inf")
    return outputs, lses


def pack_inputs(w: CombineWorkload, pin_memory: bool = False) -> tuple[torch.Tensor, torch.Tensor]:
    """Inputs of the pack step: cp_attn_out [B, H, D] (output dtype) and cp_attn_lse [B, H] (fp32),
    H = N * Hr, on the CPU."""
    gen = torch.Generator().manual_seed(w.seed)
    dt = torch_dtype(w.dtype)
    out = torch.empty((w.B, w.H, w.D), dtype=dt, pin_memory=pin_memory)
    lse = torch.empty((w.B, w.H), dtype=torch.float32, pin_memory=pin_memory)
    rows = max(1, (1 << 24) // max(1, w.H * w.D))
    for b0, b1 in _token_slices(w.B, rows):
        x = torch.empty((b1 - b0, w.H, w.D), dtype=torch.float32).normal_(0.0, w.std, generator=gen)
        out[b0:b1].copy_(x.to(dt))
    for b0, b1 in _token_slices(w.B, rows):
        lse[b0:b1].copy_(_draw_lse(gen, (b1 - b0, w.H), w))
    if w.empty_every:
        lse[:: w.empty_every, :] = float("-inf")
    return out, lse


@dataclasses.dataclass(frozen=True)
class AttentionCase:
    """Decode attention of B tokens, each with its own KV context of length L (MHA, no GQA
    grouping), split over N shards."""

    B: int = 4
    H: int = 8
    D: int = 128
    L: int = 64
    N: int = 2
    dtype: str = "bf16"
    seed: int = 0


def attention_inputs(c: AttentionCase) -> tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """q [B, H, D], k [B, L, H, D], v [B, L, H, D], normal(0, 1) rounded to the dtype."""
    gen = torch.Generator().manual_seed(c.seed)
    dt = torch_dtype(c.dtype)
    q = torch.empty((c.B, c.H, c.D)).normal_(0.0, 1.0, generator=gen).to(dt)
    k = torch.empty((c.B, c.L, c.H, c.D)).normal_(0.0, 1.0, generator=gen).to(dt)
    v = torch.empty((c.B, c.L, c.H, c.D)).normal_(0.0, 1.0, generator=gen).to(dt)
    return q, k, v


@dataclasses.dataclass(frozen=True)
class DecodeBatch:
    """Request metadata of a decode batch of B token slots: requests of 1..max_q query tokens
    each (1 = plain decode, more = speculative tokens) laid end to end from token 0, then
    `pad` padding slots that belong to no request.  Each request's KV length is drawn from a
    mix: with probability p_short uniform in [0, short_max] (0 = no KV at all), else uniform
    in [short_max + 1, max_seq]."""

    B: int
    max_q: int = 1
    pad: int = 0
    p_short: float = 0.3
    short_max: int = 16
    max_seq: int = 8192
    seed: int = 0


def decode_batch(c: DecodeBatch) -> tuple[torch.Tensor, torch.Tensor]:
    """(seq_lens [R] int32, query_start_loc [R + 1] int32) on the CPU, with
    query_start_loc[R] = B - pad.  Draws: per request its query length (uniform 1..max_q,
    cut at the last real slot), then per request one uniform u for the length class and one
    integer for the length."""
    gen = torch.Generator().manual_seed(c.seed)
    real = max(0, c.B - c.pad)
    starts = [0]
    while starts[-1] < real:
        q = int(torch.randint(1, c.max_q + 1, (1,), generator=gen))
        starts.append(min(real, starts[-1] + q))
    R = len(starts) - 1
    u = torch.rand(R, generator=gen)
    short = torch.randint(0, c.short_max + 1, (R,), generator=gen)
    long = torch.randint(c.short_max + 1, c.max_seq + 1, (R,), generator=gen)
    seq_lens = torch.where(u < c.p_short, short, long).to(torch.int32)
    return seq_lens, torch.tensor(starts, dtype=torch.int32)
