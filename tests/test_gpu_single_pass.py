"""Parity of the single-pass packed combine (dcp_unpack_combine on rows of at most 512 bytes with
3 or more shards, or 144-256 bytes with 2, and a 16-byte-multiple shard stride) with the oracle.

That kernel applies the combine rules batch by batch to a running maximum and rescales what it
has summed when the maximum grows, so the cases here are chosen to cross batch boundaries: the
only finite shards in the last batch, every finite shard in the first batch, all-empty rows,
LSE spreads wide enough that rescaling underflows, +inf / NaN LSEs, and NaN rows in shards whose
weight is 0 (the page multiplies them anyway, so the NaN must come out where the oracle has it).
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import decode_context_attention_dcp_b200 as dcp
import oracle as orc
from decode_context_attention_dcp_b200 import workloads as wl
from gpu_util import ORACLE_CODE, Guarded, assert_lse_close, assert_out_close, packed_from_split, raw

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def o() -> orc.Oracle:
    return orc.load()


def _check(o, outputs, lses, base_e, what):
    N, B, Hr, D = outputs.shape
    recv = packed_from_split(outputs, lses)
    es = outputs.element_size()
    assert (recv.stride(0) * es) % 16 == 0  # a uniform shard stride: the single-pass kernel
    ry, rg = o.lse_combine(raw(outputs), ORACLE_CODE[outputs.dtype], raw(lses), return_lse=True,
                           is_lse_base_on_e=base_e)
    res = Guarded((B, Hr, D), outputs.dtype)
    gl = Guarded((B, Hr), torch.float32)
    dcp.dcp_unpack_combine(recv.cuda(), res.tensor, gl.tensor, is_lse_base_on_e=base_e, return_lse=True)
    res.check()
    gl.check()
    assert_out_close(res.tensor, ry, what)
    assert_lse_close(gl.tensor, rg, what + " lse")
    return res.tensor.cpu(), gl.tensor.cpu()


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("fp16", 128), ("fp32", 64), ("bf16", 96), ("bf16", 64),
                                     ("fp32", 32), ("bf16", 256), ("fp16", 192), ("fp32", 128)])
@pytest.mark.parametrize("N", [2, 3, 4, 5, 8, 13, 16, 33, 64])
@pytest.mark.parametrize("base_e", [True, False])
def test_batch_boundaries(o, dtype, D, N, base_e):
    B, Hr = 12, 4
    w = wl.CombineWorkload(f"single_pass_N{N}_D{D}_{dtype}", N=N, B=B, Hr=Hr, D=D, dtype=dtype, lse_lo=-20.0,
                           lse_hi=20.0, p_neginf=0.1, p_nan=0.05, seed=N * 7 + D)
    outputs, lses = wl.split_inputs(w)
    ninf = float("-inf")
    lses[:, 0, :] = ninf                                   # all empty
    lses[:-1, 1, :] = ninf                                 # only the last shard finite
    lses[-1, 1, :] = 7.5
    lses[1:, 2, :] = ninf                                  # only the first shard finite
    lses[0, 2, :] = -3.25
    lses[:, 3, 0] = torch.linspace(-80.0, 80.0, N)         # rescaling far below / above
    lses[:, 3, 1] = torch.linspace(80.0, -80.0, N)
    lses[:, 4, :] = float("inf")                           # +inf counts as -inf: all empty
    lses[::2, 5, :] = float("nan")                         # NaN shards weigh 0
    lses[:, 6, 2] = 115.0 if not base_e else 85.0          # equal large LSEs: the plain mean
    outputs[N // 2, 7, 1] = float("nan")                   # a NaN row in a shard of weight 0 ...
    lses[N // 2, 7, 1] = ninf                              # ... propagates, as the page's 0 * NaN
    y, g = _check(o, outputs, lses, base_e, f"single pass N={N} D={D} {dtype} base_e={base_e}")
    assert bool((y[0] == 0).all()) and bool((g[0] == -math.inf).all())
    assert bool((y[4] == 0).all()) and bool((g[4] == -math.inf).all())
    assert float(g[1, 0]) == 7.5 and float(g[2, 0]) == -3.25
    assert torch.equal(y[1], outputs[-1, 1]) and torch.equal(y[2], outputs[0, 2])
    assert bool(torch.isnan(y[7, 1]).all())


def test_full_size_single_pass(o):
    """The sweep's N=16, B=16384, D=128 point through the single-pass kernel, every element."""
    from gpu_util import HOST_THREADS, compare_token_blocks
    w = wl.by_name("sweep_N16_B16384_D128")
    outputs, lses = wl.split_inputs(w)
    recv = packed_from_split(outputs, lses).cuda()
    y, g = dcp.unpack_combine(recv, return_lse=True)
    ro, rl = raw(outputs), raw(lses)

    def ref(b0, b1):
        return o.lse_combine_tokens(ro, orc.BF16, rl, b0, b1, return_lse=True, threads=HOST_THREADS)

    compare_token_blocks(w.B, w.Hr * w.D, ref, [(y, "dcp_unpack_combine")], [(g, "dcp_unpack_combine lse")],
                         "single pass full size")


@pytest.mark.parametrize("dtype,D", [("bf16", 512), ("fp16", 512), ("fp32", 256), ("bf16", 264), ("bf16", 320)])
@pytest.mark.parametrize("N", [1, 2, 3, 4, 5, 8, 15, 16])
def test_wide_rows_quarter_lanes(o, dtype, D, N):
    """Packed rows of 513 bytes to 1 KiB: with 2-4 shards the single-pass kernel with one batch
    and 16 lanes per row, with 5-15 the two-phase kernel with 16 lanes, with 16 (and 1) the
    32-lane two-phase shape; the same special rows as above, against the oracle.
    12 tokens of 3 heads keep every shard's stride a multiple of 16 bytes."""
    B, Hr = 12, 3
    w = wl.CombineWorkload(f"wide_N{N}_D{D}_{dtype}", N=N, B=B, Hr=Hr, D=D, dtype=dtype, lse_lo=-20.0,
                           lse_hi=20.0, p_neginf=0.1, p_nan=0.05, seed=N * 5 + D)
    outputs, lses = wl.split_inputs(w)
    ninf = float("-inf")
    lses[:, 0, :] = ninf
    lses[:-1, 1, :] = ninf
    lses[-1, 1, :] = 7.5
    lses[:, 2, 0] = torch.linspace(-80.0, 80.0, N)
    outputs[N // 2, 3, 1] = float("nan")
    lses[N // 2, 3, 1] = ninf
    for base_e in (True, False):
        y, g = _check(o, outputs, lses, base_e, f"wide rows N={N} D={D} {dtype} base_e={base_e}")
        assert bool((y[0] == 0).all()) and bool((g[0] == -math.inf).all())
        assert float(g[1, 0]) == 7.5 and torch.equal(y[1], outputs[-1, 1])
        assert bool(torch.isnan(y[3, 1]).all())
