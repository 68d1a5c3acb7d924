"""Parity of the 4-row group kernels with the oracle.

dcp_unpack_combine takes the group kernel when the packed buffer's shard stride is a multiple of
16 bytes and a row holds 32, 64 or 128 data words (D = 64, 128, 256 for 16-bit types; D = 32, 64,
128 for fp32); dcp_combine_pack takes it for the same row widths when the heads per rank are a
multiple of 4.  These cases are built here on purpose: capacity-strided shards whose last group
has fewer than 4 rows, shard counts 1 .. 64, NaN / +-inf / all-empty LSE rows, guard bands around
every output, and for the fused pack bit-equality with dcp_lse_combine followed by dcp_pack.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import decode_context_attention_dcp_b200 as dcp
import oracle as orc
from decode_context_attention_dcp_b200 import workloads as wl
from gpu_util import ORACLE_CODE, Guarded, assert_lse_close, assert_out_close, bits, packed_from_split, raw

pytestmark = pytest.mark.gpu

WIDTHS = [("bf16", 64), ("bf16", 128), ("bf16", 256), ("fp16", 128), ("fp16", 64), ("fp32", 32), ("fp32", 64),
          ("fp32", 128)]


@pytest.fixture(scope="module")
def o() -> orc.Oracle:
    return orc.load()


def _inputs(N, B, Hr, D, dtype, seed, specials=True):
    w = wl.CombineWorkload(f"group_N{N}_B{B}_H{Hr}_D{D}_{dtype}", N=N, B=B, Hr=Hr, D=D, dtype=dtype, lse_lo=-25.0,
                           lse_hi=25.0, p_neginf=0.08 if specials else 0.0, p_nan=0.04 if specials else 0.0,
                           empty_every=5 if specials else 0, seed=seed)
    outputs, lses = wl.split_inputs(w)
    if specials and B > 2:
        lses[:, 1, 0] = float("inf")              # +inf counts as -inf
        lses[N // 2, 2, :] = float("nan")
    return outputs, lses


def _capacity(B, Hr, W, es):
    """Rows of capacity per shard (>= B) that make the shard stride a multiple of 16 bytes."""
    cap = B
    while (cap * Hr * W * es) % 16:
        cap += 1
    return cap


@pytest.mark.parametrize("dtype,D", WIDTHS)
@pytest.mark.parametrize("N,B,Hr", [(1, 9, 3), (2, 13, 1), (3, 7, 5), (5, 37, 1), (8, 21, 3), (16, 6, 2),
                                    (33, 5, 1), (64, 3, 3), (4, 64, 4)])
def test_group_unpack_combine(o, dtype, D, N, B, Hr):
    es = 4 if dtype == "fp32" else 2
    W = D + 4 // es
    seed = N * 97 + B * 13 + Hr * 5 + D
    outputs, lses = _inputs(N, B, Hr, D, dtype, seed)
    recv = packed_from_split(outputs, lses)                      # [N, B, Hr, W]
    cap = _capacity(B, Hr, W, es)
    store = torch.full((N, cap, Hr, W), float("nan"), dtype=recv.dtype)
    store[:, :B] = recv
    d_recv = store.cuda()[:, :B]                                 # shard stride cap * Hr * W
    assert (d_recv.stride(0) * es) % 16 == 0
    for base_e in (True, False):
        ry, rg = o.lse_combine(raw(outputs), ORACLE_CODE[outputs.dtype], raw(lses), return_lse=True,
                               is_lse_base_on_e=base_e)
        res = Guarded((B, Hr, D), recv.dtype)
        gl = Guarded((B, Hr), torch.float32)
        dcp.dcp_unpack_combine(d_recv, res.tensor, gl.tensor, is_lse_base_on_e=base_e, return_lse=True)
        res.check()
        gl.check()
        assert_out_close(res.tensor, ry, f"group unpack N={N} B={B} Hr={Hr} D={D} {dtype} base_e={base_e}")
        assert_lse_close(gl.tensor, rg, f"group unpack lse N={N} B={B} Hr={Hr} D={D} {dtype}")
    # without return_lse, and the global LSE buffer untouched
    res = Guarded((B, Hr, D), recv.dtype)
    dcp.dcp_unpack_combine(d_recv, res.tensor)
    res.check()
    assert_out_close(res.tensor, o.lse_combine(raw(outputs), ORACLE_CODE[outputs.dtype], raw(lses)), "no lse")


def test_group_unpack_empty_and_single_rows(o):
    """All-empty rows give 0 and -inf exactly; a row with one finite shard is that shard's row."""
    N, B, Hr, D = 6, 8, 4, 128
    outputs, lses = _inputs(N, B, Hr, D, "bf16", 3, specials=False)
    lses[:, 0, :] = float("-inf")
    lses[:, 1, :] = torch.tensor([float("nan"), float("inf"), float("-inf"), float("nan"), float("inf"),
                                  float("-inf")]).unsqueeze(-1)
    lses[:, 2, 1] = torch.tensor([float("nan"), 3.0, float("inf"), float("-inf"), float("nan"), float("-inf")])
    y, g = dcp.unpack_combine(packed_from_split(outputs, lses).cuda(), return_lse=True)
    ry, rg = o.lse_combine(raw(outputs), orc.BF16, raw(lses), return_lse=True)
    assert_out_close(y, ry, "specials")
    assert_lse_close(g, rg, "specials lse")
    assert bool((y.cpu()[0:2] == 0).all()) and bool((g.cpu()[0:2] == -math.inf).all())
    assert torch.equal(y.cpu()[2, 1], outputs[1, 2, 1]) and float(g.cpu()[2, 1]) == 3.0


def _two_step(d_out, d_lse, ws, base_e):
    S, B, H, D = d_out.shape
    y = torch.empty((B, H, D), dtype=d_out.dtype, device="cuda")
    g = torch.empty((B, H), dtype=torch.float32, device="cuda")
    dcp.dcp_lse_combine(d_out, d_lse, y, g, is_lse_base_on_e=base_e, return_lse=True)
    send = torch.empty((ws, B, H // ws, D + dcp.dcp_lse_pack_dim(d_out.dtype)), dtype=d_out.dtype, device="cuda")
    dcp.dcp_pack(y, g, send, ws)
    return send


@pytest.mark.parametrize("dtype,D", WIDTHS)
@pytest.mark.parametrize("S,B,Hr,ws", [(1, 5, 4, 2), (2, 9, 8, 1), (3, 4, 4, 3), (4, 11, 16, 2), (8, 3, 12, 4),
                                       (16, 7, 4, 1), (33, 2, 8, 2), (64, 3, 4, 1)])
def test_group_combine_pack(o, dtype, D, S, B, Hr, ws):
    H = Hr * ws
    seed = S * 31 + B * 7 + H + D
    outputs, lses = _inputs(S, B, H, D, dtype, seed)
    d_out, d_lse = outputs.cuda(), lses.cuda()
    P = dcp.dcp_lse_pack_dim(d_out.dtype)
    for base_e in (True, False):
        send = Guarded((ws, B, Hr, D + P), d_out.dtype)
        dcp.dcp_combine_pack(d_out, d_lse, send.tensor, ws, is_lse_base_on_e=base_e)
        send.check()
        ry, rg = o.lse_combine(raw(outputs), ORACLE_CODE[outputs.dtype], raw(lses), return_lse=True,
                               is_lse_base_on_e=base_e)
        t = send.tensor
        data = t[..., :D].permute(1, 0, 2, 3).reshape(B, H, D)
        tail = t[..., D:].contiguous()
        lse = (tail.view(torch.float32) if P == 2 else tail).reshape(ws, B, Hr).permute(1, 0, 2).reshape(B, H)
        assert_out_close(data, ry, f"group pack S={S} B={B} Hr={Hr} ws={ws} D={D} {dtype}")
        assert_lse_close(lse, rg, f"group pack lse S={S} B={B} Hr={Hr} ws={ws} D={D} {dtype}")
        ref = _two_step(d_out, d_lse, ws, base_e)
        assert np.array_equal(bits(t.cpu()), bits(ref.cpu())), "differs from dcp_lse_combine + dcp_pack"


@pytest.mark.parametrize("dtype,D", [("fp32", 96), ("fp32", 160), ("bf16", 192), ("fp16", 320), ("bf16", 32)])
def test_widths_outside_the_group_kernels(o, dtype, D):
    """Rows whose data words are a multiple of 32 but not 32, 64 or 128 (and rows of 16 words)
    take the other kernels even on an aligned shard stride and with heads per rank a multiple of
    4: results match the oracle and nothing is written outside the outputs."""
    N, B, Hr, ws = 4, 8, 4, 2
    es = 4 if dtype == "fp32" else 2
    W = D + 4 // es
    outputs, lses = _inputs(N, B, Hr * ws, D, dtype, D + 1)
    recv = packed_from_split(outputs, lses)
    assert (recv.stride(0) * es) % 16 == 0
    ry, rg = o.lse_combine(raw(outputs), ORACLE_CODE[outputs.dtype], raw(lses), return_lse=True)
    res = Guarded((B, Hr * ws, D), recv.dtype)
    gl = Guarded((B, Hr * ws), torch.float32)
    dcp.dcp_unpack_combine(recv.cuda(), res.tensor, gl.tensor, return_lse=True)
    res.check()
    gl.check()
    assert_out_close(res.tensor, ry, f"unpack {dtype} D={D}")
    assert_lse_close(gl.tensor, rg, f"unpack lse {dtype} D={D}")
    P = 4 // es
    send = Guarded((ws, B, Hr, D + P), recv.dtype)
    d_out, d_lse = outputs.cuda(), lses.cuda()
    dcp.dcp_combine_pack(d_out, d_lse, send.tensor, ws)
    send.check()
    ref = _two_step(d_out, d_lse, ws, True)
    assert np.array_equal(bits(send.tensor.cpu()), bits(ref.cpu()))
    assert W == D + P
