"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, on the seeded DCP workloads.

Element by element everywhere, the full-size sweep points included (the oracle runs over token
slices on all host cores there).  Pack is compared bit for bit.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import decode_context_attention_dcp_b200 as dcp
import oracle as orc
import oracle_pins
from decode_context_attention_dcp_b200 import workloads as wl
from gpu_util import (HOST_THREADS, ORACLE_CODE, Guarded, assert_lse_close, assert_out_close, bits,
                      compare_token_blocks, packed_from_split, raw)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def o() -> orc.Oracle:
    return orc.load()


def gpu_combine(outputs, lses, w: wl.CombineWorkload, return_lse=None):
    ret = w.return_lse if return_lse is None else return_lse
    return dcp.lse_weighted_combine(outputs.cuda(), lses.cuda(), return_lse=ret,
                                    is_lse_base_on_e=w.is_lse_base_on_e)


def gpu_unpack(recv, w: wl.CombineWorkload, return_lse=None):
    ret = w.return_lse if return_lse is None else return_lse
    return dcp.unpack_combine(recv.cuda(), return_lse=ret, is_lse_base_on_e=w.is_lse_base_on_e)


def check_split(o, w, outputs, lses, ret):
    code = ORACLE_CODE[outputs.dtype]
    got = gpu_combine(outputs, lses, w, ret)
    ref = o.lse_combine(raw(outputs), code, raw(lses), return_lse=ret, is_lse_base_on_e=w.is_lse_base_on_e)
    if ret:
        assert_out_close(got[0], ref[0], f"{w.name} combine")
        assert_lse_close(got[1], ref[1], f"{w.name} combine lse")
    else:
        assert_out_close(got, ref, f"{w.name} combine")
    return got, ref


def check_packed(o, w, recv, ret):
    code = ORACLE_CODE[recv.dtype]
    got = gpu_unpack(recv, w, ret)
    ref = o.unpack_combine(raw(recv), code, w.D, return_lse=ret, is_lse_base_on_e=w.is_lse_base_on_e)
    if ret:
        assert_out_close(got[0], ref[0], f"{w.name} unpack_combine")
        assert_lse_close(got[1], ref[1], f"{w.name} unpack_combine lse")
    else:
        assert_out_close(got, ref, f"{w.name} unpack_combine")
    return got, ref


# ---- the four named workloads, element by element ------------------------------------------
def test_tiny(o):
    w = wl.TINY
    outputs, lses = wl.split_inputs(w)
    check_split(o, w, outputs, lses, True)
    check_packed(o, w, packed_from_split(outputs, lses), True)


@pytest.mark.parametrize("split", ["contiguous", "interleaved"])
@pytest.mark.parametrize("base_e", [True, False])
def test_tiny_bruteforce_attention(o, split, base_e):
    """K/V of length 64 split over 2 shards: per-shard attention + LSE (fp64, rounded to bf16 /
    fp32 as a shard would emit them), combined on the GPU, equals full attention."""
    case = wl.AttentionCase()
    q, k, v = wl.attention_inputs(case)
    scale = 1.0 / math.sqrt(case.D)
    shards = oracle_pins.shard_positions(case.L, case.N, split)
    outs = np.zeros((case.N, case.B, case.H, case.D))
    lses = np.zeros((case.N, case.B, case.H))
    full_o = np.zeros((case.B, case.H, case.D))
    full_l = np.zeros((case.B, case.H))
    for b in range(case.B):
        qb, kb, vb = raw(q[b]), raw(k[b]), raw(v[b])
        full_o[b], full_l[b] = o.attention(qb, kb, vb, orc.BF16, list(range(case.L)), scale, base_e)
        for r, pos in enumerate(shards):
            outs[r, b], lses[r, b] = o.attention(qb, kb, vb, orc.BF16, pos, scale, base_e)
    shard_out = torch.from_numpy(outs).to(torch.bfloat16)
    shard_lse = torch.from_numpy(lses).to(torch.float32)
    y, g = dcp.lse_weighted_combine(shard_out.cuda(), shard_lse.cuda(), return_lse=True, is_lse_base_on_e=base_e)
    assert_out_close(y, full_o, "combine vs full attention")
    assert_lse_close(g, full_l, "global lse vs full attention")
    # the same through the packed layout
    y2, g2 = dcp.unpack_combine(packed_from_split(shard_out, shard_lse).cuda(), return_lse=True,
                                is_lse_base_on_e=base_e)
    assert_out_close(y2, full_o, "unpack_combine vs full attention")
    assert_lse_close(g2, full_l, "unpack_combine lse vs full attention")


@pytest.mark.parametrize("ret", [False, True])
def test_gqa_packed(o, ret):
    w = wl.GQA
    outputs, lses = wl.split_inputs(w)
    assert torch.isnan(lses).any() and torch.isinf(lses).any()
    check_packed(o, w, packed_from_split(outputs, lses), ret)
    check_split(o, w, outputs, lses, ret)


def test_mla(o):
    w = wl.MLA
    outputs, lses = wl.split_inputs(w)
    (y, g), _ = check_split(o, w, outputs, lses, True)
    empty = torch.arange(w.B) % w.empty_every == 0
    assert bool((y[empty.cuda()] == 0).all())
    assert bool((g[empty.cuda()] == -math.inf).all())
    assert bool(torch.isfinite(g[~empty.cuda()]).all())


def test_mla_through_pack(o):
    """MLA shards laid out as one rank's cp_attn_out [B, N*Hr, D]: pack (bit-exact), then unpack+combine
    over the packed buffer with every shard taken from it."""
    w = wl.MLA
    outputs, lses = wl.split_inputs(w)
    cp_out = outputs.permute(1, 0, 2, 3).reshape(w.B, w.H, w.D).contiguous()
    cp_lse = lses.permute(1, 0, 2).reshape(w.B, w.H).contiguous()
    send = dcp.pack(cp_out.cuda(), cp_lse.cuda(), w.N)
    ref_send = o.pack(raw(cp_out), raw(cp_lse), w.N, orc.BF16)
    assert np.array_equal(bits(send.cpu()), bits(ref_send)), "pack is not bit-exact"
    y, g = dcp.unpack_combine(send, return_lse=True, is_lse_base_on_e=False)
    ry, rg = o.unpack_combine(ref_send, orc.BF16, w.D, return_lse=True, is_lse_base_on_e=False)
    assert_out_close(y, ry, "mla unpack_combine")
    assert_lse_close(g, rg, "mla unpack_combine lse")


def test_roundtrip_fp16(o):
    w = wl.ROUNDTRIP
    cp_out, cp_lse = wl.pack_inputs(w)
    assert cp_out.shape == (2048, 64, 128) and cp_out.dtype == torch.float16
    send = dcp.pack(cp_out.cuda(), cp_lse.cuda(), w.N)
    assert send.shape == (8, 2048, 8, 130)
    ref_send = o.pack(raw(cp_out), raw(cp_lse), w.N, orc.FP16)
    assert np.array_equal(bits(send.cpu()), bits(ref_send)), "pack is not bit-exact"
    y = dcp.unpack_combine(send)
    ry = o.unpack_combine(ref_send, orc.FP16, w.D)
    assert_out_close(y, ry, "roundtrip unpack_combine")


# ---- the bandwidth sweep -----------------------------------------------------------------
SWEEP = wl.sweep()
SWEEP_SMALL = [p for p in SWEEP if p.B == 512]
SWEEP_LARGE = [p for p in SWEEP if p.B >= 4096]


@pytest.mark.parametrize("w", SWEEP_SMALL, ids=lambda p: p.name)
def test_sweep_full_elementwise(o, w):
    outputs, lses = wl.split_inputs(w)
    check_split(o, w, outputs, lses, False)
    check_packed(o, w, packed_from_split(outputs, lses), False)


@pytest.mark.parametrize("w", SWEEP_LARGE, ids=lambda p: p.name)
def test_sweep_full_size_elementwise(o, w):
    """Full-size inputs of every B = 4096 and B = 16384 sweep point: every element of both
    entry points against the oracle (run over token slices on all host cores).  The split
    combine also returns the global LSE here, so that path is checked at full size too."""
    outputs, lses = wl.split_inputs(w)
    d_out, d_lse = outputs.cuda(), lses.cuda()
    y, g = dcp.lse_weighted_combine(d_out, d_lse, return_lse=True)
    recv = torch.cat([d_out, d_lse.unsqueeze(-1).view(d_out.dtype)], dim=-1)
    del d_out, d_lse
    y2 = dcp.unpack_combine(recv)
    del recv
    ro, rl = raw(outputs), raw(lses)

    def ref(b0, b1):
        return o.lse_combine_tokens(ro, orc.BF16, rl, b0, b1, return_lse=True, threads=HOST_THREADS)

    compare_token_blocks(w.B, w.Hr * w.D, ref, [(y, "dcp_lse_combine"), (y2, "dcp_unpack_combine")],
                         [(g, "dcp_lse_combine global lse")], w.name)


def test_bench_step_full_size(o):
    """The bench's step at full size (largest sweep point): pack of cp_attn_out [B, N*Hr, D]
    compared bit for bit everywhere, then every element of the unpack+combine of the send
    buffer against the oracle's unpack+combine of the oracle's own send buffer."""
    w = wl.by_name("sweep_N16_B16384_D512")
    cp_out, cp_lse = wl.pack_inputs(w)
    send = dcp.pack(cp_out.cuda(), cp_lse.cuda(), w.N)
    ref_send = o.pack(raw(cp_out), raw(cp_lse), w.N, orc.BF16)
    del cp_out
    got_send = bits(send.cpu())
    assert np.array_equal(got_send, bits(ref_send)), "pack is not bit-exact"
    del got_send
    y, g = dcp.unpack_combine(send, return_lse=True, is_lse_base_on_e=w.is_lse_base_on_e)

    def ref(b0, b1):
        return o.unpack_combine_tokens(ref_send, orc.BF16, w.D, b0, b1, return_lse=True, threads=HOST_THREADS)

    compare_token_blocks(w.B, w.Hr * w.D, ref, [(y, "dcp_unpack_combine")], [(g, "dcp_unpack_combine lse")],
                         "bench step")


# ---- shapes, dtypes and edge cases -----------------------------------------------------------
def _case(N, B, Hr, D, dtype, seed, p_neginf=0.1, p_nan=0.05, base_e=True):
    w = wl.CombineWorkload(f"edge_N{N}_B{B}_H{Hr}_D{D}_{dtype}", N=N, B=B, Hr=Hr, D=D, dtype=dtype,
                           p_neginf=p_neginf, p_nan=p_nan, is_lse_base_on_e=base_e, lse_lo=-30.0, lse_hi=30.0,
                           seed=seed)
    return w, *wl.split_inputs(w)


EDGE = [(N, B, Hr, D, dt)
        for (N, B, Hr, D) in [(1, 3, 2, 128), (2, 1, 1, 8), (3, 37, 3, 64), (5, 7, 5, 96), (16, 9, 2, 512),
                              (64, 3, 2, 128), (7, 2, 3, 576), (4, 5, 1, 1024), (2, 129, 4, 16), (33, 4, 3, 256),
                              # wide rows: several chunk slots per lane, several passes
                              (64, 2, 2, 1024), (33, 3, 2, 1024), (40, 2, 1, 2048), (9, 300, 1, 8192),
                              # packed rows at every offset from a 16-byte boundary in one shard stride
                              (3, 8, 4, 576), (5, 4, 4, 96), (12, 16, 2, 64)]
        for dt in ("bf16", "fp16", "fp32")]


@pytest.mark.parametrize("N,B,Hr,D,dtype", EDGE)
def test_edge_shapes(o, N, B, Hr, D, dtype):
    if dtype == "fp32" and D % 4:
        pytest.skip("fp32 rows need D % 4 == 0")
    seed = (N * 131 + B * 17 + Hr * 7 + D) % 1000
    for base_e in (True, False):
        w, outputs, lses = _case(N, B, Hr, D, dtype, seed, base_e=base_e)
        check_split(o, w, outputs, lses, True)
        check_packed(o, w, packed_from_split(outputs, lses), True)
    # the same into guarded outputs: nothing is written outside them
    ry, rg = o.lse_combine(raw(outputs), ORACLE_CODE[outputs.dtype], raw(lses), return_lse=True,
                           is_lse_base_on_e=False)
    for packed in (False, True):
        res = Guarded((B, Hr, D), outputs.dtype)
        gl = Guarded((B, Hr), torch.float32)
        if packed:
            dcp.dcp_unpack_combine(packed_from_split(outputs, lses).cuda(), res.tensor, gl.tensor,
                                   is_lse_base_on_e=False, return_lse=True)
        else:
            dcp.dcp_lse_combine(outputs.cuda(), lses.cuda(), res.tensor, gl.tensor, is_lse_base_on_e=False,
                                return_lse=True)
        res.check()
        gl.check()
        assert_out_close(res.tensor, ry, f"guarded packed={packed}")
        assert_lse_close(gl.tensor, rg, f"guarded packed={packed}")


@pytest.mark.parametrize("dtype", ["bf16", "fp16", "fp32"])
def test_single_shard_is_identity(dtype):
    w, outputs, lses = _case(1, 6, 4, 128, dtype, 5, p_neginf=0.0, p_nan=0.0)
    y, g = gpu_combine(outputs, lses, w, True)
    assert torch.equal(y.cpu().view(torch.int16 if dtype != "fp32" else torch.int32),
                       outputs[0].view(torch.int16 if dtype != "fp32" else torch.int32))
    assert torch.equal(g.cpu(), lses[0])
    y2, g2 = gpu_unpack(packed_from_split(outputs, lses), w, True)
    assert torch.equal(y2.cpu(), y.cpu()) and torch.equal(g2.cpu(), g.cpu())


def test_special_lses(o):
    """NaN, +inf and -inf LSEs, all-empty rows and single-finite-shard rows."""
    w, outputs, lses = _case(4, 8, 2, 128, "bf16", 3, p_neginf=0.0, p_nan=0.0)
    lses[:, 0, :] = float("-inf")
    lses[:, 1, :] = torch.tensor([float("nan"), float("inf"), float("-inf"), float("nan")]).unsqueeze(-1)
    lses[:, 2, 0] = torch.tensor([float("nan"), 3.0, float("inf"), float("-inf")])
    lses[:, 3, 1] = float("inf")
    lses[2, 4, :] = float("inf")
    (y, g), _ = check_split(o, w, outputs, lses, True)
    check_packed(o, w, packed_from_split(outputs, lses), True)
    assert bool((y.cpu()[0:2] == 0).all()) and bool((g.cpu()[0:2] == -math.inf).all())
    assert torch.equal(y.cpu()[2, 0], outputs[1, 2, 0])
    assert float(g.cpu()[2, 0]) == 3.0


def test_capacity_strided_shards(o):
    """Receive buffers with room for T_max > B tokens per shard (the direct-workspace layout)."""
    N, T_max, B, Hr, D = 4, 50, 37, 3, 128
    w, outputs, lses = _case(N, T_max, Hr, D, "bf16", 9)
    d_out, d_lse = outputs.cuda(), lses.cuda()
    y = torch.empty((B, Hr, D), dtype=torch.bfloat16, device="cuda")
    g = torch.empty((B, Hr), dtype=torch.float32, device="cuda")
    dcp.dcp_lse_combine(d_out[:, :B], d_lse[:, :B], y, g, return_lse=True)
    ry, rg = o.lse_combine(raw(outputs[:, :B]), orc.BF16, raw(lses[:, :B]), return_lse=True)
    assert_out_close(y, ry, "strided combine")
    assert_lse_close(g, rg, "strided combine lse")
    recv = packed_from_split(outputs, lses).cuda()
    y2 = torch.empty_like(y)
    g2 = torch.empty_like(g)
    dcp.dcp_unpack_combine(recv[:, :B], y2, g2, return_lse=True)
    assert_out_close(y2, ry, "strided unpack_combine")
    assert_lse_close(g2, rg, "strided unpack_combine lse")


def test_outputs_stay_inside_their_buffers(o):
    w, outputs, lses = _case(3, 33, 3, 96, "bf16", 11)
    res = Guarded((33, 3, 96), torch.bfloat16)
    gl = Guarded((33, 3), torch.float32)
    dcp.dcp_lse_combine(outputs.cuda(), lses.cuda(), res.tensor, gl.tensor, return_lse=True)
    res.check()
    gl.check()
    ry, rg = o.lse_combine(raw(outputs), orc.BF16, raw(lses), return_lse=True)
    assert_out_close(res.tensor, ry)
    assert_lse_close(gl.tensor, rg)
    res2 = Guarded((33, 3, 96), torch.bfloat16)
    gl2 = Guarded((33, 3), torch.float32)
    dcp.dcp_unpack_combine(packed_from_split(outputs, lses).cuda(), res2.tensor, gl2.tensor, return_lse=True)
    res2.check()
    gl2.check()
    assert_out_close(res2.tensor, ry)
    # pack: every packed-row alignment (rows are 4 bytes past a 16-byte boundary each) and ragged tiles
    for (B, H, D, ws) in [(3, 12, 8, 3), (5, 10, 128, 5), (2, 6, 520, 2), (1, 1, 64, 1), (70, 8, 128, 4)]:
        out = torch.randn(B, H, D).to(torch.bfloat16)
        lse = torch.randn(B, H)
        send = Guarded((ws, B, H // ws, D + 2), torch.bfloat16)
        dcp.dcp_pack(out.cuda(), lse.cuda(), send.tensor, ws)
        send.check()
        assert np.array_equal(bits(send.tensor.cpu()), bits(o.pack(raw(out), raw(lse), ws, orc.BF16))), (B, H, D, ws)


@pytest.mark.parametrize("dtype", ["bf16", "fp16", "fp32"])
def test_pack_bit_exact_strided_inputs(o, dtype):
    dt = wl.torch_dtype(dtype)
    B, H, D, ws = 7, 12, 64, 4
    big = torch.randn(B + 1, H + 2, D + 8).to(dt)
    out = big[1:, 1:H + 1, :D]                 # strides (H+2)*(D+8), D+8, 1
    lse_big = torch.randn(B, H + 5)
    lse_big[0, 0] = float("nan")
    lse_big.view(torch.int32)[0, 1] = 0x7FC01234    # NaN payload must survive
    lse_big[0, 2] = float("-inf")
    lse = lse_big[:, :H]
    send = dcp.pack(out.cuda(), lse.cuda(), ws)
    ref = o.pack(raw(out.contiguous()), raw(lse.contiguous()), ws, ORACLE_CODE[dt])
    assert np.array_equal(bits(send.cpu()), bits(ref))


def test_empty_batch_is_a_noop():
    outputs = torch.zeros((2, 0, 4, 128), dtype=torch.bfloat16, device="cuda")
    lses = torch.zeros((2, 0, 4), device="cuda")
    y = torch.empty((0, 4, 128), dtype=torch.bfloat16, device="cuda")
    dcp.dcp_lse_combine(outputs, lses, y)
    recv = torch.zeros((2, 0, 4, 130), dtype=torch.bfloat16, device="cuda")
    dcp.dcp_unpack_combine(recv, y)
    send = torch.empty((2, 0, 2, 130), dtype=torch.bfloat16, device="cuda")
    dcp.dcp_pack(torch.zeros((0, 4, 128), dtype=torch.bfloat16, device="cuda"),
                 torch.zeros((0, 4), device="cuda"), send, 2)
    torch.cuda.synchronize()


def test_side_stream(o):
    w, outputs, lses = _case(8, 64, 4, 128, "bf16", 21)
    s = torch.cuda.Stream()
    d_out, d_lse = outputs.cuda(), lses.cuda()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        y = dcp.lse_weighted_combine(d_out, d_lse)
    s.synchronize()
    assert_out_close(y, o.lse_combine(raw(outputs), orc.BF16, raw(lses)), "side stream")


def test_errors_raise():
    x = torch.zeros((2, 4, 8, 12), dtype=torch.bfloat16, device="cuda")     # 24-byte rows
    with pytest.raises(dcp.DCPError) as e:
        dcp.lse_weighted_combine(x, torch.zeros((2, 4, 8), device="cuda"))
    assert e.value.status == 3
    with pytest.raises(ValueError):
        dcp.pack(torch.zeros((2, 6, 128), dtype=torch.bfloat16, device="cuda"), torch.zeros((2, 6), device="cuda"), 4)


# ---- layouts of the received shards (strided combine) -------------------------------------
@pytest.mark.parametrize("token_dim", [1, 2])
@pytest.mark.parametrize("dtype", ["bf16", "fp16", "fp32"])
def test_merge_layouts(o, token_dim, dtype):
    """The merge layouts of vllm-ascend sfa_cp.py: tokens on dim 1 ([N, T, H, D], tokens scattered)
    or on dim 2 ([N, H, T, D], heads scattered); the result is [T, H, D] contiguous."""
    w, outputs, lses = _case(6, 37, 5, 128, dtype, 13)
    ref_y, ref_g = o.lse_combine(raw(outputs), ORACLE_CODE[outputs.dtype], raw(lses), return_lse=True)
    if token_dim == 2:
        recv, lrecv = outputs.permute(0, 2, 1, 3).contiguous(), lses.permute(0, 2, 1).contiguous()
    else:
        recv, lrecv = outputs, lses
    y, g = dcp.merge_dcp_outputs(recv.cuda(), lrecv.cuda(), token_dim, return_lse=True)
    assert y.is_contiguous() and tuple(y.shape) == (37, 5, 128)
    assert_out_close(y, ref_y, f"merge token_dim={token_dim}")
    assert_lse_close(g, ref_g, f"merge token_dim={token_dim} lse")


def test_strided_views(o):
    """Every operand a permuted view of storage in another order."""
    N, B, H, D = 5, 19, 6, 64
    w, outputs, lses = _case(N, B, H, D, "bf16", 17)
    ref_y, ref_g = o.lse_combine(raw(outputs), orc.BF16, raw(lses), return_lse=True)
    out_store = outputs.permute(1, 2, 0, 3).contiguous().cuda()       # [B, H, N, D]
    lse_store = lses.permute(2, 0, 1).contiguous().cuda()              # [H, N, B]
    out_view = out_store.permute(2, 0, 1, 3)                           # [N, B, H, D]
    lse_view = lse_store.permute(1, 2, 0)                              # [N, B, H]
    res_store = torch.full((H, B, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    gl_store = torch.full((H, B), float("nan"), device="cuda")
    dcp.dcp_lse_combine(out_view, lse_view, res_store.permute(1, 0, 2), gl_store.t(), return_lse=True)
    assert_out_close(res_store.permute(1, 0, 2), ref_y, "strided result")
    assert_lse_close(gl_store.t(), ref_g, "strided global lse")


def test_mla_head_scattered_full_size(o):
    """The MLA workload received head-scattered ([N, Hr, B, D]), element by element."""
    w = wl.MLA
    outputs, lses = wl.split_inputs(w)
    recv = outputs.permute(0, 2, 1, 3).contiguous().cuda()
    lrecv = lses.permute(0, 2, 1).contiguous().cuda()
    y, g = dcp.merge_dcp_outputs(recv, lrecv, 2, return_lse=True, is_lse_base_on_e=False)
    ry, rg = o.lse_combine(raw(outputs), orc.BF16, raw(lses), return_lse=True, is_lse_base_on_e=False)
    assert_out_close(y, ry, "mla head-scattered")
    assert_lse_close(g, rg, "mla head-scattered lse")


def test_c_entry_points_directly(o):
    """dcp_lse_combine and dcp_lse_combine_strided called through ctypes with raw pointers agree
    with the oracle (and with each other) on the same capacity-strided buffers."""
    lib = dcp.library()
    N, T_max, B, H, D = 3, 40, 33, 4, 128
    w, outputs, lses = _case(N, T_max, H, D, "fp16", 23)
    d_out, d_lse = outputs.cuda(), lses.cuda()
    ry, rg = o.lse_combine(raw(outputs[:, :B]), orc.FP16, raw(lses[:, :B]), return_lse=True)
    y1 = torch.empty((B, H, D), dtype=torch.float16, device="cuda")
    g1 = torch.empty((B, H), device="cuda")
    y2, g2 = torch.empty_like(y1), torch.empty_like(g1)
    s = torch.cuda.current_stream().cuda_stream
    assert lib.dcp_lse_combine(d_out.data_ptr(), d_lse.data_ptr(), y1.data_ptr(), g1.data_ptr(), N, B, H, D,
                               T_max * H * D, T_max * H, 1, 1, 1, s) == 0
    assert lib.dcp_lse_combine_strided(d_out.data_ptr(), d_lse.data_ptr(), y2.data_ptr(), g2.data_ptr(), N, B, H, D,
                                       T_max * H * D, H * D, D, T_max * H, H, 1, H * D, D, H, 1, 1, 1, 1, s) == 0
    assert_out_close(y1, ry, "dcp_lse_combine")
    assert_lse_close(g1, rg, "dcp_lse_combine lse")
    assert torch.equal(y1, y2) and torch.equal(g1, g2)


def test_cuda_graph_replay(o):
    """pack + unpack+combine captured once in a CUDA graph and replayed on new inputs: the
    library allocates nothing and never synchronises, so the captured launches stay valid."""
    N, B, Hr, D = 4, 96, 8, 128
    H = N * Hr
    cp_out = torch.empty((B, H, D), dtype=torch.bfloat16, device="cuda")
    cp_lse = torch.empty((B, H), device="cuda")
    send = torch.empty((N, B, Hr, D + 2), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((B, Hr, D), dtype=torch.bfloat16, device="cuda")
    g = torch.empty((B, Hr), device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(2):  # warm-up (first calls set up per-device state) before capture
            dcp.dcp_pack(cp_out, cp_lse, send, N)
            dcp.dcp_unpack_combine(send, y, g, return_lse=True)
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        dcp.dcp_pack(cp_out, cp_lse, send, N)
        dcp.dcp_unpack_combine(send, y, g, return_lse=True)
    for seed in (31, 32):
        w = wl.CombineWorkload("graph", N=N, B=B, Hr=Hr, D=D, lse_lo=-5.0, lse_hi=15.0, p_neginf=0.1, seed=seed)
        h_out, h_lse = wl.pack_inputs(w)
        cp_out.copy_(h_out)
        cp_lse.copy_(h_lse)
        graph.replay()
        torch.cuda.synchronize()
        ref_send = o.pack(raw(h_out), raw(h_lse), N, orc.BF16)
        assert np.array_equal(bits(send.cpu()), bits(ref_send))
        ry, rg = o.unpack_combine(ref_send, orc.BF16, D, return_lse=True)
        assert_out_close(y, ry, f"graph replay seed {seed}")
        assert_lse_close(g, rg, f"graph replay seed {seed} lse")


def test_no_wait_timed_out():
    """Every bulk-copy wait of the kernels run so far completed within its limit (a timeout
    would mean an incomplete send buffer)."""
    torch.cuda.synchronize()
    assert dcp.dcp_wait_timeouts() == 0
    assert dcp.dcp_wait_timeouts(reset=True) == 0


PACK_EDGE = [  # B, H, D, world_size, dtype
    (3, 4, 8192, 2, "bf16"), (2, 3, 8192, 3, "fp32"), (5, 6, 4096, 3, "fp32"), (9, 5, 2048, 5, "bf16"),
    (301, 7, 8, 7, "bf16"), (97, 8, 4, 2, "fp32"), (130, 16, 128, 16, "fp16"), (64, 64, 64, 1, "bf16"),
    (1, 1, 16, 1, "fp16"), (33, 12, 520, 4, "bf16"), (3, 2, 1032, 2, "fp32")]


@pytest.mark.parametrize("B,H,D,ws,dtype", PACK_EDGE)
def test_pack_edge_shapes(o, B, H, D, ws, dtype):
    """Bit-exact pack for wide rows (one bulk copy of up to 32 KiB, one row per tile), 16-byte
    rows, many ragged tiles, world sizes 1 .. H, strided inputs and NaN payloads, with guard
    bands around the send buffer."""
    dt = wl.torch_dtype(dtype)
    gen = torch.Generator().manual_seed(B * 131 + H * 17 + D)
    big = torch.randn(B, H + 1, D + 8, generator=gen).to(dt)
    lse_big = torch.randn(B, H + 3, generator=gen)
    lse_big.view(torch.int32)[0, 0] = 0x7FC0ABCD         # NaN payload must survive
    if H > 1:
        lse_big[0, 1] = float("-inf")
    out, lse = big[:, 1:, :D], lse_big[:, :H]
    out_d = big.cuda()[:, 1:, :D]                        # strides (H+1)*(D+8), D+8, 1 on the device
    lse_d = lse_big.cuda()[:, :H]                        # row stride H+3
    assert out_d.stride() == ((H + 1) * (D + 8), D + 8, 1) and lse_d.stride() == (H + 3, 1)
    P = dcp.dcp_lse_pack_dim(dt)
    send = Guarded((ws, B, H // ws, D + P), dt)
    dcp.dcp_pack(out_d, lse_d, send.tensor, ws)
    send.check()
    ref = o.pack(raw(out.contiguous()), raw(lse.contiguous()), ws, ORACLE_CODE[dt])
    assert np.array_equal(bits(send.tensor.cpu()), bits(ref))
    assert dcp.dcp_wait_timeouts() == 0


PACK_RUNS = [  # B, H, D, world_size, dtype: contiguous heads
    (5000, 42, 64, 6, "bf16"),    # 128-byte rows, 7 heads per rank: runs cut by 256-row tiles
    (2000, 20, 32, 4, "fp32"),    # 128-byte fp32 rows
    (700, 24, 16, 3, "fp16"),     # 32-byte rows
    (64, 512, 128, 2, "bf16"),    # 256 heads per rank: runs longer than a 64-row tile
    (33, 12, 520, 4, "bf16"),     # 1040-byte rows, tiles of 31 rows
    (3000, 16, 512, 2, "bf16"),   # a short launch of 1 KiB rows
    (301, 7, 8, 7, "bf16"), (97, 8, 4, 2, "fp32"), (3, 4, 8192, 2, "bf16")]


@pytest.mark.parametrize("B,H,D,ws,dtype", PACK_RUNS)
def test_pack_head_runs(o, B, H, D, ws, dtype):
    """Contiguous heads, where a (rank, token)'s rows may be copied as one run: bit-exact
    against the oracle, with guard bands around the send buffer."""
    dt = wl.torch_dtype(dtype)
    gen = torch.Generator().manual_seed(B * 7 + H * 3 + D)
    out = torch.randn(B, H, D, generator=gen).to(dt)
    lse = torch.randn(B, H, generator=gen)
    lse.view(torch.int32)[0, 0] = 0x7FC0ABCD             # NaN payload must survive
    P = dcp.dcp_lse_pack_dim(dt)
    send = Guarded((ws, B, H // ws, D + P), dt)
    dcp.dcp_pack(out.cuda(), lse.cuda(), send.tensor, ws)
    send.check()
    ref = o.pack(raw(out), raw(lse), ws, ORACLE_CODE[dt])
    assert np.array_equal(bits(send.tensor.cpu()), bits(ref))
    assert dcp.dcp_wait_timeouts() == 0


@pytest.mark.parametrize("B,H,D,ws,dtype,pad", [(3000, 96, 512, 3, "bf16", 0), (4000, 64, 512, 4, "bf16", 0),
                                               (4000, 64, 256, 4, "fp32", 0), (2000, 128, 512, 4, "fp16", 0),
                                               (4000, 64, 512, 4, "bf16", 8)])
def test_pack_rank_fast_order(o, B, H, D, ws, dtype, pad):
    """Long launches of rows of 1 KiB and more for 3 or 4 ranks, where the pack's tiles run
    in rank-fastest order and never straddle a rank (each rank's last tile is partial here):
    bit-exact against the oracle, with guard bands around the send buffer.  pad > 0: heads
    `D + pad` elements apart, so every row is a copy of its own."""
    dt = wl.torch_dtype(dtype)
    gen = torch.Generator().manual_seed(B + H + D + ws)
    big = torch.randn(B, H, D + pad, generator=gen).to(dt)
    out = big[:, :, :D]
    lse = torch.randn(B, H, generator=gen)
    lse[B // 2, H - 1] = float("-inf")
    P = dcp.dcp_lse_pack_dim(dt)
    send = Guarded((ws, B, H // ws, D + P), dt)
    dcp.dcp_pack(big.cuda()[:, :, :D], lse.cuda(), send.tensor, ws)
    assert dcp.library().dcp_testing_last_pack_kernel() == 3   # pack_kernel, rank-fastest tiles
    send.check()
    ref = o.pack(raw(out.contiguous()), raw(lse), ws, ORACLE_CODE[dt])
    assert np.array_equal(bits(send.tensor.cpu()), bits(ref))
    assert dcp.dcp_wait_timeouts() == 0


def test_concurrent_host_threads(o):
    """Four host threads, each with its own stream and inputs, pack and combine at the same
    time (first calls included, which set up each kernel instance): every result matches the
    oracle."""
    import threading
    cases = [wl.CombineWorkload(f"thr{i}", N=N, B=B, Hr=Hr, D=D, dtype=dt, lse_lo=-5.0, lse_hi=15.0, p_neginf=0.05,
                                seed=70 + i)
             for i, (N, B, Hr, D, dt) in enumerate([(4, 300, 8, 128, "bf16"), (8, 120, 4, 512, "fp16"),
                                                    (2, 500, 16, 64, "fp32"), (16, 64, 2, 256, "bf16")])]
    inputs = [wl.split_inputs(w) for w in cases]
    results = [None] * len(cases)
    errors = []
    start = threading.Barrier(len(cases))

    def work(i):
        try:
            w = cases[i]
            outputs, lses = inputs[i]
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                d_out, d_lse = outputs.cuda(), lses.cuda()
                start.wait()
                y, g = dcp.lse_weighted_combine(d_out, d_lse, return_lse=True)
                cp_out = d_out.permute(1, 0, 2, 3).reshape(w.B, w.H, w.D).contiguous()
                cp_lse = d_lse.permute(1, 0, 2).reshape(w.B, w.H).contiguous()
                y2, g2 = dcp.unpack_combine(dcp.pack(cp_out, cp_lse, w.N), return_lse=True)
            s.synchronize()
            results[i] = (y.cpu(), g.cpu(), y2.cpu(), g2.cpu())
        except Exception as e:  # reported on the main thread
            errors.append(e)

    ts = [threading.Thread(target=work, args=(i,)) for i in range(len(cases))]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    assert not errors, errors
    for w, (outputs, lses), (y, g, y2, g2) in zip(cases, inputs, results):
        ry, rg = o.lse_combine(raw(outputs), ORACLE_CODE[outputs.dtype], raw(lses), return_lse=True)
        assert_out_close(y, ry, f"{w.name} combine")
        assert_lse_close(g, rg, f"{w.name} combine lse")
        assert_out_close(y2, ry, f"{w.name} pack + unpack_combine")
        assert_lse_close(g2, rg, f"{w.name} pack + unpack_combine lse")
