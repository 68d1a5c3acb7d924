"""Parity of the combine fused with the pack (dcp_combine_pack) with the oracle.

The fused call merges a producer's S split partials and writes the merged rows, head-scattered,
into the packed send buffer, each followed by its merged fp32 LSE.  The data slots are compared
with the oracle's combine within the output tolerance and the LSE slots within the LSE
tolerance; the whole buffer must also equal, bit for bit, the two-step GPU path (dcp_lse_combine
with return_lse, then dcp_pack), which runs the same arithmetic.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import decode_context_attention_dcp_b200 as dcp
import oracle as orc
from decode_context_attention_dcp_b200 import workloads as wl
from gpu_util import (HOST_THREADS, ORACLE_CODE, Guarded, assert_lse_close, assert_out_close, bits,
                      compare_token_blocks, raw)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def o() -> orc.Oracle:
    return orc.load()


def split_packed(send: torch.Tensor, H: int):
    """A packed send buffer [N, B, Hr, D + P] back to the merged rows [B, H, D] and the fp32
    LSEs [B, H] it holds (pure reindexing and reinterpretation, no arithmetic)."""
    N, B, Hr, W = send.shape
    P = 1 if send.dtype == torch.float32 else 2
    D = W - P
    data = send[..., :D].permute(1, 0, 2, 3).reshape(B, H, D)
    tail = send[..., D:].contiguous()
    lse = (tail.view(torch.float32) if P == 2 else tail).reshape(N, B, Hr).permute(1, 0, 2).reshape(B, H)
    return data, lse


def two_step(outputs, lses, world_size, base_e):
    S, B, H, D = outputs.shape
    y = torch.empty((B, H, D), dtype=outputs.dtype, device=outputs.device)
    g = torch.empty((B, H), dtype=torch.float32, device=outputs.device)
    dcp.dcp_lse_combine(outputs, lses, y, g, is_lse_base_on_e=base_e, return_lse=True)
    send = torch.empty((world_size, B, H // world_size, D + dcp.dcp_lse_pack_dim(outputs.dtype)),
                       dtype=outputs.dtype, device=outputs.device)
    dcp.dcp_pack(y, g, send, world_size)
    return send


CASES = [  # S splits, B tokens, H heads of the producer, D, world_size
    (1, 5, 4, 64, 2), (2, 37, 12, 128, 4), (4, 9, 32, 512, 8), (3, 7, 6, 96, 3), (8, 16, 16, 128, 16),
    (5, 3, 10, 1024, 5), (2, 11, 8, 2048, 4), (16, 4, 4, 256, 1), (64, 2, 2, 128, 2), (7, 33, 5, 16, 5)]


@pytest.mark.parametrize("dtype", ["bf16", "fp16", "fp32"])
@pytest.mark.parametrize("S,B,H,D,ws", CASES)
def test_combine_pack_matches_oracle(o, dtype, S, B, H, D, ws):
    if dtype == "fp32" and D % 4:
        pytest.skip("fp32 rows need D % 4 == 0")
    seed = S * 31 + B * 7 + H + D
    for base_e in (True, False):
        w = wl.CombineWorkload(f"cp_S{S}_B{B}_H{H}_D{D}", N=S, B=B, Hr=H, D=D, dtype=dtype, lse_lo=-20.0,
                               lse_hi=20.0, p_neginf=0.1, p_nan=0.03, empty_every=5, is_lse_base_on_e=base_e,
                               seed=seed)
        outputs, lses = wl.split_inputs(w)
        d_out, d_lse = outputs.cuda(), lses.cuda()
        send = Guarded((ws, B, H // ws, D + dcp.dcp_lse_pack_dim(d_out.dtype)), d_out.dtype)
        dcp.dcp_combine_pack(d_out, d_lse, send.tensor, ws, is_lse_base_on_e=base_e)
        send.check()
        ry, rg = o.lse_combine(raw(outputs), ORACLE_CODE[outputs.dtype], raw(lses), return_lse=True,
                               is_lse_base_on_e=base_e)
        data, lse = split_packed(send.tensor, H)
        assert_out_close(data, ry, f"{w.name} base_e={base_e} rows")
        assert_lse_close(lse, rg, f"{w.name} base_e={base_e} lse")
        ref = two_step(d_out, d_lse, ws, base_e)
        assert np.array_equal(bits(send.tensor.cpu()), bits(ref.cpu())), f"{w.name}: differs from combine + pack"


def test_combine_pack_capacity_strided_splits(o):
    """Split partials with room for T_max > B tokens."""
    S, T_max, B, H, D, ws = 4, 50, 41, 8, 128, 4
    w = wl.CombineWorkload("cp_cap", N=S, B=T_max, Hr=H, D=D, lse_lo=-5.0, lse_hi=15.0, p_neginf=0.05, seed=61)
    outputs, lses = wl.split_inputs(w)
    d_out, d_lse = outputs.cuda()[:, :B], lses.cuda()[:, :B]
    send = dcp.combine_pack(d_out, d_lse, ws)
    ry, rg = o.lse_combine(raw(outputs[:, :B]), orc.BF16, raw(lses[:, :B]), return_lse=True)
    data, lse = split_packed(send, H)
    assert_out_close(data, ry, "capacity-strided combine_pack")
    assert_lse_close(lse, rg, "capacity-strided combine_pack lse")
    assert torch.equal(send.view(torch.int16), two_step(d_out, d_lse, ws, True).view(torch.int16))


def test_combine_pack_large_elementwise(o):
    """A flash-decoding-sized producer (S=4 splits, B=2048 tokens, H=256 heads, D=512, bf16,
    2.1 GB of partials) into the 16-rank send buffer: every merged row and LSE against the
    oracle (token slices on all host cores), the whole buffer against the two-step path."""
    S, B, H, D, ws = 4, 2048, 256, 512, 16
    w = wl.CombineWorkload("cp_large", N=S, B=B, Hr=H, D=D, lse_lo=-5.0, lse_hi=25.0, p_neginf=0.02, seed=62)
    outputs, lses = wl.split_inputs(w)
    d_out, d_lse = outputs.cuda(), lses.cuda()
    send = dcp.combine_pack(d_out, d_lse, ws)
    torch.cuda.synchronize()
    data, lse = split_packed(send, H)
    ro, rl = raw(outputs), raw(lses)

    def ref(b0, b1):
        return o.lse_combine_tokens(ro, orc.BF16, rl, b0, b1, return_lse=True, threads=HOST_THREADS)

    compare_token_blocks(B, H * D, ref, [(data, "dcp_combine_pack rows")], [(lse, "dcp_combine_pack lse")],
                         "large combine_pack")
    assert torch.equal(send.view(torch.int16), two_step(d_out, d_lse, ws, True).view(torch.int16))


def test_combine_pack_errors():
    x = torch.zeros(2, 4, 6, 64, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(2, 4, 6, device="cuda")
    with pytest.raises(ValueError):
        dcp.combine_pack(x, lse, 4)  # 6 heads over 4 ranks
    send = torch.empty((3, 4, 2, 66), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        dcp.dcp_combine_pack(x, lse, send[:, :2], 3)  # wrong send shape
    # a send buffer 4 bytes off a 16-byte boundary is refused before any launch
    st = dcp.library().dcp_combine_pack(x.data_ptr(), lse.data_ptr(), send.data_ptr() + 4, 2, 4, 6, 64, 4 * 6 * 64,
                                        24, 3, 0, 1, None)
    assert st == 3 and "16-byte aligned" in dcp.dcp_last_error()
