"""The pack with one tensor copy per tile (pack_tma_kernel), which long launches use when all
heads a rank holds of one token fit in 64 KiB: bit-exact against the oracle's pack, with guard
bands around the send buffer.  Every case is sized to be a long launch on a B200 and checks
which kernel ran (dcp_testing_last_pack_kernel).  A tile is k tokens with k = 64 KiB / (Hr x row
bytes); most cases leave B mod k != 0 tokens per rank, which a second launch of one tile per rank
packs.  The fallback cases check that shapes the tensor copy does not suit still take the other
kernels."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import decode_context_attention_dcp_b200 as dcp
import oracle as orc
from gpu_util import Guarded, bits, raw
from decode_context_attention_dcp_b200.workloads import torch_dtype

pytestmark = pytest.mark.gpu

ROWS, RUNS, RANK_FAST, TENSOR_3D, TENSOR_4D = 1, 2, 3, 4, 5
ORACLE_CODE = {torch.bfloat16: orc.BF16, torch.float16: orc.FP16, torch.float32: orc.FP32}


@pytest.fixture(scope="module")
def o() -> orc.Oracle:
    return orc.load()


def _pack_case(o, B, H, D, ws, dtype, pad_h=0, pad_b=0, seed=0, lse_pad=0):
    """Packs a [B, H, D] view whose heads are D + pad_h elements apart and whose tokens are
    H * (D + pad_h) + pad_b apart, with LSE rows H + lse_pad apart; returns the kernel that ran
    after checking the bits."""
    dt = torch_dtype(dtype)
    gen = torch.Generator().manual_seed(seed or B * 3 + H * 5 + D * 7 + ws)
    per_b = H * (D + pad_h) + pad_b
    flat = torch.randn(B * per_b, generator=gen).to(dt)
    view = flat.as_strided((B, H, D), (per_b, D + pad_h, 1))
    lse_big = torch.randn(B, H + lse_pad, generator=gen)
    lse = lse_big[:, :H]
    lse.view(torch.int32)[0, 0] = 0x7FC0ABCD            # NaN payload must survive
    lse[B - 1, H - 1] = float("-inf")
    d_flat = flat.cuda()
    d_view = d_flat.as_strided((B, H, D), (per_b, D + pad_h, 1))
    d_lse = lse_big.cuda()[:, :H]
    assert d_lse.stride() == (H + lse_pad, 1)
    P = dcp.dcp_lse_pack_dim(dt)
    send = Guarded((ws, B, H // ws, D + P), dt)
    dcp.dcp_pack(d_view, d_lse, send.tensor, ws)
    kernel = dcp.library().dcp_testing_last_pack_kernel()
    send.check()
    ref = o.pack(raw(view.contiguous()), raw(lse.contiguous()), ws, ORACLE_CODE[dt])
    assert np.array_equal(bits(send.tensor.cpu()), bits(ref))
    assert dcp.dcp_wait_timeouts() == 0
    return kernel


TENSOR_CASES = [  # B, H, D, world_size, dtype, kernel expected
    (2001, 128, 512, 8, "bf16", TENSOR_4D),   # 1 KiB rows split in 2 pieces of 256, k = 4
    (2048, 128, 512, 8, "bf16", TENSOR_4D),   # the same with B mod k = 0: no second launch
    (8001, 128, 128, 16, "bf16", TENSOR_3D),  # 256-byte rows, 8 heads per rank, k = 32
    (16001, 128, 64, 8, "bf16", TENSOR_3D),   # 128-byte rows, k = 32
    (4001, 128, 256, 8, "fp16", TENSOR_3D),   # 512-byte rows, k = 8
    (3001, 128, 384, 8, "bf16", TENSOR_4D),   # 768-byte rows in 2 pieces of 192, k = 5
    (6001, 128, 192, 4, "fp16", TENSOR_3D),   # 32 heads per rank of 384 bytes, k = 5
    (2001, 128, 256, 8, "fp32", TENSOR_3D),   # 1 KiB fp32 rows of 256 elements, k = 4
    (3601, 4, 8192, 2, "fp32", TENSOR_4D),    # 32 KiB rows in 32 pieces, 2 heads: one token a tile
    (2001, 128, 512, 16, "bf16", TENSOR_4D),  # 8 heads per rank, k = 8
    (8001, 128, 256, 64, "bf16", TENSOR_3D),  # 64 ranks of 2 heads, k = 64
    (8001, 256, 64, 1, "bf16", TENSOR_3D),    # 256 heads per rank (the box's limit), k = 2
    (3001, 256, 512, 4, "bf16", TENSOR_4D),   # 4 ranks of 64 heads, k = 1: 12004 tiles, over 64 per SM
    (1001, 256, 512, 4, "bf16", RANK_FAST),   # ... 4004 tiles: 4 ranks of 1 KiB rows keep the rank-fast order
    (2001, 128, 512, 1, "bf16", RANK_FAST),   # one rank: 128 KiB per token, over a tile
    (2001, 512, 128, 1, "bf16", ROWS),        # 512 heads per rank, over 256 per box
]


@pytest.mark.parametrize("B,H,D,ws,dtype,kernel", TENSOR_CASES)
def test_tensor_pack(o, B, H, D, ws, dtype, kernel):
    assert _pack_case(o, B, H, D, ws, dtype) == kernel


@pytest.mark.parametrize("B,H,D,ws,dtype,pad_h,pad_b,lse_pad,kernel", [
    (2001, 128, 512, 8, "bf16", 8, 0, 0, TENSOR_4D),    # heads D + 8 apart
    (8001, 128, 128, 16, "fp16", 0, 64, 0, TENSOR_3D),  # tokens 64 elements more than H D apart
    (2001, 128, 256, 8, "fp32", 4, 12, 0, TENSOR_3D),   # both
    (4001, 128, 256, 8, "bf16", 0, 0, 3, TENSOR_3D),    # LSE rows H + 3 apart
])
def test_tensor_pack_strided(o, B, H, D, ws, dtype, pad_h, pad_b, lse_pad, kernel):
    """The tensor map takes the head and token strides, so strided inputs keep the kernel."""
    assert _pack_case(o, B, H, D, ws, dtype, pad_h, pad_b, lse_pad=lse_pad) == kernel


def test_tensor_pack_stalled_wait_is_counted_and_the_device_stays_usable(o):
    """The timeout path of pack_tma_kernel's bounded wait: each CTA's first wait expects 16
    bytes more than its tensor copy brings and gives up after 20 ms; the kernel writes nothing,
    counts each CTA once, and the next, complete pack is bit-exact.  Here the whole tiles (k = 32
    tokens, 500 per rank) run on one CTA per SM, and the one token left per rank in a second
    launch of one CTA per rank."""
    B, H, D, ws = 16001, 128, 64, 8
    gen = torch.Generator().manual_seed(11)
    out = torch.randn(B, H, D, generator=gen).to(torch.bfloat16)
    lse = torch.randn(B, H, generator=gen)
    d_out, d_lse = out.cuda(), lse.cuda()
    send = torch.zeros((ws, B, H // ws, D + 2), dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    assert dcp.dcp_wait_timeouts(reset=True) == 0
    lib = dcp.library()
    st = lib.dcp_testing_pack_stalled(d_out.data_ptr(), d_lse.data_ptr(), send.data_ptr(), B, H, D, ws, 0,
                                      d_out.stride(0), d_out.stride(1), d_lse.stride(0),
                                      torch.cuda.current_stream().cuda_stream)
    assert st == 0, dcp.dcp_last_error()
    assert lib.dcp_testing_last_pack_kernel() == TENSOR_3D
    torch.cuda.synchronize()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert dcp.dcp_wait_timeouts(reset=True) == min(ws * (B // 32), sms) + ws
    assert bool((send.view(torch.int16) == 0).all())
    send2 = dcp.pack(d_out, d_lse, ws)
    assert lib.dcp_testing_last_pack_kernel() == TENSOR_3D
    torch.cuda.synchronize()
    assert dcp.dcp_wait_timeouts() == 0
    ref = o.pack(raw(out), raw(lse), ws, orc.BF16)
    assert np.array_equal(bits(send2.cpu()), bits(ref))


def test_tensor_pack_in_a_cuda_graph(o):
    """Both launches of a tensor-copy pack (whole tiles and the per-rank tail), captured once in
    a CUDA graph with their tensor map and replayed on new contents of the same buffers."""
    B, H, D, ws = 2001, 128, 512, 8
    cp_out = torch.empty((B, H, D), dtype=torch.bfloat16, device="cuda")
    cp_lse = torch.empty((B, H), device="cuda")
    send = torch.empty((ws, B, H // ws, D + 2), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(2):  # per-device set-up before capture
            dcp.dcp_pack(cp_out, cp_lse, send, ws)
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        dcp.dcp_pack(cp_out, cp_lse, send, ws)
    assert dcp.library().dcp_testing_last_pack_kernel() == TENSOR_4D
    for seed in (41, 42):
        gen = torch.Generator().manual_seed(seed)
        h_out = torch.randn(B, H, D, generator=gen).to(torch.bfloat16)
        h_lse = torch.randn(B, H, generator=gen)
        cp_out.copy_(h_out)
        cp_lse.copy_(h_lse)
        send.zero_()
        graph.replay()
        torch.cuda.synchronize()
        ref = o.pack(raw(h_out), raw(h_lse), ws, orc.BF16)
        assert np.array_equal(bits(send.cpu()), bits(ref))
    assert dcp.dcp_wait_timeouts() == 0
