"""The timeout path of the pack kernel's bounded wait, run on purpose without faulting or
hanging the GPU: dcp_testing_pack_stalled makes each CTA's first wait expect 16 bytes that
never arrive (every copy still lands) and gives up after 20 ms.  The kernel must return, count
each CTA once, write nothing, and leave the device usable for the next, complete pack."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import decode_context_attention_dcp_b200 as dcp
import oracle as orc
from gpu_util import bits, raw

pytestmark = pytest.mark.gpu


def test_stalled_wait_is_counted_and_the_device_stays_usable():
    B, H, D, ws = 40, 8, 128, 4          # 320 packed rows of 65 words: 5 tiles of 64 rows, one CTA each
    gen = torch.Generator().manual_seed(5)
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
    torch.cuda.synchronize()
    assert dcp.dcp_wait_timeouts(reset=True) == 5     # each of the 5 CTAs stopped once
    assert bool((send.view(torch.int16) == 0).all())  # ... before storing anything
    # the same pack without the stall: complete, bit-exact, and no wait runs out
    send2 = dcp.pack(d_out, d_lse, ws)
    torch.cuda.synchronize()
    assert dcp.dcp_wait_timeouts() == 0
    ref = orc.load().pack(raw(out), raw(lse), ws, orc.BF16)
    assert np.array_equal(bits(send2.cpu()), bits(ref))
