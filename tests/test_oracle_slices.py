"""The oracle over token slices on several host threads (used by the full-size GPU parity tests
and the bench's CPU baseline) gives exactly the whole-array results: the slices only address
rows in place, so every row is computed by the same C code on the same bits."""
from __future__ import annotations

import numpy as np
import pytest

import oracle as orc
from decode_context_attention_dcp_b200 import workloads as wl
from gpu_util import packed_from_split, raw


@pytest.fixture(scope="module")
def o() -> orc.Oracle:
    return orc.load()


@pytest.mark.parametrize("dtype", ["bf16", "fp16", "fp32"])
@pytest.mark.parametrize("threads", [1, 3, 8])
def test_token_slices_equal_whole_call(o, dtype, threads):
    w = wl.CombineWorkload("slices", N=5, B=37, Hr=3, D=64, dtype=dtype, lse_lo=-20.0, lse_hi=20.0, p_neginf=0.1,
                           p_nan=0.05, empty_every=7, seed=3)
    outputs, lses = wl.split_inputs(w)
    code = {"bf16": orc.BF16, "fp16": orc.FP16, "fp32": orc.FP32}[dtype]
    ro, rl = raw(outputs), raw(lses)
    for base_e in (True, False):
        y, g = o.lse_combine(ro, code, rl, return_lse=True, is_lse_base_on_e=base_e)
        for b0, b1 in [(0, 37), (5, 29), (36, 37), (10, 10)]:
            ys, gs = o.lse_combine_tokens(ro, code, rl, b0, b1, return_lse=True, is_lse_base_on_e=base_e,
                                          threads=threads)
            assert np.array_equal(ys, y[b0:b1]) and np.array_equal(gs, g[b0:b1])
        recv = raw(packed_from_split(outputs, lses))
        yu, gu = o.unpack_combine(recv, code, w.D, return_lse=True, is_lse_base_on_e=base_e)
        ys, gs = o.unpack_combine_tokens(recv, code, w.D, 3, 31, return_lse=True, is_lse_base_on_e=base_e,
                                         threads=threads)
        assert np.array_equal(ys, yu[3:31]) and np.array_equal(gs, gu[3:31])


@pytest.mark.parametrize("threads", [1, 4])
def test_varlen_token_slices_equal_whole_call(o, threads):
    w = wl.CombineWorkload("slices_varlen", N=4, B=61, Hr=2, D=32, lse_lo=-5.0, lse_hi=15.0, p_neginf=0.05, seed=9)
    outputs, lses = wl.split_inputs(w)
    seq_lens, qsl = wl.decode_batch(wl.DecodeBatch(B=61, max_q=3, pad=5, p_short=0.5, short_max=8, max_seq=40,
                                                   seed=9))
    ro, rl = raw(outputs), raw(lses)
    for interleave in (1, 2):
        y, g = o.lse_combine_varlen(ro, orc.BF16, rl, seq_lens.numpy(), qsl.numpy(), interleave, return_lse=True)
        for b0, b1 in [(0, 61), (7, 60), (55, 61)]:
            ys, gs = o.lse_combine_varlen_tokens(ro, orc.BF16, rl, seq_lens.numpy(), qsl.numpy(), b0, b1,
                                                 interleave, return_lse=True, threads=threads)
            assert np.array_equal(ys, y[b0:b1], equal_nan=True) and np.array_equal(gs, g[b0:b1])
