"""Parity of the variable-length combine (dcp_lse_combine_varlen) with the oracle.

A token of request r combines only the shards that hold KV of r; the rows of the other shards
are never read, so the tests fill them with NaN and give them a large finite LSE (either one,
read by mistake, changes the result).  Tokens outside every request (padding slots) must come
out as 0 with a global LSE of -inf.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import decode_context_attention_dcp_b200 as dcp
import oracle as orc
from decode_context_attention_dcp_b200 import workloads as wl
from gpu_util import HOST_THREADS, ORACLE_CODE, assert_lse_close, assert_out_close, compare_token_blocks, raw

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def o() -> orc.Oracle:
    return orc.load()


def token_requests(qsl: torch.Tensor, B: int) -> np.ndarray:
    """Request index of each of the B token slots, -1 outside every request."""
    req = np.full(B, -1, dtype=np.int64)
    q = qsl.tolist()
    for r in range(len(q) - 1):
        req[q[r]:q[r + 1]] = r
    return req


def empty_mask(o, seq_lens: torch.Tensor, qsl: torch.Tensor, N: int, B: int, interleave: int) -> torch.Tensor:
    """[N, B] bool: shard n holds no KV for token b (the oracle's local length is 0), or b is padding."""
    sl = seq_lens.tolist()
    held = np.array([[o.local_seq_len(s, N, n, interleave) > 0 for n in range(N)] for s in sl],
                    dtype=bool).reshape(len(sl), N)
    req = token_requests(qsl, B)
    mask = np.ones((N, B), dtype=bool)
    real = req >= 0
    mask[:, real] = ~held[req[real]].T
    return torch.from_numpy(mask)


def dirty(outputs: torch.Tensor, lses: torch.Tensor, mask: torch.Tensor):
    """Copies with NaN in every row of an empty shard and LSE 80 there."""
    out, l = outputs.clone(), lses.clone()
    m = mask.to(out.device)
    out[m] = float("nan")
    l[m] = 80.0
    return out, l


def check_varlen(o, outputs, lses, seq_lens, qsl, interleave, base_e=True, what=""):
    N, B = outputs.shape[:2]
    mask = empty_mask(o, seq_lens, qsl, N, B, interleave)
    d_out, d_lse = dirty(outputs, lses, mask)
    y, g = dcp.lse_weighted_combine_varlen(d_out.cuda(), d_lse.cuda(), seq_lens.cuda(), qsl.cuda(),
                                           interleave=interleave, return_lse=True, is_lse_base_on_e=base_e)
    ry, rg = o.lse_combine_varlen(raw(d_out), ORACLE_CODE[outputs.dtype], raw(d_lse), seq_lens.numpy(),
                                  qsl.numpy(), interleave, return_lse=True, is_lse_base_on_e=base_e)
    assert_out_close(y, ry, f"{what} varlen")
    assert_lse_close(g, rg, f"{what} varlen lse")
    assert not bool(torch.isnan(y).any()), f"{what}: an empty shard's row was read"
    return y, g, mask


@pytest.mark.parametrize("dtype", ["bf16", "fp16", "fp32"])
@pytest.mark.parametrize("N,interleave,max_q", [(2, 1, 1), (4, 16, 2), (8, 1, 3), (16, 4, 1), (5, 64, 1)])
def test_varlen_matches_oracle(o, dtype, N, interleave, max_q):
    B, H, D = 301, 4, 128
    seed = N * 7 + interleave + max_q
    w = wl.CombineWorkload(f"varlen_N{N}_I{interleave}", N=N, B=B, Hr=H, D=D, dtype=dtype, lse_lo=-10.0,
                           lse_hi=20.0, p_neginf=0.05, seed=seed)
    outputs, lses = wl.split_inputs(w)
    seq_lens, qsl = wl.decode_batch(wl.DecodeBatch(B=B, max_q=max_q, pad=13, p_short=0.5,
                                                   short_max=N * interleave, max_seq=4 * N * interleave,
                                                   seed=seed))
    base_e = interleave != 4
    _, g, mask = check_varlen(o, outputs, lses, seq_lens, qsl, interleave, base_e, w.name)
    assert bool(mask.any()) and not bool(mask.all())
    assert bool(torch.isinf(g[int(qsl[-1]):]).all())  # padding slots


@pytest.mark.parametrize("N,D,dtype", [(8, 256, "bf16"), (8, 128, "bf16"), (16, 128, "bf16"), (4, 128, "bf16"),
                                       (3, 512, "bf16"), (4, 512, "bf16"), (8, 512, "bf16"), (16, 256, "bf16"),
                                       (32, 256, "bf16"), (33, 512, "bf16"), (64, 128, "bf16"), (16, 64, "bf16"),
                                       (8, 64, "bf16"), (8, 128, "fp32"), (5, 96, "fp16"), (2, 128, "bf16")])
def test_varlen_with_every_shard_full_is_the_plain_combine(o, N, D, dtype):
    """Requests whose KV reaches every shard and no padding: the weights are summed as
    dcp_lse_combine sums them (the same lanes per row, or lane counts that agree for this
    shard count), so the results are identical bit for bit."""
    B, H = 200, 8
    w = wl.CombineWorkload("varlen_full", N=N, B=B, Hr=H, D=D, dtype=dtype, lse_lo=-5.0, lse_hi=15.0,
                           p_neginf=0.1, p_nan=0.02, seed=41)
    outputs, lses = [t.cuda() for t in wl.split_inputs(w)]
    seq_lens, qsl = wl.decode_batch(wl.DecodeBatch(B=B, max_q=2, p_short=0.0, short_max=N, max_seq=5000,
                                                   seed=41))
    y, g = dcp.lse_weighted_combine_varlen(outputs, lses, seq_lens.cuda(), qsl.cuda(), return_lse=True)
    yp, gp = dcp.lse_weighted_combine(outputs, lses, return_lse=True)
    word = torch.int32 if y.element_size() == 4 else torch.int16
    assert torch.equal(y.view(word), yp.view(word))
    assert torch.equal(g.view(torch.int32), gp.view(torch.int32))


def test_varlen_without_requests(o):
    """No request at all: every slot is padding (0 output, -inf LSE) and nothing is read."""
    N, B, H, D = 4, 64, 2, 64
    out = torch.full((N, B, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((N, B, H), 50.0, device="cuda")
    y, g = dcp.lse_weighted_combine_varlen(out, lse, torch.zeros(0, dtype=torch.int32, device="cuda"),
                                           torch.zeros(1, dtype=torch.int32, device="cuda"), return_lse=True)
    assert bool((y == 0).all()) and bool(torch.isneginf(g).all())


def test_varlen_zero_length_requests(o):
    """Requests whose KV length is 0 (or negative) combine no shard; their neighbours are
    unaffected."""
    N, B, H, D = 4, 6, 2, 64
    w = wl.CombineWorkload("varlen_zero", N=N, B=B, Hr=H, D=D, seed=43)
    outputs, lses = wl.split_inputs(w)
    seq_lens = torch.tensor([0, 3, -100, 100, 1], dtype=torch.int32)
    qsl = torch.tensor([0, 1, 2, 4, 5, 6], dtype=torch.int32)
    y, g, _ = check_varlen(o, outputs, lses, seq_lens, qsl, 1, what="zero-length")
    assert bool((y[0] == 0).all()) and bool((y[2:4] == 0).all())
    assert bool(torch.isneginf(g[0]).all()) and bool(torch.isneginf(g[2:4]).all())


def test_varlen_capacity_strided(o):
    """Shards with room for T_max > B tokens (the direct-workspace receive buffers)."""
    N, T_max, B, H, D = 4, 90, 70, 4, 128
    w = wl.CombineWorkload("varlen_cap", N=N, B=T_max, Hr=H, D=D, dtype="fp16", lse_lo=-5.0, lse_hi=15.0,
                           seed=44)
    outputs, lses = wl.split_inputs(w)
    seq_lens, qsl = wl.decode_batch(wl.DecodeBatch(B=B, max_q=1, pad=6, p_short=0.6, short_max=N, max_seq=50,
                                                   seed=44))
    mask = empty_mask(o, seq_lens, qsl, N, T_max, 1)
    d_out, d_lse = dirty(outputs, lses, mask)
    dd_out, dd_lse = d_out.cuda(), d_lse.cuda()
    y = torch.empty((B, H, D), dtype=torch.float16, device="cuda")
    g = torch.empty((B, H), device="cuda")
    dcp.dcp_lse_combine_varlen(dd_out[:, :B], dd_lse[:, :B], y, seq_lens.cuda(), qsl.cuda(), g, return_lse=True)
    ry, rg = o.lse_combine_varlen(raw(d_out[:, :B]), orc.FP16, raw(d_lse[:, :B]), seq_lens.numpy(), qsl.numpy(),
                                  return_lse=True)
    assert_out_close(y, ry, "capacity-strided varlen")
    assert_lse_close(g, rg, "capacity-strided varlen lse")


def test_varlen_full_size_elementwise(o):
    """The bench's largest combine shape (N=16, B=16384, H=16, D=512, bf16) with a decode batch of
    short and long requests and padding: every element against the oracle (run over token
    slices on all host cores).  The rows of shards without KV hold NaN and their LSEs 80."""
    N, B, H, D = 16, 16384, 16, 512
    w = wl.by_name("sweep_N16_B16384_D512")
    outputs, lses = wl.split_inputs(w)
    seq_lens, qsl = wl.decode_batch(wl.DecodeBatch(B=B, max_q=2, pad=300, p_short=0.4, short_max=N, max_seq=9000,
                                                   seed=45))
    mask = empty_mask(o, seq_lens, qsl, N, B, 1)
    outputs[mask] = float("nan")
    lses[mask] = 80.0
    y, g = dcp.lse_weighted_combine_varlen(outputs.cuda(), lses.cuda(), seq_lens.cuda(), qsl.cuda(),
                                           return_lse=True)
    torch.cuda.synchronize()
    assert not bool(torch.isnan(y).any())
    pad0 = int(qsl[-1])
    assert bool((y[pad0:] == 0).all()) and bool(torch.isneginf(g[pad0:]).all())
    ro, rl = raw(outputs), raw(lses)

    def ref(b0, b1):
        return o.lse_combine_varlen_tokens(ro, orc.BF16, rl, seq_lens.numpy(), qsl.numpy(), b0, b1,
                                           return_lse=True, threads=HOST_THREADS)

    compare_token_blocks(B, H * D, ref, [(y, "dcp_lse_combine_varlen")], [(g, "dcp_lse_combine_varlen lse")],
                         "full-size varlen")


def test_varlen_errors():
    x = torch.zeros(2, 4, 2, 64, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(2, 4, 2, device="cuda")
    sl = torch.ones(2, dtype=torch.int32, device="cuda")
    q = torch.tensor([0, 2, 4], dtype=torch.int32, device="cuda")
    with pytest.raises(dcp.DCPError):
        dcp.lse_weighted_combine_varlen(x, lse, sl, q, interleave=0)
    with pytest.raises(ValueError):
        dcp.lse_weighted_combine_varlen(x, lse, sl, q[:2])
    with pytest.raises(ValueError):
        dcp.lse_weighted_combine_varlen(x, lse, sl.long(), q)


@pytest.mark.parametrize("dtype,D,N", [("bf16", 2048, 4), ("fp32", 1024, 3), ("fp16", 8192, 2), ("bf16", 512, 64)])
def test_varlen_wide_rows(o, dtype, D, N):
    """Rows that take several passes per lane group (and the most shards): the shards without
    KV are skipped in every pass."""
    B, H = 23, 2
    w = wl.CombineWorkload(f"varlen_wide_{dtype}_D{D}_N{N}", N=N, B=B, Hr=H, D=D, dtype=dtype, lse_lo=-5.0,
                           lse_hi=15.0, p_neginf=0.05, seed=D + N)
    outputs, lses = wl.split_inputs(w)
    seq_lens, qsl = wl.decode_batch(wl.DecodeBatch(B=B, max_q=2, pad=3, p_short=0.6, short_max=N, max_seq=4 * N,
                                                   seed=D + N))
    check_varlen(o, outputs, lses, seq_lens, qsl, 1, True, w.name)
