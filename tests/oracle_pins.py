"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Every function takes an ``Oracle`` (one build of ``oracle/dcp_oracle.c``) and
raises AssertionError when the build disagrees with the fact it checks.  The
facts are: hand-derived worked examples (tests/golden), closed forms and
invariants of the combine defined by vllm.v1.attention.ops.dcp_alltoall
._lse_weighted_combine (vLLM API docs), brute-force softmax attention, library
conversions (numpy float16, torch bfloat16), an independent layout expression of
the packed buffer of dcp_a2a_lse_reduce, and the softmax statement of the same
merge in vllm-ascend sfa_cp.py _merge_dcp_outputs_with_torch.

The same functions run against deliberately broken builds of the oracle (see
test_oracle_pins.py) to show each plausible mistake is caught.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

import oracle as orc

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
LN2 = math.log(2.0)


def _f(x) -> float:
    """JSON number or one of the strings "nan", "inf", "-inf"."""
    return float(x)


def bf16_bits(values) -> np.ndarray:
    """Raw bf16 bits (uint16) of values that bf16 represents exactly (checked)."""
    t = torch.tensor(np.asarray(values, dtype=np.float32))
    b = t.to(torch.bfloat16)
    assert torch.equal(b.to(torch.float32), t) or bool(torch.isnan(t).any()), "not exact in bf16"
    return b.view(torch.int16).numpy().view(np.uint16)


def random_case(rng: np.random.Generator, N: int, B: int, H: int, D: int, lo=-5.0, hi=15.0,
                p_neginf=0.0, p_nan=0.0, p_posinf=0.0, dtype="bf16"):
    """Random outputs (raw bits of dtype) and fp32 LSEs for oracle-only checks."""
    vals = rng.standard_normal((N, B, H, D)).astype(np.float32)
    t = torch.from_numpy(vals)
    if dtype == "bf16":
        raw = t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        code = orc.BF16
    elif dtype == "fp16":
        raw = t.to(torch.float16).view(torch.int16).numpy().view(np.uint16)
        code = orc.FP16
    else:
        raw = vals
        code = orc.FP32
    lses = rng.uniform(lo, hi, (N, B, H)).astype(np.float32)
    u = rng.uniform(0, 1, (N, B, H))
    lses[u < p_neginf] = -np.inf
    lses[(u >= p_neginf) & (u < p_neginf + p_nan)] = np.nan
    lses[(u >= p_neginf + p_nan) & (u < p_neginf + p_nan + p_posinf)] = np.inf
    return raw, code, lses


# ------------------------------------------------------------------------------------------
def pin_golden_examples(o: orc.Oracle) -> None:
    with open(os.path.join(GOLDEN, "combine_worked_examples.json")) as fh:
        cases = json.load(fh)["cases"]
    for c in cases:
        outs = np.asarray(c["outputs"], dtype=np.float32)
        N, D = outs.shape
        raw = bf16_bits(outs).reshape(N, 1, 1, D)
        lses = np.asarray([_f(x) for x in c["lses"]], dtype=np.float32).reshape(N, 1, 1)
        y, g = o.lse_combine(raw, orc.BF16, lses, return_lse=True, is_lse_base_on_e=c["base_e"])
        exp_y = np.asarray(c["result"], dtype=np.float64)
        np.testing.assert_allclose(y.reshape(D), exp_y, rtol=0, atol=1e-12, err_msg=c["name"])
        exp_g = _f(c["global_lse"])
        if math.isinf(exp_g):
            assert g[0, 0] == exp_g, (c["name"], g[0, 0])
        else:
            assert abs(g[0, 0] - exp_g) <= 1e-12, (c["name"], g[0, 0], exp_g)


def _hexwords(a, dtype: str) -> np.ndarray:
    npdt = np.uint32 if dtype == "fp32" else np.uint16
    return np.vectorize(lambda s: int(s, 16), otypes=[np.uint64])(np.asarray(a)).astype(npdt)


def pin_pack_golden(o: orc.Oracle) -> None:
    with open(os.path.join(GOLDEN, "pack_worked_examples.json")) as fh:
        cases = json.load(fh)["cases"]
    codes = {"bf16": orc.BF16, "fp16": orc.FP16, "fp32": orc.FP32}
    for c in cases:
        out = _hexwords(c["cp_attn_out"], c["dtype"])
        if c["dtype"] == "fp32":
            out = out.view(np.float32)
        lse = _hexwords(c["cp_attn_lse"], "fp32").view(np.float32)
        send = o.pack(out, lse, c["world_size"], codes[c["dtype"]])
        want = _hexwords(c["send"], c["dtype"])
        got = send.view(np.uint32 if c["dtype"] == "fp32" else np.uint16)
        assert got.shape == want.shape, (c["name"], got.shape, want.shape)
        assert np.array_equal(got, want), (c["name"], got, want)
        assert o.lse_pack_dim(codes[c["dtype"]]) == want.shape[-1] - c["D"]


def pin_pack_layout(o: orc.Oracle) -> None:
    """Pack equals an independent numpy expression of the layout, with strided inputs too."""
    rng = np.random.default_rng(7)
    for (B, H, D, N, dt) in [(3, 8, 16, 4, "bf16"), (5, 6, 8, 3, "fp16"), (2, 4, 4, 2, "fp32"), (1, 16, 24, 16, "bf16")]:
        es = 4 if dt == "fp32" else 2
        npdt = np.float32 if dt == "fp32" else np.uint16
        big = rng.integers(0, 2 ** (8 * es), size=(B, H + 3, D + 5), dtype=np.uint64).astype(npdt)
        out = big[:, 1:H + 1, 2:D + 2]                      # strided view [B, H, D]
        lse_big = rng.standard_normal((B, H + 2)).astype(np.float32)
        lse = lse_big[:, :H]
        code = {"bf16": orc.BF16, "fp16": orc.FP16, "fp32": orc.FP32}[dt]
        send = _pack_strided(o, big, lse_big, B, H, D, N, code, es)
        Hr = H // N
        payload = np.ascontiguousarray(out).reshape(B, N, Hr, D).transpose(1, 0, 2, 3)
        lse_slots = np.ascontiguousarray(lse).view(npdt).reshape(B, N, Hr, 4 // es).transpose(1, 0, 2, 3)
        want = np.concatenate([payload, lse_slots], axis=-1)
        assert send.shape == want.shape
        assert np.array_equal(send.view(npdt), want), (B, H, D, N, dt)


def _pack_strided(o, big, lse_big, B, H, D, N, code, es):
    """Call the oracle's pack on the [:, 1:H+1, 2:D+2] view of ``big`` through explicit strides."""
    Hr = H // N
    pack = o.lse_pack_dim(code)
    send = np.zeros((N, B, Hr, D + pack), dtype=big.dtype)
    base = big.ctypes.data + (1 * big.strides[1] + 2 * big.strides[2])
    rc = o.lib.oracle_pack(base, lse_big.ctypes.data, send.ctypes.data, B, H, D, N, code,
                           big.strides[0] // es, big.strides[1] // es, lse_big.strides[0] // 4)
    assert rc == 0
    return send


def pin_unpack_inverts_pack(o: orc.Oracle) -> None:
    rng = np.random.default_rng(11)
    B, H, D, N = 3, 8, 8, 4
    out = rng.integers(0, 2 ** 16, size=(B, H, D), dtype=np.uint64).astype(np.uint16)
    lse_bits = rng.integers(0, 2 ** 32, size=(B, H), dtype=np.uint64).astype(np.uint32)
    lse_bits[0, 0] = 0x7FC01234          # NaN with a payload
    lse_bits[0, 1] = 0x80000000          # -0.0
    lse = lse_bits.view(np.float32)
    send = o.pack(out, lse, N, orc.BF16)
    outs, lses = o.unpack(send, orc.BF16, D)
    Hr = H // N
    assert np.array_equal(outs, out.reshape(B, N, Hr, D).transpose(1, 0, 2, 3))
    assert np.array_equal(lses.view(np.uint32), lse_bits.reshape(B, N, Hr).transpose(1, 0, 2))


def pin_n1_identity(o: orc.Oracle) -> None:
    rng = np.random.default_rng(1)
    for dt in ("bf16", "fp16", "fp32"):
        raw, code, lses = random_case(rng, 1, 4, 3, 16, dtype=dt)
        y, g = o.lse_combine(raw, code, lses, return_lse=True)
        assert np.array_equal(y, o.decode(raw[0], code)), dt
        assert np.array_equal(g, lses[0].astype(np.float64)), dt
        y2, g2 = o.lse_combine(raw, code, lses, return_lse=True, is_lse_base_on_e=False)
        assert np.array_equal(y2, y) and np.array_equal(g2, g), dt


def pin_equal_lse_mean(o: orc.Oracle) -> None:
    rng = np.random.default_rng(2)
    for N in (2, 3, 8):
        raw, code, lses = random_case(rng, N, 3, 2, 8)
        lses[:] = lses[0:1]
        dec = o.decode(raw, code)
        for base_e in (True, False):
            y, g = o.lse_combine(raw, code, lses, return_lse=True, is_lse_base_on_e=base_e)
            np.testing.assert_allclose(y, dec.mean(axis=0), rtol=1e-13, atol=1e-14)
            shift = math.log(N) if base_e else math.log2(N)
            np.testing.assert_allclose(g, lses[0].astype(np.float64) + shift, rtol=0, atol=1e-12)


def pin_zero_weight_shard(o: orc.Oracle) -> None:
    """A -inf, NaN or +inf shard contributes nothing: same result as with that shard removed."""
    rng = np.random.default_rng(3)
    N, B, H, D = 5, 4, 3, 8
    raw, code, lses = random_case(rng, N, B, H, D)
    for special in (-np.inf, np.nan, np.inf):
        for k in (0, 2, N - 1):
            l2 = lses.copy()
            l2[k] = special
            y, g = o.lse_combine(raw, code, l2, return_lse=True)
            keep = [i for i in range(N) if i != k]
            yr, gr = o.lse_combine(raw[keep], code, lses[keep], return_lse=True)
            np.testing.assert_allclose(y, yr, rtol=1e-15, atol=1e-15)
            np.testing.assert_allclose(g, gr, rtol=1e-15, atol=1e-15)


def pin_all_empty(o: orc.Oracle) -> None:
    rng = np.random.default_rng(4)
    for N in (1, 3):
        raw, code, lses = random_case(rng, N, 2, 2, 8)
        lses[:, 1, :] = np.array([-np.inf, np.nan, np.inf])[np.arange(N) % 3][:, None]
        for base_e in (True, False):
            y, g = o.lse_combine(raw, code, lses, return_lse=True, is_lse_base_on_e=base_e)
            assert np.all(y[1] == 0.0) and not np.any(np.isnan(y))
            assert np.all(g[1] == -np.inf)
            assert np.all(np.isfinite(g[0]))


def pin_single_finite_shard(o: orc.Oracle) -> None:
    rng = np.random.default_rng(5)
    N = 4
    raw, code, lses = random_case(rng, N, 3, 2, 8)
    lses[[0, 1, 3]] = -np.inf
    y, g = o.lse_combine(raw, code, lses, return_lse=True)
    assert np.array_equal(y, o.decode(raw[2], code))
    assert np.array_equal(g, lses[2].astype(np.float64))


def pin_two_group_merge(o: orc.Oracle) -> None:
    """Combining groups {0..k-1} and {k..N-1} and then merging the two results (with their global
    LSEs) equals combining all N at once."""
    rng = np.random.default_rng(6)
    for N, k in ((4, 1), (5, 2), (8, 4), (3, 2)):
        raw, code, lses = random_case(rng, N, 3, 4, 16, p_neginf=0.15)
        lses[:, 0, 0] = -np.inf                     # one all-empty row
        for base_e in (True, False):
            y, g = o.lse_combine(raw, code, lses, return_lse=True, is_lse_base_on_e=base_e)
            ya, ga = o.lse_combine(raw[:k], code, lses[:k], return_lse=True, is_lse_base_on_e=base_e)
            yb, gb = o.lse_combine(raw[k:], code, lses[k:], return_lse=True, is_lse_base_on_e=base_e)
            ym, gm = o.lse_combine(np.stack([ya, yb]), orc.F64, np.stack([ga, gb]), return_lse=True,
                                   is_lse_base_on_e=base_e)
            np.testing.assert_allclose(ym, y, rtol=1e-12, atol=1e-12)
            fin = np.isfinite(g)
            np.testing.assert_allclose(gm[fin], g[fin], rtol=1e-12, atol=1e-12)
            assert np.array_equal(gm[~fin], g[~fin])


def pin_base2_equivalence(o: orc.Oracle) -> None:
    rng = np.random.default_rng(8)
    raw, code, lses = random_case(rng, 6, 4, 3, 8, p_neginf=0.1)
    l_e = lses.astype(np.float64)
    y_e, g_e = o.lse_combine(raw, code, l_e, return_lse=True, is_lse_base_on_e=True)
    y_2, g_2 = o.lse_combine(raw, code, l_e / LN2, return_lse=True, is_lse_base_on_e=False)
    np.testing.assert_allclose(y_2, y_e, rtol=1e-12, atol=1e-12)
    fin = np.isfinite(g_e)
    np.testing.assert_allclose(g_2[fin], g_e[fin] / LN2, rtol=1e-12, atol=1e-12)


def pin_shift_invariance(o: orc.Oracle) -> None:
    """Adding c to every shard's LSE leaves the output unchanged and adds c to the global LSE,
    also where exp(l) alone would overflow (c = 800 in base e, 1100 in base 2): the max shift
    has to be there."""
    rng = np.random.default_rng(12)
    raw, code, lses = random_case(rng, 5, 4, 3, 8, p_neginf=0.2)
    lses[:, 1, 2] = -np.inf
    base = lses.astype(np.float64)
    for base_e, c in ((True, 800.0), (False, 1100.0), (True, -800.0)):
        y, g = o.lse_combine(raw, code, base, return_lse=True, is_lse_base_on_e=base_e)
        ys, gs = o.lse_combine(raw, code, base + c, return_lse=True, is_lse_base_on_e=base_e)
        assert np.all(np.isfinite(ys))
        np.testing.assert_allclose(ys, y, rtol=1e-12, atol=1e-12)
        fin = np.isfinite(g)
        np.testing.assert_allclose(gs[fin], g[fin] + c, rtol=1e-12, atol=1e-9)
        assert np.array_equal(gs[~fin], g[~fin])


def pin_softmax_form(o: orc.Oracle) -> None:
    """The p3 steps and the softmax-over-shards statement of the Ascend merge agree."""
    rng = np.random.default_rng(9)
    raw, code, lses = random_case(rng, 7, 5, 3, 8, p_neginf=0.2, p_nan=0.1, p_posinf=0.05)
    lses[:, 2, 1] = -np.inf
    y = o.lse_combine(raw, code, lses)
    ys = o.softmax_merge(raw, code, lses)
    np.testing.assert_allclose(y, ys, rtol=1e-12, atol=1e-13)
    assert np.all(y[2, 1] == 0.0) and np.all(ys[2, 1] == 0.0)


def pin_local_seq_len(o: orc.Oracle) -> None:
    """Interleaved KV sharding: blocks of `interleave` positions dealt round-robin to the ranks."""
    for L in (0, 1, 7, 64, 65, 100):
        for cp in (1, 2, 3, 4):
            for inter in (1, 2, 16):
                counts = [0] * cp
                for p in range(L):
                    counts[(p // inter) % cp] += 1
                got = [o.local_seq_len(L, cp, r, inter) for r in range(cp)]
                assert got == counts, (L, cp, inter, got, counts)


def shard_positions(L: int, N: int, split: str, interleave: int = 1) -> list[list[int]]:
    if split == "contiguous":
        per = -(-L // N)
        return [list(range(r * per, min(L, (r + 1) * per))) for r in range(N)]
    return [[p for p in range(L) if (p // interleave) % N == r] for r in range(N)]


def pin_bruteforce_attention(o: orc.Oracle) -> None:
    """Per-shard softmax attention + LSE, combined, equals attention over the whole context."""
    rng = np.random.default_rng(10)
    H, D, L = 3, 16, 20
    to_bits = lambda a: torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    q = to_bits(rng.standard_normal((H, D)).astype(np.float32))
    k = to_bits(rng.standard_normal((L, H, D)).astype(np.float32))
    v = to_bits(rng.standard_normal((L, H, D)).astype(np.float32))
    scale = 1.0 / math.sqrt(D)
    for N, split, inter in ((2, "contiguous", 1), (2, "interleaved", 1), (3, "interleaved", 4),
                            (4, "contiguous", 1), (8, "interleaved", 4)):
        shards = shard_positions(L, N, split, inter)
        for r, pos in enumerate(shards):
            if split == "interleaved":
                assert len(pos) == o.local_seq_len(L, N, r, inter)
        for base_e in (True, False):
            full_o, full_l = o.attention(q, k, v, orc.BF16, list(range(L)), scale, base_e)
            outs, lses = [], []
            for pos in shards:
                so, sl = o.attention(q, k, v, orc.BF16, pos, scale, base_e)
                outs.append(so)
                lses.append(sl)
            outs = np.stack(outs)[:, None]          # [N, 1, H, D]
            lses = np.stack(lses)[:, None]          # [N, 1, H]
            y, g = o.lse_combine(outs, orc.F64, lses, return_lse=True, is_lse_base_on_e=base_e)
            np.testing.assert_allclose(y[0], full_o, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(g[0], full_l, rtol=1e-12, atol=1e-12)


ALL_PINS = [
    pin_golden_examples,
    pin_pack_golden,
    pin_pack_layout,
    pin_unpack_inverts_pack,
    pin_n1_identity,
    pin_equal_lse_mean,
    pin_zero_weight_shard,
    pin_all_empty,
    pin_single_finite_shard,
    pin_two_group_merge,
    pin_base2_equivalence,
    pin_shift_invariance,
    pin_softmax_form,
    pin_local_seq_len,
    pin_bruteforce_attention,
]


def pin_varlen_reduces_to_combine(o: orc.Oracle) -> None:
    """The variable-length reading against the plain combine: with every shard holding KV it is the
    plain combine; an empty shard is the shard's LSE set to -inf with its row never read (NaN
    there changes nothing); a token outside every request gives 0 and -inf."""
    rng = np.random.default_rng(13)
    N, B, H, D = 4, 9, 3, 8
    raw, code, lses = random_case(rng, N, B, H, D)
    # three requests: tokens [0,3), [3,7), [7,8); token 8 is padding
    qsl = [0, 3, 7, 8]
    for inter in (1, 2):
        full = [N * inter * 2, 50, 100]
        y, g = o.lse_combine_varlen(raw, code, lses, full, qsl, inter, return_lse=True)
        yp, gp = o.lse_combine(raw, code, lses, return_lse=True)
        np.testing.assert_array_equal(y[:8], yp[:8])
        np.testing.assert_array_equal(g[:8], gp[:8])
        assert np.all(y[8] == 0.0) and np.all(g[8] == -np.inf)
        short = [1, 2 * inter + 1, 0]       # request 0: shard 0 only; request 1: 2-3 shards; request 2: none
        dirty = raw.copy().view(np.uint16)
        l2 = lses.copy()
        for b in range(8):
            r = 0 if b < 3 else 1 if b < 7 else 2
            for n in range(N):
                if o.local_seq_len(short[r], N, n, inter) == 0:
                    dirty[n, b] = 0x7FC0          # NaN in the rows of empty shards
                    l2[n, b] = -np.inf
        yv, gv = o.lse_combine_varlen(dirty, code, lses, short, qsl, inter, return_lse=True)
        clean = raw.copy()
        clean[l2 == -np.inf] = 0
        yr, gr = o.lse_combine(clean, code, l2, return_lse=True)
        np.testing.assert_allclose(yv[:8], yr[:8], rtol=1e-15, atol=1e-15)
        assert np.array_equal(np.isinf(gv[:8]), np.isinf(gr[:8]))
        assert not np.any(np.isnan(yv))
        assert np.all(yv[8] == 0.0) and np.all(gv[8] == -np.inf)     # padding token
        assert np.all(yv[7] == 0.0) and np.all(gv[7] == -np.inf)   # request 2 has no KV anywhere


ALL_PINS.append(pin_varlen_reduces_to_combine)


def pin_varlen_golden(o: orc.Oracle) -> None:
    """Hand-derived worked examples of the variable-length reading (tests/golden)."""
    with open(os.path.join(GOLDEN, "varlen_worked_examples.json")) as fh:
        cases = json.load(fh)["cases"]
    for c in cases:
        outs = np.asarray([[[_f(x) for x in row] for row in shard] for shard in c["outputs"]], dtype=np.float32)
        N, T, D = outs.shape
        raw = bf16_bits(outs.reshape(-1)).reshape(N, T, 1, D)
        lses = np.asarray(c["lses"], dtype=np.float32).reshape(N, T, 1)
        y, g = o.lse_combine_varlen(raw, orc.BF16, lses, c["seq_lens"], c["query_start_loc"], c["interleave"],
                                    return_lse=True, is_lse_base_on_e=c["base_e"])
        np.testing.assert_allclose(y.reshape(T, D), np.asarray(c["result"], dtype=np.float64), rtol=0, atol=1e-12,
                                   err_msg=c["name"])
        for t, want in enumerate(c["global_lse"]):
            want = _f(want)
            if math.isinf(want):
                assert g[t, 0] == want, (c["name"], t, g[t, 0])
            else:
                assert abs(g[t, 0] - want) <= 1e-12, (c["name"], t, g[t, 0], want)


ALL_PINS.append(pin_varlen_golden)
