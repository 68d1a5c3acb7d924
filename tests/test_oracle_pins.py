"""The fp64 oracle against its pins, and deliberately broken oracle builds against the same pins.

A mutant is the oracle source with one plausible mistake planted by text
substitution (a flipped sign, a dropped clamp, a transposed index, ...),
compiled to a scratch directory on the CPU.  Each must fail at least one pin.
"""
from __future__ import annotations


import numpy as np
import pytest
import torch

import oracle as orc
import oracle_pins as pins


@pytest.fixture(scope="module")
def o() -> orc.Oracle:
    return orc.load()


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(o, pin):
    pin(o)


def test_bf16_decoder_matches_torch(o):
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = o.decode(bits, orc.BF16)
    want = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(want[~nan]))


def test_fp16_decoder_matches_numpy(o):
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = o.decode(bits, orc.FP16)
    want = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(want[~nan]))


def test_rejects_bad_arguments(o):
    out = np.zeros((2, 6, 4), dtype=np.uint16)
    lse = np.zeros((2, 6), dtype=np.float32)
    with pytest.raises(ValueError):
        o.pack(out, lse, 4, orc.BF16)        # 6 heads do not split over 4 ranks
    assert o.lse_pack_dim(9) == -1


# (description, text in dcp_oracle.c, replacement)
MUTANTS = [
    ("weight exponent sign flipped", "exp(l[n] - m) : pow(2.0, l[n] - m)", "exp(m - l[n]) : pow(2.0, m - l[n])"),
    ("base-2 weight computed with exp", "pow(2.0, l[n] - m)", "exp(l[n] - m)"),
    ("global LSE uses ln in base 2", "(is_lse_base_on_e ? log(S) : log2(S)) + m", "log(S) + m"),
    ("global LSE drops the max", "(is_lse_base_on_e ? log(S) : log2(S)) + m", "(is_lse_base_on_e ? log(S) : log2(S))"),
    ("clamp of the weight sum dropped", "double denom = S < 1e-10 ? 1e-10 : S;", "double denom = S;"),
    ("normalisation dropped", "w[n] = w[n] / denom;", "w[n] = w[n];"),
    ("+inf LSE not sanitised", "l[n] = (isnan(v) || isinf(v)) ? -INFINITY : v;", "l[n] = isnan(v) ? -INFINITY : v;"),
    ("max replaced by first shard", "if (l[n] > m) m = l[n];", "(void)0;"),
    ("output index transposed (h, b)",
     "load_elem(outputs, out_dtype, n * out_stride_n + (b * H + h) * D + d) * w[n];",
     "load_elem(outputs, out_dtype, n * out_stride_n + (h * B + b) * D + d) * w[n];"),
    ("LSE index ignores the shard stride",
     ": load_elem(lses, lse_dtype, n * lse_stride_n + b * H + h);",
     ": load_elem(lses, lse_dtype, b * H + h);"),
    ("pack sends interleaved heads", "int64_t head = r * Hr + h;", "int64_t head = h * world_size + r;"),
    ("pack puts the LSE first", "memcpy(d + D * es, &cp_attn_lse[b * lse_stride_b + head], 4);",
     "memmove(d + 4, d, (size_t)(D * es - 4)); memcpy(d, &cp_attn_lse[b * lse_stride_b + head], 4);"),
    ("pack rows ordered [B, N, Hr]", "int64_t dst_row = (r * B + b) * Hr + h;",
     "int64_t dst_row = (b * world_size + r) * Hr + h;"),
    ("fp16 exponent bias off by one", "ldexp((double)(1024 + frac), expo - 25)", "ldexp((double)(1024 + frac), expo - 24)"),
    ("fp16 subnormals flushed", "v = ldexp((double)frac, -24);", "v = 0.0;"),
    ("bf16 decoded from the low bits", "uint32_t w = (uint32_t)bits << 16;", "uint32_t w = (uint32_t)bits;"),
    ("attention LSE misses the max shift", "double lse_e = npos > 0 ? log(z) + mx : -INFINITY;",
     "double lse_e = npos > 0 ? log(z) : -INFINITY;"),
    ("varlen: empty shard keeps its LSE", "double v = (empty && empty[n]) ? -INFINITY", "double v = 0 ? -INFINITY"),
    ("varlen: empty shard row still read", "if (!(empty && empty[n]))", "if (1)"),
    ("varlen: request end inclusive", "query_start_loc[r] <= b && b < query_start_loc[r + 1]",
     "query_start_loc[r] <= b && b <= query_start_loc[r + 1]"),
    ("local seq len ignores rank", "int64_t rem = seq_len - base * cp_size - rank * interleave;",
     "int64_t rem = seq_len - base * cp_size;"),
]

# A mutant the pins cannot catch, on purpose: without the "all -inf max becomes 0" rule an
# all-empty row computes exp(-inf - -inf) = NaN, and the "NaN weight becomes 0" rule then gives
# exactly the same zero output and -inf global LSE.  The two rules are redundant in exact
# arithmetic, so no test can tell them apart; both are kept as the page states them.
EQUIVALENT_MUTANTS = [("all -inf max kept", "if (m == -INFINITY) m = 0.0;", "(void)0;")]


def _extra_checks(o: orc.Oracle) -> None:
    # the decoders, through the library routines, as pins of their own
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    for code, want in ((orc.FP16, bits.view(np.float16).astype(np.float64)),
                       (orc.BF16, torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy())):
        got = o.decode(bits, code)
        nan = np.isnan(want)
        assert np.array_equal(got[~nan], want[~nan])


@pytest.mark.parametrize("desc,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, desc, old, new):
    src = open(orc.SOURCE).read()
    assert src.count(old) == 1, f"mutation site not unique or missing: {old!r}"
    mutant_src = tmp_path / "mutant.c"
    mutant_src.write_text(src.replace(old, new))
    lib = orc.compile_oracle(str(mutant_src), str(tmp_path / "libmutant.so"))
    m = orc.Oracle(lib)
    failures = []
    for pin in pins.ALL_PINS + [_extra_checks]:
        try:
            pin(m)
        except (AssertionError, ValueError, FloatingPointError):
            failures.append(pin.__name__)
    assert failures, f"no pin caught the mutant: {desc}"


@pytest.mark.parametrize("desc,old,new", EQUIVALENT_MUTANTS, ids=[m[0] for m in EQUIVALENT_MUTANTS])
def test_equivalent_mutant_documented(tmp_path, desc, old, new):
    src = open(orc.SOURCE).read()
    assert src.count(old) == 1
    mutant_src = tmp_path / "mutant.c"
    mutant_src.write_text(src.replace(old, new))
    m = orc.Oracle(orc.compile_oracle(str(mutant_src), str(tmp_path / "libmutant.so")))
    for pin in pins.ALL_PINS:
        pin(m)      # passes: the two rules coincide, as the comment above explains
