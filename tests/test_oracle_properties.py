"""Randomised properties of the fp64 oracle's combine (CPU only).

The combine of vllm.v1.attention.ops.dcp_alltoall._lse_weighted_combine (vLLM API docs) is a
softmax-weighted mean over the shard axis.  Whatever the shapes, values, base and special LSEs,
it must be invariant under a permutation of the shards, invariant (output) and equivariant
(global LSE) under one shift of every LSE, agree with the softmax statement of the same merge
in vllm-ascend sfa_cp.py _merge_dcp_outputs_with_torch, and treat a shard repeated k times
like one shard whose LSE is larger by log k.  The interleaved sharding of the variable-length
reading puts KV on a prefix of the shards.  Hypothesis draws the cases.
"""
from __future__ import annotations

import math

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle as orc
from oracle_pins import random_case

_O = None


def o() -> orc.Oracle:
    global _O
    if _O is None:
        _O = orc.load()
    return _O


cases = st.fixed_dictionaries({
    "N": st.integers(1, 9), "B": st.integers(1, 4), "H": st.integers(1, 3), "D": st.sampled_from([8, 16, 24]),
    "dtype": st.sampled_from(["bf16", "fp16", "fp32"]), "base_e": st.booleans(),
    "p_neginf": st.sampled_from([0.0, 0.2, 0.6]), "p_nan": st.sampled_from([0.0, 0.1]),
    "p_posinf": st.sampled_from([0.0, 0.1]), "seed": st.integers(0, 2**31 - 1)})


def _draw(c):
    rng = np.random.default_rng(c["seed"])
    return random_case(rng, c["N"], c["B"], c["H"], c["D"], lo=-20.0, hi=20.0, p_neginf=c["p_neginf"],
                       p_nan=c["p_nan"], p_posinf=c["p_posinf"], dtype=c["dtype"])


def _close(a, b, tol=1e-12):
    a, b = np.asarray(a), np.asarray(b)
    inf = np.isinf(b)
    assert np.array_equal(np.isinf(a), inf) and np.array_equal(a[inf], b[inf])
    np.testing.assert_allclose(a[~inf], b[~inf], rtol=tol, atol=tol)


@settings(max_examples=60, deadline=None)
@given(cases)
def test_shard_permutation_invariance(c):
    raw, code, lses = _draw(c)
    perm = np.random.default_rng(c["seed"] + 1).permutation(c["N"])
    y, g = o().lse_combine(raw, code, lses, return_lse=True, is_lse_base_on_e=c["base_e"])
    yp, gp = o().lse_combine(np.ascontiguousarray(raw[perm]), code, np.ascontiguousarray(lses[perm]),
                             return_lse=True, is_lse_base_on_e=c["base_e"])
    _close(yp, y)
    _close(gp, g)


@settings(max_examples=60, deadline=None)
@given(cases, st.sampled_from([-37.5, -3.0, 0.75, 12.0]))
def test_common_shift(c, shift):
    """Adding the same constant to every LSE leaves the output and moves the global LSE by it
    (f64 LSEs, so the shifted inputs are exact)."""
    raw, code, lses = _draw(c)
    l64 = lses.astype(np.float64)
    y, g = o().lse_combine(raw, code, l64, return_lse=True, is_lse_base_on_e=c["base_e"])
    ys, gs = o().lse_combine(raw, code, l64 + shift, return_lse=True, is_lse_base_on_e=c["base_e"])
    _close(ys, y, 1e-12)
    fin = np.isfinite(g)
    assert np.array_equal(np.isfinite(gs), fin)
    np.testing.assert_allclose(gs[fin], g[fin] + shift, rtol=1e-12, atol=1e-11)


@settings(max_examples=60, deadline=None)
@given(cases)
def test_softmax_statement(c):
    """The [ASCEND] softmax statement gives the same merge (base e)."""
    raw, code, lses = _draw(c)
    y = o().lse_combine(raw, code, lses)
    ys = o().softmax_merge(raw, code, lses)
    _close(ys, y, 1e-12)


@settings(max_examples=40, deadline=None)
@given(cases, st.integers(2, 4))
def test_repeated_shard_is_a_larger_lse(c, k):
    """Shard 0 repeated k times (k identical copies) merges like one shard 0 whose LSE is
    larger by log k (ln k in base e, log2 k in base 2)."""
    raw, code, lses = _draw(c)
    l64 = lses.astype(np.float64)
    rep = np.concatenate([np.repeat(raw[:1], k, axis=0), raw[1:]])
    lrep = np.concatenate([np.repeat(l64[:1], k, axis=0), l64[1:]])
    y, g = o().lse_combine(rep, code, lrep, return_lse=True, is_lse_base_on_e=c["base_e"])
    bumped = l64.copy()
    fin0 = np.isfinite(bumped[0])
    bumped[0][fin0] += math.log(k) if c["base_e"] else math.log2(k)
    yb, gb = o().lse_combine(raw, code, bumped, return_lse=True, is_lse_base_on_e=c["base_e"])
    _close(y, yb, 1e-12)
    _close(g, gb, 1e-12)


@settings(max_examples=200, deadline=None)
@given(st.integers(0, 20000), st.integers(1, 64), st.sampled_from([1, 2, 3, 4, 16, 64, 128]))
def test_shards_holding_kv_are_a_prefix(seq, N, interleave):
    """Under interleaved sharding (vllm-ascend sfa_cp.py _get_dcp_local_seq_lens) shard n holds
    positions of a request of length seq exactly when n * interleave < seq, so the shards
    holding KV are shards [0, k) with k = min(N, ceil(seq / interleave)) -- the criterion the
    variable-length kernels evaluate instead of the local length -- and the local lengths add
    up to seq."""
    lens = [o().local_seq_len(seq, N, n, interleave) for n in range(N)]
    assert sum(lens) == seq
    assert all(ln >= 0 for ln in lens)
    for n, ln in enumerate(lens):
        assert (ln > 0) == (n * interleave < seq), (seq, N, interleave, n, ln)
    k = min(N, -(-seq // interleave))
    assert [ln > 0 for ln in lens] == [n < k for n in range(N)]
