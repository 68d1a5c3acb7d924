"""The host's launch-shape rules for the split-layout combine, checked without a GPU through
dcp_testing_split_shape, over every shard count and every row length the library accepts.

The property that matters for correctness: dcp_lse_combine, dcp_lse_combine_varlen (when
every shard holds KV) and dcp_combine_pack (against dcp_lse_combine followed by dcp_pack) give
the same bits because they sum each row's weights the same way. Lane j of G sums shards j,
j + G, ... in order, then the G lanes reduce by halving; two lane counts G1 < G2 therefore
add the same pairs in the same order exactly when N <= 2 * G1. The first test checks that
arithmetic fact directly in fp32 on adversarial weights. The second checks that the shapes
the host picks only ever differ where it holds.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest

import decode_context_attention_dcp_b200 as dcp

MAX_SHARDS = 64
MAX_CHUNKS = 2048          # D * elemsize / 16 for D = 8192 fp32
PLAIN, VARLEN, PACK = 0, 1, 2


def lane_sum(w: np.ndarray, G: int) -> np.float32:
    """The device's weight sum with G lanes, in fp32: sequential per lane, then xor halving."""
    lanes = [np.float32(0.0)] * G
    for n, x in enumerate(w):
        lanes[n % G] = np.float32(lanes[n % G] + x)
    off = G // 2
    while off:
        lanes = [np.float32(lanes[j] + lanes[j ^ off]) for j in range(G)]
        off //= 2
    return lanes[0]


@pytest.mark.parametrize("G1,G2", [(4, 8), (4, 16), (8, 16), (8, 32), (16, 32), (4, 32)])
def test_lane_counts_agree_up_to_twice_the_smaller(G1, G2):
    """The reduction fact the shape rules rely on, with weights spread over 40 binades so that
    any change of summation order shows in the last bit."""
    rng = np.random.default_rng(G1 * 100 + G2)
    for N in range(1, 2 * G1 + 1):
        for _ in range(50):
            w = (rng.random(N) * np.exp2(rng.integers(-20, 20, N))).astype(np.float32)
            assert lane_sum(w, G1) == lane_sum(w, G2), (N, w)
    differs = 0
    for _ in range(200):
        w = (rng.random(2 * G1 + 1) * np.exp2(rng.integers(-20, 20, 2 * G1 + 1))).astype(np.float32)
        differs += lane_sum(w, G1) != lane_sum(w, G2)
    assert differs > 0      # beyond 2 * G1 shards the orders really differ


@pytest.fixture(scope="module")
def shapes():
    lib = dcp.library()
    fn = lib.dcp_testing_split_shape
    fn.restype = ctypes.c_int32
    fn.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32)]
    out = (ctypes.c_int32 * 4)()
    table = {}
    for kind in (PLAIN, VARLEN, PACK):
        for N in range(1, MAX_SHARDS + 1):
            for c in range(1, MAX_CHUNKS + 1):
                assert fn(kind, N, c, out) == 0
                table[kind, N, c] = tuple(out)
    return table


def test_invalid_arguments():
    lib = dcp.library()
    out = (ctypes.c_int32 * 4)()
    fn = lib.dcp_testing_split_shape
    for args in [(3, 8, 16), (-1, 8, 16), (0, 0, 16), (0, MAX_SHARDS + 1, 16), (0, 8, 0)]:
        assert fn(*args, out) == 1
    assert fn(0, 8, 16, None) == 1


def test_shapes_are_instantiated_and_bounded(shapes):
    """Every shape is one the launcher has a kernel instance for, with 4-16 loads in flight per
    lane; single-slot shapes have at most 8 lanes, the 2 x 2 shape 4, the 2 x 8 shape occurs
    only for the variable-length rows of 8 lanes and the fused pack."""
    for (kind, N, c), (G, cpl, nb, pf) in shapes.items():
        assert G in (4, 8, 16, 32) and cpl in (1, 2, 4) and nb in (2, 4, 8) and pf in (0, 1)
        assert 4 <= cpl * nb <= 16
        if cpl == 1:
            assert nb == 8 and G <= 8
        if (cpl, nb) == (2, 2):
            assert G == 4
        if (cpl, nb) == (2, 8):
            assert kind == PACK or (kind == VARLEN and G == 8 and 8 < c <= 16 and N >= 8)
        if kind == PACK:
            assert pf == 0
        if kind == VARLEN:
            assert pf == 1
        slots = -(-c // G)
        assert cpl <= max(slots, 1) or (cpl == 4 and slots == 3), (kind, N, c, G, cpl)


def test_weight_sums_match_the_plain_combine(shapes):
    """Wherever the variable-length or fused-pack shape differs from the plain one in lanes per
    row, N <= 2 * the smaller lane count, so every entry point sums the weights alike."""
    for N in range(1, MAX_SHARDS + 1):
        for c in range(1, MAX_CHUNKS + 1):
            Gp = shapes[PLAIN, N, c][0]
            for kind in (VARLEN, PACK):
                G = shapes[kind, N, c][0]
                assert G == Gp or N <= 2 * min(G, Gp), (kind, N, c, G, Gp)


# ---- the tensor-copy pack's tile shape (dcp_testing_pack_tensor_shape) ----------------------

BOX_BYTES = 65536


@pytest.fixture(scope="module")
def tensor_shape():
    fn = dcp.library().dcp_testing_pack_tensor_shape
    fn.restype = ctypes.c_int32
    fn.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, ctypes.c_int64, ctypes.POINTER(ctypes.c_int32)]
    out = (ctypes.c_int32 * 3)()

    def shape(Hr, D, dtype, B):
        assert fn(Hr, D, dtype, B, out) == 0
        return tuple(out)
    return shape


def test_tensor_shape_invalid_arguments():
    fn = dcp.library().dcp_testing_pack_tensor_shape
    out = (ctypes.c_int32 * 3)()
    for args in [(0, 128, 0, 16), (4, 0, 0, 16), (4, 128, 3, 16), (4, 128, -1, 16), (4, 128, 0, 0)]:
        assert fn(*args, out) == 1
    assert fn(4, 128, 0, 16, None) == 1


@pytest.mark.parametrize("dtype,es", [(0, 2), (1, 2), (2, 4)])
def test_tensor_shape_rules(tensor_shape, dtype, es):
    """For every row length the API accepts (D * elemsize a multiple of 16, up to 8192) and a
    spread of head and token counts: the tile is the largest k <= min(256, B) whose k x Hr rows
    fit 64 KiB, and each row is split into the fewest m pieces of at most 256 elements and a
    multiple of 16 bytes; no tile at all past 256 heads or one token's heads over 64 KiB."""
    step = 16 // es
    for D in range(step, 8193, step):
        # the expected split, by brute force over every divisor
        m_ref = next((m for m in range(1, 257) if D % m == 0 and D // m <= 256 and (D // m * es) % 16 == 0), None)
        for Hr in (1, 2, 3, 4, 7, 16, 64, 128, 255, 256, 257):
            for B in (1, 3, 1000, 100000):
                k, m, dims = tensor_shape(Hr, D, dtype, B)
                if Hr > 256 or Hr * D * es > BOX_BYTES or m_ref is None:
                    assert (k, m, dims) == (0, 0, 0), (D, Hr, B)
                    continue
                assert 1 <= k <= min(256, B) and k * Hr * D * es <= BOX_BYTES, (D, Hr, B, k)
                assert k == min(256, B) or (k + 1) * Hr * D * es > BOX_BYTES, (D, Hr, B, k)
                assert m == m_ref and dims == (3 if m == 1 else 4), (D, m, m_ref)


def test_tensor_shape_examples(tensor_shape):
    """The shapes the bench and sweep workloads take (16 heads per rank, bf16)."""
    assert tensor_shape(16, 512, 0, 16384) == (4, 2, 4)     # 4 tokens x 16 heads x 2 pieces of 256
    assert tensor_shape(16, 128, 0, 16384) == (16, 1, 3)
    assert tensor_shape(16, 64, 0, 32768) == (32, 1, 3)
    assert tensor_shape(2, 8192, 2, 3601) == (1, 32, 4)     # fp32: 32 KiB rows in 32 pieces
    assert tensor_shape(64, 512, 0, 3001) == (1, 2, 4)      # exactly 64 KiB per token
    assert tensor_shape(128, 512, 0, 2001) == (0, 0, 0)     # 128 KiB per token: no tile
