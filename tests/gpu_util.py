"""Shared helpers of the GPU parity tests: raw views for the oracle, the packed-buffer
construction for tests, tolerance checks, and guarded output buffers."""
from __future__ import annotations

import os

import numpy as np
import torch

import oracle as orc

# Tolerances.  Output: |err| <= 1e-2 * max(1, |ref|) for 16-bit outputs (one bf16/fp16 rounding
# of an fp32 accumulation); fp32 outputs: 2e-5 * max(1, |ref|) (fp32 accumulation of N terms).
# Global LSE (fp32): |err| <= 1e-4, and -inf must be exactly -inf.
OUT_TOL = {torch.bfloat16: 1e-2, torch.float16: 1e-2, torch.float32: 2e-5}
LSE_TOL = 1e-4
ORACLE_CODE = {torch.bfloat16: orc.BF16, torch.float16: orc.FP16, torch.float32: orc.FP32}
# Host threads the oracle may use on full-size inputs (token slices, see oracle.Oracle.*_tokens).
HOST_THREADS = max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1))


def raw(t: torch.Tensor) -> np.ndarray:
    """The bits of a CPU tensor as a numpy array the oracle reads (uint16 for 16-bit types)."""
    t = t.contiguous().cpu()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def bits(a) -> np.ndarray:
    """Integer view of a tensor's or array's elements (uint16 / uint32), for bit-exact comparison."""
    if isinstance(a, torch.Tensor):
        a = raw(a)
    return a.view(np.uint32) if a.dtype.itemsize == 4 else a.view(np.uint16)


def as_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().to(torch.float64).numpy()


def packed_from_split(outputs: torch.Tensor, lses: torch.Tensor) -> torch.Tensor:
    """A receive buffer [N, B, Hr, D + P] holding each row of ``outputs`` followed by the bit
    pattern of its fp32 LSE (memory order), built on the CPU from split inputs."""
    es = outputs.element_size()
    slots = lses.contiguous().unsqueeze(-1).view(outputs.dtype) if es == 2 else lses.contiguous().unsqueeze(-1)
    return torch.cat([outputs, slots.reshape(*lses.shape, 4 // es)], dim=-1).contiguous()


def assert_out_close(gpu: torch.Tensor, ref: np.ndarray, what: str = "") -> None:
    got = as_f64(gpu)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    tol = OUT_TOL[gpu.dtype]
    nan_ref, nan_got = np.isnan(ref), np.isnan(got)
    assert np.array_equal(nan_ref, nan_got), f"{what}: NaN positions differ"
    err = np.abs(got - ref)[~nan_ref]
    bound = (tol * np.maximum(1.0, np.abs(ref)))[~nan_ref]
    bad = err > bound
    if bad.any():
        idx = np.argmax(err / bound)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outputs beyond tolerance; worst err "
                             f"{err.flat[idx]:.3g} vs bound {bound.flat[idx]:.3g}")


def assert_lse_close(gpu: torch.Tensor, ref: np.ndarray, what: str = "") -> None:
    got = as_f64(gpu)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    inf_ref = np.isinf(ref)
    assert np.array_equal(np.isinf(got), inf_ref), f"{what}: infinite global LSEs differ"
    assert np.array_equal(got[inf_ref], ref[inf_ref]), f"{what}: -inf must stay -inf"
    assert not np.isnan(got).any(), f"{what}: NaN global LSE"
    err = np.abs(got[~inf_ref] - ref[~inf_ref])
    assert err.size == 0 or err.max() <= LSE_TOL, f"{what}: global LSE err {err.max():.3g} > {LSE_TOL}"


class Guarded:
    """A device buffer with sentinel-filled margins before and after it, to catch writes
    outside the output (stands in for a memory checker)."""

    MARGIN = 4096  # bytes on each side (a multiple of 256, so the middle stays aligned)

    def __init__(self, shape, dtype, device="cuda"):
        n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        self.nbytes = n
        self.store = torch.full((n + 2 * self.MARGIN,), 0xA5, dtype=torch.uint8, device=device)
        self.tensor = self.store[self.MARGIN:self.MARGIN + n].view(dtype).view(shape)

    def check(self) -> None:
        head = self.store[:self.MARGIN]
        tail = self.store[self.MARGIN + self.nbytes:]
        assert bool((head == 0xA5).all()), "write before the start of the output"
        assert bool((tail == 0xA5).all()), "write past the end of the output"


def compare_token_blocks(B: int, per_token_elems: int, ref_fn, outs, lses=(), what: str = "") -> None:
    """Element-by-element comparison of full-size device results with the oracle, one block of
    tokens at a time so host memory stays bounded.  ``ref_fn(b0, b1)`` returns the oracle's
    (result, global LSE) of tokens [b0, b1); ``outs`` and ``lses`` list (device tensor, label)
    pairs of [B, ...] results and global LSEs to check against them."""
    block = max(1, (1 << 24) // max(1, per_token_elems))
    for b0 in range(0, B, block):
        b1 = min(B, b0 + block)
        ry, rg = ref_fn(b0, b1)
        for t, label in outs:
            assert_out_close(t[b0:b1], ry, f"{what} {label} tokens [{b0}, {b1})")
        for t, label in lses:
            assert_lse_close(t[b0:b1], rg, f"{what} {label} tokens [{b0}, {b1})")
