"""The C ABI of libdcpcombine.so without a GPU: every declared symbol is exported, and the
host-side argument checks reject bad calls before any CUDA work.

Validation runs before any CUDA call, so these tests pass fake (never dereferenced)
device addresses and need no device.
"""
from __future__ import annotations

import ctypes
import os
import re
import subprocess

import pytest

import decode_context_attention_dcp_b200 as dcp
from decode_context_attention_dcp_b200 import _build

HEADER = os.path.join(_build.INCLUDE, "dcp_combine.h")
HEADERS = sorted(os.path.join(_build.INCLUDE, f) for f in os.listdir(_build.INCLUDE) if f.endswith(".h"))

OK, INVALID, DTYPE, MISALIGNED, SHAPE = 0, 1, 2, 3, 4
A = 0x10000          # a fake 16-byte aligned address (never dereferenced: the calls fail validation)


def declared_functions(headers=(HEADER,)) -> list[str]:
    names = set()
    for h in headers:
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names.update(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(dcp_[a-z0-9_]+)\s*\(", text,
                                flags=re.M))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    return dcp.library()


def test_header_declares_the_entry_points():
    names = declared_functions()
    for need in ("dcp_pack", "dcp_lse_combine", "dcp_unpack_combine", "dcp_lse_pack_dim", "dcp_last_error"):
        assert need in names, names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions(HEADERS)
    assert "dcp_testing_pack_stalled" in names
    out = subprocess.run(["nm", "-D", "--defined-only", _build.LIBRARY], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in names:
        assert name in exported, f"{name} declared in include/ but not exported"
        assert hasattr(lib, name)


def test_pack_dim_and_version(lib):
    assert lib.dcp_lse_pack_dim(0) == 2
    assert lib.dcp_lse_pack_dim(1) == 2
    assert lib.dcp_lse_pack_dim(2) == 1
    assert lib.dcp_lse_pack_dim(3) == -1
    assert dcp.dcp_version() >= 10000


def _combine(lib, **kw):
    a = dict(outputs=A, lses=A, result=A, glse=A, N=2, B=4, H=8, D=128, sn=None, ln=None, dtype=0, base_e=1,
             ret=1)
    a.update(kw)
    sn = a["sn"] if a["sn"] is not None else a["B"] * a["H"] * a["D"]
    ln = a["ln"] if a["ln"] is not None else a["B"] * a["H"]
    return lib.dcp_lse_combine(a["outputs"], a["lses"], a["result"], a["glse"], a["N"], a["B"], a["H"], a["D"], sn,
                               ln, a["dtype"], a["base_e"], a["ret"], None)


def _unpack(lib, **kw):
    a = dict(recv=A, result=A, glse=A, N=4, B=8, Hr=8, D=128, sn=None, dtype=0, base_e=1, ret=0)
    a.update(kw)
    P = 1 if a["dtype"] == 2 else 2
    sn = a["sn"] if a["sn"] is not None else a["B"] * a["Hr"] * (a["D"] + P)
    return lib.dcp_unpack_combine(a["recv"], a["result"], a["glse"], a["N"], a["B"], a["Hr"], a["D"], sn,
                                  a["dtype"], a["base_e"], a["ret"], None)


def _pack(lib, **kw):
    a = dict(out=A, lse=A, send=A, B=4, H=16, D=128, ws=4, dtype=0, sb=None, sh=None, lb=None)
    a.update(kw)
    sh = a["sh"] if a["sh"] is not None else a["D"]
    sb = a["sb"] if a["sb"] is not None else a["H"] * sh
    lb = a["lb"] if a["lb"] is not None else a["H"]
    return lib.dcp_pack(a["out"], a["lse"], a["send"], a["B"], a["H"], a["D"], a["ws"], a["dtype"], sb, sh, lb,
                        None)


@pytest.mark.parametrize("call", [_combine, _unpack, _pack], ids=["combine", "unpack_combine", "pack"])
def test_common_rejections(lib, call):
    key_n = "ws" if call is _pack else "N"
    assert call(lib, dtype=3) == DTYPE
    assert call(lib, dtype=-1) == DTYPE
    assert call(lib, **{key_n: 0}) == INVALID
    assert call(lib, **{key_n: 65}) == INVALID
    assert call(lib, B=-1) == INVALID
    assert call(lib, D=0) == INVALID
    assert call(lib, D=8193 * 8) == INVALID
    assert call(lib, D=12) == MISALIGNED          # 24 bytes per bf16 row
    assert call(lib, D=6, dtype=2) == MISALIGNED  # 24 bytes per fp32 row
    assert "dcp_" in dcp.dcp_last_error()
    assert call(lib, B=0) == OK                   # empty batch: a no-op, no CUDA call
    assert dcp.dcp_last_error() == ""


def test_combine_rejections(lib):
    assert _combine(lib, outputs=None) == INVALID
    assert _combine(lib, lses=None) == INVALID
    assert _combine(lib, result=None) == INVALID
    assert _combine(lib, glse=None, ret=1) == INVALID
    assert _combine(lib, outputs=A + 8) == MISALIGNED
    assert _combine(lib, result=A + 4) == MISALIGNED
    assert _combine(lib, lses=A + 2) == MISALIGNED
    assert _combine(lib, sn=4 * 8 * 128 - 8) == INVALID      # shard stride smaller than a shard
    assert _combine(lib, sn=4 * 8 * 128 + 4) == MISALIGNED   # shard stride of 8 bytes extra
    assert _combine(lib, ln=31) == INVALID
    assert _combine(lib, H=0) == INVALID


def test_unpack_rejections(lib):
    assert _unpack(lib, recv=None) == INVALID
    assert _unpack(lib, result=None) == INVALID
    assert _unpack(lib, glse=None, ret=1) == INVALID
    assert _unpack(lib, recv=A + 4) == MISALIGNED
    assert _unpack(lib, sn=8 * 8 * 130 - 2) == INVALID
    assert _unpack(lib, sn=8 * 8 * 130 + 1) == MISALIGNED    # odd bf16 stride: not 4-byte aligned
    assert _unpack(lib, Hr=0) == INVALID


def test_pack_rejections(lib):
    assert _pack(lib, H=18, ws=4) == SHAPE        # 18 heads over 4 ranks
    assert _pack(lib, out=None) == INVALID
    assert _pack(lib, lse=None) == INVALID
    assert _pack(lib, send=None) == INVALID
    assert _pack(lib, out=A + 2) == MISALIGNED
    assert _pack(lib, send=A + 4) == MISALIGNED
    assert _pack(lib, lse=A + 1) == MISALIGNED
    assert _pack(lib, sh=132) == MISALIGNED       # head stride of 264 bytes
    assert _pack(lib, sh=0) == INVALID
    assert _pack(lib, lb=15) == INVALID


def test_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(2, 4, 8, 128, dtype=torch.bfloat16)
    lse = torch.zeros(2, 4, 8)
    with pytest.raises(ValueError):
        dcp.lse_weighted_combine(x, lse)
    with pytest.raises((dcp.DCPError, ValueError)):
        dcp.dcp_lse_pack_dim(torch.int8)


def _strided(lib, **kw):
    a = dict(outputs=A, lses=A, result=A, glse=A, N=2, B=4, H=8, D=128, dtype=0, ret=1)
    B, H, D = kw.get("B", 4), kw.get("H", 8), kw.get("D", 128)
    st = dict(os_n=B * H * D, os_b=D, os_h=B * D, ls_n=B * H, ls_b=1, ls_h=B, rs_b=H * D, rs_h=D, gs_b=H, gs_h=1)
    a.update(st)
    a.update(kw)
    return lib.dcp_lse_combine_strided(a["outputs"], a["lses"], a["result"], a["glse"], a["N"], a["B"], a["H"],
                                       a["D"], a["os_n"], a["os_b"], a["os_h"], a["ls_n"], a["ls_b"], a["ls_h"],
                                       a["rs_b"], a["rs_h"], a["gs_b"], a["gs_h"], a["dtype"], 1, a["ret"], None)


def test_strided_rejections(lib):
    assert _strided(lib, B=0) == OK
    assert _strided(lib, dtype=5) == DTYPE
    assert _strided(lib, N=0) == INVALID
    assert _strided(lib, os_b=-128) == INVALID
    assert _strided(lib, ls_h=-1) == INVALID
    assert _strided(lib, os_b=132) == MISALIGNED          # 264-byte token stride
    assert _strided(lib, os_n=4 * 8 * 128 + 4) == MISALIGNED
    assert _strided(lib, rs_h=130) == MISALIGNED
    assert _strided(lib, result=A + 8) == MISALIGNED
    assert _strided(lib, glse=None) == INVALID
    assert _strided(lib, B=1 << 22, H=1 << 10) == INVALID  # 2^32 result rows
    assert "dcp_lse_combine_strided" in dcp.dcp_last_error()


def _varlen(lib, **kw):
    a = dict(outputs=A, lses=A, result=A, glse=A, N=2, B=4, H=8, D=128, sn=None, ln=None, seq=A, qsl=A, R=3,
             inter=1, dtype=0, ret=1)
    a.update(kw)
    sn = a["sn"] if a["sn"] is not None else a["B"] * a["H"] * a["D"]
    ln = a["ln"] if a["ln"] is not None else a["B"] * a["H"]
    return lib.dcp_lse_combine_varlen(a["outputs"], a["lses"], a["result"], a["glse"], a["N"], a["B"], a["H"],
                                      a["D"], sn, ln, a["seq"], a["qsl"], a["R"], a["inter"], a["dtype"], 1,
                                      a["ret"], None)


def test_varlen_rejections(lib):
    assert _varlen(lib, B=0) == OK
    assert _varlen(lib, dtype=3) == DTYPE
    assert _varlen(lib, N=65) == INVALID
    assert _varlen(lib, sn=4 * 8 * 128 - 8) == INVALID
    assert _varlen(lib, sn=4 * 8 * 128 + 4) == MISALIGNED
    assert _varlen(lib, R=-1) == INVALID
    assert _varlen(lib, inter=0) == INVALID
    assert _varlen(lib, seq=None) == INVALID
    assert _varlen(lib, qsl=None) == INVALID
    assert _varlen(lib, seq=A + 2) == MISALIGNED
    assert _varlen(lib, qsl=A + 1) == MISALIGNED
    assert _varlen(lib, outputs=A + 8) == MISALIGNED
    assert _varlen(lib, glse=None, ret=1) == INVALID
    assert "dcp_lse_combine_varlen" in dcp.dcp_last_error()


def _combine_pack(lib, **kw):
    a = dict(outputs=A, lses=A, send=A, S=2, B=4, H=16, D=128, ss=None, ls=None, ws=4, dtype=0)
    a.update(kw)
    ss = a["ss"] if a["ss"] is not None else a["B"] * a["H"] * a["D"]
    ls = a["ls"] if a["ls"] is not None else a["B"] * a["H"]
    return lib.dcp_combine_pack(a["outputs"], a["lses"], a["send"], a["S"], a["B"], a["H"], a["D"], ss, ls, a["ws"],
                                a["dtype"], 1, None)


def test_combine_pack_rejections(lib):
    assert _combine_pack(lib, B=0) == OK
    assert _combine_pack(lib, dtype=7) == DTYPE
    assert _combine_pack(lib, S=0) == INVALID
    assert _combine_pack(lib, S=65) == INVALID
    assert _combine_pack(lib, ws=0) == INVALID
    assert _combine_pack(lib, ws=65) == INVALID
    assert _combine_pack(lib, H=18, ws=4) == SHAPE
    assert _combine_pack(lib, D=12) == MISALIGNED
    assert _combine_pack(lib, ss=4 * 16 * 128 - 8) == INVALID
    assert _combine_pack(lib, ss=4 * 16 * 128 + 4) == MISALIGNED
    assert _combine_pack(lib, ls=63) == INVALID
    assert _combine_pack(lib, send=None) == INVALID
    assert _combine_pack(lib, send=A + 4) == MISALIGNED
    assert _combine_pack(lib, outputs=None) == INVALID
    assert _combine_pack(lib, lses=A + 2) == MISALIGNED
    assert "dcp_combine_pack" in dcp.dcp_last_error()


def test_error_text_is_per_thread(lib):
    """dcp_last_error belongs to the calling thread: a failing call on one thread does not
    change what another thread sees."""
    import threading
    seen = {}
    barrier = threading.Barrier(2)

    def failing():
        assert _combine(lib, dtype=9) == DTYPE
        barrier.wait()
        barrier.wait()
        seen["failing"] = dcp.dcp_last_error()

    def clean():
        assert _combine(lib, B=0) == OK
        barrier.wait()
        seen["clean"] = dcp.dcp_last_error()
        barrier.wait()

    ts = [threading.Thread(target=failing), threading.Thread(target=clean)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    assert "unsupported dtype" in seen["failing"]
    assert seen["clean"] == ""
