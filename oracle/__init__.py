"""fp64 CPU oracle for the DCP LSE-weighted combine (pack, combine, unpack+combine).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the bench's CPU
baseline leg import this package; the product (``decode_context_attention_dcp_b200``)
never does.  The arithmetic lives in ``dcp_oracle.c`` (plain C loops in double
precision, built here with gcc -O2 -fno-fast-math); this module only compiles
it and marshals numpy arrays in and out.

Sources, by page and section:
  * vLLM API docs, ``vllm.v1.attention.ops.dcp_alltoall``: ``_lse_weighted_combine``
    (the combine) and ``dcp_a2a_lse_reduce`` (the packed [N, B, H/N, D+pack] layout).
  * vllm-ascend ``attention/context_parallel/sfa_cp.py``: ``_merge_dcp_outputs_with_torch``
    (the softmax form of the merge) and ``_get_dcp_local_seq_lens`` (interleaved KV shards).
  * vLLM API docs, ``vllm.v1.attention.ops.dcp``: ``DirectDCPA2AWorkspace.lse_reduce`` takes
    optional ``seq_lens`` / ``query_start_loc``; what it does with them is not on the pages, so
    ``lse_combine_varlen`` implements a stated reading (parity unpinned for that reading).
"""
from __future__ import annotations

import concurrent.futures
import ctypes
import hashlib
import os
import subprocess
import tempfile

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "dcp_oracle.c")
LIBRARY = os.path.join(_HERE, "liboracle.so")

# The oracle's own dtype codes (see dcp_oracle.c).
BF16, FP16, FP32, F64 = 0, 1, 2, 3

_c_i64 = ctypes.c_int64
_c_int = ctypes.c_int
_c_ptr = ctypes.c_void_p


_GCC_FLAGS = ["-O2", "-fno-fast-math", "-std=c11", "-fPIC", "-shared"]


def _digest(source: str) -> str:
    h = hashlib.sha256(" ".join(_GCC_FLAGS).encode() + b"\0")
    with open(source, "rb") as fh:
        h.update(fh.read())
    return h.hexdigest()


def compile_oracle(source: str = SOURCE, output: str = LIBRARY) -> str:
    """Compile the C oracle into a shared library (atomically replaces ``output``; the source's
    digest is kept beside it)."""
    fd, tmp = tempfile.mkstemp(suffix=".so", dir=os.path.dirname(output))
    os.close(fd)
    try:
        subprocess.run(["gcc", *_GCC_FLAGS, "-o", tmp, source, "-lm"], check=True)
        os.replace(tmp, output)
        with open(output + ".sha256", "w") as fh:
            fh.write(_digest(source) + "\n")
    finally:
        if os.path.exists(tmp):
            os.unlink(tmp)
    return output


def _stale(lib: str, src: str) -> bool:
    """True unless ``lib`` was built from exactly the current source and flags."""
    if not os.path.exists(lib) or not os.path.exists(lib + ".sha256"):
        return True
    with open(lib + ".sha256") as fh:
        return fh.read().strip() != _digest(src)


class Oracle:
    """ctypes view of one build of ``dcp_oracle.c``."""

    def __init__(self, library: str):
        self.path = library
        lib = ctypes.CDLL(library)
        lib.oracle_lse_pack_dim.argtypes = [_c_int]
        lib.oracle_lse_pack_dim.restype = _c_int
        lib.oracle_decode.argtypes = [_c_ptr, _c_int, _c_i64]
        lib.oracle_decode.restype = ctypes.c_double
        lib.oracle_pack.argtypes = [_c_ptr, _c_ptr, _c_ptr, _c_i64, _c_i64, _c_i64, _c_int, _c_int,
                                    _c_i64, _c_i64, _c_i64]
        lib.oracle_pack.restype = _c_int
        lib.oracle_unpack.argtypes = [_c_ptr, _c_ptr, _c_ptr, _c_int, _c_i64, _c_i64, _c_i64, _c_i64, _c_int]
        lib.oracle_unpack.restype = _c_int
        lib.oracle_lse_combine.argtypes = [_c_ptr, _c_int, _c_ptr, _c_int, _c_ptr, _c_ptr, _c_int,
                                           _c_i64, _c_i64, _c_i64, _c_i64, _c_i64, _c_int, _c_int]
        lib.oracle_lse_combine.restype = _c_int
        lib.oracle_unpack_combine.argtypes = [_c_ptr, _c_int, _c_ptr, _c_ptr, _c_int, _c_i64, _c_i64,
                                              _c_i64, _c_i64, _c_int, _c_int]
        lib.oracle_unpack_combine.restype = _c_int
        lib.oracle_softmax_merge.argtypes = [_c_ptr, _c_int, _c_ptr, _c_int, _c_ptr, _c_int, _c_i64,
                                             _c_i64, _c_i64, _c_i64, _c_i64]
        lib.oracle_softmax_merge.restype = _c_int
        lib.oracle_attention.argtypes = [_c_ptr, _c_ptr, _c_ptr, _c_int, _c_ptr, _c_ptr, _c_i64, _c_i64,
                                         _c_ptr, _c_i64, ctypes.c_double, _c_int]
        lib.oracle_attention.restype = _c_int
        lib.oracle_lse_combine_varlen.argtypes = [_c_ptr, _c_int, _c_ptr, _c_int, _c_ptr, _c_ptr, _c_int, _c_i64,
                                                  _c_i64, _c_i64, _c_i64, _c_i64, _c_ptr, _c_ptr, _c_int, _c_int,
                                                  _c_int, _c_int]
        lib.oracle_lse_combine_varlen.restype = _c_int
        lib.oracle_local_seq_len.argtypes = [_c_i64, _c_i64, _c_i64, _c_i64]
        lib.oracle_local_seq_len.restype = _c_i64
        self.lib = lib

    # ---- helpers -------------------------------------------------------------------
    @staticmethod
    def _ptr(a: np.ndarray) -> int:
        return a.ctypes.data

    @staticmethod
    def _check(rc: int, what: str) -> None:
        if rc != 0:
            raise ValueError(f"oracle {what} rejected its arguments")

    # ---- API -----------------------------------------------------------------------
    def lse_pack_dim(self, dtype: int) -> int:
        return self.lib.oracle_lse_pack_dim(dtype)

    def decode(self, raw: np.ndarray, dtype: int) -> np.ndarray:
        """Decode raw element bits (uint16 for bf16/fp16) to float64, element by element."""
        raw = np.ascontiguousarray(raw)
        flat = raw.reshape(-1)
        out = np.empty(flat.shape[0], dtype=np.float64)
        for i in range(flat.shape[0]):
            out[i] = self.lib.oracle_decode(self._ptr(flat), dtype, i)
        return out.reshape(raw.shape)

    def pack(self, cp_attn_out: np.ndarray, cp_attn_lse: np.ndarray, world_size: int, dtype: int,
             out_strides: tuple[int, int] | None = None, lse_stride_b: int | None = None) -> np.ndarray:
        """cp_attn_out [B, H, D] raw elements (uint16 / float32), cp_attn_lse [B, H] float32 ->
        send buffer [world_size, B, H/world_size, D + pack] of raw elements."""
        B, H, D = cp_attn_out.shape
        es = cp_attn_out.dtype.itemsize
        if out_strides is None:
            out_strides = (cp_attn_out.strides[0] // es, cp_attn_out.strides[1] // es)
        if lse_stride_b is None:
            lse_stride_b = cp_attn_lse.strides[0] // 4
        assert cp_attn_out.strides[2] == es and cp_attn_lse.strides[1] == 4
        pack = self.lse_pack_dim(dtype)
        send = np.zeros((world_size, B, H // max(world_size, 1), D + pack), dtype=cp_attn_out.dtype)
        rc = self.lib.oracle_pack(self._ptr(cp_attn_out), self._ptr(cp_attn_lse), self._ptr(send), B, H, D,
                                  world_size, dtype, out_strides[0], out_strides[1], lse_stride_b)
        self._check(rc, "pack")
        return send

    def unpack(self, recv: np.ndarray, dtype: int, D: int) -> tuple[np.ndarray, np.ndarray]:
        N, B, Hr, W = recv.shape
        recv = np.ascontiguousarray(recv)
        outs = np.zeros((N, B, Hr, D), dtype=recv.dtype)
        lses = np.zeros((N, B, Hr), dtype=np.float32)
        rc = self.lib.oracle_unpack(self._ptr(recv), self._ptr(outs), self._ptr(lses), N, B, Hr, D,
                                    B * Hr * W, dtype)
        self._check(rc, "unpack")
        return outs, lses

    def lse_combine(self, outputs: np.ndarray, out_dtype: int, lses: np.ndarray, return_lse: bool = False,
                    is_lse_base_on_e: bool = True):
        """outputs [N, B, H, D] raw elements (or float64 with out_dtype=F64), lses [N, B, H]
        float32 or float64 -> result [B, H, D] float64 (+ global LSE [B, H] float64)."""
        outputs = np.ascontiguousarray(outputs)
        lses = np.ascontiguousarray(lses)
        N, B, H, D = outputs.shape
        assert lses.shape == (N, B, H)
        lse_dtype = F64 if lses.dtype == np.float64 else FP32
        assert lses.dtype in (np.float32, np.float64)
        result = np.zeros((B, H, D), dtype=np.float64)
        glse = np.zeros((B, H), dtype=np.float64)
        rc = self.lib.oracle_lse_combine(self._ptr(outputs), out_dtype, self._ptr(lses), lse_dtype,
                                         self._ptr(result), self._ptr(glse), N, B, H, D, B * H * D, B * H,
                                         int(is_lse_base_on_e), int(return_lse))
        self._check(rc, "lse_combine")
        return (result, glse) if return_lse else result

    def unpack_combine(self, recv: np.ndarray, dtype: int, D: int, return_lse: bool = False,
                       is_lse_base_on_e: bool = True):
        recv = np.ascontiguousarray(recv)
        N, B, Hr, W = recv.shape
        result = np.zeros((B, Hr, D), dtype=np.float64)
        glse = np.zeros((B, Hr), dtype=np.float64)
        rc = self.lib.oracle_unpack_combine(self._ptr(recv), dtype, self._ptr(result), self._ptr(glse), N, B, Hr,
                                            D, B * Hr * W, int(is_lse_base_on_e), int(return_lse))
        self._check(rc, "unpack_combine")
        return (result, glse) if return_lse else result

    # ---- token slices on several host threads ------------------------------------------
    # Every (token, head) row of the combine is independent, so a token range can be split
    # over threads: each thread runs the unchanged C function on its own slice, addressed in
    # place through the full arrays' shard strides.  ctypes releases the GIL during the call.
    @staticmethod
    def _split_run(fn, b0: int, b1: int, threads: int) -> None:
        threads = max(1, min(threads, b1 - b0))
        if threads == 1:
            fn(b0, b1)
            return
        step = (b1 - b0 + threads - 1) // threads
        bounds = [(s, min(b1, s + step)) for s in range(b0, b1, step)]
        with concurrent.futures.ThreadPoolExecutor(max_workers=len(bounds)) as ex:
            for f in [ex.submit(fn, s, e) for s, e in bounds]:
                f.result()

    def lse_combine_tokens(self, outputs: np.ndarray, out_dtype: int, lses: np.ndarray, b0: int, b1: int,
                           return_lse: bool = False, is_lse_base_on_e: bool = True, threads: int = 1):
        """``lse_combine`` of tokens [b0, b1) only, read in place from C-contiguous full-size
        outputs [N, B, H, D] / lses [N, B, H]; ``threads`` host threads share the tokens.
        Returns [b1 - b0, H, D] float64 (+ [b1 - b0, H] float64)."""
        assert outputs.flags.c_contiguous and lses.flags.c_contiguous
        N, B, H, D = outputs.shape
        assert lses.shape == (N, B, H) and 0 <= b0 <= b1 <= B
        lse_dtype = F64 if lses.dtype == np.float64 else FP32
        es, ls = outputs.dtype.itemsize, lses.dtype.itemsize
        result = np.zeros((b1 - b0, H, D), dtype=np.float64)
        glse = np.zeros((b1 - b0, H), dtype=np.float64)

        def run(s: int, e: int) -> None:
            rc = self.lib.oracle_lse_combine(self._ptr(outputs) + s * H * D * es, out_dtype,
                                             self._ptr(lses) + s * H * ls, lse_dtype,
                                             self._ptr(result) + (s - b0) * H * D * 8,
                                             self._ptr(glse) + (s - b0) * H * 8, N, e - s, H, D, B * H * D, B * H,
                                             int(is_lse_base_on_e), int(return_lse))
            self._check(rc, "lse_combine")

        self._split_run(run, b0, b1, threads)
        return (result, glse) if return_lse else result

    def unpack_combine_tokens(self, recv: np.ndarray, dtype: int, D: int, b0: int, b1: int,
                              return_lse: bool = False, is_lse_base_on_e: bool = True, threads: int = 1):
        """``unpack_combine`` of tokens [b0, b1) only, read in place from a C-contiguous
        [N, B, Hr, W] buffer; ``threads`` host threads share the tokens."""
        assert recv.flags.c_contiguous
        N, B, Hr, W = recv.shape
        assert 0 <= b0 <= b1 <= B
        es = recv.dtype.itemsize
        result = np.zeros((b1 - b0, Hr, D), dtype=np.float64)
        glse = np.zeros((b1 - b0, Hr), dtype=np.float64)

        def run(s: int, e: int) -> None:
            rc = self.lib.oracle_unpack_combine(self._ptr(recv) + s * Hr * W * es, dtype,
                                                self._ptr(result) + (s - b0) * Hr * D * 8,
                                                self._ptr(glse) + (s - b0) * Hr * 8, N, e - s, Hr, D, B * Hr * W,
                                                int(is_lse_base_on_e), int(return_lse))
            self._check(rc, "unpack_combine")

        self._split_run(run, b0, b1, threads)
        return (result, glse) if return_lse else result

    def lse_combine_varlen_tokens(self, outputs: np.ndarray, out_dtype: int, lses: np.ndarray, seq_lens,
                                  query_start_loc, b0: int, b1: int, interleave: int = 1, return_lse: bool = False,
                                  is_lse_base_on_e: bool = True, threads: int = 1):
        """``lse_combine_varlen`` of tokens [b0, b1) only, read in place from C-contiguous
        full-size outputs [N, B, H, D] / lses [N, B, H].  A slice starting at token s sees
        query_start_loc - s (the same requests, indexed from the slice's first token)."""
        assert outputs.flags.c_contiguous and lses.flags.c_contiguous
        N, B, H, D = outputs.shape
        assert lses.shape == (N, B, H) and 0 <= b0 <= b1 <= B
        sl = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
        qsl = np.asarray(query_start_loc, dtype=np.int64)
        assert qsl.shape[0] == sl.shape[0] + 1
        lse_dtype = F64 if lses.dtype == np.float64 else FP32
        es, ls = outputs.dtype.itemsize, lses.dtype.itemsize
        result = np.zeros((b1 - b0, H, D), dtype=np.float64)
        glse = np.zeros((b1 - b0, H), dtype=np.float64)

        def run(s: int, e: int) -> None:
            q = np.ascontiguousarray(qsl - s, dtype=np.int32)
            rc = self.lib.oracle_lse_combine_varlen(self._ptr(outputs) + s * H * D * es, out_dtype,
                                                    self._ptr(lses) + s * H * ls, lse_dtype,
                                                    self._ptr(result) + (s - b0) * H * D * 8,
                                                    self._ptr(glse) + (s - b0) * H * 8, N, e - s, H, D, B * H * D,
                                                    B * H, self._ptr(sl) if len(sl) else None, self._ptr(q), len(sl),
                                                    int(interleave), int(is_lse_base_on_e), int(return_lse))
            self._check(rc, "lse_combine_varlen")

        self._split_run(run, b0, b1, threads)
        return (result, glse) if return_lse else result

    def softmax_merge(self, outputs: np.ndarray, out_dtype: int, lses: np.ndarray) -> np.ndarray:
        outputs = np.ascontiguousarray(outputs)
        lses = np.ascontiguousarray(lses)
        N, B, H, D = outputs.shape
        lse_dtype = F64 if lses.dtype == np.float64 else FP32
        result = np.zeros((B, H, D), dtype=np.float64)
        rc = self.lib.oracle_softmax_merge(self._ptr(outputs), out_dtype, self._ptr(lses), lse_dtype,
                                           self._ptr(result), N, B, H, D, B * H * D, B * H)
        self._check(rc, "softmax_merge")
        return result

    def attention(self, q: np.ndarray, k: np.ndarray, v: np.ndarray, dtype: int, positions,
                  scale: float, is_lse_base_on_e: bool = True) -> tuple[np.ndarray, np.ndarray]:
        """One token: q [H, D], k/v [L, H, D] -> (out [H, D] f64, lse [H] f64) over ``positions``."""
        q, k, v = (np.ascontiguousarray(x) for x in (q, k, v))
        H, D = q.shape
        pos = np.ascontiguousarray(np.asarray(positions, dtype=np.int64))
        out = np.zeros((H, D), dtype=np.float64)
        lse = np.zeros(H, dtype=np.float64)
        rc = self.lib.oracle_attention(self._ptr(q), self._ptr(k), self._ptr(v), dtype, self._ptr(out),
                                       self._ptr(lse), H, D, self._ptr(pos) if len(pos) else None, len(pos),
                                       float(scale), int(is_lse_base_on_e))
        self._check(rc, "attention")
        return out, lse

    def lse_combine_varlen(self, outputs: np.ndarray, out_dtype: int, lses: np.ndarray, seq_lens, query_start_loc,
                           interleave: int = 1, return_lse: bool = False, is_lse_base_on_e: bool = True):
        """The combine with empty shards skipped (see oracle_lse_combine_varlen for the reading):
        outputs [N, T, H, D], lses [N, T, H]; seq_lens [R], query_start_loc [R + 1] (int32)."""
        outputs = np.ascontiguousarray(outputs)
        lses = np.ascontiguousarray(lses)
        N, B, H, D = outputs.shape
        sl = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
        qsl = np.ascontiguousarray(np.asarray(query_start_loc, dtype=np.int32))
        assert qsl.shape[0] == sl.shape[0] + 1
        lse_dtype = F64 if lses.dtype == np.float64 else FP32
        result = np.zeros((B, H, D), dtype=np.float64)
        glse = np.zeros((B, H), dtype=np.float64)
        rc = self.lib.oracle_lse_combine_varlen(self._ptr(outputs), out_dtype, self._ptr(lses), lse_dtype,
                                                self._ptr(result), self._ptr(glse), N, B, H, D, B * H * D, B * H,
                                                self._ptr(sl) if len(sl) else None, self._ptr(qsl), len(sl),
                                                int(interleave), int(is_lse_base_on_e), int(return_lse))
        self._check(rc, "lse_combine_varlen")
        return (result, glse) if return_lse else result

    def local_seq_len(self, seq_len: int, cp_size: int, rank: int, interleave: int) -> int:
        return self.lib.oracle_local_seq_len(seq_len, cp_size, rank, interleave)


_default: Oracle | None = None


def load() -> Oracle:
    """The oracle built from ``dcp_oracle.c`` (compiled on first use or when the source changed)."""
    global _default
    if _default is None:
        if _stale(LIBRARY, SOURCE):
            compile_oracle()
        _default = Oracle(LIBRARY)
    return _default
