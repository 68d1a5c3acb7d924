"""B200 (sm_100a) DCP LSE-weighted combine: thin Python binding of libdcpcombine.so.

The three device steps of the decode-context-parallel combine (vLLM API docs,
vllm.v1.attention.ops.dcp_alltoall: _lse_weighted_combine and
dcp_a2a_lse_reduce) run in hand-written CUDA kernels behind a C ABI
(include/dcp_combine.h).  This module only marshals torch CUDA tensors into
pointers, sizes, strides and the current stream; every step of the
computation happens in the library.  There is no fallback: if the library
cannot be built or loaded, every call raises.

Low-level calls (same names as the C ABI, caller-allocated outputs):
    dcp_pack(cp_attn_out, cp_attn_lse, send_buf, world_size)
    dcp_lse_combine(outputs, lses, result, global_lse=None, ...)
    dcp_lse_combine_varlen(outputs, lses, result, seq_lens, query_start_loc, ...)
    dcp_combine_pack(partial_outputs, partial_lses, send_buf, world_size, ...)
    dcp_unpack_combine(recv_buf, result, global_lse=None, ...)
    dcp_lse_pack_dim(dtype), dcp_last_error(), dcp_wait_timeouts(reset=False)

Allocating helpers with the pages' argument conventions:
    lse_weighted_combine(outputs, lses, return_lse=False, is_lse_base_on_e=True)
    merge_dcp_outputs(output_recv, lse_recv, token_dim)   (head- or token-scattered layouts)
    lse_weighted_combine_varlen(outputs, lses, seq_lens, query_start_loc, interleave=1, ...)
    pack(cp_attn_out, cp_attn_lse, world_size)
    combine_pack(partial_outputs, partial_lses, world_size)   (split merge + pack in one pass)
    unpack_combine(recv_buf, return_lse=False, is_lse_base_on_e=True)
"""
from __future__ import annotations

import ctypes
import threading

import torch

from . import _build

__all__ = [
    "DCPError", "library", "dcp_lse_pack_dim", "dcp_pack", "dcp_lse_combine", "dcp_lse_combine_varlen",
    "dcp_combine_pack", "dcp_unpack_combine", "combine_pack", "dcp_last_error", "dcp_version", "dcp_wait_timeouts", "lse_weighted_combine", "lse_weighted_combine_varlen",
    "merge_dcp_outputs", "pack", "unpack_combine",
    "DTYPE_CODES",
]

DTYPE_CODES = {torch.bfloat16: 0, torch.float16: 1, torch.float32: 2}
STATUS_NAMES = {0: "DCP_OK", 1: "DCP_ERR_INVALID_ARG", 2: "DCP_ERR_UNSUPPORTED_DTYPE", 3: "DCP_ERR_MISALIGNED",
                4: "DCP_ERR_SHAPE", 5: "DCP_ERR_CUDA"}

_i32, _i64, _ptr = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p
_lib: ctypes.CDLL | None = None
_lock = threading.Lock()


class DCPError(RuntimeError):
    """A non-OK status from libdcpcombine.so (``status`` holds the dcp_status code)."""

    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def library() -> ctypes.CDLL:
    """The loaded C library (built in-tree first if it is missing or older than its sources)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                path = _build.build()
                lib = ctypes.CDLL(path)
                lib.dcp_lse_pack_dim.argtypes = [_i32]
                lib.dcp_lse_pack_dim.restype = _i32
                lib.dcp_pack.argtypes = [_ptr, _ptr, _ptr, _i64, _i64, _i64, _i32, _i32, _i64, _i64, _i64, _ptr]
                lib.dcp_pack.restype = _i32
                lib.dcp_testing_pack_stalled.argtypes = lib.dcp_pack.argtypes
                lib.dcp_testing_pack_stalled.restype = _i32
                lib.dcp_testing_last_pack_kernel.argtypes = []
                lib.dcp_testing_last_pack_kernel.restype = _i32
                lib.dcp_lse_combine.argtypes = [_ptr, _ptr, _ptr, _ptr, _i32, _i64, _i64, _i64, _i64, _i64, _i32,
                                                _i32, _i32, _ptr]
                lib.dcp_lse_combine.restype = _i32
                lib.dcp_lse_combine_strided.argtypes = [_ptr, _ptr, _ptr, _ptr, _i32, _i64, _i64, _i64,
                                                        _i64, _i64, _i64, _i64, _i64, _i64, _i64, _i64, _i64, _i64,
                                                        _i32, _i32, _i32, _ptr]
                lib.dcp_lse_combine_strided.restype = _i32
                lib.dcp_lse_combine_varlen.argtypes = [_ptr, _ptr, _ptr, _ptr, _i32, _i64, _i64, _i64, _i64, _i64,
                                                       _ptr, _ptr, _i32, _i32, _i32, _i32, _i32, _ptr]
                lib.dcp_lse_combine_varlen.restype = _i32
                lib.dcp_combine_pack.argtypes = [_ptr, _ptr, _ptr, _i32, _i64, _i64, _i64, _i64, _i64, _i32, _i32,
                                                 _i32, _ptr]
                lib.dcp_combine_pack.restype = _i32
                lib.dcp_unpack_combine.argtypes = [_ptr, _ptr, _ptr, _i32, _i64, _i64, _i64, _i64, _i32, _i32, _i32,
                                                   _ptr]
                lib.dcp_unpack_combine.restype = _i32
                lib.dcp_last_error.argtypes = []
                lib.dcp_last_error.restype = ctypes.c_char_p
                lib.dcp_wait_timeouts.argtypes = [ctypes.POINTER(ctypes.c_uint64), _i32]
                lib.dcp_wait_timeouts.restype = _i32
                lib.dcp_version.argtypes = []
                lib.dcp_version.restype = _i32
                _lib = lib
    return _lib


def dcp_last_error() -> str:
    return library().dcp_last_error().decode()


def dcp_wait_timeouts(reset: bool = False) -> int:
    """Pack CTAs whose wait for their copies timed out on the current device since the last
    reset (synchronises the device).  Nonzero means some dcp_pack result is incomplete."""
    c = ctypes.c_uint64(0)
    _check(library().dcp_wait_timeouts(ctypes.byref(c), int(bool(reset))))
    return int(c.value)


def dcp_version() -> int:
    return library().dcp_version()


def _check(status: int) -> None:
    if status != 0:
        raise DCPError(status, dcp_last_error())


def _code(dtype: torch.dtype) -> int:
    if dtype not in DTYPE_CODES:
        raise DCPError(2, f"unsupported dtype {dtype}")
    return DTYPE_CODES[dtype]


def _cuda(*tensors: torch.Tensor | None) -> torch.device:
    dev = None
    for t in tensors:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError("all tensors must be on the same device")
    return dev


def _stream(device: torch.device, stream) -> int:
    s = torch.cuda.current_stream(device) if stream is None else stream
    return s.cuda_stream if isinstance(s, torch.cuda.Stream) else int(s)


def _inner_contiguous(t: torch.Tensor, dims: int, what: str) -> None:
    """The last ``dims`` dimensions of ``t`` must be laid out contiguously."""
    expect = 1
    for d in range(t.dim() - 1, t.dim() - 1 - dims, -1):
        if t.size(d) != 1 and t.stride(d) != expect:
            raise ValueError(f"{what}: the last {dims} dimensions must be contiguous (strides {t.stride()})")
        expect *= t.size(d)


def dcp_lse_pack_dim(dtype: torch.dtype) -> int:
    """Output-dtype slots that carry one fp32 LSE in a packed row (2 for bf16/fp16, 1 for fp32)."""
    return library().dcp_lse_pack_dim(_code(dtype))


def dcp_pack(cp_attn_out: torch.Tensor, cp_attn_lse: torch.Tensor, send_buf: torch.Tensor, world_size: int,
             stream=None) -> None:
    """cp_attn_out [B, H, D] + cp_attn_lse [B, H] fp32 -> send_buf [world_size, B, H/world_size, D + P].

    Asynchronous: the kernel's bounded waits for its copies cannot report to this call.  If one
    ran out (never, while the copies work), send_buf is incomplete and dcp_wait_timeouts()
    (which synchronises) is nonzero; callers that must be sure read it before trusting send_buf."""
    dev = _cuda(cp_attn_out, cp_attn_lse, send_buf)
    B, H, D = cp_attn_out.shape
    if cp_attn_lse.shape != (B, H) or cp_attn_lse.dtype != torch.float32:
        raise ValueError(f"cp_attn_lse must be fp32 [{B}, {H}], got {cp_attn_lse.dtype} {tuple(cp_attn_lse.shape)}")
    if cp_attn_out.stride(2) != 1 or cp_attn_lse.stride(1) != 1:
        raise ValueError("cp_attn_out and cp_attn_lse must be contiguous in their last dimension")
    if send_buf.dtype != cp_attn_out.dtype or not send_buf.is_contiguous():
        raise ValueError("send_buf must be contiguous and of the output dtype")
    code = _code(cp_attn_out.dtype)
    lib = library()
    P = lib.dcp_lse_pack_dim(code)
    if world_size >= 1 and H % world_size == 0 and send_buf.shape != (world_size, B, H // world_size, D + P):
        raise ValueError(f"send_buf must have shape {(world_size, B, H // world_size, D + P)}")
    with torch.cuda.device(dev):
        _check(lib.dcp_pack(cp_attn_out.data_ptr(), cp_attn_lse.data_ptr(), send_buf.data_ptr(), B, H, D,
                            int(world_size), code, cp_attn_out.stride(0), cp_attn_out.stride(1),
                            cp_attn_lse.stride(0), _stream(dev, stream)))


def dcp_lse_combine(outputs: torch.Tensor, lses: torch.Tensor, result: torch.Tensor,
                    global_lse: torch.Tensor | None = None, is_lse_base_on_e: bool = True,
                    return_lse: bool = False, stream=None) -> None:
    """outputs [N, B, H, D] + lses [N, B, H] fp32 -> result [B, H, D] (+ global_lse [B, H] fp32).

    Any strides are accepted (views in token- or head-major order, capacity-strided shards) as
    long as the last dimension of outputs and result is contiguous: the canonical layout goes to
    dcp_lse_combine, every other one to dcp_lse_combine_strided."""
    dev = _cuda(outputs, lses, result, global_lse)
    N, B, H, D = outputs.shape
    if lses.shape != (N, B, H) or lses.dtype != torch.float32:
        raise ValueError(f"lses must be fp32 [{N}, {B}, {H}], got {lses.dtype} {tuple(lses.shape)}")
    if outputs.stride(3) != 1 and D > 1:
        raise ValueError("outputs must be contiguous in its last dimension")
    if result.shape != (B, H, D) or result.dtype != outputs.dtype or (result.stride(2) != 1 and D > 1):
        raise ValueError("result must be a [B, H, D] tensor of the output dtype, contiguous in its last dimension")
    if return_lse and (global_lse is None or global_lse.shape != (B, H) or global_lse.dtype != torch.float32):
        raise ValueError("return_lse needs an fp32 [B, H] global_lse")
    gs = global_lse.stride() if (return_lse and global_lse is not None) else (0, 0)
    canonical = (outputs.stride()[1:] == (H * D, D, 1) or B * H == 1) and lses.stride()[1:] == (H, 1) \
        and result.is_contiguous() and (not return_lse or global_lse.is_contiguous())
    if canonical:
        with torch.cuda.device(dev):
            _check(library().dcp_lse_combine(
                outputs.data_ptr(), lses.data_ptr(), result.data_ptr(),
                global_lse.data_ptr() if (return_lse and global_lse is not None) else None,
                N, B, H, D, outputs.stride(0) if N > 1 else B * H * D, lses.stride(0) if N > 1 else B * H,
                _code(outputs.dtype), int(bool(is_lse_base_on_e)), int(bool(return_lse)), _stream(dev, stream)))
        return
    with torch.cuda.device(dev):
        _check(library().dcp_lse_combine_strided(
            outputs.data_ptr(), lses.data_ptr(), result.data_ptr(),
            global_lse.data_ptr() if (return_lse and global_lse is not None) else None,
            N, B, H, D, *outputs.stride()[:3], *lses.stride(), *result.stride()[:2], gs[0], gs[1],
            _code(outputs.dtype), int(bool(is_lse_base_on_e)), int(bool(return_lse)), _stream(dev, stream)))


def dcp_lse_combine_varlen(outputs: torch.Tensor, lses: torch.Tensor, result: torch.Tensor, seq_lens: torch.Tensor,
                           query_start_loc: torch.Tensor, global_lse: torch.Tensor | None = None,
                           interleave: int = 1, is_lse_base_on_e: bool = True, return_lse: bool = False,
                           stream=None) -> None:
    """Variable-length combine: outputs [N, B, H, D] + lses [N, B, H] fp32 -> result [B, H, D], where
    token b of request r (query_start_loc[r] <= b < query_start_loc[r+1]) combines only the shards
    n with n * interleave < seq_lens[r]; rows of the other shards are never read.  seq_lens
    [R] and query_start_loc [R + 1] are int32 tensors on the same device.  Shards may be
    capacity-strided (outputs.stride(0) >= B*H*D); dims 1..3 must be contiguous."""
    dev = _cuda(outputs, lses, result, global_lse, seq_lens, query_start_loc)
    N, B, H, D = outputs.shape
    if lses.shape != (N, B, H) or lses.dtype != torch.float32:
        raise ValueError(f"lses must be fp32 [{N}, {B}, {H}], got {lses.dtype} {tuple(lses.shape)}")
    if (outputs.stride()[1:] != (H * D, D, 1) and B * H > 1) or lses.stride()[1:] != (H, 1):
        raise ValueError("outputs and lses must be contiguous within a shard")
    if result.shape != (B, H, D) or result.dtype != outputs.dtype or not result.is_contiguous():
        raise ValueError(f"result must be a contiguous [{B}, {H}, {D}] tensor of the output dtype")
    if return_lse and (global_lse is None or global_lse.shape != (B, H) or global_lse.dtype != torch.float32
                       or not global_lse.is_contiguous()):
        raise ValueError("return_lse needs a contiguous fp32 [B, H] global_lse")
    R = seq_lens.numel()
    for t, n, what in ((seq_lens, R, "seq_lens"), (query_start_loc, R + 1, "query_start_loc")):
        if t.dtype != torch.int32 or t.dim() != 1 or t.numel() != n or not t.is_contiguous():
            raise ValueError(f"{what} must be a contiguous 1-D int32 tensor of {n} entries")
    with torch.cuda.device(dev):
        _check(library().dcp_lse_combine_varlen(
            outputs.data_ptr(), lses.data_ptr(), result.data_ptr(),
            global_lse.data_ptr() if (return_lse and global_lse is not None) else None,
            N, B, H, D, outputs.stride(0) if N > 1 else B * H * D, lses.stride(0) if N > 1 else B * H,
            seq_lens.data_ptr() if R else None, query_start_loc.data_ptr(), R, int(interleave),
            _code(outputs.dtype), int(bool(is_lse_base_on_e)), int(bool(return_lse)), _stream(dev, stream)))


def dcp_combine_pack(partial_outputs: torch.Tensor, partial_lses: torch.Tensor, send_buf: torch.Tensor,
                     world_size: int, is_lse_base_on_e: bool = True, stream=None) -> None:
    """partial_outputs [S, B, H, D] + partial_lses [S, B, H] fp32 (a producer's S KV splits)
    -> send_buf [world_size, B, H/world_size, D + P]: the merged rows, head-scattered, each
    followed by its merged fp32 LSE.  Splits may be capacity-strided; dims 1..3 contiguous."""
    dev = _cuda(partial_outputs, partial_lses, send_buf)
    S, B, H, D = partial_outputs.shape
    code = _code(partial_outputs.dtype)
    if partial_lses.shape != (S, B, H) or partial_lses.dtype != torch.float32:
        raise ValueError(f"partial_lses must be fp32 [{S}, {B}, {H}], got {partial_lses.dtype} "
                         f"{tuple(partial_lses.shape)}")
    if (partial_outputs.stride()[1:] != (H * D, D, 1) and B * H > 1) or partial_lses.stride()[1:] != (H, 1):
        raise ValueError("partial_outputs and partial_lses must be contiguous within a split")
    if world_size < 1 or H % world_size:
        raise ValueError(f"H={H} heads do not split over world_size={world_size}")
    P = library().dcp_lse_pack_dim(code)
    want = (world_size, B, H // world_size, D + P)
    if tuple(send_buf.shape) != want or send_buf.dtype != partial_outputs.dtype or not send_buf.is_contiguous():
        raise ValueError(f"send_buf must be a contiguous {want} tensor of the output dtype")
    with torch.cuda.device(dev):
        _check(library().dcp_combine_pack(
            partial_outputs.data_ptr(), partial_lses.data_ptr(), send_buf.data_ptr(), S, B, H, D,
            partial_outputs.stride(0) if S > 1 else B * H * D, partial_lses.stride(0) if S > 1 else B * H,
            int(world_size), code, int(bool(is_lse_base_on_e)), _stream(dev, stream)))


def dcp_unpack_combine(recv_buf: torch.Tensor, result: torch.Tensor, global_lse: torch.Tensor | None = None,
                       is_lse_base_on_e: bool = True, return_lse: bool = False, stream=None) -> None:
    """recv_buf [N, B, Hr, D + P] -> result [B, Hr, D] (+ global_lse [B, Hr] fp32)."""
    dev = _cuda(recv_buf, result, global_lse)
    N, B, Hr, W = recv_buf.shape
    code = _code(recv_buf.dtype)
    D = W - library().dcp_lse_pack_dim(code)
    _inner_contiguous(recv_buf, 3, "recv_buf")
    if result.shape != (B, Hr, D) or result.dtype != recv_buf.dtype or not result.is_contiguous():
        raise ValueError(f"result must be a contiguous [{B}, {Hr}, {D}] tensor of the buffer dtype")
    if return_lse and (global_lse is None or global_lse.shape != (B, Hr) or global_lse.dtype != torch.float32
                       or not global_lse.is_contiguous()):
        raise ValueError("return_lse needs a contiguous fp32 [B, Hr] global_lse")
    with torch.cuda.device(dev):
        _check(library().dcp_unpack_combine(
            recv_buf.data_ptr(), result.data_ptr(),
            global_lse.data_ptr() if (return_lse and global_lse is not None) else None,
            N, B, Hr, D, recv_buf.stride(0) if N > 1 else B * Hr * W, code, int(bool(is_lse_base_on_e)),
            int(bool(return_lse)), _stream(dev, stream)))


# ---- allocating helpers ------------------------------------------------------------------
def lse_weighted_combine(outputs: torch.Tensor, lses: torch.Tensor, return_lse: bool = False,
                         is_lse_base_on_e: bool = True):
    """Same arguments and results as the pages' _lse_weighted_combine, computed on the GPU:
    outputs [N, B, H, D], lses [N, B, H] -> [B, H, D] (and the global LSE [B, H] fp32)."""
    N, B, H, D = outputs.shape
    result = torch.empty((B, H, D), dtype=outputs.dtype, device=outputs.device)
    glse = torch.empty((B, H), dtype=torch.float32, device=outputs.device) if return_lse else None
    dcp_lse_combine(outputs, lses, result, glse, is_lse_base_on_e=is_lse_base_on_e, return_lse=return_lse)
    return (result, glse) if return_lse else result


def lse_weighted_combine_varlen(outputs: torch.Tensor, lses: torch.Tensor, seq_lens: torch.Tensor,
                                query_start_loc: torch.Tensor, interleave: int = 1, return_lse: bool = False,
                                is_lse_base_on_e: bool = True):
    """The receive-side reduce with the batch's request metadata (seq_lens [R], query_start_loc
    [R + 1], int32 on the device): shards that hold no KV of a token's request are skipped,
    tokens outside every request give 0 (and LSE -inf).  Returns [B, H, D] (and [B, H] fp32)."""
    N, B, H, D = outputs.shape
    result = torch.empty((B, H, D), dtype=outputs.dtype, device=outputs.device)
    glse = torch.empty((B, H), dtype=torch.float32, device=outputs.device) if return_lse else None
    dcp_lse_combine_varlen(outputs, lses, result, seq_lens, query_start_loc, glse, interleave=interleave,
                           is_lse_base_on_e=is_lse_base_on_e, return_lse=return_lse)
    return (result, glse) if return_lse else result


def merge_dcp_outputs(output_recv: torch.Tensor, lse_recv: torch.Tensor, token_dim: int,
                      return_lse: bool = False, is_lse_base_on_e: bool = True):
    """The merge of received shards in the layouts of vllm-ascend sfa_cp.py
    _merge_dcp_outputs_with_torch: output_recv [N, X, Y, D], lse_recv [N, X, Y] fp32, with the
    tokens on dim ``token_dim`` (1: [N, T, H, D], tokens scattered; 2: [N, H, T, D], heads
    scattered).  Returns the combine as a contiguous [T, H, D] tensor of the output dtype (and
    the global LSE [T, H] fp32)."""
    if token_dim not in (1, 2):
        raise ValueError(f"token_dim must be 1 or 2, got {token_dim}")
    if output_recv.dim() != 4 or lse_recv.dim() != 3 or tuple(output_recv.shape[:3]) != tuple(lse_recv.shape):
        raise ValueError(f"expected [N, X, Y, D] outputs and [N, X, Y] LSEs, got {tuple(output_recv.shape)} and "
                         f"{tuple(lse_recv.shape)}")
    if token_dim == 2:
        output_recv = output_recv.transpose(1, 2)
        lse_recv = lse_recv.transpose(1, 2)
    return lse_weighted_combine(output_recv, lse_recv, return_lse=return_lse, is_lse_base_on_e=is_lse_base_on_e)


def pack(cp_attn_out: torch.Tensor, cp_attn_lse: torch.Tensor, world_size: int) -> torch.Tensor:
    """The packed send buffer [world_size, B, H/world_size, D + P] of cp_attn_out / cp_attn_lse."""
    B, H, D = cp_attn_out.shape
    if world_size < 1 or H % world_size != 0:
        raise ValueError(f"H={H} heads do not split evenly over {world_size} ranks")
    P = dcp_lse_pack_dim(cp_attn_out.dtype)
    send = torch.empty((world_size, B, H // world_size, D + P), dtype=cp_attn_out.dtype, device=cp_attn_out.device)
    dcp_pack(cp_attn_out, cp_attn_lse, send, world_size)
    return send


def combine_pack(partial_outputs: torch.Tensor, partial_lses: torch.Tensor, world_size: int,
                 is_lse_base_on_e: bool = True) -> torch.Tensor:
    """A producer's S split partials [S, B, H, D] (+ [S, B, H] fp32 LSEs) merged and packed in
    one pass: the send buffer [world_size, B, H/world_size, D + P] that pack() would build from
    the merged result and its LSE."""
    S, B, H, D = partial_outputs.shape
    P = dcp_lse_pack_dim(partial_outputs.dtype)
    send = torch.empty((world_size, B, H // world_size, D + P), dtype=partial_outputs.dtype,
                       device=partial_outputs.device)
    dcp_combine_pack(partial_outputs, partial_lses, send, world_size, is_lse_base_on_e=is_lse_base_on_e)
    return send


def unpack_combine(recv_buf: torch.Tensor, return_lse: bool = False, is_lse_base_on_e: bool = True):
    """Combine of a packed receive buffer [N, B, Hr, D + P] -> [B, Hr, D] (and [B, Hr] fp32)."""
    N, B, Hr, W = recv_buf.shape
    D = W - dcp_lse_pack_dim(recv_buf.dtype)
    result = torch.empty((B, Hr, D), dtype=recv_buf.dtype, device=recv_buf.device)
    glse = torch.empty((B, Hr), dtype=torch.float32, device=recv_buf.device) if return_lse else None
    dcp_unpack_combine(recv_buf, result, glse, is_lse_base_on_e=is_lse_base_on_e, return_lse=return_lse)
    return (result, glse) if return_lse else result
