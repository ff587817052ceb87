"""ctypes binding of libmla_b200.so (the C ABI in include/mla_b200.h).

Argument marshalling only: tensors are passed as raw device pointers with the
current CUDA stream; every step of the decode runs in the library's kernels.
The functions keep the C names.  There is no CPU fallback: if the library is
missing, or a call returns a non-zero status, a RuntimeError is raised.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmla_b200.so")

MLA_OK = 0
MLA_ERR_ARG = -1
MLA_ERR_UNSUPPORTED = -2
MLA_ERR_CUDA = -3
MLA_ERR_WORKSPACE = -4
MLA_ERR_DEVICE = -5
MLA_ERR_SCRATCH = -6

MLA_DEVERR_SEQLEN = 0x1
MLA_DEVERR_PAGE = 0x2
MLA_DEVERR_TIMEOUT = 0x4
MLA_DEVERR_PLAN = 0x8
MLA_DEVERR_FP8_RANGE = 0x10

EXPORTED = (
    "mla_metadata_bytes",
    "mla_workspace_bytes",
    "mla_num_sm_pairs",
    "mla_get_metadata",
    "mla_decode",
    "mla_decode_f32",
    "mla_decode_fp8",
    "mla_decode_fp8_timed",
    "mla_decode_timed",
    "mla_decode_noalloc",
    "mla_absorb_q",
    "mla_up_project",
    "mla_merge_splits",
    "mla_merge_splits_f32",
    "mla_selftest_bounded_wait",
    "mla_check_device_error",
    "mla_take_device_errors",
    "mla_error_string",
)

_lib = None
_vp = ctypes.c_void_p
_i32p = ctypes.POINTER(ctypes.c_int32)


class MLAError(RuntimeError):
    def __init__(self, func: str, status: int):
        self.status = status
        super().__init__(f"{func} failed: {status} ({mla_error_string(status)})")


def lib() -> ctypes.CDLL:
    """Open the library once (RuntimeError if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m mla_decode_attention_13_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.mla_metadata_bytes.restype = ctypes.c_size_t
        L.mla_metadata_bytes.argtypes = [ctypes.c_int] * 3
        L.mla_workspace_bytes.restype = ctypes.c_size_t
        L.mla_workspace_bytes.argtypes = [ctypes.c_int] * 3
        L.mla_num_sm_pairs.restype = ctypes.c_int
        L.mla_num_sm_pairs.argtypes = []
        L.mla_get_metadata.restype = ctypes.c_int
        L.mla_get_metadata.argtypes = [_vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, _vp, _vp]
        dec = [_vp, _vp, ctypes.c_int64, _vp, ctypes.c_int, _vp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
               ctypes.c_float, ctypes.c_int, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
        L.mla_decode.restype = ctypes.c_int
        L.mla_decode.argtypes = dec
        L.mla_decode_f32.restype = ctypes.c_int
        L.mla_decode_f32.argtypes = dec
        L.mla_decode_fp8.restype = ctypes.c_int
        L.mla_decode_fp8.argtypes = [_vp, _vp, _vp, _vp] + dec[2:]
        L.mla_decode_fp8_timed.restype = ctypes.c_int
        L.mla_decode_fp8_timed.argtypes = [_vp, _vp, _vp, _vp] + dec[2:] + [_vp, _vp]
        L.mla_decode_timed.restype = ctypes.c_int
        L.mla_decode_timed.argtypes = dec + [_vp, _vp]
        L.mla_decode_noalloc.restype = ctypes.c_int
        L.mla_decode_noalloc.argtypes = dec[:14] + [_vp]
        L.mla_absorb_q.restype = ctypes.c_int
        L.mla_absorb_q.argtypes = [_vp, _vp, _vp, ctypes.c_int, ctypes.c_int, _vp, _vp]
        L.mla_up_project.restype = ctypes.c_int
        L.mla_up_project.argtypes = [_vp, _vp, ctypes.c_int, ctypes.c_int, _vp, _vp]
        L.mla_merge_splits.restype = ctypes.c_int
        L.mla_merge_splits.argtypes = [_vp, _vp] + [ctypes.c_int] * 4 + [_vp, _vp, _vp]
        L.mla_merge_splits_f32.restype = ctypes.c_int
        L.mla_merge_splits_f32.argtypes = [_vp, _vp] + [ctypes.c_int] * 4 + [_vp, _vp, _vp]
        L.mla_selftest_bounded_wait.restype = ctypes.c_int
        L.mla_selftest_bounded_wait.argtypes = [_vp]
        L.mla_check_device_error.restype = ctypes.c_int
        L.mla_check_device_error.argtypes = [_vp, _vp, ctypes.POINTER(ctypes.c_uint32)]
        L.mla_take_device_errors.restype = ctypes.c_int
        L.mla_take_device_errors.argtypes = [_vp, ctypes.POINTER(ctypes.c_uint32)]
        L.mla_error_string.restype = ctypes.c_char_p
        L.mla_error_string.argtypes = [ctypes.c_int]
        _lib = L
    return _lib


def mla_error_string(status: int) -> str:
    return lib().mla_error_string(int(status)).decode()


def mla_metadata_bytes(batch: int, h_q: int, s_q: int) -> int:
    return int(lib().mla_metadata_bytes(batch, h_q, s_q))


def mla_workspace_bytes(batch: int, h_q: int, s_q: int) -> int:
    return int(lib().mla_workspace_bytes(batch, h_q, s_q))


def mla_num_sm_pairs() -> int:
    n = int(lib().mla_num_sm_pairs())
    if n < 0:
        raise MLAError("mla_num_sm_pairs", n)
    return n


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


def _check(func: str, status: int) -> None:
    if status != MLA_OK:
        raise MLAError(func, status)


def mla_get_metadata(seqlens: torch.Tensor, h_q: int, s_q: int, metadata: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """Split-KV plan for one decode step; returns the (device) metadata buffer."""
    batch = int(seqlens.shape[0])
    nbytes = mla_metadata_bytes(batch, h_q, s_q)
    if nbytes == 0:
        raise MLAError("mla_metadata_bytes", MLA_ERR_UNSUPPORTED)
    if metadata is None:
        metadata = torch.empty(nbytes // 4, dtype=torch.int32, device=seqlens.device)
    _check("mla_get_metadata",
           lib().mla_get_metadata(_ptr(seqlens), batch, h_q, s_q, _ptr(metadata), _stream_ptr(stream)))
    return metadata


def mla_decode(q: torch.Tensor, kv_cache: torch.Tensor, block_table: torch.Tensor, seqlens: torch.Tensor,
               softmax_scale: float, causal: bool, metadata: torch.Tensor, workspace: Optional[torch.Tensor] = None,
               out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None, stream=None,
               events: Optional[Tuple] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """MLA decode; returns (out [b, s_q, h_q, 512] bf16, lse [b, h_q, s_q] fp32).

    ``events`` = (before, after) torch.cuda.Event recorded around the split-KV
    kernel (timing only).
    """
    batch, s_q, h_q, d = q.shape
    if d != 576 or kv_cache.shape[-1] != 576 or q.dtype != torch.bfloat16 or kv_cache.dtype != torch.bfloat16:
        raise MLAError("mla_decode", MLA_ERR_ARG)
    for t in (q, kv_cache, block_table, seqlens):
        if not t.is_contiguous():
            raise MLAError("mla_decode", MLA_ERR_ARG)
    if out is None:
        out = torch.empty(batch, s_q, h_q, 512, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty(batch, h_q, s_q, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(max(mla_workspace_bytes(batch, h_q, s_q), 16), dtype=torch.uint8, device=q.device)
    args = [_ptr(q), _ptr(kv_cache), int(kv_cache.shape[0]), _ptr(block_table), int(block_table.shape[1]),
            _ptr(seqlens), batch, s_q, h_q, float(softmax_scale), int(bool(causal)), _ptr(out), _ptr(lse),
            _ptr(metadata), _ptr(workspace), int(workspace.numel() * workspace.element_size()), _stream_ptr(stream)]
    if events is None:
        status = lib().mla_decode(*args)
    else:
        ev = []
        for e in events:
            if e is not None and int(e.cuda_event) == 0:
                e.record()  # torch creates the CUDA event lazily, on first record
            ev.append(None if e is None else int(e.cuda_event))
        status = lib().mla_decode_timed(*args, *ev)
    _check("mla_decode", status)
    return out, lse


def mla_decode_f32(q: torch.Tensor, kv_cache: torch.Tensor, block_table: torch.Tensor, seqlens: torch.Tensor,
                   softmax_scale: float, causal: bool, metadata: torch.Tensor, workspace: Optional[torch.Tensor] = None,
                   out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                   stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """mla_decode with an fp32 output: returns (out [b, s_q, h_q, 512] fp32,
    lse [b, h_q, s_q] fp32), for results that are merged again before they are
    rounded (mla_merge_splits_f32)."""
    batch, s_q, h_q, d = q.shape
    if d != 576 or kv_cache.shape[-1] != 576 or q.dtype != torch.bfloat16 or kv_cache.dtype != torch.bfloat16:
        raise MLAError("mla_decode_f32", MLA_ERR_ARG)
    for t in (q, kv_cache, block_table, seqlens):
        if not t.is_contiguous():
            raise MLAError("mla_decode_f32", MLA_ERR_ARG)
    if out is None:
        out = torch.empty(batch, s_q, h_q, 512, dtype=torch.float32, device=q.device)
    elif tuple(out.shape) != (batch, s_q, h_q, 512) or out.dtype != torch.float32 or not out.is_contiguous():
        raise MLAError("mla_decode_f32", MLA_ERR_ARG)
    if lse is None:
        lse = torch.empty(batch, h_q, s_q, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(max(mla_workspace_bytes(batch, h_q, s_q), 16), dtype=torch.uint8, device=q.device)
    _check("mla_decode_f32",
           lib().mla_decode_f32(_ptr(q), _ptr(kv_cache), int(kv_cache.shape[0]), _ptr(block_table),
                                int(block_table.shape[1]), _ptr(seqlens), batch, s_q, h_q, float(softmax_scale),
                                int(bool(causal)), _ptr(out), _ptr(lse), _ptr(metadata), _ptr(workspace),
                                int(workspace.numel() * workspace.element_size()), _stream_ptr(stream)))
    return out, lse


def mla_decode_fp8(q: torch.Tensor, latent_codes: torch.Tensor, rope: torch.Tensor, exps: torch.Tensor,
                   block_table: torch.Tensor, seqlens: torch.Tensor, softmax_scale: float, causal: bool,
                   metadata: torch.Tensor, workspace: Optional[torch.Tensor] = None,
                   out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None, stream=None,
                   events: Optional[Tuple] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """MLA decode over an FP8 latent cache: latent_codes [pages, 64, 512]
    uint8 (E4M3), rope [pages, 64, 64] bf16, exps [pages, 64] int8 (token
    scale 2^exp).  Returns (out [b, s_q, h_q, 512] bf16, lse [b, h_q, s_q]).

    ``events`` = (before, after) torch.cuda.Event recorded around the split-KV
    kernel (timing only: mla_decode_fp8_timed)."""
    batch, s_q, h_q, d = q.shape
    pages = int(latent_codes.shape[0])
    if d != 576 or q.dtype != torch.bfloat16:
        raise MLAError("mla_decode_fp8", MLA_ERR_ARG)
    if tuple(latent_codes.shape) != (pages, 64, 512) or latent_codes.dtype != torch.uint8:
        raise MLAError("mla_decode_fp8", MLA_ERR_ARG)
    if tuple(rope.shape) != (pages, 64, 64) or rope.dtype != torch.bfloat16:
        raise MLAError("mla_decode_fp8", MLA_ERR_ARG)
    if tuple(exps.shape) != (pages, 64) or exps.dtype != torch.int8:
        raise MLAError("mla_decode_fp8", MLA_ERR_ARG)
    for t in (q, latent_codes, rope, exps, block_table, seqlens):
        if not t.is_contiguous():
            raise MLAError("mla_decode_fp8", MLA_ERR_ARG)
    if out is None:
        out = torch.empty(batch, s_q, h_q, 512, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty(batch, h_q, s_q, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(max(mla_workspace_bytes(batch, h_q, s_q), 16), dtype=torch.uint8, device=q.device)
    args = [_ptr(q), _ptr(latent_codes), _ptr(rope), _ptr(exps), pages, _ptr(block_table),
            int(block_table.shape[1]), _ptr(seqlens), batch, s_q, h_q, float(softmax_scale), int(bool(causal)),
            _ptr(out), _ptr(lse), _ptr(metadata), _ptr(workspace), int(workspace.numel() * workspace.element_size()),
            _stream_ptr(stream)]
    if events is None:
        status = lib().mla_decode_fp8(*args)
    else:
        ev = []
        for e in events:
            if e is not None and int(e.cuda_event) == 0:
                e.record()  # torch creates the CUDA event lazily, on first record
            ev.append(None if e is None else int(e.cuda_event))
        status = lib().mla_decode_fp8_timed(*args, *ev)
    _check("mla_decode_fp8", status)
    return out, lse


def mla_decode_noalloc(q: torch.Tensor, kv_cache: torch.Tensor, block_table: torch.Tensor, seqlens: torch.Tensor,
                       softmax_scale: float, causal: bool, metadata: torch.Tensor, out: torch.Tensor,
                       lse: torch.Tensor, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """MLA decode with the library's fixed scratch instead of a workspace.

    For callers that cannot allocate device memory in the decode loop: every
    buffer (q, cache, table, lengths, metadata, out, lse) is passed in, and
    nothing is allocated here or in the library.  Calls that overlap on the GPU
    share the one scratch array and race.
    """
    batch, s_q, h_q, d = q.shape
    if d != 576 or kv_cache.shape[-1] != 576 or q.dtype != torch.bfloat16 or kv_cache.dtype != torch.bfloat16:
        raise MLAError("mla_decode_noalloc", MLA_ERR_ARG)
    for t in (q, kv_cache, block_table, seqlens, out, lse):
        if not t.is_contiguous():
            raise MLAError("mla_decode_noalloc", MLA_ERR_ARG)
    if tuple(out.shape) != (batch, s_q, h_q, 512) or out.dtype != torch.bfloat16:
        raise MLAError("mla_decode_noalloc", MLA_ERR_ARG)
    if tuple(lse.shape) != (batch, h_q, s_q) or lse.dtype != torch.float32:
        raise MLAError("mla_decode_noalloc", MLA_ERR_ARG)
    _check("mla_decode_noalloc",
           lib().mla_decode_noalloc(_ptr(q), _ptr(kv_cache), int(kv_cache.shape[0]), _ptr(block_table),
                                    int(block_table.shape[1]), _ptr(seqlens), batch, s_q, h_q, float(softmax_scale),
                                    int(bool(causal)), _ptr(out), _ptr(lse), _ptr(metadata), _stream_ptr(stream)))
    return out, lse


def _projection_shapes(func: str, x: torch.Tensor, cols: int, w: torch.Tensor) -> Tuple[int, int]:
    """(tokens, h_q) of x [..., h_q, cols] against weights [h_q, 512, 128]."""
    if x.dim() < 2 or x.shape[-1] != cols or x.dtype != torch.bfloat16 or not x.is_contiguous():
        raise MLAError(func, MLA_ERR_ARG)
    h_q = int(x.shape[-2])
    if tuple(w.shape) != (h_q, 512, 128) or w.dtype != torch.bfloat16 or not w.is_contiguous():
        raise MLAError(func, MLA_ERR_ARG)
    tokens = x.numel() // (h_q * cols)
    return tokens, h_q


def mla_absorb_q(q_nope: torch.Tensor, q_rope: torch.Tensor, w_uk: torch.Tensor, out: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    """Absorbed query [..., h_q, 576] = [W_UK^h q_nope, q_rope] per token and head.

    q_nope [..., h_q, 128], q_rope [..., h_q, 64], w_uk [h_q, 512, 128] (latent
    index first), all bf16 on the device.
    """
    tokens, h_q = _projection_shapes("mla_absorb_q", q_nope, 128, w_uk)
    if tuple(q_rope.shape) != tuple(q_nope.shape[:-1]) + (64,) or q_rope.dtype != torch.bfloat16 \
            or not q_rope.is_contiguous():
        raise MLAError("mla_absorb_q", MLA_ERR_ARG)
    if out is None:
        out = torch.empty(*q_nope.shape[:-1], 576, dtype=torch.bfloat16, device=q_nope.device)
    elif tuple(out.shape) != tuple(q_nope.shape[:-1]) + (576,) or out.dtype != torch.bfloat16 \
            or not out.is_contiguous():
        raise MLAError("mla_absorb_q", MLA_ERR_ARG)
    if tokens == 0:
        return out
    _check("mla_absorb_q", lib().mla_absorb_q(_ptr(q_nope), _ptr(q_rope), _ptr(w_uk), tokens, h_q, _ptr(out),
                                              _stream_ptr(stream)))
    return out


def mla_up_project(o_latent: torch.Tensor, w_uv: torch.Tensor, out: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """Per-head output [..., h_q, 128] = o_latent W_UV^h.

    o_latent [..., h_q, 512] (mla_decode's out), w_uv [h_q, 512, 128] (latent
    index first), bf16 on the device.
    """
    tokens, h_q = _projection_shapes("mla_up_project", o_latent, 512, w_uv)
    if out is None:
        out = torch.empty(*o_latent.shape[:-1], 128, dtype=torch.bfloat16, device=o_latent.device)
    elif tuple(out.shape) != tuple(o_latent.shape[:-1]) + (128,) or out.dtype != torch.bfloat16 \
            or not out.is_contiguous():
        raise MLAError("mla_up_project", MLA_ERR_ARG)
    if tokens == 0:
        return out
    _check("mla_up_project", lib().mla_up_project(_ptr(o_latent), _ptr(w_uv), tokens, h_q, _ptr(out),
                                                  _stream_ptr(stream)))
    return out


def mla_merge_splits(outs: torch.Tensor, lses: torch.Tensor, out: Optional[torch.Tensor] = None,
                     lse: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Merge decode results over disjoint token ranges of the same rows.

    outs [splits, batch, s_q, h_q, 512] bf16 and lses [splits, batch, h_q, s_q]
    fp32 (the splits' mla_decode results, stacked); returns (out, lse) as
    mla_decode would over the union of the ranges.
    """
    if outs.dim() != 5 or outs.shape[-1] != 512 or outs.dtype != torch.bfloat16 or not outs.is_contiguous():
        raise MLAError("mla_merge_splits", MLA_ERR_ARG)
    splits, batch, s_q, h_q, _ = outs.shape
    if tuple(lses.shape) != (splits, batch, h_q, s_q) or lses.dtype != torch.float32 or not lses.is_contiguous():
        raise MLAError("mla_merge_splits", MLA_ERR_ARG)
    if out is None:
        out = torch.empty(batch, s_q, h_q, 512, dtype=torch.bfloat16, device=outs.device)
    if lse is None:
        lse = torch.empty(batch, h_q, s_q, dtype=torch.float32, device=outs.device)
    _check("mla_merge_splits", lib().mla_merge_splits(_ptr(outs), _ptr(lses), splits, batch, s_q, h_q, _ptr(out),
                                                      _ptr(lse), _stream_ptr(stream)))
    return out, lse


def mla_merge_splits_f32(outs: torch.Tensor, lses: torch.Tensor, out: Optional[torch.Tensor] = None,
                         lse: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """mla_merge_splits over fp32 partial outputs (mla_decode_f32's out):
    outs [splits, batch, s_q, h_q, 512] fp32; returns (out bf16, lse fp32)."""
    if outs.dim() != 5 or outs.shape[-1] != 512 or outs.dtype != torch.float32 or not outs.is_contiguous():
        raise MLAError("mla_merge_splits_f32", MLA_ERR_ARG)
    splits, batch, s_q, h_q, _ = outs.shape
    if tuple(lses.shape) != (splits, batch, h_q, s_q) or lses.dtype != torch.float32 or not lses.is_contiguous():
        raise MLAError("mla_merge_splits_f32", MLA_ERR_ARG)
    if out is None:
        out = torch.empty(batch, s_q, h_q, 512, dtype=torch.bfloat16, device=outs.device)
    if lse is None:
        lse = torch.empty(batch, h_q, s_q, dtype=torch.float32, device=outs.device)
    _check("mla_merge_splits_f32", lib().mla_merge_splits_f32(_ptr(outs), _ptr(lses), splits, batch, s_q, h_q,
                                                              _ptr(out), _ptr(lse), _stream_ptr(stream)))
    return out, lse


def mla_selftest_bounded_wait(stream=None) -> None:
    """Enqueue one bounded wait that runs out (raises MLA_DEVERR_TIMEOUT after ~1 s)."""
    _check("mla_selftest_bounded_wait", lib().mla_selftest_bounded_wait(_stream_ptr(stream)))


def mla_take_device_errors(stream=None) -> int:
    """Read and clear the device's sticky error bits (raised by any call
    since the last take); synchronises the stream."""
    word = ctypes.c_uint32(0)
    status = lib().mla_take_device_errors(_stream_ptr(stream), ctypes.byref(word))
    if status not in (MLA_OK, MLA_ERR_DEVICE):
        raise MLAError("mla_take_device_errors", status)
    return int(word.value)


def mla_check_device_error(metadata: torch.Tensor, stream=None) -> int:
    """Synchronise and return the device error word (0 = no error)."""
    word = ctypes.c_uint32(0)
    status = lib().mla_check_device_error(_ptr(metadata), _stream_ptr(stream), ctypes.byref(word))
    if status not in (MLA_OK, MLA_ERR_DEVICE):
        raise MLAError("mla_check_device_error", status)
    return int(word.value)
