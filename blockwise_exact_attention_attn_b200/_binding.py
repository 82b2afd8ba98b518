"""ctypes binding of libringattn.so (include/ring_attn.h).

Argument marshalling only: tensors become device pointers, enums become
ints, the stream defaults to torch's current CUDA stream.  Every step of the
computation runs in the library's CUDA kernels; when the library is missing
the calls raise (there is no fallback).
"""

from __future__ import annotations

import ctypes
import math
import os
import threading
from typing import Optional

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libringattn.so")

RA_OK, RA_ERR_INVALID, RA_ERR_UNSUPPORTED, RA_ERR_CUDA, RA_ERR_TIMEOUT = range(5)
CONTIGUOUS, STRIPED = 0, 1
F32, BF16, F16 = 0, 1, 2

EXPORTS = (
    "ring_attn_fwd",
    "ring_attn_gqa_fwd",
    "ring_attn_fwd_fp8",
    "ring_attn_fwd_step",
    "ring_attn_bwd",
    "ring_attn_bwd_simt",
    "ring_attn_qkvpacked_fwd",
    "ring_attn_fwd_simt",
    "ring_attn_fwd_noalloc",
    "ring_attn_noalloc_status",
    "ring_attn_fwd_host",
    "ring_attn_fwd_host_workspace",
    "ring_attn_merge",
    "ring_attn_status",
    "ring_attn_status_string",
    "ring_attn_schedule",
    "ring_attn_test_withhold_q",
    "ring_attn_test_dump_schedule",
)


class RingAttnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {status_string(status)} ({status})")


_lib = None
_lock = threading.Lock()

_c_int = ctypes.c_int
_c_float = ctypes.c_float
_c_vp = ctypes.c_void_p
_c_i64 = ctypes.c_int64

_FWD_ARGS = [_c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_int, _c_int, _c_int, _c_int, _c_int,
             _c_int, _c_int, _c_float, _c_int, _c_vp, _c_int, _c_vp]
# ring_attn_gqa_fwd: heads_kv follows heads
_GQA_ARGS = _FWD_ARGS[:7] + [_c_int] + _FWD_ARGS[7:]


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load (once) and return the CUDA library; raise when it was not built."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(
                f"{path} is missing: build it with "
                "`python -m blockwise_exact_attention_attn_b200.build`")
        lib = ctypes.CDLL(path)
        lib.ring_attn_fwd.argtypes = _FWD_ARGS
        lib.ring_attn_fwd.restype = _c_int
        lib.ring_attn_fwd_step.argtypes = [_c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_int, _c_int,
                                           _c_int, _c_int, _c_int, _c_int, _c_int, _c_float,
                                           _c_int, _c_int, _c_int, _c_int, _c_vp]
        lib.ring_attn_fwd_step.restype = _c_int
        lib.ring_attn_bwd.argtypes = [_c_vp] * 9 + _GQA_ARGS[5:]
        lib.ring_attn_bwd.restype = _c_int
        lib.ring_attn_bwd_simt.argtypes = [_c_vp] * 9 + _GQA_ARGS[5:]
        lib.ring_attn_bwd_simt.restype = _c_int
        lib.ring_attn_gqa_fwd.argtypes = _GQA_ARGS
        lib.ring_attn_gqa_fwd.restype = _c_int
        lib.ring_attn_fwd_fp8.argtypes = _GQA_ARGS[:16] + [_c_float] * 3 + [_c_vp]
        lib.ring_attn_fwd_fp8.restype = _c_int
        lib.ring_attn_fwd_simt.argtypes = _FWD_ARGS
        lib.ring_attn_fwd_simt.restype = _c_int
        lib.ring_attn_fwd_noalloc.argtypes = _FWD_ARGS
        lib.ring_attn_fwd_noalloc.restype = _c_int
        lib.ring_attn_noalloc_status.argtypes = [_c_vp]
        lib.ring_attn_noalloc_status.restype = _c_int
        lib.ring_attn_fwd_host.argtypes = (_FWD_ARGS[:14] + [_c_int, _c_int, _c_vp,
                                                             ctypes.c_size_t, _c_vp])
        lib.ring_attn_fwd_host.restype = _c_int
        lib.ring_attn_fwd_host_workspace.argtypes = [_c_int] * 6
        lib.ring_attn_fwd_host_workspace.restype = ctypes.c_size_t
        lib.ring_attn_qkvpacked_fwd.argtypes = [_c_vp, _c_vp, _c_vp] + _FWD_ARGS[5:]
        lib.ring_attn_qkvpacked_fwd.restype = _c_int
        lib.ring_attn_merge.argtypes = [_c_vp, _c_vp, _c_vp, _c_vp, _c_int, _c_int, _c_int,
                                        _c_int, _c_int, _c_vp]
        lib.ring_attn_merge.restype = _c_int
        lib.ring_attn_status.argtypes = [_c_vp]
        lib.ring_attn_status.restype = _c_int
        lib.ring_attn_status_string.argtypes = [_c_int]
        lib.ring_attn_status_string.restype = ctypes.c_char_p
        lib.ring_attn_schedule.argtypes = [_c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                           _c_int, _c_int, _c_vp, _c_vp, _c_vp, _c_i64]
        lib.ring_attn_schedule.restype = _c_i64
        lib.ring_attn_test_withhold_q.argtypes = [_c_int]
        lib.ring_attn_test_withhold_q.restype = _c_int
        lib.ring_attn_test_dump_schedule.argtypes = [_c_vp, _c_i64]
        lib.ring_attn_test_dump_schedule.restype = _c_int
        _lib = lib
        return lib


def library_path() -> str:
    return LIB_PATH


def status_string(status: int) -> str:
    return load_library().ring_attn_status_string(int(status)).decode()


ring_attn_status_string = status_string


# --------------------------------------------------------------------- helpers

def _ptr(t, name: str) -> int:
    if t is None:
        return 0
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float16:
        return F16
    raise ValueError(f"unsupported dtype {t.dtype}")


def _layout_code(layout) -> int:
    if isinstance(layout, str):
        return {"contiguous": CONTIGUOUS, "striped": STRIPED}[layout]
    return int(layout)


def _check(fn: str, st: int):
    if st != RA_OK:
        raise RingAttnError(fn, st)


# --------------------------------------------------------------------- C ABI

def ring_attn_fwd(q, k, v, out, lse, batch: int, heads: int, seqlen: int, d_head: int,
                  n_ring_blocks: int, layout=CONTIGUOUS, causal: bool = False,
                  softmax_scale: Optional[float] = None, max_ring_passes: Optional[int] = None,
                  cu_seqlens=None, dtype: Optional[int] = None, stream=None) -> None:
    """Exact ring-ordered blockwise attention forward (see ring_attn.h)."""
    lib = load_library()
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d_head)
    if max_ring_passes is None:
        max_ring_passes = n_ring_blocks
    st = lib.ring_attn_fwd(
        _ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _ptr(out, "out"), _ptr(lse, "lse"),
        int(batch), int(heads), int(seqlen), int(d_head), int(n_ring_blocks),
        _layout_code(layout), int(bool(causal)), float(softmax_scale), int(max_ring_passes),
        _ptr(cu_seqlens, "cu_seqlens"), _dtype_code(q) if dtype is None else int(dtype),
        _stream(stream))
    _check("ring_attn_fwd", st)


def ring_attn_gqa_fwd(q, k, v, out, lse, batch: int, heads: int, heads_kv: int, seqlen: int,
                      d_head: int, n_ring_blocks: int, layout=CONTIGUOUS, causal: bool = False,
                      softmax_scale: Optional[float] = None,
                      max_ring_passes: Optional[int] = None, cu_seqlens=None,
                      dtype: Optional[int] = None, stream=None) -> None:
    """ring_attn_fwd with heads_kv key/value heads shared by consecutive
    groups of heads / heads_kv query heads (see ring_attn.h)."""
    lib = load_library()
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d_head)
    if max_ring_passes is None:
        max_ring_passes = n_ring_blocks
    st = lib.ring_attn_gqa_fwd(
        _ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _ptr(out, "out"), _ptr(lse, "lse"),
        int(batch), int(heads), int(heads_kv), int(seqlen), int(d_head), int(n_ring_blocks),
        _layout_code(layout), int(bool(causal)), float(softmax_scale), int(max_ring_passes),
        _ptr(cu_seqlens, "cu_seqlens"), _dtype_code(q) if dtype is None else int(dtype),
        _stream(stream))
    _check("ring_attn_gqa_fwd", st)


def ring_attn_fwd_fp8(q, k, v, out, lse, batch: int, heads: int, heads_kv: int, seqlen: int,
                      d_head: int, n_ring_blocks: int, layout=CONTIGUOUS, causal: bool = False,
                      softmax_scale: Optional[float] = None,
                      max_ring_passes: Optional[int] = None, cu_seqlens=None,
                      descale_q: float = 1.0, descale_k: float = 1.0, descale_v: float = 1.0,
                      stream=None) -> None:
    """Forward on e4m3 q/k/v (torch.float8_e4m3fn or uint8 tensors) with
    per-tensor descale factors; out is bf16 (see ring_attn.h)."""
    lib = load_library()
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d_head)
    if max_ring_passes is None:
        max_ring_passes = n_ring_blocks
    st = lib.ring_attn_fwd_fp8(
        _ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _ptr(out, "out"), _ptr(lse, "lse"),
        int(batch), int(heads), int(heads_kv), int(seqlen), int(d_head), int(n_ring_blocks),
        _layout_code(layout), int(bool(causal)), float(softmax_scale), int(max_ring_passes),
        _ptr(cu_seqlens, "cu_seqlens"), float(descale_q), float(descale_k), float(descale_v),
        _stream(stream))
    _check("ring_attn_fwd_fp8", st)


def ring_attn_fwd_step(q, k, v, out, lse, batch: int, heads: int, seqlen: int, d_head: int,
                       n_ring_blocks: int, q_block: int, kv_block: int, accumulate: bool,
                       layout=CONTIGUOUS, causal: bool = False,
                       softmax_scale: Optional[float] = None, dtype: Optional[int] = None,
                       stream=None) -> None:
    """Fold ring block kv_block's keys into the running fp32 (out, lse) of
    ring block q_block's queries (see ring_attn.h)."""
    lib = load_library()
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d_head)
    st = lib.ring_attn_fwd_step(
        _ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _ptr(out, "out"), _ptr(lse, "lse"),
        int(batch), int(heads), int(seqlen), int(d_head), int(n_ring_blocks),
        _layout_code(layout), int(bool(causal)), float(softmax_scale), int(q_block),
        int(kv_block), int(bool(accumulate)), _dtype_code(q) if dtype is None else int(dtype),
        _stream(stream))
    _check("ring_attn_fwd_step", st)


def ring_attn_bwd(q, k, v, out, lse, dout, dq, dk, dv, batch: int, heads: int, heads_kv: int,
                  seqlen: int, d_head: int, n_ring_blocks: int, layout=CONTIGUOUS,
                  causal: bool = False, softmax_scale: Optional[float] = None,
                  max_ring_passes: Optional[int] = None, cu_seqlens=None,
                  dtype: Optional[int] = None, stream=None) -> None:
    """Gradients dq, dk, dv of the forward (see ring_attn.h)."""
    _bwd("ring_attn_bwd", q, k, v, out, lse, dout, dq, dk, dv, batch, heads, heads_kv, seqlen,
         d_head, n_ring_blocks, layout, causal, softmax_scale, max_ring_passes, cu_seqlens,
         dtype, stream)


def ring_attn_bwd_simt(q, k, v, out, lse, dout, dq, dk, dv, batch: int, heads: int,
                       heads_kv: int, seqlen: int, d_head: int, n_ring_blocks: int,
                       layout=CONTIGUOUS, causal: bool = False,
                       softmax_scale: Optional[float] = None,
                       max_ring_passes: Optional[int] = None, cu_seqlens=None,
                       dtype: Optional[int] = None, stream=None) -> None:
    """Same contract as ring_attn_bwd on the CUDA-core kernels."""
    _bwd("ring_attn_bwd_simt", q, k, v, out, lse, dout, dq, dk, dv, batch, heads, heads_kv,
         seqlen, d_head, n_ring_blocks, layout, causal, softmax_scale, max_ring_passes,
         cu_seqlens, dtype, stream)


def _bwd(fn, q, k, v, out, lse, dout, dq, dk, dv, batch, heads, heads_kv, seqlen, d_head,
         n_ring_blocks, layout, causal, softmax_scale, max_ring_passes, cu_seqlens, dtype,
         stream) -> None:
    lib = load_library()
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d_head)
    if max_ring_passes is None:
        max_ring_passes = n_ring_blocks
    st = getattr(lib, fn)(
        _ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _ptr(out, "out"), _ptr(lse, "lse"),
        _ptr(dout, "dout"), _ptr(dq, "dq"), _ptr(dk, "dk"), _ptr(dv, "dv"),
        int(batch), int(heads), int(heads_kv), int(seqlen), int(d_head), int(n_ring_blocks),
        _layout_code(layout), int(bool(causal)), float(softmax_scale), int(max_ring_passes),
        _ptr(cu_seqlens, "cu_seqlens"), _dtype_code(q) if dtype is None else int(dtype),
        _stream(stream))
    _check(fn, st)


def ring_attn_fwd_simt(q, k, v, out, lse, batch: int, heads: int, seqlen: int, d_head: int,
                       n_ring_blocks: int, layout=CONTIGUOUS, causal: bool = False,
                       softmax_scale: Optional[float] = None,
                       max_ring_passes: Optional[int] = None, cu_seqlens=None,
                       dtype: Optional[int] = None, stream=None) -> None:
    """Same contract as ring_attn_fwd on the CUDA-core kernel."""
    lib = load_library()
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d_head)
    if max_ring_passes is None:
        max_ring_passes = n_ring_blocks
    st = lib.ring_attn_fwd_simt(
        _ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _ptr(out, "out"), _ptr(lse, "lse"),
        int(batch), int(heads), int(seqlen), int(d_head), int(n_ring_blocks),
        _layout_code(layout), int(bool(causal)), float(softmax_scale), int(max_ring_passes),
        _ptr(cu_seqlens, "cu_seqlens"), _dtype_code(q) if dtype is None else int(dtype),
        _stream(stream))
    _check("ring_attn_fwd_simt", st)


def ring_attn_fwd_noalloc(q, k, v, out, lse, batch: int, heads: int, seqlen: int,
                          d_head: int, n_ring_blocks: int, layout=CONTIGUOUS,
                          causal: bool = False, softmax_scale: Optional[float] = None,
                          max_ring_passes: Optional[int] = None, cu_seqlens=None,
                          dtype: Optional[int] = None, stream=None) -> None:
    """ring_attn_fwd without any device allocation (see ring_attn.h)."""
    lib = load_library()
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d_head)
    if max_ring_passes is None:
        max_ring_passes = n_ring_blocks
    st = lib.ring_attn_fwd_noalloc(
        _ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _ptr(out, "out"), _ptr(lse, "lse"),
        int(batch), int(heads), int(seqlen), int(d_head), int(n_ring_blocks),
        _layout_code(layout), int(bool(causal)), float(softmax_scale), int(max_ring_passes),
        _ptr(cu_seqlens, "cu_seqlens"), _dtype_code(q) if dtype is None else int(dtype),
        _stream(stream))
    _check("ring_attn_fwd_noalloc", st)


def ring_attn_noalloc_status(stream=None) -> int:
    """Synchronize the stream; return and clear the status word of the
    allocation-free calls (see ring_attn.h)."""
    return int(load_library().ring_attn_noalloc_status(_stream(stream)))


def _host_ptr(t, name: str) -> int:
    if t.is_cuda:
        raise ValueError(f"{name} must be a host tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def ring_attn_fwd_host_workspace(batch: int, heads: int, seqlen: int, d_head: int,
                                 dtype: int, head_chunk: int = 0) -> int:
    """Bytes of device workspace ring_attn_fwd_host needs (see ring_attn.h)."""
    return int(load_library().ring_attn_fwd_host_workspace(
        int(batch), int(heads), int(seqlen), int(d_head), int(dtype), int(head_chunk)))


def ring_attn_fwd_host(q, k, v, out, lse, batch: int, heads: int, seqlen: int, d_head: int,
                       n_ring_blocks: int, layout=CONTIGUOUS, causal: bool = False,
                       softmax_scale: Optional[float] = None,
                       max_ring_passes: Optional[int] = None, workspace=None,
                       head_chunk: int = 0, dtype: Optional[int] = None, stream=None) -> None:
    """Forward on page-locked HOST tensors through a caller-owned device
    workspace (a uint8 CUDA tensor); asynchronous on the stream (see
    ring_attn.h)."""
    lib = load_library()
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d_head)
    if max_ring_passes is None:
        max_ring_passes = n_ring_blocks
    if workspace is None:
        raise ValueError("workspace is required (see ring_attn_fwd_host_workspace)")
    st = lib.ring_attn_fwd_host(
        _host_ptr(q, "q"), _host_ptr(k, "k"), _host_ptr(v, "v"), _host_ptr(out, "out"),
        _host_ptr(lse, "lse"), int(batch), int(heads), int(seqlen), int(d_head),
        int(n_ring_blocks), _layout_code(layout), int(bool(causal)), float(softmax_scale),
        int(max_ring_passes), _dtype_code(q) if dtype is None else int(dtype), int(head_chunk),
        _ptr(workspace, "workspace"), int(workspace.numel() * workspace.element_size()),
        _stream(stream))
    _check("ring_attn_fwd_host", st)


def ring_attn_qkvpacked_fwd(qkv, out, lse, batch: int, heads: int, seqlen: int, d_head: int,
                            n_ring_blocks: int, layout=CONTIGUOUS, causal: bool = False,
                            softmax_scale: Optional[float] = None,
                            max_ring_passes: Optional[int] = None, cu_seqlens=None,
                            dtype: Optional[int] = None, stream=None) -> None:
    """q/k/v packed as [..., 3, heads, d_head] (see ring_attn.h)."""
    lib = load_library()
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d_head)
    if max_ring_passes is None:
        max_ring_passes = n_ring_blocks
    st = lib.ring_attn_qkvpacked_fwd(
        _ptr(qkv, "qkv"), _ptr(out, "out"), _ptr(lse, "lse"),
        int(batch), int(heads), int(seqlen), int(d_head), int(n_ring_blocks),
        _layout_code(layout), int(bool(causal)), float(softmax_scale), int(max_ring_passes),
        _ptr(cu_seqlens, "cu_seqlens"), _dtype_code(qkv) if dtype is None else int(dtype),
        _stream(stream))
    _check("ring_attn_qkvpacked_fwd", st)


def ring_attn_merge(out_a, lse_a, out_b, lse_b, batch: int, heads: int, seqlen: int,
                    d_head: int, dtype: Optional[int] = None, stream=None) -> None:
    """Fold (out_b, lse_b) into (out_a, lse_a) in place (see ring_attn.h)."""
    lib = load_library()
    st = lib.ring_attn_merge(
        _ptr(out_a, "out_a"), _ptr(lse_a, "lse_a"), _ptr(out_b, "out_b"), _ptr(lse_b, "lse_b"),
        int(batch), int(heads), int(seqlen), int(d_head),
        _dtype_code(out_a) if dtype is None else int(dtype), _stream(stream))
    _check("ring_attn_merge", st)


def ring_attn_status(stream=None) -> int:
    """Synchronize the stream; return and clear the device status word."""
    return int(load_library().ring_attn_status(_stream(stream)))


def ring_attn_test_withhold_q(on: bool) -> bool:
    """Failure-detection test hook: while on, tensor-core forward launches load
    no query tile, so their bounded wait expires and RA_ERR_TIMEOUT is latched.
    Returns the previous setting."""
    return bool(load_library().ring_attn_test_withhold_q(1 if on else 0))


def ring_attn_test_dump_schedule(buf) -> None:
    """Schedule-dump test hook: a CUDA int32 tensor of 4 + 4 * capacity
    elements receives one record per visited kv tile of every tensor-core
    forward launch while set; None turns it off (see ring_attn.h)."""
    lib = load_library()
    if buf is None:
        st = lib.ring_attn_test_dump_schedule(None, 0)
    else:
        n = buf.numel()
        if n < 4 or (n - 4) % 4:
            raise ValueError("buf must hold 4 + 4 * capacity int32 elements")
        st = lib.ring_attn_test_dump_schedule(_ptr(buf, "buf"), (n - 4) // 4)
    _check("ring_attn_test_dump_schedule", st)


def ring_attn_schedule(seqlen: int, n_ring_blocks: int, layout=CONTIGUOUS,
                       causal: bool = False, max_ring_passes: Optional[int] = None,
                       q_tile: int = 128, kv_tile: int = 128, q_tiles_per_item: int = 1):
    """Visited (q_tile, kv_tile, class) triples of the ring scheduler, as
    three numpy arrays in visit order (class 1 = FULL, 2 = PARTIAL).  With
    q_tiles_per_item = 2, pairs of q-tiles walk one key/value stream, as the
    tensor-core kernel's work items do."""
    lib = load_library()
    if max_ring_passes is None:
        max_ring_passes = n_ring_blocks
    args = (int(seqlen), int(n_ring_blocks), _layout_code(layout), int(bool(causal)),
            int(max_ring_passes), int(q_tile), int(kv_tile), int(q_tiles_per_item))
    n = lib.ring_attn_schedule(*args, None, None, None, 0)
    if n < 0:
        raise RingAttnError("ring_attn_schedule", RA_ERR_INVALID)
    qt = np.zeros(n, dtype=np.int32)
    kt = np.zeros(n, dtype=np.int32)
    cl = np.zeros(n, dtype=np.int8)
    if n:
        lib.ring_attn_schedule(*args, qt.ctypes.data, kt.ctypes.data, cl.ctypes.data, n)
    return qt, kt, cl


# --------------------------------------------------------------------- user API

def _alloc_out(q_like, rows_shape, heads, d_head, lse_shape):
    import torch
    out = torch.empty(*rows_shape, heads, d_head, dtype=q_like.dtype, device=q_like.device)
    lse = torch.empty(*lse_shape, dtype=torch.float32, device=q_like.device)
    return out, lse


def ring_attn_func(q, k, v, n_ring_blocks: int, causal: bool = False, layout=CONTIGUOUS,
                   softmax_scale: Optional[float] = None, max_ring_passes: Optional[int] = None,
                   stream=None):
    """q: [batch, seqlen, heads, d_head], k, v: [batch, seqlen, heads_kv, d_head]
    CUDA tensors (heads_kv a divisor of heads; fewer key/value heads is
    grouped-query attention) -> (out, lse[batch, heads, seqlen])."""
    B, S, H, D = q.shape
    Hkv = k.shape[2]
    out, lse = _alloc_out(q, (B, S), H, D, (B, H, S))
    if Hkv == H:
        ring_attn_fwd(q, k, v, out, lse, B, H, S, D, n_ring_blocks, layout, causal,
                      softmax_scale, max_ring_passes, None, None, stream)
    else:
        ring_attn_gqa_fwd(q, k, v, out, lse, B, H, Hkv, S, D, n_ring_blocks, layout, causal,
                          softmax_scale, max_ring_passes, None, None, stream)
    return out, lse


def ring_attn_func_host(q, k, v, n_ring_blocks: int, causal: bool = False, layout=CONTIGUOUS,
                        softmax_scale: Optional[float] = None,
                        max_ring_passes: Optional[int] = None, out=None, lse=None,
                        head_chunk: int = 0, workspace=None, device=None):
    """ring_attn_func on page-locked HOST tensors q, k, v [batch, seqlen,
    heads, d_head] (same head count): returns (out, lse) on the host
    (page-locked).  Runs ring_attn_fwd_host, which moves chunks of heads in
    and out on its own streams while other chunks compute; `workspace`
    (a uint8 CUDA tensor of ring_attn_fwd_host_workspace bytes) is allocated
    when not given.  Returns after the results are on the host."""
    import torch
    B, S, H, D = q.shape
    if k.shape[2] != H:
        raise ValueError("the host-input forward takes as many key/value heads as query heads")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    if out is None:
        out = torch.empty(B, S, H, D, dtype=q.dtype).pin_memory()
    if lse is None:
        lse = torch.empty(B, H, S, dtype=torch.float32).pin_memory()
    code = _dtype_code(q)
    if workspace is None:
        nbytes = ring_attn_fwd_host_workspace(B, H, S, D, code, head_chunk)
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        stream = torch.cuda.current_stream(dev)
        ring_attn_fwd_host(q, k, v, out, lse, B, H, S, D, n_ring_blocks, layout, causal,
                           softmax_scale, max_ring_passes, workspace, head_chunk, code, stream)
        stream.synchronize()
    return out, lse


def ring_attn_qkvpacked_func(qkv, n_ring_blocks: int, causal: bool = False,
                             layout=CONTIGUOUS, softmax_scale: Optional[float] = None,
                             max_ring_passes: Optional[int] = None, stream=None):
    """qkv: [batch, seqlen, 3, heads, d_head] -> (out, lse[batch, heads, seqlen])."""
    B, S, _, H, D = qkv.shape
    out, lse = _alloc_out(qkv, (B, S), H, D, (B, H, S))
    ring_attn_qkvpacked_fwd(qkv, out, lse, B, H, S, D, n_ring_blocks, layout, causal,
                            softmax_scale, max_ring_passes, None, None, stream)
    return out, lse


def ring_attn_varlen_qkvpacked_func(qkv, cu_seqlens, n_ring_blocks: int, causal: bool = False,
                                    layout=CONTIGUOUS, softmax_scale: Optional[float] = None,
                                    max_ring_passes: Optional[int] = None, stream=None):
    """qkv: [total, 3, heads, d_head], cu_seqlens: int32 [batch + 1] (device) ->
    (out [total, heads, d_head], lse [heads, total])."""
    T, _, H, D = qkv.shape
    B = cu_seqlens.numel() - 1
    out, lse = _alloc_out(qkv, (T,), H, D, (H, T))
    ring_attn_qkvpacked_fwd(qkv, out, lse, B, H, T, D, n_ring_blocks, layout, causal,
                            softmax_scale, max_ring_passes, cu_seqlens, None, stream)
    return out, lse
