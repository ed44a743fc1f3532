"""B200 (sm_100a) sink attention: the Python binding of ``libattn_sink.so``.

Fused flash attention whose softmax denominator carries a per-head sink logit
(Huawei CANN ops-transformer ``flash_attn`` doc, "Function":
``out = sum e^{S-m} V / (sum e^{S-m} + e^{sink-m})``, ``m = max(sink, max S)``).  The same
call covers slime's learnable softmax offset (``softmax(S) * sigmoid(lse - offset)``) and
softmax_n (``sink = log n``).

This module only marshals arguments: it checks tensors, allocates outputs and the
workspace with torch (device memory and streams are all torch provides), and calls the
C ABI declared in ``include/attn_sink.h``.  Every step of the computation runs in the
library's CUDA kernels; there is no CPU or PyTorch fallback, and importing the entry
points fails loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
# ATTN_SINK_LIBRARY selects another build of the library (e.g. the bounds-checking
# libattn_sink_debug.so); by default the in-tree release build is loaded.
LIB_PATH = os.environ.get("ATTN_SINK_LIBRARY") or os.path.join(_HERE, "libattn_sink.so")

ATTN_SINK_BF16, ATTN_SINK_FP32, ATTN_SINK_FP16 = 0, 1, 2
STATUS = {0: "OK", 1: "ERR_INVALID_ARG", 2: "ERR_UNSUPPORTED", 3: "ERR_WORKSPACE", 4: "ERR_CUDA",
          5: "ERR_TIMEOUT", 6: "ERR_BAD_INDEX"}

_SYMBOLS = ("attn_sink_fwd", "attn_sink_bwd", "attn_sink_decode", "attn_sink_fwd_workspace_size",
            "attn_sink_bwd_workspace_size", "attn_sink_decode_workspace_size",
            "attn_sink_decode_num_splits", "attn_sink_status_string",
            "attn_sink_get_device_status", "attn_sink_selftest_wait_timeout", "attn_sink_version",
            "attn_sink_decode_paged", "attn_sink_decode_noalloc")


class AttnSinkParams(ctypes.Structure):
    """Mirror of ``attn_sink_params`` (include/attn_sink.h)."""

    _fields_ = [("batch", ctypes.c_int), ("total_q", ctypes.c_int), ("total_k", ctypes.c_int),
                ("max_seqlen_q", ctypes.c_int), ("max_seqlen_k", ctypes.c_int),
                ("num_heads_q", ctypes.c_int), ("num_heads_kv", ctypes.c_int),
                ("head_dim_qk", ctypes.c_int), ("head_dim_v", ctypes.c_int),
                ("softmax_scale", ctypes.c_float), ("causal", ctypes.c_int),
                ("window_left", ctypes.c_int), ("window_right", ctypes.c_int),
                ("dtype", ctypes.c_int)]


class AttnSinkDropout(ctypes.Structure):
    """Mirror of ``attn_sink_dropout`` (include/attn_sink.h)."""

    _fields_ = [("p", ctypes.c_float), ("seed", ctypes.c_uint64), ("offset", ctypes.c_uint32)]


def _dropout(dropout):
    """(p, seed, offset) -> AttnSinkDropout, or None."""
    if dropout is None:
        return None
    p, seed, offset = dropout
    return AttnSinkDropout(float(p), int(seed) & 0xFFFFFFFFFFFFFFFF, int(offset) & 0xFFFFFFFF)


class AttnSinkError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS.get(status, status)} ({_status_text(status)})")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libattn_sink.so once (raises ImportError if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m softmax_attn_sink_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER(AttnSinkParams)
        vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
        L.attn_sink_fwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.attn_sink_bwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.attn_sink_decode.argtypes = [P, vp, vp, vp, vp, vp, i32, vp, vp, vp, sz, vp]
        L.attn_sink_bwd_deterministic.argtypes = list(L.attn_sink_bwd.argtypes)
        L.attn_sink_bwd_deterministic.restype = i32
        D = ctypes.POINTER(AttnSinkDropout)
        L.attn_sink_fwd_dropout.argtypes = [P, vp, vp, vp, vp, vp, vp, D, vp, vp, vp, sz, vp]
        L.attn_sink_fwd_dropout.restype = i32
        L.attn_sink_bwd_dropout.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, D, vp, vp, vp, vp, vp, sz, vp]
        L.attn_sink_bwd_dropout.restype = i32
        L.attn_sink_decode_paged.argtypes = [P, vp, vp, vp, vp, vp, i32, i32, i32, vp, i32, vp, vp, vp, sz, vp]
        for f in (L.attn_sink_fwd, L.attn_sink_bwd, L.attn_sink_decode, L.attn_sink_decode_paged):
            f.restype = i32
        for f in (L.attn_sink_fwd_workspace_size, L.attn_sink_bwd_workspace_size):
            f.argtypes, f.restype = [P], sz
        L.attn_sink_decode_workspace_size.argtypes = [P, i32]
        L.attn_sink_decode_workspace_size.restype = sz
        L.attn_sink_decode_num_splits.argtypes = [P]
        L.attn_sink_decode_num_splits.restype = i32
        L.attn_sink_status_string.argtypes = [i32]
        L.attn_sink_status_string.restype = ctypes.c_char_p
        L.attn_sink_get_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
        L.attn_sink_get_device_status.restype = i32
        L.attn_sink_check_seqlens.argtypes = [P, vp, vp, vp]
        L.attn_sink_check_seqlens.restype = i32
        L.attn_sink_selftest_wait_timeout.argtypes = [vp]
        L.attn_sink_selftest_wait_timeout.restype = i32
        L.attn_sink_version.argtypes = []
        L.attn_sink_version.restype = i32
        _lib = L
    return _lib


def _status_text(status: int) -> str:
    try:
        return lib().attn_sink_status_string(int(status)).decode()
    except Exception:  # pragma: no cover
        return "?"


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise AttnSinkError(fn, status)


def make_params(*, batch, total_q, total_k, max_seqlen_q, max_seqlen_k, num_heads_q, num_heads_kv,
                head_dim_qk, head_dim_v, softmax_scale, causal=False, window_left=-1,
                window_right=-1, dtype=ATTN_SINK_BF16) -> AttnSinkParams:
    return AttnSinkParams(int(batch), int(total_q), int(total_k), int(max_seqlen_q),
                          int(max_seqlen_k), int(num_heads_q), int(num_heads_kv), int(head_dim_qk),
                          int(head_dim_v), float(softmax_scale), int(bool(causal)),
                          int(window_left), int(window_right), int(dtype))


# --- torch-facing entry points ------------------------------------------------------------

def _torch():
    import torch
    return torch


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return ATTN_SINK_BF16
    if t.dtype == torch.float32:
        return ATTN_SINK_FP32
    if t.dtype == torch.float16:
        return ATTN_SINK_FP16
    raise TypeError(f"unsupported dtype {t.dtype}; use bfloat16, float16 or float32")


def _require(t, name, dtype=None, ndim=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims")


def _stream(stream) -> int:
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _common(q, k, v, cu_seqlens_q, cu_seqlens_k, sink, max_seqlen_q, max_seqlen_k, softmax_scale,
            causal, window_size):
    torch = _torch()
    _require(q, "q", ndim=3)
    _require(k, "k", q.dtype, 3)
    _require(v, "v", q.dtype, 3)
    if cu_seqlens_q is not None:
        _require(cu_seqlens_q, "cu_seqlens_q", torch.int32, 1)
    _require(cu_seqlens_k, "cu_seqlens_k", torch.int32, 1)
    if sink is not None:
        _require(sink, "sink", torch.float32, 1)
        if sink.shape[0] != q.shape[1]:
            raise ValueError("sink must have one value per q head")
    scale = 1.0 / math.sqrt(q.shape[-1]) if softmax_scale is None else float(softmax_scale)
    wl, wr = window_size
    return make_params(batch=cu_seqlens_k.shape[0] - 1, total_q=q.shape[0], total_k=k.shape[0],
                       max_seqlen_q=max_seqlen_q, max_seqlen_k=max_seqlen_k,
                       num_heads_q=q.shape[1], num_heads_kv=k.shape[1], head_dim_qk=q.shape[2],
                       head_dim_v=v.shape[2], softmax_scale=scale, causal=causal,
                       window_left=wl, window_right=wr, dtype=_dtype_code(q))


def attn_sink_fwd(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                  sink=None, softmax_scale: Optional[float] = None, causal: bool = False,
                  window_size: Sequence[int] = (-1, -1), out=None, lse=None, return_lse=True,
                  stream=None, dropout=None):
    """Sink-attention forward on packed THD tensors.  Returns (out, lse).  dropout, when
    given, is (p, seed, offset) (tensor-core path; see attn_sink_dropout).

    q [T_q, Hq, dk], k [T_k, Hkv, dk], v [T_k, Hkv, dv] (bf16, fp16 or fp32, CUDA, contiguous);
    cu_seqlens_q / cu_seqlens_k int32 [B + 1]; sink fp32 [Hq] or None (= -inf);
    softmax_scale defaults to 1/sqrt(dk); window_size (left, right), -1 = unbounded;
    causal is bottom-right aligned.  lse [Hq, T_q] fp32 excludes the sink.
    """
    torch = _torch()
    p = _common(q, k, v, cu_seqlens_q, cu_seqlens_k, sink, max_seqlen_q, max_seqlen_k,
                softmax_scale, causal, window_size)
    if out is None:
        out = torch.empty((q.shape[0], q.shape[1], v.shape[2]), dtype=q.dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((q.shape[1], q.shape[0]), dtype=torch.float32, device=q.device)
    ws_bytes = lib().attn_sink_fwd_workspace_size(ctypes.byref(p))
    if ws_bytes == ctypes.c_size_t(-1).value:
        raise AttnSinkError("attn_sink_fwd_workspace_size", 1)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device) if ws_bytes else None
    if dropout is None:
        st = lib().attn_sink_fwd(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                 cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), _ptr(sink),
                                 out.data_ptr(), _ptr(lse), _ptr(ws), ws_bytes, _stream(stream))
        _check("attn_sink_fwd", st)
    else:
        d = _dropout(dropout)
        st = lib().attn_sink_fwd_dropout(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                         cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), _ptr(sink),
                                         ctypes.byref(d), out.data_ptr(), _ptr(lse), _ptr(ws), ws_bytes,
                                         _stream(stream))
        _check("attn_sink_fwd_dropout", st)
    return out, lse


def attn_sink_bwd(q, k, v, out, dout, lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int,
                  max_seqlen_k: int, sink=None, softmax_scale: Optional[float] = None,
                  causal: bool = False, window_size: Sequence[int] = (-1, -1), dq=None, dk=None,
                  dv=None, dsink=None, stream=None, deterministic: bool = False, dropout=None):
    """Backward for the loss sum(dout * out).  Returns (dq, dk, dv, dsink).  With
    deterministic=True the results are bit-identical from run to run (slower).  dropout:
    the forward's (p, seed, offset) (implies the deterministic path)."""
    torch = _torch()
    p = _common(q, k, v, cu_seqlens_q, cu_seqlens_k, sink, max_seqlen_q, max_seqlen_k,
                softmax_scale, causal, window_size)
    _require(out, "out", q.dtype, 3)
    _require(dout, "dout", q.dtype, 3)
    _require(lse, "lse", torch.float32, 2)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if dsink is None:
        dsink = torch.empty(q.shape[1], dtype=torch.float32, device=q.device)
    ws_bytes = lib().attn_sink_bwd_workspace_size(ctypes.byref(p))
    if ws_bytes == ctypes.c_size_t(-1).value:
        raise AttnSinkError("attn_sink_bwd_workspace_size", 1)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q.device)
    if dropout is not None:
        d = _dropout(dropout)
        st = lib().attn_sink_bwd_dropout(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                         out.data_ptr(), dout.data_ptr(), lse.data_ptr(),
                                         cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), _ptr(sink),
                                         ctypes.byref(d), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                         dsink.data_ptr(), ws.data_ptr(), ws_bytes, _stream(stream))
        _check("attn_sink_bwd_dropout", st)
        return dq, dk, dv, dsink
    fn = lib().attn_sink_bwd_deterministic if deterministic else lib().attn_sink_bwd
    st = fn(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(),
            out.data_ptr(), dout.data_ptr(), lse.data_ptr(),
            cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), _ptr(sink),
            dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), dsink.data_ptr(),
            ws.data_ptr(), ws_bytes, _stream(stream))
    _check("attn_sink_bwd_deterministic" if deterministic else "attn_sink_bwd", st)
    return dq, dk, dv, dsink


def attn_sink_decode(q, k, v, cu_seqlens_k, max_seqlen_k: int, sink=None,
                     softmax_scale: Optional[float] = None, causal: bool = True,
                     window_size: Sequence[int] = (-1, -1), num_splits: int = 0, out=None,
                     lse=None, return_lse=True, workspace=None, stream=None):
    """Split-KV decode: q [B, Hq, dk], one query per sequence.  Returns (out, lse)."""
    torch = _torch()
    p = _common(q, k, v, None, cu_seqlens_k, sink, 1, max_seqlen_k, softmax_scale, causal,
                window_size)
    if out is None:
        out = torch.empty((q.shape[0], q.shape[1], v.shape[2]), dtype=q.dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((q.shape[1], q.shape[0]), dtype=torch.float32, device=q.device)
    ws_bytes = lib().attn_sink_decode_workspace_size(ctypes.byref(p), int(num_splits))
    if ws_bytes == ctypes.c_size_t(-1).value:
        raise AttnSinkError("attn_sink_decode_workspace_size", 1)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q.device)
    st = lib().attn_sink_decode(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                cu_seqlens_k.data_ptr(), _ptr(sink), int(num_splits),
                                out.data_ptr(), _ptr(lse), workspace.data_ptr(),
                                workspace.numel(), _stream(stream))
    _check("attn_sink_decode", st)
    return out, lse


def attn_sink_decode_paged(q, k_cache, v_cache, block_table, seqused_k, max_seqlen_k: int, sink=None,
                           softmax_scale: Optional[float] = None, causal: bool = True,
                           window_size: Sequence[int] = (-1, -1), num_splits: int = 0, out=None,
                           lse=None, return_lse=True, workspace=None, stream=None):
    """Split-KV decode over a paged K/V cache: q [B, Hq, dk], k_cache [num_blocks,
    block_size, Hkv, dk], v_cache [num_blocks, block_size, Hkv, dv], block_table int32
    [B, max_blocks_per_seq], seqused_k int32 [B].  Returns (out, lse)."""
    torch = _torch()
    _require(q, "q", ndim=3)
    _require(k_cache, "k_cache", q.dtype, 4)
    _require(v_cache, "v_cache", q.dtype, 4)
    _require(block_table, "block_table", torch.int32, 2)
    _require(seqused_k, "seqused_k", torch.int32, 1)
    if sink is not None:
        _require(sink, "sink", torch.float32, 1)
        if sink.shape[0] != q.shape[1]:
            raise ValueError("sink must have one value per q head")
    num_blocks, block_size = k_cache.shape[0], k_cache.shape[1]
    if tuple(v_cache.shape[:3]) != (num_blocks, block_size, k_cache.shape[2]):
        raise ValueError("k_cache and v_cache must share [num_blocks, block_size, Hkv]")
    if block_table.shape[0] != q.shape[0] or seqused_k.shape[0] != q.shape[0]:
        raise ValueError("block_table and seqused_k need one row / entry per sequence")
    scale = 1.0 / math.sqrt(q.shape[-1]) if softmax_scale is None else float(softmax_scale)
    wl, wr = window_size
    p = make_params(batch=q.shape[0], total_q=q.shape[0], total_k=num_blocks * block_size,
                    max_seqlen_q=1, max_seqlen_k=max_seqlen_k, num_heads_q=q.shape[1],
                    num_heads_kv=k_cache.shape[2], head_dim_qk=q.shape[2], head_dim_v=v_cache.shape[3],
                    softmax_scale=scale, causal=causal, window_left=wl, window_right=wr,
                    dtype=_dtype_code(q))
    if out is None:
        out = torch.empty((q.shape[0], q.shape[1], v_cache.shape[3]), dtype=q.dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((q.shape[1], q.shape[0]), dtype=torch.float32, device=q.device)
    ws_bytes = lib().attn_sink_decode_workspace_size(ctypes.byref(p), int(num_splits))
    if ws_bytes == ctypes.c_size_t(-1).value:
        raise AttnSinkError("attn_sink_decode_workspace_size", 1)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q.device)
    st = lib().attn_sink_decode_paged(ctypes.byref(p), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                      block_table.data_ptr(), seqused_k.data_ptr(), int(num_blocks),
                                      int(block_size), int(block_table.shape[1]), _ptr(sink),
                                      int(num_splits), out.data_ptr(), _ptr(lse), workspace.data_ptr(),
                                      workspace.numel(), _stream(stream))
    _check("attn_sink_decode_paged", st)
    return out, lse


def decode_num_splits(batch, max_seqlen_k, total_k, num_heads_q, num_heads_kv, head_dim_qk,
                      head_dim_v, dtype=ATTN_SINK_BF16) -> int:
    p = make_params(batch=batch, total_q=batch, total_k=total_k, max_seqlen_q=1,
                    max_seqlen_k=max_seqlen_k, num_heads_q=num_heads_q, num_heads_kv=num_heads_kv,
                    head_dim_qk=head_dim_qk, head_dim_v=head_dim_v, softmax_scale=1.0,
                    causal=True, dtype=dtype)
    return int(lib().attn_sink_decode_num_splits(ctypes.byref(p)))


def device_status(stream=None) -> Tuple[int, int]:
    """Synchronise, then read and clear the device status word: (status, raw bits)."""
    bits = ctypes.c_uint32(0)
    st = lib().attn_sink_get_device_status(_stream(stream), ctypes.byref(bits))
    return int(st), int(bits.value)


def check_seqlens(cu_seqlens_q, cu_seqlens_k, total_q: int, total_k: int, max_seqlen_q: int,
                  max_seqlen_k: int, stream=None) -> Tuple[int, int]:
    """Check the cu_seqlens contract on the device (cu_seqlens_q may be None), then read and
    clear the device status: (status, raw bits); status 6 means a broken contract."""
    torch = _torch()
    _require(cu_seqlens_k, "cu_seqlens_k", torch.int32, 1)
    if cu_seqlens_q is not None:
        _require(cu_seqlens_q, "cu_seqlens_q", torch.int32, 1)
    p = make_params(batch=cu_seqlens_k.shape[0] - 1, total_q=total_q, total_k=total_k,
                    max_seqlen_q=max_seqlen_q, max_seqlen_k=max_seqlen_k, num_heads_q=1, num_heads_kv=1,
                    head_dim_qk=128, head_dim_v=128, softmax_scale=1.0)
    _check("attn_sink_check_seqlens", lib().attn_sink_check_seqlens(
        ctypes.byref(p), _ptr(cu_seqlens_q), cu_seqlens_k.data_ptr(), _stream(stream)))
    return device_status(stream)


def selftest_wait_timeout(stream=None) -> None:
    """Launch the diagnostics kernel whose bounded wait runs out (about 2 s)."""
    _check("attn_sink_selftest_wait_timeout", lib().attn_sink_selftest_wait_timeout(_stream(stream)))


class SinkAttention:
    """Autograd wrapper: ``SinkAttention.apply(q, k, v, sink, cu_q, cu_k, max_q, max_k,
    scale, causal, window_left, window_right[, dropout[, deterministic]])`` -> out, with
    gradients for q, k, v and the sink (the learnable offset of slime's
    learnable_softmax_flash_attn_varlen).  dropout is None or (p, seed, offset); the backward
    redraws the forward's keep decisions from it."""

    _fn = None

    @classmethod
    def apply(cls, *args):
        if cls._fn is None:
            torch = _torch()

            class _F(torch.autograd.Function):
                @staticmethod
                def forward(ctx, q, k, v, sink, cu_q, cu_k, max_q, max_k, scale, causal, wl, wr,
                            dropout=None, deterministic=False):
                    out, lse = attn_sink_fwd(q, k, v, cu_q, cu_k, max_q, max_k, sink, scale,
                                             causal, (wl, wr), dropout=dropout)
                    ctx.save_for_backward(q, k, v, sink, cu_q, cu_k, out, lse)
                    ctx.cfg = (max_q, max_k, scale, causal, wl, wr, dropout, deterministic)
                    return out

                @staticmethod
                def backward(ctx, dout):
                    q, k, v, sink, cu_q, cu_k, out, lse = ctx.saved_tensors
                    max_q, max_k, scale, causal, wl, wr, dropout, deterministic = ctx.cfg
                    dq, dk, dv, ds = attn_sink_bwd(q, k, v, out, dout.contiguous(), lse, cu_q,
                                                   cu_k, max_q, max_k, sink, scale, causal,
                                                   (wl, wr), deterministic=deterministic,
                                                   dropout=dropout)
                    return (dq, dk, dv, ds) + (None,) * 10

            cls._fn = _F
        return cls._fn.apply(*args)


__all__ = ["attn_sink_fwd", "attn_sink_bwd", "attn_sink_decode", "attn_sink_decode_paged", "decode_num_splits",
           "check_seqlens",
           "device_status", "selftest_wait_timeout", "SinkAttention", "AttnSinkError", "AttnSinkParams", "make_params",
           "lib", "LIB_PATH", "ATTN_SINK_BF16", "ATTN_SINK_FP32", "ATTN_SINK_FP16", "AttnSinkDropout"]
