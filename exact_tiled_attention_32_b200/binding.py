"""Python binding of libfa.so (argument marshalling only).

The names follow the C ABI in ``include/fa.h`` (``fa_fwd``, ``fa_fwd_kvcache``,
``fa_fwd_splitkv``, ``fa_get_device_status``, ``fa_status_string`` ...).  ``attention_forward`` is
the convenience call on torch tensors: it checks shapes, allocates O and the
logsumexp with torch, and calls ``fa_fwd`` on the current CUDA stream.  Every
step of the computation runs in the CUDA kernels of libfa.so; there is no other
implementation behind this module.  If the library is missing, importing this
module raises.
"""
from __future__ import annotations

import ctypes
import math
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfa.so")

FA_OK = 0
FA_ERR_NULL = -1
FA_ERR_SHAPE = -2
FA_ERR_HEADDIM = -3
FA_ERR_GQA = -4
FA_ERR_ALIGN = -5
FA_ERR_ARCH = -6
FA_ERR_LAUNCH = -7
FA_ERR_DEVICE_TIMEOUT = -8
FA_ERR_SEQLENS = -9

EXPORTED = ("fa_fwd", "fa_get_device_status", "fa_status_string", "fa_fwd_noalloc", "fa_fwd_kvcache",
            "fa_selftest_watchdog", "fa_fwd_splitkv", "fa_splitkv_num_splits", "fa_splitkv_workspace_bytes",
            "fa_bwd", "fa_bwd_workspace_bytes", "fa_fwd_fp8", "fa_fwd_partial", "fa_merge_partials",
            "fa_get_noalloc_status", "fa_fwd_fp8_varlen", "fa_fwd_kvcache_varlen")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m exact_tiled_attention_32_b200.build` "
        "(there is no fallback implementation)")

_lib = ctypes.CDLL(LIB_PATH)
_lib.fa_fwd.restype = ctypes.c_int
_lib.fa_fwd.argtypes = [
    ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
    ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
    ctypes.c_float, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
]
_lib.fa_fwd_noalloc.restype = ctypes.c_int
_lib.fa_fwd_noalloc.argtypes = _lib.fa_fwd.argtypes
_lib.fa_fwd_kvcache.restype = ctypes.c_int
_lib.fa_fwd_kvcache.argtypes = [
    ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
    ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
    ctypes.c_float, ctypes.c_int, ctypes.c_void_p,
]
_lib.fa_fwd_kvcache_varlen.restype = ctypes.c_int
_lib.fa_fwd_kvcache_varlen.argtypes = _lib.fa_fwd_kvcache.argtypes[:-1] + [ctypes.c_void_p] * 3
_lib.fa_fwd_splitkv.restype = ctypes.c_int
_lib.fa_fwd_splitkv.argtypes = _lib.fa_fwd_kvcache.argtypes[:-1] + [
    ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
]
_lib.fa_splitkv_num_splits.restype = ctypes.c_int
_lib.fa_splitkv_num_splits.argtypes = [ctypes.c_int] * 6
_lib.fa_splitkv_workspace_bytes.restype = ctypes.c_size_t
_lib.fa_splitkv_workspace_bytes.argtypes = [ctypes.c_int] * 5
_lib.fa_bwd.restype = ctypes.c_int
_lib.fa_bwd.argtypes = [ctypes.c_void_p] * 9 + [ctypes.c_int] * 5 + [
    ctypes.c_float, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
]
_lib.fa_bwd_workspace_bytes.restype = ctypes.c_size_t
_lib.fa_bwd_workspace_bytes.argtypes = [ctypes.c_int] * 5
_lib.fa_fwd_fp8.restype = ctypes.c_int
_lib.fa_fwd_fp8.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 5 + [ctypes.c_float, ctypes.c_int] + \
    [ctypes.c_float] * 3 + [ctypes.c_void_p]
_lib.fa_fwd_fp8_varlen.restype = ctypes.c_int
_lib.fa_fwd_fp8_varlen.argtypes = _lib.fa_fwd_fp8.argtypes[:-1] + [ctypes.c_void_p, ctypes.c_void_p]
_lib.fa_fwd_partial.restype = ctypes.c_int
_lib.fa_fwd_partial.argtypes = _lib.fa_fwd_kvcache.argtypes
_lib.fa_merge_partials.restype = ctypes.c_int
_lib.fa_merge_partials.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_int,
                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
_lib.fa_selftest_watchdog.restype = ctypes.c_int
_lib.fa_selftest_watchdog.argtypes = [ctypes.c_int, ctypes.c_void_p]
_lib.fa_get_device_status.restype = ctypes.c_int
_lib.fa_get_device_status.argtypes = [ctypes.c_void_p]
_lib.fa_get_noalloc_status.restype = ctypes.c_int
_lib.fa_get_noalloc_status.argtypes = [ctypes.c_void_p]
_lib.fa_status_string.restype = ctypes.c_char_p
_lib.fa_status_string.argtypes = [ctypes.c_int]


class FAError(RuntimeError):
    def __init__(self, code: int, where: str = "fa_fwd"):
        self.code = code
        super().__init__(f"{where}: {fa_status_string(code)} ({code})")


def _addr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s) -> int | None:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def fa_fwd(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal, cu_seqlens=None, stream=None) -> int:
    """The C entry point; tensors or raw device addresses.  Returns the status."""
    return _lib.fa_fwd(_addr(q), _addr(k), _addr(v), _addr(o), _addr(lse), int(B), int(Hq),
                       int(Hkv), int(N), int(d), float(scale), int(bool(causal)),
                       _addr(cu_seqlens), _stream(stream))


def fa_fwd_noalloc(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal, cu_seqlens=None, stream=None) -> int:
    """The C entry point that allocates no device memory (for callers that
    cannot allocate: its scratch is a fixed array inside the library).  Same
    arguments and result as fa_fwd; returns the status."""
    return _lib.fa_fwd_noalloc(_addr(q), _addr(k), _addr(v), _addr(o), _addr(lse), int(B), int(Hq),
                               int(Hkv), int(N), int(d), float(scale), int(bool(causal)),
                               _addr(cu_seqlens), _stream(stream))


def fa_fwd_kvcache(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, stream=None) -> int:
    """The C entry point for a chunk of Nq queries (the last Nq positions)
    against Nk keys; returns the status."""
    return _lib.fa_fwd_kvcache(_addr(q), _addr(k), _addr(v), _addr(o), _addr(lse), int(B), int(Hq),
                               int(Hkv), int(Nq), int(Nk), int(d), float(scale), int(bool(causal)),
                               _stream(stream))


def fa_fwd_kvcache_varlen(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, cu_seqlens_q, cu_seqlens_k,
                          stream=None) -> int:
    """The C entry point for packed query chunks against packed keys."""
    return _lib.fa_fwd_kvcache_varlen(_addr(q), _addr(k), _addr(v), _addr(o), _addr(lse), int(B), int(Hq),
                                      int(Hkv), int(Nq), int(Nk), int(d), float(scale), int(bool(causal)),
                                      _addr(cu_seqlens_q), _addr(cu_seqlens_k), _stream(stream))


def attention_forward_kvcache(q, k, v, *, causal: bool = False, scale: float | None = None,
                              cu_seqlens_q=None, cu_seqlens_k=None):
    """O, lse for q [B, Hq, Nq, d] against k/v [B, Hkv, Nk, d] (bf16 CUDA
    tensors); query row i sits at key position Nk - Nq + i.  Packed
    (``cu_seqlens_q`` and ``cu_seqlens_k``, int32 [B+1] CUDA tensors): q
    [Nq, Hq, d] against k/v [Nk, Hkv, d], sequence s's rows the last of its
    key positions; returns O [Nq, Hq, d] and lse [Hq, Nq]."""
    import torch

    if q.dtype != torch.bfloat16 or k.dtype != torch.bfloat16 or v.dtype != torch.bfloat16:
        raise TypeError("q, k, v must be bfloat16")
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    if (cu_seqlens_q is None) != (cu_seqlens_k is None):
        raise ValueError("give both cu_seqlens_q and cu_seqlens_k, or neither")
    if cu_seqlens_q is not None:
        for c in (cu_seqlens_q, cu_seqlens_k):
            if c.dtype != torch.int32 or not c.is_cuda or c.dim() != 1:
                raise ValueError("cu_seqlens: int32 CUDA tensors [B+1]")
        if cu_seqlens_q.numel() != cu_seqlens_k.numel():
            raise ValueError("cu_seqlens_q and cu_seqlens_k must have the same length")
        if q.dim() != 3 or k.dim() != 3 or k.shape != v.shape:
            raise ValueError("packed layout: q [Nq,Hq,d], k/v [Nk,Hkv,d]")
        Nq, Hq, d = q.shape
        Nk, Hkv = k.shape[0], k.shape[1]
        if k.shape[2] != d:
            raise ValueError("k/v shape does not match q")
        if scale is None:
            scale = 1.0 / math.sqrt(d)
        out = torch.empty_like(q)
        lse = torch.empty((Hq, Nq), dtype=torch.float32, device=q.device)
        rc = fa_fwd_kvcache_varlen(q, k, v, out, lse, cu_seqlens_q.numel() - 1, Hq, Hkv, Nq, Nk, d, scale, causal,
                                   cu_seqlens_q, cu_seqlens_k, torch.cuda.current_stream(q.device))
        if rc != FA_OK:
            raise FAError(rc, "fa_fwd_kvcache_varlen")
        return out, lse
    if q.dim() != 4 or k.dim() != 4 or k.shape != v.shape:
        raise ValueError("q [B,Hq,Nq,d], k/v [B,Hkv,Nk,d]")
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if k.shape[0] != B or k.shape[3] != d:
        raise ValueError("k/v shape does not match q")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = torch.empty_like(q)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    rc = fa_fwd_kvcache(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal,
                        torch.cuda.current_stream(q.device))
    if rc != FA_OK:
        raise FAError(rc, "fa_fwd_kvcache")
    return out, lse


def fa_fwd_splitkv(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, num_splits, workspace,
                   workspace_bytes, stream=None) -> int:
    """The C entry point for decode-shaped problems (keys cut into
    ``num_splits`` ranges merged through the logsumexp); returns the status."""
    return _lib.fa_fwd_splitkv(_addr(q), _addr(k), _addr(v), _addr(o), _addr(lse), int(B), int(Hq),
                               int(Hkv), int(Nq), int(Nk), int(d), float(scale), int(bool(causal)),
                               int(num_splits), _addr(workspace), int(workspace_bytes), _stream(stream))


def fa_splitkv_num_splits(B, Hq, Hkv, Nq, Nk, d) -> int:
    """Split count for this shape on the current device (or a negative status)."""
    return _lib.fa_splitkv_num_splits(int(B), int(Hq), int(Hkv), int(Nq), int(Nk), int(d))


def fa_splitkv_workspace_bytes(B, Hq, Nq, d, num_splits) -> int:
    """Workspace bytes fa_fwd_splitkv needs (0 for one split or bad arguments)."""
    return int(_lib.fa_splitkv_workspace_bytes(int(B), int(Hq), int(Nq), int(d), int(num_splits)))


def attention_forward_splitkv(q, k, v, *, causal: bool = False, scale: float | None = None,
                              num_splits: int | None = None, workspace=None):
    """``attention_forward_kvcache`` through fa_fwd_splitkv: O, lse for
    q [B, Hq, Nq, d] against k/v [B, Hkv, Nk, d] (bf16 CUDA tensors).
    ``num_splits`` defaults to the library's choice for the current device;
    the workspace is allocated with torch unless one (a CUDA tensor of at least
    the required bytes) is passed."""
    import torch

    if q.dtype != torch.bfloat16 or k.dtype != torch.bfloat16 or v.dtype != torch.bfloat16:
        raise TypeError("q, k, v must be bfloat16")
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    if q.dim() != 4 or k.dim() != 4 or k.shape != v.shape:
        raise ValueError("q [B,Hq,Nq,d], k/v [B,Hkv,Nk,d]")
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if k.shape[0] != B or k.shape[3] != d:
        raise ValueError("k/v shape does not match q")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if num_splits is None:
        num_splits = fa_splitkv_num_splits(B, Hq, Hkv, Nq, Nk, d)
        if num_splits < 0:
            raise FAError(num_splits, "fa_splitkv_num_splits")
    need = fa_splitkv_workspace_bytes(B, Hq, Nq, d, num_splits)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    out = torch.empty_like(q)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    rc = fa_fwd_splitkv(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, num_splits, workspace,
                        wbytes, torch.cuda.current_stream(q.device))
    if rc != FA_OK:
        raise FAError(rc, "fa_fwd_splitkv")
    return out, lse


def fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, N, d, scale, causal, cu_seqlens, workspace,
           workspace_bytes, stream=None) -> int:
    """The C entry point of the backward pass; returns the status."""
    return _lib.fa_bwd(_addr(q), _addr(k), _addr(v), _addr(o), _addr(lse), _addr(dout), _addr(dq), _addr(dk),
                       _addr(dv), int(B), int(Hq), int(Hkv), int(N), int(d), float(scale), int(bool(causal)),
                       _addr(cu_seqlens), _addr(workspace), int(workspace_bytes), _stream(stream))


def fa_bwd_workspace_bytes(B, Hq, N, d, packed=False) -> int:
    """Workspace bytes fa_bwd needs (0 for bad arguments)."""
    return int(_lib.fa_bwd_workspace_bytes(int(B), int(Hq), int(N), int(d), int(bool(packed))))


def attention_backward(q, k, v, o, lse, dout, *, causal: bool = False, scale: float | None = None,
                       cu_seqlens=None, workspace=None):
    """dq, dk, dv for the forward O, lse = attention_forward(q, k, v, ...)
    and the upstream gradient ``dout`` (bf16 CUDA tensors, layouts of the
    forward: dense, or packed with ``cu_seqlens``).  The workspace is
    allocated with torch unless given."""
    import torch

    for t in (q, k, v, o, dout):
        if t.dtype != torch.bfloat16:
            raise TypeError("q, k, v, o, dout must be bfloat16")
    if lse.dtype != torch.float32:
        raise TypeError("lse must be float32")
    q, k, v, o, dout, lse = (t.contiguous() for t in (q, k, v, o, dout, lse))
    if k.shape != v.shape or o.shape != q.shape or dout.shape != q.shape:
        raise ValueError("o, dout must have q's shape and v k's")
    if cu_seqlens is None:
        if q.dim() != 4:
            raise ValueError("dense layout: q, o, dout [B,Hq,N,d], k/v [B,Hkv,N,d]")
        B, Hq, N, d = q.shape
        Hkv = k.shape[1]
    else:
        if q.dim() != 3:
            raise ValueError("packed layout: q, o, dout [N,Hq,d], k/v [N,Hkv,d]")
        if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda:
            raise ValueError("cu_seqlens must be an int32 CUDA tensor")
        N, Hq, d = q.shape
        Hkv = k.shape[1]
        B = cu_seqlens.numel() - 1
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = fa_bwd_workspace_bytes(B, Hq, N, d, cu_seqlens is not None)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    rc = fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, N, d, scale, causal, cu_seqlens, workspace,
                workspace.numel() * workspace.element_size(), torch.cuda.current_stream(q.device))
    if rc != FA_OK:
        raise FAError(rc, "fa_bwd")
    return dq, dk, dv


def fa_fwd_fp8(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal, q_scale, k_scale, v_scale, stream=None) -> int:
    """The C entry point of the FP8 (E4M3) forward; returns the status."""
    return _lib.fa_fwd_fp8(_addr(q), _addr(k), _addr(v), _addr(o), _addr(lse), int(B), int(Hq), int(Hkv), int(N),
                           int(d), float(scale), int(bool(causal)), float(q_scale), float(k_scale), float(v_scale),
                           _stream(stream))


def fa_fwd_fp8_varlen(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal, q_scale, k_scale, v_scale, cu_seqlens,
                      stream=None) -> int:
    """The C entry point of the FP8 (E4M3) forward on packed sequences."""
    return _lib.fa_fwd_fp8_varlen(_addr(q), _addr(k), _addr(v), _addr(o), _addr(lse), int(B), int(Hq), int(Hkv),
                                  int(N), int(d), float(scale), int(bool(causal)), float(q_scale), float(k_scale),
                                  float(v_scale), _addr(cu_seqlens), _stream(stream))


def attention_forward_fp8(q, k, v, q_scale: float, k_scale: float, v_scale: float, *, causal: bool = False,
                          scale: float | None = None, cu_seqlens=None):
    """O (bf16), lse for E4M3 q, k, v (CUDA tensors of dtype
    torch.float8_e4m3fn or uint8 holding E4M3 codes) with per-tensor scales:
    the values are code * scale.  Dense: q [B, Hq, N, d], k/v [B, Hkv, N, d];
    packed (``cu_seqlens`` int32 [B+1] on the device): q [N, Hq, d], k/v
    [N, Hkv, d], returning O [N, Hq, d] and lse [Hq, N]."""
    import torch

    for t in (q, k, v):
        if t.dtype not in (torch.uint8, getattr(torch, "float8_e4m3fn", torch.uint8)):
            raise TypeError("q, k, v must be float8_e4m3fn (or uint8 E4M3 codes)")
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    stream = torch.cuda.current_stream(q.device)
    if cu_seqlens is not None:
        if q.dim() != 3 or k.dim() != 3 or k.shape != v.shape:
            raise ValueError("packed layout: q [N,Hq,d], k/v [N,Hkv,d]")
        if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda or cu_seqlens.dim() != 1:
            raise ValueError("cu_seqlens: int32 CUDA tensor [B+1]")
        N, Hq, d = q.shape
        Hkv = k.shape[1]
        if k.shape[0] != N or k.shape[2] != d:
            raise ValueError("k/v shape does not match q")
        if scale is None:
            scale = 1.0 / math.sqrt(d)
        B = cu_seqlens.numel() - 1
        out = torch.empty((N, Hq, d), dtype=torch.bfloat16, device=q.device)
        lse = torch.empty((Hq, N), dtype=torch.float32, device=q.device)
        rc = fa_fwd_fp8_varlen(q, k, v, out, lse, B, Hq, Hkv, N, d, scale, causal, q_scale, k_scale, v_scale,
                               cu_seqlens, stream)
        if rc != FA_OK:
            raise FAError(rc, "fa_fwd_fp8_varlen")
        return out, lse
    if q.dim() != 4 or k.dim() != 4 or k.shape != v.shape:
        raise ValueError("dense layout: q [B,Hq,N,d], k/v [B,Hkv,N,d]")
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if k.shape[0] != B or k.shape[2] != N or k.shape[3] != d:
        raise ValueError("k/v shape does not match q")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = torch.empty((B, Hq, N, d), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    rc = fa_fwd_fp8(q, k, v, out, lse, B, Hq, Hkv, N, d, scale, causal, q_scale, k_scale, v_scale, stream)
    if rc != FA_OK:
        raise FAError(rc, "fa_fwd_fp8")
    return out, lse


def fa_fwd_partial(q, k, v, o_part, lse_part, B, Hq, Hkv, Nq, Nk, d, scale, causal, stream=None) -> int:
    """The C entry point writing one key range's fp32 share (O / l, lse)."""
    return _lib.fa_fwd_partial(_addr(q), _addr(k), _addr(v), _addr(o_part), _addr(lse_part), int(B), int(Hq),
                               int(Hkv), int(Nq), int(Nk), int(d), float(scale), int(bool(causal)), _stream(stream))


def fa_merge_partials(o_parts, lse_parts, nparts, rows, d, o, lse, stream=None) -> int:
    """The C entry point merging shares of the same rows."""
    return _lib.fa_merge_partials(_addr(o_parts), _addr(lse_parts), int(nparts), int(rows), int(d), _addr(o),
                                  _addr(lse), _stream(stream))


def fa_selftest_watchdog(timeout_ms: int, stream=None) -> int:
    """Launches the watchdog self-test (a bounded wait that runs out)."""
    return _lib.fa_selftest_watchdog(int(timeout_ms), _stream(stream))


def fa_get_device_status(stream=None) -> int:
    return _lib.fa_get_device_status(_stream(stream))


def fa_get_noalloc_status(stream=None) -> int:
    """Reads and clears the device-side status of fa_fwd_noalloc (kept in the
    library's fixed array); allocates no device memory."""
    return _lib.fa_get_noalloc_status(_stream(stream))


def fa_status_string(code: int) -> str:
    return _lib.fa_status_string(int(code)).decode()


def attention_forward(q, k, v, *, causal: bool = False, scale: float | None = None,
                      cu_seqlens=None, out=None, lse=None):
    """O, lse = attention_forward(q, k, v) on bf16 CUDA tensors.

    Dense: q [B, Hq, N, d], k/v [B, Hkv, N, d]; returns O [B, Hq, N, d] and
    lse [B, Hq, N] (fp32).  Packed (``cu_seqlens`` int32 [B+1] on the device):
    q [N, Hq, d], k/v [N, Hkv, d]; returns O [N, Hq, d] and lse [Hq, N].
    """
    import torch

    if q.dtype != torch.bfloat16 or k.dtype != torch.bfloat16 or v.dtype != torch.bfloat16:
        raise TypeError("q, k, v must be bfloat16")
    if not (q.is_cuda and k.is_cuda and v.is_cuda):
        raise ValueError("q, k, v must be CUDA tensors")
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    if cu_seqlens is None:
        if q.dim() != 4 or k.shape != v.shape or k.dim() != 4:
            raise ValueError("dense layout: q [B,Hq,N,d], k/v [B,Hkv,N,d]")
        B, Hq, N, d = q.shape
        Hkv = k.shape[1]
        if k.shape[0] != B or k.shape[2] != N or k.shape[3] != d:
            raise ValueError("k/v shape does not match q")
        lse_shape = (B, Hq, N)
    else:
        if q.dim() != 3 or k.dim() != 3 or k.shape != v.shape:
            raise ValueError("packed layout: q [N,Hq,d], k/v [N,Hkv,d]")
        N, Hq, d = q.shape
        Hkv = k.shape[1]
        B = cu_seqlens.numel() - 1
        if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda:
            raise ValueError("cu_seqlens must be an int32 CUDA tensor")
        lse_shape = (Hq, N)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(lse_shape, dtype=torch.float32, device=q.device)
    rc = fa_fwd(q, k, v, out, lse, B, Hq, Hkv, N, d, scale, causal, cu_seqlens,
                torch.cuda.current_stream(q.device))
    if rc != FA_OK:
        raise FAError(rc)
    return out, lse
