"""fp64 CPU oracle for exact attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (the CUDA library and its Python binding) never
imports, links or runs anything here, and this package imports nothing from the
product package.

The arithmetic lives in ``oracle.c`` (plain C, fp64, one OpenMP loop over query
rows); this module only compiles it and marshals numpy arrays through ctypes.
Every function cites the passage of the pages it follows in ``oracle.c``:

* ``softmax``          -- the whole-row softmax (xspy.com, section 3).
* ``online_softmax``   -- the two-pass streaming softmax over blocks
                          (xspy.com, section 3; 14cs17 page, Theorem 2).
* ``attention``        -- standard attention with every score row
                          materialised (14cs17 page, "Standard Attention
                          Memory Analysis").
* ``attention_tiled``  -- the tiled forward with the online-softmax update
                          (14cs17 page, "Flash Attention Algorithm"), in fp64.
* ``attention_kv``     -- a chunk of queries against a longer key sequence,
                          the chunk's rows being its last positions (xspy.com,
                          section 1, chunked prefill).
* ``attention_bwd``    -- dQ, dK, dV of standard attention: the derivative of
                          the forward's definition (the pages name only the
                          recomputation of the backward pass).
* ``e4m3_decode``, ``attention_fp8`` -- FP8 (E4M3) inputs: each code decoded
                          by the format's definition and multiplied by its
                          tensor's scale, then standard attention in fp64
                          (the pages name FP8 only as FlashAttention-3's; the
                          reading is attention of the dequantised inputs).

Pins (in ``tests/test_oracle.py``): the worked examples of both pages, row sums
of one, torch's fp64 scaled-dot-product attention as an independent library
routine, brute force on tiny shapes with no max shift, closed forms (causal row
0, all-zero queries, one dominant key) and the tiled == untiled identity.
The GQA head mapping, the packed-sequence layout and the lse definition rest on
readings of the pages (stated in oracle.c) and are pinned only through the
library routine and brute force that encode the same reading.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", _SRC, "-o", tmp, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def bind(path: str):
    """Load an oracle library from ``path`` and declare its signatures."""
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    i64p = ctypes.POINTER(ctypes.c_int64)
    u16p = ctypes.POINTER(ctypes.c_uint16)
    i32p = ctypes.POINTER(ctypes.c_int32)
    lib.oracle_softmax.restype = ctypes.c_double
    lib.oracle_softmax.argtypes = [dp, ctypes.c_int64, dp]
    lib.oracle_online_softmax.restype = ctypes.c_double
    lib.oracle_online_softmax.argtypes = [dp, i64p, ctypes.c_int64, i64p, dp]
    lib.oracle_attention.restype = ctypes.c_int
    lib.oracle_attention.argtypes = [
        u16p, u16p, u16p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_int, ctypes.c_double, ctypes.c_int, i32p, i64p, ctypes.c_int64,
        dp, dp, ctypes.c_int,
    ]
    lib.oracle_attention_tiled.restype = ctypes.c_int
    lib.oracle_attention_tiled.argtypes = [
        u16p, u16p, u16p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_int, ctypes.c_double, ctypes.c_int, i32p, ctypes.c_int, ctypes.c_int,
        i64p, dp, dp,
    ]
    lib.oracle_attention_kv.restype = ctypes.c_int
    lib.oracle_attention_kv.argtypes = [
        u16p, u16p, u16p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_int, ctypes.c_double, ctypes.c_int, i64p, ctypes.c_int64, dp, dp, ctypes.c_int,
    ]
    lib.oracle_attention_bwd.restype = ctypes.c_int
    lib.oracle_attention_bwd.argtypes = [
        u16p, u16p, u16p, u16p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_double, ctypes.c_int, i64p, ctypes.c_int64, dp, dp, dp, ctypes.c_int,
    ]
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_num_threads.argtypes = []
    return lib


def _load(lib=None):
    global _lib
    if lib is not None:
        return lib
    if _lib is None:
        build()
        _lib = bind(_LIB_PATH)
    return _lib


def _ptr(a: np.ndarray | None, ctype):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def softmax(x, lib=None) -> tuple[np.ndarray, float]:
    """Whole-row softmax in fp64; returns (p, lse)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    p = np.empty_like(x)
    lse = _load(lib).oracle_softmax(_ptr(x, ctypes.c_double), x.size, _ptr(p, ctypes.c_double))
    return p, lse


def online_softmax(x, block_lens, order=None, lib=None) -> tuple[np.ndarray, float]:
    """Two-pass streaming softmax of ``x`` cut into consecutive blocks of
    ``block_lens``, visiting the blocks in ``order``; returns (p, lse)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    bl = np.ascontiguousarray(block_lens, dtype=np.int64)
    if int(bl.sum()) != x.size:
        raise ValueError("block lengths must add up to len(x)")
    od = None if order is None else np.ascontiguousarray(order, dtype=np.int64)
    p = np.empty_like(x)
    lse = _load(lib).oracle_online_softmax(
        _ptr(x, ctypes.c_double), _ptr(bl, ctypes.c_int64), bl.size,
        _ptr(od, ctypes.c_int64), _ptr(p, ctypes.c_double))
    return p, lse


def _as_bits(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("q, k, v are passed as bf16 bit patterns (uint16)")
    return a


def attention(q, k, v, B, Hq, Hkv, N, d, scale, causal, cu_seqlens=None,
              rows=None, nthreads=0, lib=None) -> tuple[np.ndarray, np.ndarray]:
    """Materialised fp64 attention.

    q, k, v: bf16 bit patterns (uint16).  Dense: q [B,Hq,N,d], k/v [B,Hkv,N,d].
    Packed (``cu_seqlens`` given, B+1 int32 offsets): q [N,Hq,d], k/v
    [N,Hkv,d], N = total tokens.  ``rows``: row ids (dense (b*Hq+h)*N+t,
    packed h*N+token) or None for all rows.  Returns (o [nrows, d] fp64,
    lse [nrows] fp64).
    """
    q, k, v = _as_bits(q), _as_bits(k), _as_bits(v)
    cu = None if cu_seqlens is None else np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    total = Hq * N if cu is not None else B * Hq * N
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nrows = total if r is None else r.size
    o = np.zeros((nrows, d), dtype=np.float64)
    lse = np.zeros(nrows, dtype=np.float64)
    rc = _load(lib).oracle_attention(
        _ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16), _ptr(v, ctypes.c_uint16),
        B, Hq, Hkv, N, d, float(scale), int(bool(causal)), _ptr(cu, ctypes.c_int32),
        _ptr(r, ctypes.c_int64), nrows, _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double),
        int(nthreads))
    if rc != 0:
        raise ValueError("oracle_attention: bad arguments or row id out of range")
    return o, lse


def attention_tiled(q, k, v, B, Hq, Hkv, N, d, scale, causal, cu_seqlens=None,
                    br=128, bc=128, kv_order=None, lib=None) -> tuple[np.ndarray, np.ndarray]:
    """The tiled forward with the online-softmax update, in fp64; every row.
    Same arguments and outputs as ``attention`` (rows=None)."""
    q, k, v = _as_bits(q), _as_bits(k), _as_bits(v)
    cu = None if cu_seqlens is None else np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    total = Hq * N if cu is not None else B * Hq * N
    o = np.zeros((total, d), dtype=np.float64)
    lse = np.zeros(total, dtype=np.float64)
    ko = None if kv_order is None else np.ascontiguousarray(kv_order, dtype=np.int64)
    rc = _load(lib).oracle_attention_tiled(
        _ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16), _ptr(v, ctypes.c_uint16),
        B, Hq, Hkv, N, d, float(scale), int(bool(causal)), _ptr(cu, ctypes.c_int32),
        int(br), int(bc), _ptr(ko, ctypes.c_int64), _ptr(o, ctypes.c_double),
        _ptr(lse, ctypes.c_double))
    if rc != 0:
        raise ValueError("oracle_attention_tiled: bad arguments")
    return o, lse


def attention_kv(q, k, v, B, Hq, Hkv, Nq, Nk, d, scale, causal, rows=None, nthreads=0,
                 lib=None) -> tuple[np.ndarray, np.ndarray]:
    """Materialised fp64 attention of a chunk of Nq queries (the last Nq
    positions) against Nk keys.  q [B,Hq,Nq,d], k/v [B,Hkv,Nk,d] bf16 bits;
    row ids (b*Hq+h)*Nq+i.  Returns (o [nrows, d], lse [nrows])."""
    q, k, v = _as_bits(q), _as_bits(k), _as_bits(v)
    total = B * Hq * Nq
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nrows = total if r is None else r.size
    o = np.zeros((nrows, d), dtype=np.float64)
    lse = np.zeros(nrows, dtype=np.float64)
    rc = _load(lib).oracle_attention_kv(
        _ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16), _ptr(v, ctypes.c_uint16),
        B, Hq, Hkv, Nq, Nk, d, float(scale), int(bool(causal)), _ptr(r, ctypes.c_int64), nrows,
        _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_attention_kv: bad arguments or row id out of range")
    return o, lse


def attention_bwd(q, k, v, dout, B, Hq, Hkv, N, d, scale, causal, units=None, nthreads=0,
                  lib=None) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """fp64 gradients (dq, dk, dv) of dense attention for the upstream
    gradient ``dout``.  q, dout [B,Hq,N,d], k/v [B,Hkv,N,d] as bf16 bits.
    ``units``: (batch, kv head) units b*Hkv+hk to compute, or None for all.
    With units=None: dq [B,Hq,N,d], dk/dv [B,Hkv,N,d]; otherwise dq
    [nunits, Hq/Hkv, N, d] and dk/dv [nunits, N, d]."""
    q, k, v, dout = _as_bits(q), _as_bits(k), _as_bits(v), _as_bits(dout)
    g = Hq // Hkv
    u = None if units is None else np.ascontiguousarray(units, dtype=np.int64)
    nunits = B * Hkv if u is None else u.size
    dq = np.zeros((nunits, g, N, d), dtype=np.float64)
    dk = np.zeros((nunits, N, d), dtype=np.float64)
    dv = np.zeros((nunits, N, d), dtype=np.float64)
    rc = _load(lib).oracle_attention_bwd(
        _ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16), _ptr(v, ctypes.c_uint16),
        _ptr(dout, ctypes.c_uint16), B, Hq, Hkv, N, d, float(scale), int(bool(causal)),
        _ptr(u, ctypes.c_int64), nunits, _ptr(dq, ctypes.c_double), _ptr(dk, ctypes.c_double),
        _ptr(dv, ctypes.c_double), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_attention_bwd: bad arguments or unit out of range")
    if u is None:
        return dq.reshape(B, Hq, N, d), dk.reshape(B, Hkv, N, d), dv.reshape(B, Hkv, N, d)
    return dq, dk, dv


def e4m3_decode(codes) -> np.ndarray:
    """FP8 E4M3 codes -> fp64 by the format's definition: sign bit 7,
    exponent bits 6..3 with bias 7, mantissa bits 2..0; exponent field 0 is
    subnormal (mantissa * 2^-9); exponent 15 with mantissa 7 is NaN (no
    infinities)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    val = np.where((e == 15) & ((c & 0x7) == 7), np.nan, val)
    return sign * val


def _exact_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Bit patterns of values that bf16 holds exactly (checked)."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    if not np.array_equal(f.astype(np.float64), x):
        raise ValueError("value not exact in fp32")
    u = f.view(np.uint32)
    if np.any(u & 0xFFFF):
        raise ValueError("dequantised value not exact in bf16: use a power-of-two scale")
    return (u >> 16).astype(np.uint16)


def attention_fp8(q8, k8, v8, q_scale, k_scale, v_scale, B, Hq, Hkv, N, d, scale, causal, rows=None,
                  nthreads=0, lib=None, abs_v=False, cu_seqlens=None) -> tuple[np.ndarray, np.ndarray]:
    """Standard attention, in fp64, of the dequantised E4M3 inputs
    (value = e4m3_decode(code) * tensor scale).  Dense or packed
    (``cu_seqlens``) layouts as ``attention``.  With power-of-two scales every
    dequantised value is exact in bf16, so the fp64 materialised attention of
    ``oracle.c`` runs on them unchanged.  ``abs_v``: use |V| (gives
    sum_j p_j |v_j| per row, the weight the FP8 tolerance is stated in)."""
    qb = _exact_bf16_bits(e4m3_decode(q8) * q_scale)
    kb = _exact_bf16_bits(e4m3_decode(k8) * k_scale)
    vv = e4m3_decode(v8) * v_scale
    vb = _exact_bf16_bits(np.abs(vv) if abs_v else vv)
    return attention(qb, kb, vb, B, Hq, Hkv, N, d, scale, causal, cu_seqlens=cu_seqlens, rows=rows,
                     nthreads=nthreads, lib=lib)


def num_threads() -> int:
    """OpenMP threads the oracle uses."""
    return int(_load().oracle_num_threads())
