"""Seeded synthetic inputs for the attention forward.

This module holds no attention arithmetic: it only draws numbers.  Both the
oracle (through the tests and the bench) and the CUDA path are fed from it, so
they see bit-identical bf16 inputs.

Generator (stated here so that any other implementation can reproduce it):

* SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014): draw i (i = 1, 2, ...) of a stream seeded with
  ``seed`` is ``mix(seed + i * 0x9E3779B97F4A7C15 mod 2^64)`` with the
  published two-multiply finaliser.  Being counter-based, any range of draws
  can be produced independently, which is how large tensors are generated in
  parallel chunks.
* Uniforms: ``u = (x >> 11) * 2^-53`` in [0, 1).
* Normals: Box-Muller on consecutive draws (x_2i, x_2i+1):
  ``r = sqrt(-2 ln(1 - u_2i))``, ``z_2i = r cos(2 pi u_2i+1)``,
  ``z_2i+1 = r sin(2 pi u_2i+1)``; a tensor of n values consumes
  n rounded up to even draws.
* Integers in [lo, hi]: ``lo + x mod (hi - lo + 1)``, one draw each.
* bf16: the fp64 normal rounded to nearest-even directly to bf16 (8
  significant bits), then stored as its 16-bit pattern.

Workloads (seed = 1000 + config index; tensors drawn in the order Q, K, V from
one stream; for the packed batch the sequence lengths are drawn first):

* c1: B=1, H=1, N=256, d=64, non-causal
* c2: B=2, H=8, N=4096, d=64, non-causal and causal (same inputs)
* c3: B=1, H=32, N=16384, d=128, causal
* c4: B=1, Hq=32, Hkv=8, N=32768, d=128, causal
* c5: 16 sequences, lengths uniform in [512, 8192], H=16, d=128, causal
* p3: a query chunk of 2048 rows (the last positions) against 16384 keys,
  B=1, H=32, d=128, causal -- the chunked-prefill shape
* dec: one decode step -- 1 query row per (batch, head) against a 32768-key
  cache, B=8, Hq=32, Hkv=8, d=128 (with one row, causal allows every key)
* c3f8: c3's shape with Q, K, V drawn as N(0,1) times 32 and rounded to
  nearest-even FP8 E4M3 (per-tensor scale 1/32); c5f8: c5's batch, c2f8:
  c2's non-causal shape (d = 64), drawn the same way
* E4M3: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits, subnormals in
  steps of 2^-9; the encoder rounds half to even and saturates at 448
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
FP8_SCALE = 1.0 / 32.0      # per-tensor scale of the E4M3 workloads (a power of two)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def splitmix64(seed: int, start: int, count: int) -> np.ndarray:
    """Draws start+1 .. start+count of the SplitMix64 stream seeded ``seed``."""
    with np.errstate(over="ignore"):
        i = np.arange(start + 1, start + 1 + count, dtype=np.uint64)
        return _mix(np.uint64(seed) + i * GAMMA)


def _normals_chunk(seed: int, start: int, count: int) -> np.ndarray:
    # count is even and start is even: pairs never straddle chunks
    x = splitmix64(seed, start, count)
    u = (x >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    u1 = 1.0 - u[0::2]
    u2 = u[1::2]
    r = np.sqrt(-2.0 * np.log(u1))
    t = 2.0 * math.pi * u2
    out = np.empty(count, dtype=np.float64)
    out[0::2] = r * np.cos(t)
    out[1::2] = r * np.sin(t)
    return out


def fp64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to nearest-even bf16 and return the bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    b = x.view(np.uint64)
    lsb = (b >> np.uint64(45)) & np.uint64(1)
    with np.errstate(over="ignore"):
        r = (b + np.uint64((1 << 44) - 1) + lsb) & ~np.uint64((1 << 45) - 1)
    f32 = r.view(np.float64).astype(np.float32)     # exact: 8 significant bits
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def fp64_to_e4m3_bits(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to nearest-even FP8 E4M3 (OCP FP8: 1 sign, 4
    exponent bits with bias 7, 3 mantissa bits, subnormals, no infinities, the
    one NaN pattern per sign never produced): finite values beyond 448 saturate
    to +-448.  Returns the 8-bit patterns."""
    x = np.asarray(x, dtype=np.float64)
    sign = (np.signbit(x)).astype(np.uint8) << np.uint8(7)
    a = np.abs(x)
    code = np.zeros(a.shape, dtype=np.int64)
    sub = a < 2.0 ** -6
    # subnormals (and zero): multiples of 2^-9, rounded half to even
    code[sub] = np.rint(a[sub] * 512.0).astype(np.int64)
    norm = ~sub
    if norm.any():
        f, ex = np.frexp(a[norm])                      # a = f 2^ex, f in [0.5, 1)
        e = ex.astype(np.int64) - 1                     # a = (1 + m) 2^e
        mq = np.rint((2.0 * f - 1.0) * 8.0).astype(np.int64)
        carry = mq == 8
        e[carry] += 1
        mq[carry] = 0
        c = ((e + 7) << 3) | mq
        code[norm] = np.minimum(c, 0x7E)               # 0x7E = 448; larger values saturate
    return (code.astype(np.uint8) | sign).astype(np.uint8)


def bf16_bits_to_float(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


class Stream:
    """One seeded SplitMix64 stream; draws are consumed in order."""

    def __init__(self, seed: int):
        self.seed = int(seed)
        self.pos = 0

    def integers(self, lo: int, hi: int, n: int) -> np.ndarray:
        x = splitmix64(self.seed, self.pos, n)
        self.pos += n
        span = np.uint64(hi - lo + 1)
        return (x % span).astype(np.int64) + lo

    def normal_e4m3(self, shape, inv_scale: float, threads: int = 8) -> np.ndarray:
        """E4M3 bit patterns of i.i.d. N(0,1) draws times ``inv_scale`` (the
        tensor's quantisation: value = code * (1 / inv_scale)), C order."""
        n = int(np.prod(shape))
        draws = n + (n & 1)
        if self.pos & 1:
            self.pos += 1
        base = self.pos
        out = np.empty(n, dtype=np.uint8)

        def work(c0):
            c1 = min(c0 + _CHUNK, draws)
            z = _normals_chunk(self.seed, base + c0, c1 - c0)
            e = min(c1, n)
            out[c0:e] = fp64_to_e4m3_bits(z[: e - c0] * inv_scale)

        starts = range(0, draws, _CHUNK)
        if threads > 1 and draws > _CHUNK:
            with ThreadPoolExecutor(threads) as ex:
                list(ex.map(work, starts))
        else:
            for c0 in starts:
                work(c0)
        self.pos += draws
        return out.reshape(shape)

    def normal_bf16(self, shape, threads: int = 8) -> np.ndarray:
        """bf16 bit patterns of i.i.d. N(0,1) draws, in C order of ``shape``."""
        n = int(np.prod(shape))
        draws = n + (n & 1)
        if self.pos & 1:                 # keep Box-Muller pairs aligned
            self.pos += 1
        base = self.pos
        out = np.empty(n, dtype=np.uint16)

        def work(c0):
            c1 = min(c0 + _CHUNK, draws)
            z = _normals_chunk(self.seed, base + c0, c1 - c0)
            e = min(c1, n)
            out[c0:e] = fp64_to_bf16_bits(z[: e - c0])

        starts = range(0, draws, _CHUNK)
        if threads > 1 and draws > _CHUNK:
            with ThreadPoolExecutor(threads) as ex:
                list(ex.map(work, starts))
        else:
            for c0 in starts:
                work(c0)
        self.pos += draws
        return out.reshape(shape)


@dataclass
class Workload:
    """One attention forward problem: shapes, flags and (once drawn) inputs."""
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int                  # dense: per-sequence length; packed: total tokens
    d: int
    causal: bool
    seed: int
    seqlens: list[int] | None = None
    Nk: int | None = None   # dense query chunk: keys per sequence (the chunk is the last N positions)
    fp8: bool = False       # Q, K, V as E4M3 codes with per-tensor scale FP8_SCALE (see draw)
    q: np.ndarray | None = field(default=None, repr=False)
    k: np.ndarray | None = field(default=None, repr=False)
    v: np.ndarray | None = field(default=None, repr=False)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def packed(self) -> bool:
        return self.seqlens is not None

    @property
    def cu_seqlens(self) -> np.ndarray | None:
        if self.seqlens is None:
            return None
        return np.concatenate([[0], np.cumsum(self.seqlens)]).astype(np.int32)

    @property
    def lengths(self) -> list[int]:
        return list(self.seqlens) if self.packed else [self.N] * self.B

    @property
    def chunk(self) -> bool:
        return self.Nk is not None and not self.packed

    def flops(self) -> float:
        """4*L^2*d per (sequence, head), halved when causal (the convention of
        the metric; the count is of the dense score matrix).  A query chunk
        counts 4*d per attended key per row: 4*d*Nq*Nk, or under the causal
        mask 4*d*sum_i (Nk - Nq + i + 1)."""
        if self.chunk:
            Nq, Nk = self.N, self.Nk
            keys = Nq * (Nk - Nq) + Nq * (Nq + 1) / 2 if self.causal else Nq * Nk
            return 4.0 * self.d * keys * self.B * self.Hq
        f = sum(4.0 * L * L * self.d for L in self.lengths) * self.Hq
        return f / 2 if self.causal else f

    @property
    def decode(self) -> bool:
        """A query chunk of fewer than 128 rows: the split-key path."""
        return self.chunk and self.N < 128

    def hbm_bytes(self) -> float:
        """Bytes the forward must move at least: Q, K, V read once, O (bf16)
        and lse (fp32) written once."""
        nq = self.B * self.Hq * self.N if not self.packed else self.Hq * self.N
        nk = self.B * self.Hkv * (self.Nk if self.chunk else self.N) if not self.packed else self.Hkv * self.N
        return 2.0 * self.d * (2 * nq + 2 * nk) + 4.0 * nq

    def q_shape(self):
        return (self.N, self.Hq, self.d) if self.packed else (self.B, self.Hq, self.N, self.d)

    def kv_shape(self):
        if self.chunk:
            return (self.B, self.Hkv, self.Nk, self.d)
        return (self.N, self.Hkv, self.d) if self.packed else (self.B, self.Hkv, self.N, self.d)

    def total_rows(self) -> int:
        return self.Hq * self.N if self.packed else self.B * self.Hq * self.N

    def draw(self, threads: int = 8) -> "Workload":
        s = Stream(self.seed)
        if self.packed:
            s.pos = self._len_draws
        if self.fp8:
            # N(0,1) samples times 1 / FP8_SCALE = 32 use E4M3's range (|x| <= ~180
            # of 448) while keeping small values out of the subnormals
            inv = 1.0 / FP8_SCALE
            self.q = s.normal_e4m3(self.q_shape(), inv, threads)
            self.k = s.normal_e4m3(self.kv_shape(), inv, threads)
            self.v = s.normal_e4m3(self.kv_shape(), inv, threads)
            return self
        self.q = s.normal_bf16(self.q_shape(), threads)
        self.k = s.normal_bf16(self.kv_shape(), threads)
        self.v = s.normal_bf16(self.kv_shape(), threads)
        return self

    _len_draws: int = 0


def packed_workload(name, nseq, lo, hi, H, d, causal, seed, Hkv=None) -> Workload:
    """Packed batch whose nseq lengths are the first nseq draws of the stream."""
    s = Stream(seed)
    lens = [int(x) for x in s.integers(lo, hi, nseq)]
    w = Workload(name, nseq, H, Hkv or H, int(sum(lens)), d, causal, seed, seqlens=lens)
    w._len_draws = s.pos
    return w


def packed_from_lengths(name, lens, H, d, causal, seed, Hkv=None) -> Workload:
    """Packed batch with given lengths (edge cases); inputs from ``seed``."""
    return Workload(name, len(lens), H, Hkv or H, int(sum(lens)), d, causal, seed,
                    seqlens=[int(x) for x in lens])


def config(name: str) -> Workload:
    """The named workloads c1, c2nc, c2c, c3, c4, c5, p3, dec, c3f8, c5f8, c2f8 (inputs not yet drawn)."""
    if name == "c1":
        return Workload("c1", 1, 1, 1, 256, 64, False, 1001)
    if name == "c2nc":
        return Workload("c2nc", 2, 8, 8, 4096, 64, False, 1002)
    if name == "c2c":
        return Workload("c2c", 2, 8, 8, 4096, 64, True, 1002)
    if name == "c3":
        return Workload("c3", 1, 32, 32, 16384, 128, True, 1003)
    if name == "c4":
        return Workload("c4", 1, 32, 8, 32768, 128, True, 1004)
    if name == "c5":
        return packed_workload("c5", 16, 512, 8192, 16, 128, True, 1005)
    if name == "p3":
        # a 2048-row prefill chunk at the end of a 16384-token sequence,
        # c3's heads and head size
        return Workload("p3", 1, 32, 32, 2048, 128, True, 1006, Nk=16384)
    if name == "c3f8":
        # c3 with Q, K, V in E4M3 (per-tensor scale 1/32)
        return Workload("c3f8", 1, 32, 32, 16384, 128, True, 1008, fp8=True)
    if name == "c2f8":
        # c2's non-causal shape (d = 64) with E4M3 inputs
        return Workload("c2f8", 2, 8, 8, 4096, 64, False, 1009, fp8=True)
    if name == "c5f8":
        # c5's packed batch (same lengths) with E4M3 inputs
        w = packed_workload("c5f8", 16, 512, 8192, 16, 128, True, 1005)
        w.fp8 = True
        return w
    if name == "dec":
        # one new token per sequence of a batch of 8 against a 32768-token
        # cache, c4's grouped heads
        return Workload("dec", 8, 32, 8, 1, 128, True, 1007, Nk=32768)
    raise KeyError(name)


CONFIGS = ("c1", "c2nc", "c2c", "c3", "c4", "c5", "p3", "dec", "c3f8", "c5f8", "c2f8")
