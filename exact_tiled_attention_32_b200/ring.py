"""Ring attention: the attention forward of one long sequence split over ranks.

The "Flash Attention" page (14cs17.netlify.app, *Research Perspective*) names
ring attention for distributed long context.  The sequence is cut into
``world`` contiguous shards; rank r holds query, key and value positions
[r L, (r+1) L).  Over ``world`` steps every rank keeps its queries and passes
its current key/value shard to rank r+1 while receiving the next one from
rank r-1, so that at step t it holds shard (r - t) mod world.  Each step
writes this rank's fp32 share (O / l and the logsumexp over the step's keys,
``fa_fwd_partial``); the shares are merged at the end with the online-softmax
rescale applied to whole key ranges (``fa_merge_partials``).

Under the causal mask a query at position p sees keys at positions <= p, so a
shard from a lower rank is seen in full, the rank's own shard through the
causal diagonal, and a shard from a higher rank not at all (its step adds
nothing and no kernel runs).

Every kernel is in libfa.so; this module only schedules them and moves the
key/value shards with torch.distributed point-to-point operations (NCCL on
GPUs), which run on the communication stream while the step's kernel runs on
the compute stream.

With contiguous shards the causal work is uneven: rank r has r + 1 non-empty
steps.  The zig-zag assignment (``ring_attention_forward_zigzag``) cuts the
sequence into 2 world chunks of C positions and gives rank r chunks r and
2 world - 1 - r; at every step each rank then has the same work (two full
C x C blocks, or at step 0 two diagonal blocks and one full one).
"""
from __future__ import annotations

import math

FULL, DIAG, SKIP = "full", "diag", "skip"


def ring_schedule(rank: int, world: int, causal: bool) -> list[tuple[int, str]]:
    """(source shard, mode) of each step of ``rank``: at step t the rank
    holds shard (rank - t) mod world; mode is FULL (every key allowed), DIAG
    (the causal diagonal shard) or SKIP (no key allowed)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    out = []
    for t in range(world):
        src = (rank - t) % world
        if not causal or src < rank:
            out.append((src, FULL))
        elif src == rank:
            out.append((src, DIAG))
        else:
            out.append((src, SKIP))
    return out


class DistExchange:
    """Passes key/value shards around the ring with torch.distributed
    point-to-point operations: send to rank+1, receive from rank-1."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def start(self, send, recv):
        """Starts sending the tensors ``send`` and receiving into ``recv``;
        returns the requests."""
        dist = self.dist
        nxt = (self.rank + 1) % self.world
        prv = (self.rank - 1) % self.world
        if self.group is not None:
            nxt = dist.get_global_rank(self.group, nxt)
            prv = dist.get_global_rank(self.group, prv)
        ops = []
        # even ranks send first, odd ranks receive first, so that a blocking
        # backend pairs the operations without a cycle
        pairs = [(dist.isend, t, nxt) for t in send], [(dist.irecv, t, prv) for t in recv]
        order = pairs if self.rank % 2 == 0 else pairs[::-1]
        for group_ops in order:
            for fn, t, peer in group_ops:
                ops.append(dist.P2POp(fn, t, peer, self.group))
        return dist.batch_isend_irecv(ops)

    @staticmethod
    def wait(reqs):
        for r in reqs:
            r.wait()


def _shapes(q, k, v):
    if q.dim() != 4 or k.dim() != 4 or k.shape != v.shape:
        raise ValueError("dense shards: q [B,Hq,L,d], k/v [B,Hkv,L,d]")
    B, Hq, L, d = q.shape
    if k.shape[0] != B or k.shape[2] != L or k.shape[3] != d:
        raise ValueError("k/v shard shape does not match q")
    return B, Hq, k.shape[1], L, d


def ring_attention_forward(q, k, v, *, causal: bool = False, scale: float | None = None, group=None):
    """O, lse of this rank's query shard against the whole sequence.

    q [B, Hq, L, d], k/v [B, Hkv, L, d]: bf16 CUDA tensors, this rank's
    shard (positions [rank L, (rank+1) L)).  Every rank of ``group`` calls it
    with shards of the same shape.  Returns O [B, Hq, L, d] (bf16) and lse
    [B, Hq, L] (fp32) of the rank's rows."""
    import torch
    from . import binding as fa

    B, Hq, Hkv, L, d = _shapes(q, k, v)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    ex = DistExchange(group)
    world, rank = ex.world, ex.rank
    rows = B * Hq * L
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    o_parts = torch.empty((world, rows, d), dtype=torch.float32, device=q.device)
    lse_parts = torch.empty((world, rows), dtype=torch.float32, device=q.device)
    stream = torch.cuda.current_stream(q.device)
    # step t computes on bufs[cur] while sending it on and receiving the next
    # shard into bufs[1 - cur]; the caller's k, v are only ever sent
    bufs = [(k, v), (torch.empty_like(k), torch.empty_like(v))]
    cur = 0
    for t, (src, mode) in enumerate(ring_schedule(rank, world, causal)):
        reqs = None
        if t + 1 < world:
            reqs = ex.start(list(bufs[cur]), list(bufs[1 - cur]))
        kc, vc = bufs[cur]
        if mode == SKIP:
            lse_parts[t].fill_(-math.inf)
        else:
            rc = fa.fa_fwd_partial(q, kc, vc, o_parts[t], lse_parts[t], B, Hq, Hkv, L, L, d, scale, mode == DIAG,
                                   stream)
            if rc != fa.FA_OK:
                raise fa.FAError(rc, "fa_fwd_partial")
        if reqs is not None:
            ex.wait(reqs)
            cur = 1 - cur
            if t == 0:
                # the next receive goes into a fresh pair, not the caller's k, v
                bufs[1 - cur] = (torch.empty_like(k), torch.empty_like(v))
    o = torch.empty((B, Hq, L, d), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device)
    rc = fa.fa_merge_partials(o_parts, lse_parts, world, rows, d, o, lse, stream)
    if rc != fa.FA_OK:
        raise fa.FAError(rc, "fa_merge_partials")
    return o, lse


def emulate_ring_forward(q, k, v, world: int, *, causal: bool = False, scale: float | None = None):
    """Every rank of a ``world``-rank ring run one after the other on this
    device, each step's shard taken directly from the full tensors (no
    communication): the ring's schedule, per-step kernels and merge, checked
    on one GPU.  q [B, Hq, N, d], k/v [B, Hkv, N, d] with N = world * L.
    Returns the full O and lse."""
    import torch
    from . import binding as fa

    B, Hq, Hkv, N, d = _shapes(q, k, v)
    if N % world:
        raise ValueError("N must be a multiple of world")
    L = N // world
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    stream = torch.cuda.current_stream(q.device)
    rows = B * Hq * L
    o = torch.empty((B, Hq, N, d), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    for rank in range(world):
        qs = q[:, :, rank * L:(rank + 1) * L].contiguous()
        o_parts = torch.empty((world, rows, d), dtype=torch.float32, device=q.device)
        lse_parts = torch.empty((world, rows), dtype=torch.float32, device=q.device)
        for t, (src, mode) in enumerate(ring_schedule(rank, world, causal)):
            if mode == SKIP:
                lse_parts[t].fill_(-math.inf)
                continue
            ks = k[:, :, src * L:(src + 1) * L].contiguous()
            vs = v[:, :, src * L:(src + 1) * L].contiguous()
            rc = fa.fa_fwd_partial(qs, ks, vs, o_parts[t], lse_parts[t], B, Hq, Hkv, L, L, d, scale, mode == DIAG,
                                   stream)
            if rc != fa.FA_OK:
                raise fa.FAError(rc, "fa_fwd_partial")
        os_ = torch.empty((B, Hq, L, d), dtype=torch.bfloat16, device=q.device)
        ls_ = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device)
        rc = fa.fa_merge_partials(o_parts, lse_parts, world, rows, d, os_, ls_, stream)
        if rc != fa.FA_OK:
            raise fa.FAError(rc, "fa_merge_partials")
        o[:, :, rank * L:(rank + 1) * L] = os_
        lse[:, :, rank * L:(rank + 1) * L] = ls_
    return o, lse


# ---------------------------------------------------------------- zig-zag
def zigzag_chunks(rank: int, world: int) -> tuple[int, int]:
    """The two chunks (of 2 world equal chunks of the sequence) that ``rank``
    holds, in the order of its local shard."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    return rank, 2 * world - 1 - rank


def zigzag_schedule(rank: int, world: int, causal: bool) -> list[tuple[int, list[tuple[int, int, str]]]]:
    """Per step t: (source rank, [(query half, key half, mode), ...]) for the
    four chunk pairs of the rank's two query chunks and the two key chunks it
    holds at that step (those of rank (rank - t) mod world).  Mode as
    ``ring_schedule``: a key chunk below the query chunk is FULL, the same
    chunk DIAG, a later one SKIP."""
    qa = zigzag_chunks(rank, world)
    out = []
    for t in range(world):
        src = (rank - t) % world
        kb = zigzag_chunks(src, world)
        pairs = []
        for qi, a in enumerate(qa):
            for ki, b in enumerate(kb):
                mode = FULL if (not causal or b < a) else DIAG if b == a else SKIP
                pairs.append((qi, ki, mode))
        out.append((src, pairs))
    return out


def zigzag_shard(x, rank: int, world: int):
    """The zig-zag local shard of a full-sequence tensor x [B, H, N, d]
    (N = 2 world C): chunks rank and 2 world - 1 - rank, concatenated along
    the sequence, contiguous [B, H, 2C, d]."""
    import torch
    N = x.shape[2]
    if N % (2 * world):
        raise ValueError("N must be a multiple of 2 * world")
    C = N // (2 * world)
    a, b = zigzag_chunks(rank, world)
    return torch.cat([x[:, :, a * C:(a + 1) * C], x[:, :, b * C:(b + 1) * C]], dim=2).contiguous()


def zigzag_unshard(shards, world: int):
    """Inverse of ``zigzag_shard``: the full-sequence tensor from the local
    shards of ranks 0 .. world - 1 (each [B, H, 2C, ...])."""
    import torch
    C = shards[0].shape[2] // 2
    chunks = [None] * (2 * world)
    for r, x in enumerate(shards):
        a, b = zigzag_chunks(r, world)
        chunks[a], chunks[b] = x[:, :, :C], x[:, :, C:]
    return torch.cat(chunks, dim=2)


def _halves(x):
    C = x.shape[2] // 2
    return x[:, :, :C].contiguous(), x[:, :, C:].contiguous()


def _zigzag_step(fa, qh, kh, vh, pairs, t, o_parts, lse_parts, B, Hq, Hkv, C, d, scale, stream):
    """The four chunk pairs of one step: each query half's share of each key
    half goes to part 2 t + key half of that query half."""
    for qi, ki, mode in pairs:
        slot = 2 * t + ki
        if mode == SKIP:
            lse_parts[qi][slot].fill_(-math.inf)
            continue
        rc = fa.fa_fwd_partial(qh[qi], kh[ki], vh[ki], o_parts[qi][slot], lse_parts[qi][slot], B, Hq, Hkv, C, C, d,
                               scale, mode == DIAG, stream)
        if rc != fa.FA_OK:
            raise fa.FAError(rc, "fa_fwd_partial")


def _zigzag_merge(fa, o_parts, lse_parts, world, B, Hq, C, d, device, stream):
    import torch
    rows = B * Hq * C
    outs, lses = [], []
    for qi in range(2):
        o = torch.empty((B, Hq, C, d), dtype=torch.bfloat16, device=device)
        lse = torch.empty((B, Hq, C), dtype=torch.float32, device=device)
        rc = fa.fa_merge_partials(o_parts[qi], lse_parts[qi], 2 * world, rows, d, o, lse, stream)
        if rc != fa.FA_OK:
            raise fa.FAError(rc, "fa_merge_partials")
        outs.append(o)
        lses.append(lse)
    return torch.cat(outs, dim=2), torch.cat(lses, dim=2)


def ring_attention_forward_zigzag(q, k, v, *, causal: bool = False, scale: float | None = None, group=None):
    """Ring attention with the zig-zag assignment.  q [B, Hq, 2C, d], k/v
    [B, Hkv, 2C, d]: bf16 CUDA tensors, this rank's zig-zag shard (chunks
    rank and 2 world - 1 - rank of the sequence, see ``zigzag_shard``).
    Returns O [B, Hq, 2C, d] (bf16) and lse [B, Hq, 2C] (fp32) in the same
    local layout."""
    import torch
    from . import binding as fa

    B, Hq, Hkv, L, d = _shapes(q, k, v)
    if L % 2:
        raise ValueError("a zig-zag shard holds two chunks of equal length")
    C = L // 2
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    ex = DistExchange(group)
    world, rank = ex.world, ex.rank
    rows = B * Hq * C
    qh = _halves(q)
    o_parts = [torch.empty((2 * world, rows, d), dtype=torch.float32, device=q.device) for _ in range(2)]
    lse_parts = [torch.empty((2 * world, rows), dtype=torch.float32, device=q.device) for _ in range(2)]
    stream = torch.cuda.current_stream(q.device)
    k0, k1 = _halves(k)
    v0, v1 = _halves(v)
    bufs = [(k0, k1, v0, v1), tuple(torch.empty_like(x) for x in (k0, k1, v0, v1))]
    cur = 0
    for t, (src, pairs) in enumerate(zigzag_schedule(rank, world, causal)):
        reqs = None
        if t + 1 < world:
            reqs = ex.start(list(bufs[cur]), list(bufs[1 - cur]))
        kc0, kc1, vc0, vc1 = bufs[cur]
        _zigzag_step(fa, qh, (kc0, kc1), (vc0, vc1), pairs, t, o_parts, lse_parts, B, Hq, Hkv, C, d, scale, stream)
        if reqs is not None:
            ex.wait(reqs)
            cur = 1 - cur
    return _zigzag_merge(fa, o_parts, lse_parts, world, B, Hq, C, d, q.device, stream)


def emulate_zigzag_forward(q, k, v, world: int, *, causal: bool = False, scale: float | None = None):
    """Every rank of a ``world``-rank zig-zag ring run one after the other on
    this device, each step's chunks taken directly from the full tensors (no
    communication).  q [B, Hq, N, d], k/v [B, Hkv, N, d] with N = 2 world C.
    Returns the full O and lse."""
    import torch
    from . import binding as fa

    B, Hq, Hkv, N, d = _shapes(q, k, v)
    if N % (2 * world):
        raise ValueError("N must be a multiple of 2 * world")
    C = N // (2 * world)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    stream = torch.cuda.current_stream(q.device)
    rows = B * Hq * C
    o_shards, lse_shards = [], []
    for rank in range(world):
        qh = _halves(zigzag_shard(q, rank, world))
        o_parts = [torch.empty((2 * world, rows, d), dtype=torch.float32, device=q.device) for _ in range(2)]
        lse_parts = [torch.empty((2 * world, rows), dtype=torch.float32, device=q.device) for _ in range(2)]
        for t, (src, pairs) in enumerate(zigzag_schedule(rank, world, causal)):
            kh = _halves(zigzag_shard(k, src, world))
            vh = _halves(zigzag_shard(v, src, world))
            _zigzag_step(fa, qh, kh, vh, pairs, t, o_parts, lse_parts, B, Hq, Hkv, C, d, scale, stream)
        o, lse = _zigzag_merge(fa, o_parts, lse_parts, world, B, Hq, C, d, q.device, stream)
        o_shards.append(o)
        lse_shards.append(lse.unsqueeze(-1))
    return zigzag_unshard(o_shards, world), zigzag_unshard(lse_shards, world).squeeze(-1)

