"""Context-parallel attention: the token sequence of one video split over G ranks.

The pages name two schemes for sequences too long for one GPU (kwkr.cn Wan
explainer, section 3.2: the token sequence is split over GPUs and recombined
with Ulysses and Ring Attention; "Wan: Open and Advanced Large-Scale Video
Generative Models", section 5: the DiT trains with FSDP + 2-D context parallel,
converting layouts at module boundaries).  Each rank holds S_loc consecutive
tokens of Q, K, V (and dO) with all H heads, [B, S_loc, H, D] bf16.

Ulysses (H divisible by G): one all-to-all turns the sequence shard into all
G*S_loc tokens of Hg = H/G heads; the local full attention (wan_attn_fwd /
wan_attn_bwd) runs unchanged; a second all-to-all turns O (or dQ, dK, dV) back
into sequence shards.  ``wan_attn_cp_layout`` does the block permutations around
the exchanges (none are needed for B = 1 on the head side).

Ring (any H): the K, V shards travel around the ring; at step t rank r attends
its queries to the block of rank (r - t) mod G (wan_attn_cross_fwd) and folds
the partial (O_t, lse_t) into an fp32 running result (wan_attn_cp_merge); the
next block's transfer overlaps the current block's attention.  The backward
recomputes each block's share with the final O and LSE (wan_attn_cross_bwd):
dQ parts add up locally, dK and dV parts add up in fp32 accumulators that
travel with their block and arrive home after G steps (wan_attn_cp_accumulate).

Every compute step is one call of the CUDA library (``LibraryOps``); the
exchanges are torch.distributed calls (``TorchComm``: NCCL on GPUs).  Both are
parameters so the schedule itself can be exercised with other communicators.
"""
from __future__ import annotations

from . import wan_attn as _wa


class LibraryOps:
    """The compute steps of the schedules, each one call of libwan_attn."""

    acc_dtype = None   # torch.float32, set on first use (torch imported lazily)

    def __init__(self):
        import torch
        self.acc_dtype = torch.float32

    def attn_fwd(self, q, k, v):
        return _wa.fwd(q, k, v)

    def attn_bwd(self, q, k, v, o, do, lse):
        return _wa.bwd(q, k, v, o, do, lse)

    def cross_fwd(self, q, k, v):
        return _wa.cross_fwd(q, k, v)

    def cross_bwd(self, q, k, v, o, do, lse):
        return _wa.cross_bwd(q, k, v, o, do, lse)

    def merge(self, o_acc, lse_acc, o_part, lse_part, first, o_out=None):
        _wa.cp_merge(o_acc, lse_acc, o_part, lse_part, first, o_out)

    def accumulate(self, acc, part, first, out=None):
        _wa.cp_accumulate(acc, part, first, out)

    def layout(self, dst, src, B, S_loc, G, Hg, which):
        _wa.cp_layout(dst, src, B, S_loc, G, Hg, which, D=src.shape[-1])


class TorchComm:
    """Exchanges over a torch.distributed process group (the default group if None).

    Without an initialised process group it is a single rank and never communicates."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        if dist.is_available() and dist.is_initialized():
            self.size = dist.get_world_size(group)
            self.rank = dist.get_rank(group)
        else:
            self.size, self.rank = 1, 0

    def _global(self, group_rank: int) -> int:
        if self.group is None:
            return group_rank
        return self.dist.get_global_rank(self.group, group_rank)

    def all_to_all(self, out, inp):
        """Equal chunks along dim 0: chunk g of inp goes to rank g; chunk g of out comes from rank g."""
        self.dist.all_to_all_single(out, inp, group=self.group)

    def ring_start(self, sends, recvs):
        """Start sending each of `sends` to rank + 1 and receiving each of `recvs` from rank - 1;
        returns a handle for ring_wait."""
        d = self.dist
        nxt, prv = self._global((self.rank + 1) % self.size), self._global((self.rank - 1) % self.size)
        ops = [d.P2POp(d.isend, t, nxt, group=self.group) for t in sends]
        ops += [d.P2POp(d.irecv, t, prv, group=self.group) for t in recvs]
        return d.batch_isend_irecv(ops)

    def ring_wait(self, handle):
        for h in handle:
            h.wait()


def _defaults(comm, ops):
    return (comm if comm is not None else TorchComm()), (ops if ops is not None else LibraryOps())


# ---------------------------------------------------------------------------
# Ulysses
# ---------------------------------------------------------------------------
def _to_heads(x, comm, ops):
    """[B, S_loc, H, D] sequence shard -> [B, G*S_loc, H/G, D] head shard (one all-to-all)."""
    import torch
    B, S_loc, H, D = x.shape
    G = comm.size
    Hg = H // G
    send = torch.empty((G, B, S_loc, Hg, D), dtype=x.dtype, device=x.device)
    ops.layout(send, x, B, S_loc, G, Hg, _wa.CP_SEQ_TO_SEND)
    recv = torch.empty_like(send)
    comm.all_to_all(recv, send)
    if B == 1:                                   # [G, 1, S_loc, Hg, D] is already [1, G*S_loc, Hg, D]
        return recv.view(B, G * S_loc, Hg, D)
    out = torch.empty((B, G * S_loc, Hg, D), dtype=x.dtype, device=x.device)
    ops.layout(out, recv, B, S_loc, G, Hg, _wa.CP_RECV_TO_HEADS)
    return out


def _to_seq(xh, comm, ops):
    """[B, G*S_loc, Hg, D] head shard -> [B, S_loc, G*Hg, D] sequence shard (one all-to-all)."""
    import torch
    B, S, Hg, D = xh.shape
    G = comm.size
    S_loc = S // G
    if B == 1:
        send = xh.reshape(G, B, S_loc, Hg, D)
    else:
        send = torch.empty((G, B, S_loc, Hg, D), dtype=xh.dtype, device=xh.device)
        ops.layout(send, xh, B, S_loc, G, Hg, _wa.CP_HEADS_TO_SEND)
    recv = torch.empty_like(send)
    comm.all_to_all(recv, send.contiguous())
    out = torch.empty((B, S_loc, G * Hg, D), dtype=xh.dtype, device=xh.device)
    ops.layout(out, recv, B, S_loc, G, Hg, _wa.CP_RECV_TO_SEQ)
    return out


def ulysses_attn_fwd(q, k, v, comm=None, ops=None):
    """Full attention of the G ranks' joint sequence; returns (o shard, ctx for the backward).

    q, k, v: this rank's [B, S_loc, H, D] shard (equal S_loc on every rank, H % G == 0)."""
    comm, ops = _defaults(comm, ops)
    B, S_loc, H, D = q.shape
    if H % comm.size:
        raise ValueError(f"Ulysses needs the head count ({H}) divisible by the ranks ({comm.size})")
    if comm.size == 1:
        o, lse = ops.attn_fwd(q, k, v)
        return o, (q, k, v, o, lse)
    qh, kh, vh = (_to_heads(x, comm, ops) for x in (q, k, v))
    oh, lse_h = ops.attn_fwd(qh, kh, vh)
    return _to_seq(oh, comm, ops), (qh, kh, vh, oh, lse_h)


def ulysses_attn_bwd(do, ctx, comm=None, ops=None):
    """dQ, dK, dV shards of sum(O * dO) for the forward that returned ctx."""
    comm, ops = _defaults(comm, ops)
    qh, kh, vh, oh, lse_h = ctx
    if comm.size == 1:
        return ops.attn_bwd(qh, kh, vh, oh, do, lse_h)
    doh = _to_heads(do, comm, ops)
    grads = ops.attn_bwd(qh, kh, vh, oh, doh, lse_h)
    return tuple(_to_seq(g, comm, ops) for g in grads)


# ---------------------------------------------------------------------------
# Ring
# ---------------------------------------------------------------------------
def ring_attn_fwd(q, k, v, comm=None, ops=None):
    """Full attention of the joint sequence by Ring Attention; returns (o, lse) of this rank's queries.

    q, k, v: this rank's [B, S_loc, H, D] shard (equal shapes on every rank)."""
    import torch
    comm, ops = _defaults(comm, ops)
    G = comm.size
    B, S_loc, H, D = q.shape
    o = torch.empty_like(q)
    o_acc = torch.empty(q.shape, dtype=ops.acc_dtype, device=q.device)
    lse = torch.empty((B, H, S_loc), dtype=ops.acc_dtype, device=q.device)
    cur = [k, v]                                # the key block held now
    nxt = [torch.empty_like(k), torch.empty_like(v)] if G > 1 else None
    spare = [torch.empty_like(k), torch.empty_like(v)] if G > 2 else None
    for t in range(G):
        more = t + 1 < G
        handle = comm.ring_start(cur, nxt) if more else None          # next block in flight
        o_t, lse_t = ops.cross_fwd(q, cur[0], cur[1])
        ops.merge(o_acc, lse, o_t, lse_t, t == 0, None if more else o)
        if more:
            comm.ring_wait(handle)
            # the block just sent is free again (never the caller's k, v)
            cur, nxt = nxt, (spare if t == 0 else cur)
    return o, lse


def ring_attn_bwd(q, k, v, o, do, lse, comm=None, ops=None):
    """dQ, dK, dV of this rank's shard for the ring forward that returned (o, lse)."""
    import torch
    comm, ops = _defaults(comm, ops)
    G = comm.size
    if G == 1:
        return ops.cross_bwd(q, k, v, o, do, lse)
    dq = torch.empty_like(q)
    dq_acc = torch.empty(q.shape, dtype=ops.acc_dtype, device=q.device)
    cur = [k, v]
    nxt = [torch.empty_like(k), torch.empty_like(v)]
    spare = [torch.empty_like(k), torch.empty_like(v)] if G > 2 else None
    # fp32 dK, dV sums of the block held now; they travel with it and reach home after G passes,
    # the last pass in bf16
    acc = [torch.empty(k.shape, dtype=ops.acc_dtype, device=k.device) for _ in range(2)]
    acc_in = [torch.empty_like(a) for a in acc]
    fin = [torch.empty_like(k), torch.empty_like(v)]
    fin_in = [torch.empty_like(k), torch.empty_like(v)]
    acc_handle = None
    for t in range(G):
        last = t + 1 == G
        kv_handle = comm.ring_start(cur, nxt) if not last else None
        dq_t, dk_t, dv_t = ops.cross_bwd(q, cur[0], cur[1], o, do, lse)
        ops.accumulate(dq_acc, dq_t, t == 0, dq if last else None)
        if t > 0:                               # this block's sums so far, from rank - 1
            comm.ring_wait(acc_handle)
            acc, acc_in = acc_in, acc
        ops.accumulate(acc[0], dk_t, t == 0, fin[0] if last else None)
        ops.accumulate(acc[1], dv_t, t == 0, fin[1] if last else None)
        acc_handle = comm.ring_start(fin, fin_in) if last else comm.ring_start(acc, acc_in)
        if not last:
            comm.ring_wait(kv_handle)
            cur, nxt = nxt, (spare if t == 0 else cur)
    comm.ring_wait(acc_handle)
    return dq, fin_in[0], fin_in[1]
