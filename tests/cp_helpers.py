"""Test stand-ins for the context-parallel schedules (video_dit_full_b200.context_parallel).

* ``HostOps``: the schedules' compute steps on the CPU in fp64, so the schedules
  can run on gloo ranks without a GPU.  Attention comes from the oracle; a key
  block's share of the backward is written out from its definition with the
  given (global) O and LSE:  P = exp(s - lse), D_i = dO_i . o_i,
  dS = P (dP - D), dQ = dS K / sqrt(D), dK = dS^T Q / sqrt(D), dV = P^T dO.
  Merge, accumulate and the layout permutations are restated with numpy / torch.
* ``ThreadComm``: G ranks as G threads of one process (one GPU), exchanging
  tensors by host-synchronised copies: no kernel ever waits for another.
"""
import threading

import numpy as np

import oracle


class HostOps:
    def __init__(self):
        import torch
        self.torch = torch
        self.acc_dtype = torch.float64

    def _t(self, a):
        return self.torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))

    def attn_fwd(self, q, k, v):
        o, lse = oracle.attn_fwd(q.numpy(), k.numpy(), v.numpy())
        return self._t(o), self._t(lse)

    cross_fwd = attn_fwd

    def cross_bwd(self, q, k, v, o, do, lse):
        q, k, v, o, do, lse = (x.numpy() for x in (q, k, v, o, do, lse))
        B, S, H, D = q.shape
        dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
        for b in range(B):
            for h in range(H):
                Q, K, V, O, dO = (x[b, :, h, :] for x in (q, k, v, o, do))
                p = np.exp(Q @ K.T / np.sqrt(D) - lse[b, h][:, None])
                ds = p * (dO @ V.T - (dO * O).sum(axis=1)[:, None])
                dq[b, :, h] = ds @ K / np.sqrt(D)
                dk[b, :, h] = ds.T @ Q / np.sqrt(D)
                dv[b, :, h] = p.T @ dO
        return self._t(dq), self._t(dk), self._t(dv)

    def attn_bwd(self, q, k, v, o, do, lse):
        return self.cross_bwd(q, k, v, o, do, lse)

    def merge(self, o_acc, lse_acc, o_part, lse_part, first, o_out=None):
        if first:
            o_acc.copy_(o_part)
            lse_acc.copy_(lse_part)
        else:
            la, lp = lse_acc.numpy(), lse_part.numpy()
            ln = np.logaddexp(la, lp)
            wa = np.exp(la - ln).transpose(0, 2, 1)[..., None]     # [B, S, H, 1]
            wp = np.exp(lp - ln).transpose(0, 2, 1)[..., None]
            o_acc.copy_(self._t(wa * o_acc.numpy() + wp * o_part.numpy()))
            lse_acc.copy_(self._t(ln))
        if o_out is not None:
            o_out.copy_(o_acc)

    def accumulate(self, acc, part, first, out=None):
        if first:
            acc.copy_(part)
        else:
            acc.add_(part)
        if out is not None:
            out.copy_(acc)

    def layout(self, dst, src, B, S_loc, G, Hg, which):
        D = src.shape[-1]
        if which == 0:      # [B, S_loc, G, Hg, D] -> [G, B, S_loc, Hg, D]
            y = src.reshape(B, S_loc, G, Hg, D).permute(2, 0, 1, 3, 4)
        elif which in (1, 2):   # [G, B, ...] <-> [B, G, ...]
            y = src.reshape(G if which == 1 else B, B if which == 1 else G, S_loc, Hg, D).permute(1, 0, 2, 3, 4)
        else:               # [G, B, S_loc, Hg, D] -> [B, S_loc, G, Hg, D]
            y = src.reshape(G, B, S_loc, Hg, D).permute(1, 2, 0, 3, 4)
        dst.view(-1).copy_(y.reshape(-1))


class ThreadWorld:
    def __init__(self, G):
        self.G = G
        self.barrier = threading.Barrier(G, timeout=120)
        self.slots = [None] * G


class ThreadComm:
    def __init__(self, world, rank):
        self.world, self.rank, self.size = world, rank, world.G

    def _sync(self):
        import torch
        if torch.cuda.is_available():
            torch.cuda.synchronize()

    def all_to_all(self, out, inp):
        w, G = self.world, self.size
        self._sync()
        w.slots[self.rank] = inp
        w.barrier.wait()
        chunks = out.view(G, -1)
        for g in range(G):
            chunks[g].copy_(w.slots[g].view(G, -1)[self.rank])
        self._sync()
        w.barrier.wait()

    def ring_start(self, sends, recvs):
        w, G = self.world, self.size
        self._sync()
        w.slots[self.rank] = list(sends)
        w.barrier.wait()
        for r, s in zip(recvs, w.slots[(self.rank - 1) % G]):
            r.copy_(s)
        self._sync()
        w.barrier.wait()
        return None

    def ring_wait(self, handle):
        pass


def run_threads(G, fn):
    """Run fn(rank, comm) for every rank on its own thread; returns the results in rank order."""
    world = ThreadWorld(G)
    out, errs = [None] * G, []

    def body(r):
        try:
            out[r] = fn(r, ThreadComm(world, r))
        except BaseException as e:      # noqa: BLE001 - re-raised below
            errs.append(e)
            world.barrier.abort()

    threads = [threading.Thread(target=body, args=(r,)) for r in range(G)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    if errs:
        raise errs[0]
    return out
