"""The context-parallel schedules on gloo ranks (CPU): every rank holds one
sequence shard, runs Ring and Ulysses attention forward and backward with the
fp64 host stand-ins, and the gathered shards must equal the oracle's result on
the whole sequence (kwkr.cn Wan explainer, section 3.2: sequence split over GPUs,
recombined with Ulysses and Ring Attention)."""
import os

import numpy as np
import pytest

import oracle

CASES = [(2, 1, 5, 4, 8), (3, 2, 4, 6, 8), (4, 1, 3, 4, 16)]   # G, B, S_loc, H, D


def _problem(B, S, H, D):
    rng = np.random.default_rng(1000 + S)
    return [rng.standard_normal((B, S, H, D)) for _ in range(4)]   # q, k, v, dO


def _rank_main(rank, G, case, port, outdir):
    import torch
    import torch.distributed as dist
    from cp_helpers import HostOps
    from video_dit_full_b200 import context_parallel as cp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=G)
    try:
        _, B, S_loc, H, D = case
        q, k, v, do = (torch.from_numpy(np.ascontiguousarray(x[:, rank * S_loc:(rank + 1) * S_loc]))
                       for x in _problem(B, G * S_loc, H, D))
        ops, comm = HostOps(), cp.TorchComm()
        assert comm.size == G and comm.rank == rank
        o_r, lse_r = cp.ring_attn_fwd(q, k, v, comm, ops)
        dq_r, dk_r, dv_r = cp.ring_attn_bwd(q, k, v, o_r, do, lse_r, comm, ops)
        o_u, ctx = cp.ulysses_attn_fwd(q, k, v, comm, ops)
        dq_u, dk_u, dv_u = cp.ulysses_attn_bwd(do, ctx, comm, ops)
        np.savez(os.path.join(outdir, f"r{rank}.npz"), o_r=o_r, lse_r=lse_r, dq_r=dq_r, dk_r=dk_r, dv_r=dv_r,
                 o_u=o_u, dq_u=dq_u, dk_u=dk_u, dv_u=dv_u)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", CASES)
def test_ring_and_ulysses_match_the_unsharded_oracle(case, tmp_path):
    import torch.multiprocessing as mp
    G, B, S_loc, H, D = case
    port = 29600 + 7 * G + S_loc
    mp.spawn(_rank_main, args=(G, case, port, str(tmp_path)), nprocs=G, join=True)
    res = [np.load(tmp_path / f"r{r}.npz") for r in range(G)]
    cat = lambda key, axis=1: np.concatenate([x[key] for x in res], axis=axis)
    q, k, v, do = _problem(B, G * S_loc, H, D)
    o, lse = oracle.attn_fwd(q, k, v)
    g = oracle.attn_bwd(q, k, v, do)
    for scheme in ("r", "u"):
        np.testing.assert_allclose(cat("o_" + scheme), o, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(cat("dq_" + scheme), g["dq"], rtol=1e-9, atol=1e-11)
        np.testing.assert_allclose(cat("dk_" + scheme), g["dk"], rtol=1e-9, atol=1e-11)
        np.testing.assert_allclose(cat("dv_" + scheme), g["dv"], rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(cat("lse_r", axis=2), lse, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("G,B,S_loc,H,D", [(3, 1, 5, 3, 8), (4, 2, 3, 4, 8)])
def test_schedules_with_a_synchronous_communicator(G, B, S_loc, H, D):
    """The same schedules over in-process ranks whose exchanges finish inside the call."""
    import torch
    from cp_helpers import HostOps, run_threads
    from video_dit_full_b200 import context_parallel as cp
    q, k, v, do = _problem(B, G * S_loc, H, D)

    def rank(r, comm):
        sh = [torch.from_numpy(np.ascontiguousarray(x[:, r * S_loc:(r + 1) * S_loc])) for x in (q, k, v, do)]
        o, lse = cp.ring_attn_fwd(*sh[:3], comm, HostOps())
        gr = cp.ring_attn_bwd(*sh[:3], o, sh[3], lse, comm, HostOps())
        o_u, ctx = cp.ulysses_attn_fwd(*sh[:3], comm, HostOps())
        return o, gr, o_u, cp.ulysses_attn_bwd(sh[3], ctx, comm, HostOps())

    res = run_threads(G, rank)
    o, _ = oracle.attn_fwd(q, k, v)
    g = oracle.attn_bwd(q, k, v, do)
    for oi, gi in ((0, 1), (2, 3)):
        np.testing.assert_allclose(torch.cat([r[oi] for r in res], dim=1).numpy(), o, rtol=1e-10, atol=1e-12)
        for i, name in enumerate(("dq", "dk", "dv")):
            got = torch.cat([r[gi][i] for r in res], dim=1).numpy()
            np.testing.assert_allclose(got, g[name], rtol=1e-9, atol=1e-11)
