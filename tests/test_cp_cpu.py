"""Time-sharded context parallelism (frame_wise_gated_b200.cp): the host
logic -- per-rank maps, the all-gather, the prefix and the local scan -- on
CPU with gloo ranks. The per-rank compute runs through a stand-in backend
built on the oracle (test infrastructure), since the CUDA kernels need a GPU;
the GPU test of the kernels' side is tests/test_gpu_cp.py."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class OracleBackend:
    """Same contract as cp.KernelBackend, computed by the float64 oracle."""

    def shard_composite(self, k, v, beta, gamma):
        from oracle import gdn_oracle as O
        B, H, T, S, D = k.shape
        E = torch.empty((B, H, D, D), dtype=torch.float64)
        Hm = torch.empty_like(E)
        g = torch.empty((B, H), dtype=torch.float64)
        for b in range(B):
            for h in range(H):
                C, Hc = O.chunk_composites(k[b, h].numpy(), v[b, h].numpy(), beta[b, h].numpy(),
                                           gamma[b, h].numpy(), list(range(T)), [False] * T)
                gp = float(np.prod(gamma[b, h].numpy()))
                g[b, h] = gp
                E[b, h] = torch.from_numpy(np.eye(D) - C / gp)
                Hm[b, h] = torch.from_numpy(Hc)
        return E, Hm, g

    def prefix(self, E_all, H_all, g_all, state_in, r):
        R, B, H, D = E_all.shape[:4]
        St = torch.zeros((B, H, D, D), dtype=torch.float64) if state_in is None else state_in.clone()
        for p in range(r):
            St = g_all[p][..., None, None] * (St - St @ E_all[p]) + H_all[p]
        return St

    def scan(self, q, k, v, beta, gamma, state_in, *, bidir=False, block_reset=False, block=3,
             state_in_rev=...):
        from oracle import gdn_oracle as O
        a = (q.numpy(), k.numpy(), v.numpy(), beta.numpy(), gamma.numpy())
        o, st = O.gdn_frame_scan(*a, None if state_in is None else state_in.numpy())
        if not bidir:
            return torch.from_numpy(o), torch.from_numpy(st)
        seed = state_in if state_in_rev is ... else state_in_rev
        o_r, st_r = O.gdn_frame_scan(*a, None if seed is None else seed.numpy(), reverse=True,
                                     block=block if block_reset else 0)
        return (torch.from_numpy(o), torch.from_numpy(st), torch.from_numpy(o_r),
                torch.from_numpy(st_r))


def _case(B=1, H=2, T=8, S=5, D=4, seed=3):
    rng = np.random.default_rng(seed)
    return dict(q=rng.standard_normal((B, H, T, S, D)), k=rng.standard_normal((B, H, T, S, D)),
                v=rng.standard_normal((B, H, T, S, D)), beta=rng.random((B, H, T, S)),
                gamma=0.85 + 0.15 * rng.random((B, H, T)),
                s0=0.3 * rng.standard_normal((B, H, D, D)))


def _worker(rank, world, port, q):
    import torch.distributed as dist
    from frame_wise_gated_b200 import cp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = _case()
        T = x["q"].shape[2]
        per = T // world
        sl = slice(rank * per, (rank + 1) * per)
        part = {n: torch.from_numpy(np.ascontiguousarray(x[n][:, :, sl])) for n in
                ("q", "k", "v", "beta", "gamma")}
        out, st = cp.frame_scan_fwd_cp(part["q"], part["k"], part["v"], part["beta"],
                                       part["gamma"], torch.from_numpy(x["s0"]),
                                       backend=OracleBackend())
        dist.barrier()
        q.put((rank, out.numpy(), st.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_cp_ranks_equal_one_sequence(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    from oracle import gdn_oracle as O
    x = _case()
    o_ref, s_ref = O.gdn_frame_scan(x["q"], x["k"], x["v"], x["beta"], x["gamma"], x["s0"])
    got = np.concatenate([r[1] for r in res], axis=2)
    assert np.max(np.abs(got - o_ref)) < 1e-10 * max(1.0, np.max(np.abs(o_ref)))
    assert np.max(np.abs(res[-1][2] - s_ref)) < 1e-10 * max(1.0, np.max(np.abs(s_ref)))


def _worker_bidir(rank, world, port, q, rev_seed):
    import torch.distributed as dist
    from frame_wise_gated_b200 import cp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = _case(T=12, seed=5)
        per = 12 // world
        sl = slice(rank * per, (rank + 1) * per)
        part = {n: torch.from_numpy(np.ascontiguousarray(x[n][:, :, sl])) for n in
                ("q", "k", "v", "beta", "gamma")}
        kw = {} if rev_seed == "default" else dict(state_in_rev=None)
        out, st, out_r, st_r = cp.frame_scan_bidir_cp(
            part["q"], part["k"], part["v"], part["beta"], part["gamma"],
            torch.from_numpy(x["s0"]), block=3, backend=OracleBackend(), **kw)
        dist.barrier()
        q.put((rank, out.numpy(), st.numpy(), out_r.numpy(), st_r.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,rev_seed", [(2, "default"), (4, "default"), (4, "zeros")])
def test_cp_bidirectional_ranks_equal_one_sequence(world, rev_seed):
    """The bidirectional chunk-causal form over 12 frames in blocks of 3, split
    over 2 or 4 gloo ranks (shards of 6 or 3 frames: whole blocks), equals the
    oracle's forward scan and block-reset reverse scan of the whole sequence;
    the reverse seed (state_in, or zeros) reaches only the last block."""
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker_bidir, args=(r, world, port, q, rev_seed))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    from oracle import gdn_oracle as O
    x = _case(T=12, seed=5)
    a = (x["q"], x["k"], x["v"], x["beta"], x["gamma"])
    o_ref, s_ref = O.gdn_frame_scan(*a, x["s0"])
    o_rr, s_rr = O.gdn_frame_scan(*a, x["s0"] if rev_seed == "default" else None, reverse=True,
                                  block=3)
    scale = lambda r: 1e-10 * max(1.0, np.max(np.abs(r)))
    assert np.max(np.abs(np.concatenate([r[1] for r in res], axis=2) - o_ref)) < scale(o_ref)
    assert np.max(np.abs(res[-1][2] - s_ref)) < scale(s_ref)
    assert np.max(np.abs(np.concatenate([r[3] for r in res], axis=2) - o_rr)) < scale(o_rr)
    assert np.max(np.abs(res[0][4] - s_rr)) < scale(s_rr)


def test_cp_bidirectional_rejects_split_blocks():
    from frame_wise_gated_b200 import cp
    x = {n: torch.zeros((1, 1, 4, 2, 4)) for n in ("q", "k", "v")}
    with pytest.raises(ValueError):
        cp.frame_scan_bidir_cp(x["q"], x["k"], x["v"], torch.zeros((1, 1, 4, 2)),
                               torch.ones((1, 1, 4)), block=3, backend=OracleBackend())
