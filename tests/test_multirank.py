"""Row sharding across ranks, on the CPU with gloo and world_size 2.

The forward needs no exchange: each rank's rows give the same codes, scales
and G as the full tensor's rows.  The backward's dgamma is a sum over rows, so
the all-reduced per-rank partials equal the full-tensor dgamma.  The per-rank
arithmetic here is the oracle's (this checks the partition and the collective,
not the kernels).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from normalisation_row_bf16_b200.shard import allreduce_dgamma, max_over_ranks, row_range


def test_row_range_partition():
    for T in (0, 1, 7, 8192, 8193):
        for world in (1, 2, 3, 8):
            spans = [row_range(T, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == T
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            sizes = [hi - lo for lo, hi in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        row_range(10, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from normalisation_row_bf16_b200 import synthetic
        T, D = 37, 256
        x = synthetic.activations(T, D, "outliers", seed=3)
        g = synthetic.gamma(D, seed=3)
        dy = synthetic.upstream_grad(T, D, seed=3)
        lo, hi = row_range(T, rank, world)
        rows = np.arange(lo, hi)
        q, s, G = oracle.mxnorm_fwd(x, g, 2.0, rows=rows)
        _, dg = oracle.mxnorm_bwd(x, dy, g, G, rows=rows)
        dgt = torch.from_numpy(dg)
        allreduce_dgamma(dgt)
        t = max_over_ranks(float(rank + 1))
        out.put((rank, lo, hi, q, s, G, dgt.numpy(), t))
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    import oracle
    from normalisation_row_bf16_b200 import synthetic
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    T, D = 37, 256
    x = synthetic.activations(T, D, "outliers", seed=3)
    g = synthetic.gamma(D, seed=3)
    dy = synthetic.upstream_grad(T, D, seed=3)
    q, s, G = oracle.mxnorm_fwd(x, g, 2.0)
    _, dg = oracle.mxnorm_bwd(x, dy, g, G)
    for rank, lo, hi, qr, sr, Gr, dgr, t in res:
        assert np.array_equal(qr, q[lo:hi]) and np.array_equal(sr, s[lo:hi])
        assert np.array_equal(Gr, G[lo:hi])
        assert np.allclose(dgr, dg, rtol=1e-12, atol=1e-14)
        assert t == 2.0
