"""The N > 1 host logic on CPU: world-size-2 gloo process groups check batch
sharding and the parameter-gradient all-reduce against the oracle on the full
batch, and the max-over-ranks timing reduction."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from discrete_selective_ssm_b200.parallel import (allreduce_param_grads, max_over_ranks,
                                                  shard_batch)


def test_shard_batch_covers_disjointly():
    for B in (0, 1, 5, 16, 17):
        for W in (1, 2, 3, 8):
            parts = [shard_batch(B, r, W) for r in range(W)]
            assert parts[0][0] == 0 and parts[-1][1] == B
            for (a, b), (c, _) in zip(parts, parts[1:]):
                assert b == c and a <= b
            sizes = [b - a for a, b in parts]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_batch(4, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        import oracle
        r = np.random.default_rng(5)
        Bt, L, d, N = 3, 12, 4, 8
        t = dict(u=r.normal(size=(Bt, L, d)), a=r.normal(3, 1, size=(Bt, L, d)),
                 b=r.normal(-1, 1, size=(Bt, L, d)), B=r.normal(size=(Bt, L, N)),
                 C=r.normal(size=(Bt, L, N)), z=r.normal(size=(Bt, L, d)),
                 dout=r.normal(size=(Bt, L, d)))
        w, bias, D = r.normal(0, .5, (d, 4)), r.normal(size=(d,)), r.normal(size=(d,))
        s0, s1 = shard_batch(Bt, rank, world)
        sl = {k: v[s0:s1] for k, v in t.items()}
        g = oracle.block_bwd(sl["u"], w, bias, sl["a"], sl["b"], sl["B"], sl["C"], sl["z"], D,
                             None, sl["dout"])
        tg = {k: torch.tensor(g[k]) for k in ("dD", "dconv_w", "dconv_b")}
        allreduce_param_grads(tg)
        full = oracle.block_bwd(t["u"], w, bias, t["a"], t["b"], t["B"], t["C"], t["z"], D,
                                None, t["dout"])
        ok = all(np.allclose(tg[k].numpy(), full[k], rtol=1e-12, atol=1e-12)
                 for k in ("dD", "dconv_w", "dconv_b"))
        m = max_over_ranks(10.0 + rank)
        q.put((rank, ok, m))
        dist.barrier()
        dist.destroy_process_group()
    except Exception as e:  # report instead of hanging the parent
        q.put((rank, repr(e), None))


def test_two_rank_gloo_param_grads_and_timing():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    for rank, ok, m in res:
        assert ok is True, f"rank {rank}: {ok}"
        assert m == 11.0
