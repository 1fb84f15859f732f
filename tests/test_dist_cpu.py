"""Token-sharded replicas on CPU (gloo, world size 2): the expert counts are
summed over ranks, the slowest rank's time is reported, and the global bias
step computed from the summed counts is identical on every rank."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle
    from mixture_experts_layer_limited_b200 import dist as mdist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        E, T, k = 16, 64, 4
        rng = np.random.default_rng(100 + rank)
        # each replica routes its own tokens
        L = rng.standard_normal((T, E)).astype(np.float32)
        r = oracle.route_from_logits(L, k, 1, 1, "sigmoid", True, 1.0, np.zeros(E, np.float32))
        local = torch.from_numpy(r.counts.astype(np.int32))
        counts = local.clone()
        mdist.allreduce_counts_(counts)
        t = mdist.max_over_ranks(1.0 + rank)
        bias = oracle.bias_update(counts.numpy(), np.zeros(E, np.float32), 0.001, T * world, k)
        out[rank] = (local.numpy().tolist(), counts.numpy().tolist(), t, bias.tolist())
        mdist.barrier()
    finally:
        dist.destroy_process_group()


def test_replicas_sum_counts_and_agree_on_bias():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    l0, c0, t0, b0 = out[0]
    l1, c1, t1, b1 = out[1]
    assert c0 == c1 == (np.array(l0) + np.array(l1)).tolist()
    assert sum(c0) == 2 * 64 * 4
    assert t0 == t1 == 2.0                      # max over ranks
    assert b0 == b1                             # replicas keep one bias
