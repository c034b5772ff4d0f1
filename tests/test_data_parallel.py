"""Data-parallel host logic on CPU with two gloo ranks: token sharding, replicated weight
quantisation, and the weight-gradient all-reduce equal the single-process result."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bit_ternary_qat_b200 import dp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_token_shard_covers_everything():
    for T in (1, 7, 4096, 4099):
        for world in (1, 2, 3, 8):
            spans = [dp.token_shard(T, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == T
            for (a, b), (c, d) in zip(spans, spans[1:]):
                assert b == c
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from bit_ternary_qat_b200 import synth
        li = synth.random_case(37, 64, 48, seed=5, dtype="f32")
        a, b = dp.token_shard(37, world, rank)
        gamma, wq = oracle.quant_weight(li.W)
        ok_rep = dp.check_replicated(torch.from_numpy(wq)) and dp.check_replicated(torch.tensor([gamma]))
        r = oracle.rmsnorm_rinv(li.X[a:b], 1e-6)
        _, _, xdq = oracle.act_quant(li.X[a:b], r, None)
        dW = torch.from_numpy(oracle.grad_weight(li.dY[a:b], xdq)).double()
        dp.allreduce_weight_grad(dW)
        q.put((rank, ok_rep, dW.numpy()))
    finally:
        dist.destroy_process_group()


def test_weight_grad_allreduce_matches_single_process():
    import oracle
    from bit_ternary_qat_b200 import synth
    oracle.build()
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    li = synth.random_case(37, 64, 48, seed=5, dtype="f32")
    f = oracle.forward(li.X, li.W)
    dW_full = oracle.grad_weight(li.dY, f["xdq"])
    for rank, ok_rep, dW in res:
        assert ok_rep
        assert np.allclose(dW, dW_full, rtol=1e-6, atol=1e-7)
