"""Data-parallel bias control over two ranks (gloo, CPU).

The T_i and T_all of the bias-update equation (LongCat-Flash llm-wiki entity page, section 2.1)
are global-batch quantities. When each rank routes its own shard of the batch, all-reducing the
per-rank expert counts and updating with T_all = all tokens must give, on every rank, exactly the
biases of one process that routed the whole batch: the bias trajectory of a few control steps is
compared bit for bit. This is the one cross-rank exchange of the layer (routing, grouping, the
expert GEMMs and the combine are per token).
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle

N, Z, K, K_E, D, T_RANK, STEPS, MU = 16, 8, 6, 4, 64, 96, 3, 3e-2


def _bf16(a):
    return torch.as_tensor(np.asarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _batches(world):
    rng = np.random.default_rng(21)
    wr = _bf16(rng.standard_normal((N + Z, D)) * 0.05)
    xs = [_bf16(rng.standard_normal((T_RANK * world, D))) for _ in range(STEPS)]
    return wr, xs


def _bias0():
    b = np.zeros(N + Z, np.float32)
    b[N:] = 2.0 / (N + Z)
    return b


def _rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        wr, xs = _batches(world)
        b = _bias0()
        traj = []
        for x in xs:
            shard = np.ascontiguousarray(x[rank * T_RANK:(rank + 1) * T_RANK])
            z = oracle.router_logits(shard, wr)
            _, _, counts, bad = oracle.route(z, b, K)
            assert bad == 0
            c = torch.from_numpy(counts.astype(np.int64))
            dist.all_reduce(c)
            b = oracle.bias_update(b, c.numpy().astype(np.int32), T_RANK * world, N, Z, K, K_E, MU)
            traj.append(b.copy())
        q.put((rank, np.stack(traj)))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_rank_count_allreduce_equals_single_process_control():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # one process routing every token of each global batch
    wr, xs = _batches(world)
    b = _bias0()
    ref = []
    for x in xs:
        z = oracle.router_logits(x, wr)
        _, _, counts, _ = oracle.route(z, b, K)
        b = oracle.bias_update(b, counts, T_RANK * world, N, Z, K, K_E, MU)
        ref.append(b.copy())
    ref = np.stack(ref)
    for r in range(world):
        np.testing.assert_array_equal(results[r].view(np.uint32), ref.view(np.uint32))
    # the control moved the biases (the check is not vacuous)
    assert np.any(ref[-1] != _bias0())
