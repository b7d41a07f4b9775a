"""Expert parallelism over CPU ranks (gloo): the orchestration of mixture_experts_zero_b200.ep
(who sends which rows where, the expert-major regrouping, the return exchange, the combine) with
each rank's compute done by the oracle, against one process running the oracle's layer on the
whole batch with all experts.

Ranks hold disjoint experts (rank r: FFN experts [r N/G, (r+1) N/G)) and their own tokens. Only
rows routed to FFN experts travel; zero-computation picks stay on their rank (LongCat-Flash
llm-wiki entity page, section 2.1: E_i(x) = x). Routing indices, gates and counts must be
bit-exact, every output bit-identical to the single-process oracle (each row's expert arithmetic
and each token's rank-order combine are the same computations, only moved between ranks), and
the bias update after the counts all-reduce equal to the single-process update.

The regrouping is restated here from its definition (a stable sort of the received rows by local
expert), independently of the CUDA kernel that does it on the GPU; that kernel is checked against
the same definition in tests/test_gpu_ep.py.
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
from mixture_experts_zero_b200 import ep

N, Z, K, K_E, D, I, T_RANK, MU = 16, 8, 6, 4, 64, 64, 40, 3e-2


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


class OracleOps:
    """Each step of one rank on the CPU: the oracle, or plain index operations."""

    def route(self, x, wr, bias, K, N, counts):
        z = oracle.router_logits(_bits(x), _bits(wr))
        c = np.zeros(wr.shape[0], np.int32)
        idx, gate, c, bad = oracle.route(z, bias.numpy(), K, counts=c)
        assert bad == 0
        if counts is not None:
            counts += torch.from_numpy(c)
        return torch.from_numpy(idx), torch.from_numpy(gate)

    def permute(self, idx, N, E, x):
        T, K = idx.shape
        off, row_token, pair_row = oracle.permute(idx.numpy(), N)
        x_perm = torch.zeros(T * K, x.shape[1], dtype=torch.bfloat16)
        x_perm[: len(row_token)] = x[torch.from_numpy(row_token).long()]
        return torch.from_numpy(off), torch.from_numpy(row_token), torch.from_numpy(pair_row), x_perm

    def regroup_plan(self, cnt_recv, m):
        G, n_local = cnt_recv.shape
        c = cnt_recv.numpy()
        # expert of every received row, in arrival order (source-major, then expert)
        expert_of = np.concatenate([np.repeat(np.arange(n_local), c[s]) for s in range(G)]).astype(np.int64)
        assert expert_of.size == m
        perm = np.argsort(expert_of, kind="stable").astype(np.int32)
        off = np.concatenate([[0], np.cumsum(np.bincount(expert_of, minlength=n_local))]).astype(np.int32)
        return torch.from_numpy(perm), torch.from_numpy(off)

    def copy_rows(self, src, index, scatter):
        idx = index.long()
        if scatter:
            out = torch.empty_like(src[: len(idx)])
            out[idx] = src[: len(idx)]
            return out
        return src[idx].contiguous()

    def expert_ffn(self, x_rows, offsets, w13, w2):
        m = x_rows.shape[0]
        experts = np.repeat(np.arange(w13.shape[0]), np.diff(offsets.numpy())).astype(np.int32)
        assert experts.size == m
        if m == 0:
            return torch.empty(0, w2.shape[1], dtype=torch.bfloat16)
        _, y = oracle.expert_rows(_bits(x_rows), experts, _bits(w13), _bits(w2), want_h=False)
        return _bf16(y)

    def combine(self, x, y, idx, gate, pair_row):
        return _bf16(oracle.combine(_bits(x), _bits(y), idx.numpy(), gate.numpy(), pair_row.numpy(), N))

    def bias_update(self, bias, counts, T_all, N_, Z_, K_, K_e, mu):
        bias.copy_(torch.from_numpy(oracle.bias_update(bias.numpy(), counts.numpy(), T_all, N_, Z_, K_, K_e, mu)))
        counts.zero_()


def _problem(world):
    rng = np.random.default_rng(37)
    x = _bits(torch.from_numpy(rng.standard_normal((T_RANK * world, D)).astype(np.float32)).to(torch.bfloat16))
    wr = _bits(torch.from_numpy((rng.standard_normal((N + Z, D)) * 0.2).astype(np.float32)).to(torch.bfloat16))
    w13 = _bits(torch.from_numpy((rng.standard_normal((N, 2 * I, D)) / D ** 0.5).astype(np.float32)).to(torch.bfloat16))
    w2 = _bits(torch.from_numpy((rng.standard_normal((N, D, I)) / I ** 0.5).astype(np.float32)).to(torch.bfloat16))
    bias = np.zeros(N + Z, np.float32)
    bias[N:] = 1.0 / (N + Z)  # some zero-expert picks on every rank
    return x, wr, w13, w2, bias


def _rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        x, wr, w13, w2, bias = _problem(world)
        comm = ep.TorchComm()
        ops = OracleOps()
        layer = ep.ExpertParallelMoE(N, Z, K, comm, ops=ops)
        lo, hi = layer.lo, layer.hi
        xs = _bf16(x[rank * T_RANK:(rank + 1) * T_RANK])
        counts = torch.zeros(N + Z, dtype=torch.int32)
        out, idx, gate = layer.forward(xs, _bf16(wr), torch.from_numpy(bias), _bf16(w13[lo:hi]),
                                       _bf16(w2[lo:hi]), counts=counts)
        local_counts = counts.clone()
        b = torch.from_numpy(bias.copy())
        layer.bias_update(b, counts, T_RANK * world, K_E, MU)
        q.put((rank, _bits(out), idx.numpy(), gate.numpy(), local_counts.numpy(), b.numpy()))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 4])
def test_expert_parallel_layer_equals_the_single_process_oracle(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        r, *vals = q.get(timeout=180)
        got[r] = vals
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x, wr, w13, w2, bias = _problem(world)
    ref = oracle.forward(x, wr, bias, w13, w2, N, Z, K)
    assert ref["bad"] == 0
    out = np.concatenate([got[r][0] for r in range(world)])
    idx = np.concatenate([got[r][1] for r in range(world)])
    gate = np.concatenate([got[r][2] for r in range(world)])
    np.testing.assert_array_equal(idx, ref["idx"])
    np.testing.assert_array_equal(gate.view(np.uint32), ref["gate"].view(np.uint32))
    np.testing.assert_array_equal(sum(got[r][3] for r in range(world)), ref["counts"])
    # some picks went to zero-computation experts, and some rows crossed ranks
    assert (idx >= N).any()
    owner = idx // (N // world)
    assert any(((owner[r * T_RANK:(r + 1) * T_RANK] != r) & (idx[r * T_RANK:(r + 1) * T_RANK] < N)).any()
               for r in range(world))
    np.testing.assert_array_equal(out, ref["out"])
    b_ref = oracle.bias_update(bias, ref["counts"], T_RANK * world, N, Z, K, K_E, MU)
    for r in range(world):
        np.testing.assert_array_equal(got[r][4].view(np.uint32), b_ref.view(np.uint32))
