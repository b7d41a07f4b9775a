"""GPU parity of the expert-parallel pieces: the regroup plan and the row copies against their
definitions, and the whole expert-parallel layer, with G ranks emulated on one GPU, against the
single-GPU layer.

The emulated ranks are host threads, one CUDA stream each; their exchanges are host-side copies
between the ranks' buffers behind a barrier, with the device synchronised on both sides, so no
kernel ever waits on another rank's kernel (the exchanges a real run does with NCCL).
"""
import threading

import numpy as np
import pytest
import torch

from mixture_experts_zero_b200 import binding as B
from mixture_experts_zero_b200 import ep

from tests.gpu_util import assert_out_close, make, np_bits, oracle_tokens

pytestmark = pytest.mark.gpu


def _plan_ref(cnt: np.ndarray):
    """Expert-major order of rows that arrived source-major: a stable sort by local expert."""
    G, n_local = cnt.shape
    expert_of = np.concatenate([np.repeat(np.arange(n_local), cnt[s]) for s in range(G)]).astype(np.int64)
    perm = np.argsort(expert_of, kind="stable").astype(np.int32)
    off = np.concatenate([[0], np.cumsum(np.bincount(expert_of, minlength=n_local))]).astype(np.int32)
    return perm, off


@pytest.mark.parametrize("G,n_local,hi", [(1, 512, 40), (4, 128, 30), (8, 256, 3), (2048, 1, 5), (3, 5, 0)])
def test_regroup_plan_equals_a_stable_sort_by_expert(cuda_device, G, n_local, hi):
    rng = np.random.default_rng(G * 1000 + n_local)
    cnt = rng.integers(0, hi + 1, size=(G, n_local)).astype(np.int32)
    if hi:
        cnt[rng.integers(G), :] = 0  # a source with nothing for this rank
    ws = B._status_ws("cuda")
    perm, off = B.lc_moe_ep_regroup_plan(torch.from_numpy(cnt).cuda(), ws=ws)
    r_perm, r_off = _plan_ref(cnt)
    np.testing.assert_array_equal(off.cpu().numpy(), r_off)
    np.testing.assert_array_equal(perm.cpu().numpy(), r_perm)
    assert B.lc_moe_read_status(ws) == 0


def test_copy_rows_gather_and_scatter(cuda_device):
    g = torch.Generator(device="cuda").manual_seed(3)
    for n, d in [(1, 64), (1000, 6144), (777, 192), (5, 8)]:
        src = torch.randn(n, d, generator=g, device="cuda").to(torch.bfloat16)
        perm = torch.randperm(n, generator=g, device="cuda").to(torch.int32)
        ws = B._status_ws("cuda")
        got = B.lc_moe_copy_rows(src, perm, ws=ws)
        assert torch.equal(got, src[perm.long()])
        back = B.lc_moe_copy_rows(got, perm, scatter=True, ws=ws)
        assert torch.equal(back, src)
        assert B.lc_moe_read_status(ws) == 0
    # an index outside [0, n) is reported and its row skipped
    src = torch.ones(4, 64, dtype=torch.bfloat16, device="cuda")
    bad = torch.tensor([0, 1, 7, 2], dtype=torch.int32, device="cuda")
    ws = B._status_ws("cuda")
    B.lc_moe_copy_rows(src, bad, ws=ws)
    assert B.lc_moe_read_status(ws, raise_on_error=False) == B.DEV_IDX_RANGE


class ThreadComm:
    """G emulated ranks in one process: exchanges are device copies between the ranks' buffers,
    synchronised on the host."""

    class Shared:
        def __init__(self, G):
            self.G = G
            self.barrier = threading.Barrier(G)
            self.slots = [None] * G

    def __init__(self, shared, rank):
        self.sh, self.rank, self.size = shared, rank, shared.G

    def all_to_all_single(self, out, inp, out_splits, in_splits):
        torch.cuda.synchronize()
        self.sh.slots[self.rank] = (inp, [int(v) for v in in_splits])
        self.sh.barrier.wait()
        pos = 0
        for s in range(self.size):
            src, splits = self.sh.slots[s]
            lo = sum(splits[: self.rank])
            n = splits[self.rank]
            assert n == int(out_splits[s])
            out[pos:pos + n].copy_(src[lo:lo + n])
            pos += n
        torch.cuda.synchronize()
        self.sh.barrier.wait()

    def all_reduce(self, t):
        torch.cuda.synchronize()
        self.sh.slots[self.rank] = (t.clone(), None)
        self.sh.barrier.wait()
        total = sum(self.sh.slots[s][0] for s in range(self.size))
        self.sh.barrier.wait()
        t.copy_(total)
        torch.cuda.synchronize()


@pytest.mark.parametrize("G", [2, 4])
def test_expert_parallel_layer_on_emulated_ranks(cuda_device, G):
    """The small workload split over G emulated ranks (tokens and experts): routing equal to the
    single-GPU layer's bit for bit, outputs within the layer's tolerance of the oracle's MoE
    equation on that routing, expert counts and biases after the update equal."""
    d = make("small", grid=True)
    w = d["w"]
    T_r = w.T // G
    shared = ThreadComm.Shared(G)
    results = [None] * G
    errors = []

    def rank_main(r):
        try:
            with torch.cuda.stream(torch.cuda.Stream()):
                layer = ep.ExpertParallelMoE(w.N, w.Z, w.K, ThreadComm(shared, r))
                counts = torch.zeros(w.E, dtype=torch.int32, device="cuda")
                xs = d["x"][r * T_r:(r + 1) * T_r].contiguous()
                out, idx, gate = layer.forward(xs, d["wr"], d["bias"], d["w13"][layer.lo:layer.hi].contiguous(),
                                               d["w2"][layer.lo:layer.hi].contiguous(), counts=counts)
                local = counts.clone()
                bias = d["bias"].clone()
                layer.bias_update(bias, counts, w.T, w.K_e, w.mu)
                torch.cuda.synchronize()
                results[r] = (out, idx, gate, local, bias)
        except Exception as e:  # noqa: BLE001
            errors.append(e)
            shared.barrier.abort()

    threads = [threading.Thread(target=rank_main, args=(r,)) for r in range(G)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not errors, errors
    out = torch.cat([results[r][0] for r in range(G)])
    idx = torch.cat([results[r][1] for r in range(G)])
    gate = torch.cat([results[r][2] for r in range(G)])
    counts = sum(results[r][3] for r in range(G))
    # the single-GPU layer on the whole batch
    ref_counts = torch.zeros(w.E, dtype=torch.int32, device="cuda")
    ref_idx = torch.empty(w.T, w.K, dtype=torch.int32, device="cuda")
    ref_gate = torch.empty(w.T, w.K, dtype=torch.float32, device="cuda")
    ref_out = B.lc_moe_forward(d["x"], d["wr"], d["bias"], d["w13"], d["w2"], w.K, idx=ref_idx, gate=ref_gate,
                               counts=ref_counts)
    assert torch.equal(idx, ref_idx) and torch.equal(gate, ref_gate) and torch.equal(counts, ref_counts)
    ref_bias = d["bias"].clone()
    B.lc_moe_bias_update(ref_bias, ref_counts, w.T, w.N, w.Z, w.K, w.K_e, w.mu, reset_counts=True)
    for r in range(G):
        assert torch.equal(results[r][4], ref_bias)
    tokens = np.arange(0, w.T, 5)
    exact = oracle_tokens(np_bits(d["x"]), tokens, idx.cpu().numpy(), gate.cpu().numpy(), w.N, d["w13"], d["w2"])
    assert_out_close(np_bits(out)[tokens], exact, what=f"expert-parallel out, G={G}")
    # the same per-row arithmetic as the single-GPU layer: nearly all outputs bit-identical
    assert (out == ref_out).float().mean().item() > 0.99
