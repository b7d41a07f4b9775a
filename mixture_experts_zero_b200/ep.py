"""Expert parallelism for the MoE layer with zero-computation experts.

The LongCat-Flash pages deploy the layer with its experts spread over GPUs (llm-wiki entity page,
section 2.2 ScMoE: expert-parallel dispatch and combine; section 5: multi-GPU deployments). Here
G ranks each hold N/G of the N FFN experts, rank r the experts [r N/G, (r+1) N/G), and each rank
routes its own tokens. One forward on every rank:

  1. route and group its tokens' picks by expert over all N experts (lc_moe_route, lc_moe_permute);
     the rows of rank r's experts are one contiguous slice of the grouped rows;
  2. exchange the per-expert row counts (an all-to-all of G x N/G int32), then the rows
     themselves (an all-to-all of bf16 rows). Picks of the zero-computation experts (E_i(x) = x,
     section 2.1) never leave the rank: only FFN rows travel, about K_e/K of the picks;
  3. put the received rows in expert order (lc_moe_ep_regroup_plan + lc_moe_copy_rows), run the
     grouped SwiGLU GEMMs of the local experts (lc_moe_expert_ffn), put the outputs back in
     arrival order (lc_moe_copy_rows, scatter);
  4. return every output row to its source (the inverse all-to-all), where it lands at the
     position the source's grouping gave the input row, and combine with the zero-expert term
     in rank order (lc_moe_combine), exactly as the single-GPU layer does.

The expert counts T_i of the bias update are global-batch quantities: the caller all-reduces the
counts across ranks before lc_moe_bias_update, as in data parallelism.

Every step of the layer runs in the library's kernels (``CudaOps``); the exchanges go through a
``comm`` object with ``rank``, ``size``, ``all_to_all_single(out, inp, out_splits, in_splits)`` and
``all_reduce(t)``: ``TorchComm`` wraps a torch.distributed process group (NCCL over NVLink on
B200s). Both are parameters so that the orchestration can be checked on CPU ranks.
"""
from __future__ import annotations

import numpy as np
import torch

from . import binding as B


def expert_range(N: int, G: int, rank: int) -> tuple[int, int]:
    """FFN experts [lo, hi) held by ``rank`` of ``G`` (N must be a multiple of G)."""
    if N % G:
        raise ValueError(f"N = {N} experts do not split evenly over {G} ranks")
    n_local = N // G
    return rank * n_local, (rank + 1) * n_local


class TorchComm:
    """The exchanges over a torch.distributed process group (default: the world)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.size = dist.get_world_size(group)

    def all_to_all_single(self, out, inp, out_splits, in_splits):
        self.dist.all_to_all_single(out, inp, list(map(int, out_splits)), list(map(int, in_splits)),
                                    group=self.group)

    def all_reduce(self, t):
        self.dist.all_reduce(t, group=self.group)


class CudaOps:
    """The layer's steps on the GPU: the C-ABI kernels through the binding."""

    def route(self, x, wr, bias, K, N, counts):
        idx, gate = B.lc_moe_route(x, wr, bias, K, N, counts=counts)[:2]
        return idx, gate

    def permute(self, idx, N, E, x):
        return B.lc_moe_permute(idx, N, E, x=x)

    def regroup_plan(self, cnt_recv, m):
        return B.lc_moe_ep_regroup_plan(cnt_recv, m_cap=m)

    def copy_rows(self, src, index, scatter):
        return B.lc_moe_copy_rows(src, index, scatter=scatter)

    def expert_ffn(self, x_rows, offsets, w13, w2):
        m = x_rows.shape[0]
        if m == 0:
            return torch.empty(0, w2.shape[1], dtype=torch.bfloat16, device=x_rows.device)
        _, y = B.lc_moe_expert_ffn(x_rows, offsets, w13, w2, m, 1)
        return y

    def combine(self, x, y, idx, gate, pair_row):
        # zero-computation picks are the ones with pair_row = -1; idx is not needed on the GPU
        return B.lc_moe_combine(x, y, gate, pair_row)

    def bias_update(self, bias, counts, T_all, N, Z, K, K_e, mu):
        B.lc_moe_bias_update(bias, counts, T_all, N, Z, K, K_e, mu, reset_counts=True)


class ExpertParallelMoE:
    """One rank of the expert-parallel layer: N FFN experts split over ``comm.size`` ranks, Z
    zero-computation experts, K picks per token. ``w13_local`` / ``w2_local`` hold this rank's
    experts only ([N/G, 2I, d] and [N/G, d, I])."""

    def __init__(self, N: int, Z: int, K: int, comm, ops=None):
        self.N, self.Z, self.K = N, Z, K
        self.comm = comm
        self.ops = ops if ops is not None else CudaOps()
        self.lo, self.hi = expert_range(N, comm.size, comm.rank)
        self.n_local = self.hi - self.lo

    def forward(self, x, wr, bias, w13_local, w2_local, counts=None):
        """MoE(x) for this rank's tokens. Returns (out [T, d], idx [T, K], gate [T, K]);
        ``counts`` ([N + Z] int32) is added to with this rank's picks."""
        G, n_local, N, K = self.comm.size, self.n_local, self.N, self.K
        E = N + self.Z
        T, d = x.shape
        if w13_local.shape[0] != n_local or w2_local.shape[0] != n_local:
            raise ValueError(f"this rank holds {n_local} experts; got {w13_local.shape[0]} / {w2_local.shape[0]}")
        dev = x.device
        # 1. route and group over all N experts
        idx, gate = self.ops.route(x, wr, bias, K, N, counts)
        offsets, row_token, pair_row, x_perm = self.ops.permute(idx, N, E, x)
        # 2. per-expert counts of the rows bound for each rank, then the rows
        off_h = offsets.cpu().numpy().astype(np.int64)
        cnt_send = np.diff(off_h).reshape(G, n_local).astype(np.int32)
        send_splits = cnt_send.sum(axis=1)
        cnt_recv = torch.empty(G, n_local, dtype=torch.int32, device=dev)
        self.comm.all_to_all_single(cnt_recv.view(-1), torch.from_numpy(cnt_send).view(-1).to(dev),
                                    [n_local] * G, [n_local] * G)
        cnt_recv_h = cnt_recv.cpu().numpy().astype(np.int64)
        recv_splits = cnt_recv_h.sum(axis=1)
        m_send, m_recv = int(send_splits.sum()), int(recv_splits.sum())
        recv = torch.empty(m_recv, d, dtype=torch.bfloat16, device=dev)
        self.comm.all_to_all_single(recv, x_perm[:m_send], recv_splits, send_splits)
        # 3. expert order, the local experts, arrival order
        perm, loc_off = self.ops.regroup_plan(cnt_recv, m_recv)
        x_loc = self.ops.copy_rows(recv, perm, False)
        y_loc = self.ops.expert_ffn(x_loc, loc_off, w13_local, w2_local)
        y_recv = self.ops.copy_rows(y_loc, perm, True)
        # 4. outputs back to their sources, then the combine with the zero-expert term
        y = torch.empty(T * K, d, dtype=torch.bfloat16, device=dev)
        self.comm.all_to_all_single(y[:m_send], y_recv, send_splits, recv_splits)
        out = self.ops.combine(x, y, idx, gate, pair_row)
        return out, idx, gate

    def bias_update(self, bias, counts, T_all: int, K_e: int, mu: float):
        """Global expert counts (all-reduced over the ranks), then the bias update of section 2.1
        on the device; ``counts`` is reset."""
        self.comm.all_reduce(counts)
        self.ops.bias_update(bias, counts, T_all, self.N, self.Z, self.K, K_e, mu)
