"""Every tile kind the grouped expert GEMMs build at the full prefill workload, checked against the
oracle element by element, and end to end through the layer.

The grouped GEMMs (LongCat-Flash llm-wiki entity page, section 2.1: only the N FFN experts do
work) split each expert's rows into tiles by its row count c:
  GEMM 1 (gate/up + SwiGLU): c < 128: weight tiles only ("cold"); otherwise floor(c/256) full
    256-row tiles, a remainder of 128..255 rows as one more (padded) row tile, and a remainder
    below 128 rows as leftover weight tiles;
  GEMM 2 (down): the same row rules as GEMM 1 (weight tiles below 128 rows, a padded
    128..255-row remainder tile, leftover weight tiles below 128 rows); its weight tiles take the
    double form of 512 output features per tile (d is a multiple of 512 here).
The rules are restated here from that description, independently of the kernel, to pick rows: for
each kind, the first and the last row of one tile of that kind (every output column of those rows
is checked, so every feature tile of both accumulators is covered). The test fails if the
workload does not produce a kind at all, so it cannot pass vacuously.
"""
import numpy as np
import pytest
import torch

from mixture_experts_zero_b200 import binding as B

from tests.gpu_util import (assert_out_close, assert_within_ulp, expert_down_sampled,
                            expert_rows_sampled, make, np_bits, oracle_tokens)

pytestmark = pytest.mark.gpu


def tile_rows(off: np.ndarray):
    """{(gemm, kind): (expert, first row, last row)} for one tile of each kind."""
    found = {}

    def note(key, e, r0, r1):
        found.setdefault(key, (e, int(r0), int(r1)))

    for e in range(len(off) - 1):
        o, c = int(off[e]), int(off[e + 1] - off[e])
        if c == 0:
            continue
        # GEMM 1
        if c < 128:
            note((1, "cold weight tile"), e, o, o + c - 1)
        else:
            nfull, rem = divmod(c, 256)
            if nfull:
                note((1, "full 256-row tile"), e, o, o + 255)
                if nfull > 1:
                    note((1, "full 256-row tile, last block"), e, o + (nfull - 1) * 256, o + nfull * 256 - 1)
            if rem >= 128:
                note((1, "padded 128..255-row remainder tile"), e, o + nfull * 256, o + c - 1)
            elif rem > 0:
                note((1, "leftover weight tile"), e, o + nfull * 256, o + c - 1)
        # GEMM 2
        if c < 128:
            note((2, "cold double weight tile"), e, o, o + c - 1)
        else:
            nfull, rem = divmod(c, 256)
            if nfull:
                note((2, "full 256-row tile"), e, o, o + 255)
            if rem >= 128:
                note((2, "padded 128..255-row remainder tile"), e, o + nfull * 256, o + c - 1)
            elif rem > 0:
                note((2, "leftover double weight tile"), e, o + nfull * 256, o + c - 1)
    return found


KINDS = {(1, "cold weight tile"), (1, "full 256-row tile"), (1, "full 256-row tile, last block"),
         (1, "padded 128..255-row remainder tile"), (1, "leftover weight tile"),
         (2, "cold double weight tile"), (2, "full 256-row tile"),
         (2, "padded 128..255-row remainder tile"), (2, "leftover double weight tile")}


def _selected_rows(off):
    found = tile_rows(off)
    missing = KINDS - set(found)
    assert not missing, f"the workload builds no tile of kind(s) {sorted(missing)}"
    rows = sorted({r for _, r0, r1 in found.values() for r in (r0, r1)})
    return found, np.array(rows)


def test_every_tile_kind_of_the_prefill_schedule(cuda_device):
    d = make("prefill")
    w = d["w"]
    idx, _ = B.lc_moe_route(d["x"], d["wr"], d["bias"], w.K, w.N)
    offsets, row_token, pair_row, x_perm = B.lc_moe_permute(idx, w.N, w.E, x=d["x"])
    h, y = B.lc_moe_expert_ffn(x_perm, offsets, d["w13"], d["w2"], w.T, w.K)
    off = offsets.cpu().numpy()
    found, rows = _selected_rows(off)
    experts = np.repeat(np.arange(w.N), np.diff(off))[rows]
    H, _ = expert_rows_sampled(np_bits(x_perm)[rows], experts, d["w13"], d["w2"])
    assert_within_ulp(np_bits(h)[rows], H, what="H at the rows of every tile kind")
    Y = expert_down_sampled(np_bits(h)[rows], experts, d["w2"])
    assert_within_ulp(np_bits(y)[rows], Y, what="Y at the rows of every tile kind")


def test_every_tile_kind_end_to_end_prefill(cuda_device):
    """Grid activations (exact logits, so the GPU's routing is the oracle's): the layer output of
    one token routed through each tile kind equals the oracle's MoE equation for that token."""
    d = make("prefill", grid=True)
    w = d["w"]
    s = B.Shape(w.T, w.d, w.N, w.Z, w.K, w.I)
    ws = B.new_workspace(s)
    idx = torch.empty(w.T, w.K, dtype=torch.int32, device="cuda")
    gate = torch.empty(w.T, w.K, dtype=torch.float32, device="cuda")
    out = B.lc_moe_forward(d["x"], d["wr"], d["bias"], d["w13"], d["w2"], w.K, idx=idx, gate=gate, ws=ws)
    assert B.lc_moe_read_status(ws) == 0
    offsets, row_token, _, _ = B.lc_moe_permute(idx, w.N, w.E)
    off = offsets.cpu().numpy()
    found, _ = _selected_rows(off)
    rt = row_token.cpu().numpy()
    tokens = np.unique([rt[r1] for _, _, r1 in found.values()])
    ref = oracle_tokens(np_bits(d["x"]), tokens, idx.cpu().numpy(), gate.cpu().numpy(), w.N,
                        d["w13"], d["w2"])
    assert_out_close(np_bits(out)[tokens], ref, what="out of tokens through every tile kind")
