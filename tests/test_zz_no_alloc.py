"""dsa_sparse_attn_noalloc against dsa_sparse_attn (needs a B200).

The no-allocation entry point is for callers that cannot call cudaMalloc when
they run the layer (a fixed memory pool, a runtime that only hands kernels
its own tensors).  It keeps its scratch in a static device array instead of
a caller workspace.  Its results must agree with the workspace entry point on
the same inputs, on two calls in a row (the array keeps the previous call's
contents, which must not leak into the next result).

This file is named to be collected last, so a run that stops at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from dsa_lightning_indexer_b200 import synth
from tests import parity

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from dsa_lightning_indexer_b200 import binding as bd


def _args(wl):
    return (wl.q_offsets, wl.kv_offsets, wl.ctx_lens)


CASES = {
    # few rows: the selected set is split over CTAs, partials in the static array
    "decode_split": lambda: synth.custom([3000, 2500, 700], [1, 1, 1], 64, 2048, seed=150),
    # many rows, 16 heads: one CTA per (row, head block), no partials
    "prefill_rows": lambda: synth.prefill(300, 16, 64, seed=151),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_noalloc_matches_workspace_entry_point(name):
    wl = CASES[name]()
    _, idx_np, _, _ = oracle.dsa_layer(*_args(wl), wl.q_idx, wl.w, wl.k_idx, wl.q, wl.kv,
                                       wl.top_k, wl.scale)
    dw = bd.DeviceWorkload(wl)
    idx = torch.from_numpy(idx_np).cuda()
    ref_out = torch.empty(wl.Nq, wl.H, 512, device="cuda")
    ref_lse = torch.empty(wl.Nq, wl.H, device="cuda")
    bd.sparse_attn(dw.batch, dw.q, dw.kv, idx, wl.top_k, wl.scale, ref_out, ref_lse, dw.ws)
    ref_out, ref_lse = ref_out.cpu().numpy(), ref_lse.cpu().numpy()
    runs = []
    for _ in range(2):
        out = torch.full((wl.Nq, wl.H, 512), float("nan"), device="cuda")
        lse = torch.full((wl.Nq, wl.H), float("nan"), device="cuda")
        bd.sparse_attn_noalloc(dw.batch, dw.q, dw.kv, idx, wl.top_k, wl.scale, out, lse)
        torch.cuda.synchronize()
        runs.append((out.cpu().numpy(), lse.cpu().numpy()))
    for out, lse in runs:
        parity.check_attention(out, lse, ref_out, ref_lse.astype(np.float64))
    assert np.array_equal(runs[0][0], runs[1][0]) and np.array_equal(runs[0][1], runs[1][1])
