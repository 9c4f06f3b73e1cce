"""Kernel-side failure reporting and the device-side index check (needs a B200).

* A wait that runs out: with the test-only DSA_FLAG_TEST_STALL the indexer's
  TMA producer issues no load at all (so no copy is in flight when the CTAs
  give up), every wait of the indexer runs out after its time limit (about a
  second), the call returns, and dsa_check_device_status reports
  DSA_ERR_DEVICE_TIMEOUT and clears the word; the next call is correct.
* Index entries outside -1..p are skipped and reported as DSA_ERR_BAD_INDEX.
  The bad entries used here still fall inside the allocated cache rows (the
  batches have spare capacity past each context, and negative entries are
  only used where rows of an earlier sequence precede them), so even a
  missed check could only read valid memory.
* The standalone calls with DSA_FLAG_SCORE_HISTOGRAM run the fused layer's
  histogram-driven selection and give exactly the layer's index sets.
"""
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


def _up4(x):
    return (int(x) + 3) // 4 * 4


def test_stalled_indexer_reports_timeout_then_recovers():
    wl = synth.custom([9000, 3000, 700], [1, 1, 1], 16, 256, seed=160)
    dw = bd.DeviceWorkload(wl)
    out, lse, idx = dw.new_outputs()
    idx.fill_(-1)
    dw.forward(out, lse, idx, flags=bd.FLAG_TEST_STALL)
    with pytest.raises(bd.DsaError) as e:
        bd.check_device_status(dw.ws)
    assert e.value.status == bd.ERR_DEVICE_TIMEOUT
    assert not dw.ws[:256].any().item()        # read and cleared
    bd.check_device_status(dw.ws)              # nothing left to report
    # the next call on the same workspace is correct
    got_out, got_lse, got_idx = (t.cpu().numpy() for t in dw.forward())
    bd.check_device_status(dw.ws)
    ld = _up4(wl.ctx_lens.max())
    ref_scores, ref_idx, _, _ = oracle.dsa_layer(*_args(wl), wl.q_idx, wl.w, wl.k_idx, wl.q,
                                                 wl.kv, wl.top_k, wl.scale, ld=ld)
    parity.check_selection(got_idx, ref_idx, ref_scores, wl)
    att_out, att_lse = oracle.sparse_attn(*_args(wl), wl.q, wl.kv, got_idx, wl.scale)
    parity.check_attention(got_out, got_lse, att_out, att_lse)


def _corrupted(wl, bad):
    """The oracle's index sets with the entries `bad` {(row, slot): value}
    written in, and the same sets with those entries as -1 (what the kernels
    must compute)."""
    _, idx, _, _ = oracle.dsa_layer(*_args(wl), wl.q_idx, wl.w, wl.k_idx, wl.q, wl.kv, wl.top_k,
                                    wl.scale)
    given, expect = idx.copy(), idx.copy()
    pos = wl.positions()
    for (r, slot), v in bad.items():
        b = int(np.searchsorted(wl.q_offsets, r, side="right") - 1)
        row = int(wl.kv_offsets[b]) + v
        assert v < -1 or v > pos[r]                       # outside -1..p
        assert 0 <= row < int(wl.kv_offsets[-1])         # but inside the cache allocation
        given[r, slot] = v
        expect[r, slot] = -1
    return given, expect


# (workload, bad entries): few rows take the single-tile decode kernel, many
# rows the many-row kernel.
BAD = {
    "decode_kernel": (lambda: synth.custom([700, 900, 400], [1, 2, 1], 16, 64, seed=161,
                                           caps=[760, 950, 420]),
                      {(0, 3): 705, (1, 10): -4, (3, 0): 410}),
    "many_row_kernel": (lambda: synth.custom([300, 50], [300, 50], 16, 64, seed=162,
                                             caps=[340, 60]),
                        {(299, 5): 310, (300, 1): -3, (349, 63): 55, (120, 0): 121}),
}


@pytest.mark.parametrize("name", sorted(BAD))
def test_out_of_range_indices_are_skipped_and_reported(name):
    make, bad = BAD[name]
    wl = make()
    given, expect = _corrupted(wl, bad)
    ref_out, ref_lse = oracle.sparse_attn(*_args(wl), wl.q, wl.kv, expect, wl.scale)
    dw = bd.DeviceWorkload(wl)
    idx = torch.from_numpy(given).cuda()
    out = torch.full((wl.Nq, wl.H, 512), float("nan"), device="cuda")
    lse = torch.full((wl.Nq, wl.H), float("nan"), device="cuda")
    bd.sparse_attn(dw.batch, dw.q, dw.kv, idx, wl.top_k, wl.scale, out, lse, dw.ws)
    with pytest.raises(bd.DsaError) as e:
        bd.check_device_status(dw.ws)
    assert e.value.status == bd.ERR_BAD_INDEX
    parity.check_attention(out.cpu().numpy(), lse.cpu().numpy(), ref_out, ref_lse)
    # valid sets raise nothing
    bd.sparse_attn(dw.batch, dw.q, dw.kv, torch.from_numpy(expect).cuda(), wl.top_k, wl.scale,
                   out, lse, dw.ws)
    bd.check_device_status(dw.ws)
    # the workspace-free entry point skips them too (it has no error word)
    out2 = torch.full_like(out, float("nan"))
    lse2 = torch.full_like(lse, float("nan"))
    bd.sparse_attn_noalloc(dw.batch, dw.q, dw.kv, idx, wl.top_k, wl.scale, out2, lse2)
    torch.cuda.synchronize()
    parity.check_attention(out2.cpu().numpy(), lse2.cpu().numpy(), ref_out, ref_lse)


def _hist_decode():
    # six single-token rows: the layer takes the fused tail
    return synth.custom([9000, 1500, 20000, 40000, 7000, 12000], [1] * 6, 16, 2048, seed=163)


def test_standalone_histogram_path_matches_the_layer():
    wl = _hist_decode()
    dw = bd.DeviceWorkload(wl)
    lay_out, lay_lse, lay_idx = (t.cpu().numpy() for t in dw.forward())
    ld = _up4(wl.ctx_lens.max())
    scores = torch.full((wl.Nq, ld), float("nan"), device="cuda")
    bd.indexer_score(dw.batch, dw.q_idx, dw.w, dw.k_idx, scores, ld, dw.ws,
                     flags=bd.FLAG_SCORE_HISTOGRAM)
    sets = []
    for _ in range(2):  # the same histograms serve repeated selections
        idx = torch.full((wl.Nq, wl.top_k), -7, dtype=torch.int32, device="cuda")
        bd.topk(dw.batch, scores, ld, wl.top_k, idx, dw.ws, flags=bd.FLAG_SCORE_HISTOGRAM)
        sets.append(idx.cpu().numpy())
    bd.check_device_status(dw.ws)
    for s in sets:
        assert np.array_equal(s, lay_idx)
    # and the selection is the oracle's on the kernel's own scores
    want = oracle.topk(*_args(wl), np.nan_to_num(scores.cpu().numpy(), nan=0.0), wl.top_k)
    assert np.array_equal(sets[0], want)


def test_multi_token_decode_takes_the_histogram_path():
    """Several new tokens per sequence (items of 2, 4 and 8 queries): the
    indexer builds every row's histogram, the fused layer and the standalone
    histogram path give the same index sets, and they are the oracle's."""
    wl = synth.custom([20000, 9000, 30000], [2, 4, 8], 64, 2048, seed=164)
    dw = bd.DeviceWorkload(wl)
    lay_out, lay_lse, lay_idx = (t.cpu().numpy() for t in dw.forward())
    bd.check_device_status(dw.ws)
    ld = _up4(wl.ctx_lens.max())
    scores = torch.full((wl.Nq, ld), float("nan"), device="cuda")
    bd.indexer_score(dw.batch, dw.q_idx, dw.w, dw.k_idx, scores, ld, dw.ws,
                     flags=bd.FLAG_SCORE_HISTOGRAM)
    idx = torch.full((wl.Nq, wl.top_k), -7, dtype=torch.int32, device="cuda")
    bd.topk(dw.batch, scores, ld, wl.top_k, idx, dw.ws, flags=bd.FLAG_SCORE_HISTOGRAM)
    bd.check_device_status(dw.ws)
    assert np.array_equal(idx.cpu().numpy(), lay_idx)
    ref_scores, ref_idx, _, _ = oracle.dsa_layer(*_args(wl), wl.q_idx, wl.w, wl.k_idx, wl.q,
                                                 wl.kv, wl.top_k, wl.scale, ld=ld)
    parity.check_selection(lay_idx, ref_idx, ref_scores, wl)
    att_out, att_lse = oracle.sparse_attn(*_args(wl), wl.q, wl.kv, lay_idx, wl.scale)
    parity.check_attention(lay_out, lay_lse, att_out, att_lse)
