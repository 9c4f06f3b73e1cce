"""Paged (block-table) caches (needs a B200).

The same workloads with their caches cut into pages placed in a random
order among unused pages: every call must give exactly what it gives on the
contiguous caches (the kernels read the same values in the same order, only
the rows' addresses differ), and so match the oracle on the contiguous data.
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


CASES = {
    # decode, fused tail (six rows): ragged lengths, pages of 64 rows
    "decode_fused_p64": (lambda: synth.custom([20000, 9000, 3000, 50000, 15000, 8000], [1] * 6,
                                              64, 2048, seed=200), 64),
    # decode, separate selection and attention kernels (four rows), pages of 64
    "decode_chain_p64": (lambda: synth.custom([20000, 9000, 3000, 50000], [1] * 4, 64, 2048,
                                              seed=204), 64),
    # multi-token decode (items of 2 and 4 queries), pages of 256 rows
    "multi_token_p256": (lambda: synth.custom([12000, 30000], [2, 4], 64, 2048, seed=201), 256),
    # prefill-like rows: many-row attention, one-CTA-per-row selection, pages of 128
    "prefill_p128": (lambda: synth.custom([700, 300], [700, 120], 16, 256, seed=202,
                                          caps=[760, 300]), 128),
    # the few-row attention kernel with slices and the merge (no histogram path)
    "decode_short_p64": (lambda: synth.custom([5000, 777, 129], [1, 1, 1], 64, 128, seed=203),
                         64),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_paged_layer_equals_contiguous(name):
    make, ps = CASES[name]
    wl = make()
    pw = synth.paged(wl, ps, seed=210)
    got = [t.cpu().numpy() for t in bd.DeviceWorkload(pw).forward()]
    dw = bd.DeviceWorkload(wl)
    want = [t.cpu().numpy() for t in dw.forward()]
    bd.check_device_status(dw.ws)
    for a, b in zip(got, want):
        assert np.array_equal(a, b)
    ld = _up4(wl.ctx_lens.max())
    ref_scores, ref_idx, _, _ = oracle.dsa_layer(*_args(wl), wl.q_idx, wl.w, wl.k_idx, wl.q,
                                                 wl.kv, wl.top_k, wl.scale, ld=ld)
    parity.check_selection(got[2], ref_idx, ref_scores, wl)
    att_out, att_lse = oracle.sparse_attn(*_args(wl), wl.q, wl.kv, got[2], wl.scale)
    parity.check_attention(got[0], got[1], att_out, att_lse)


def test_paged_standalone_calls():
    wl = synth.custom([20000, 40000, 900], [1, 1, 1], 64, 2048, seed=204)
    pw = synth.paged(wl, 128, seed=211)
    pd, cd = bd.DeviceWorkload(pw), bd.DeviceWorkload(wl)
    ld = _up4(wl.ctx_lens.max())
    res = []
    for d in (pd, cd):
        scores = torch.full((wl.Nq, ld), float("nan"), device="cuda")
        bd.indexer_score(d.batch, d.q_idx, d.w, d.k_idx, scores, ld, d.ws,
                         flags=bd.FLAG_SCORE_HISTOGRAM)
        out, lse, idx = d.new_outputs()
        bd.topk(d.batch, scores, ld, wl.top_k, idx, d.ws, flags=bd.FLAG_SCORE_HISTOGRAM)
        bd.sparse_attn(d.batch, d.q, d.kv, idx, wl.top_k, wl.scale, out, lse, d.ws)
        o2, l2 = torch.empty_like(out), torch.empty_like(lse)
        bd.sparse_attn_noalloc(d.batch, d.q, d.kv, idx, wl.top_k, wl.scale, o2, l2)
        bd.check_device_status(d.ws)
        res.append([t.cpu().numpy() for t in (scores, idx, out, lse, o2, l2)])
    for a, b in zip(*res):
        assert np.array_equal(np.nan_to_num(a, nan=7.0), np.nan_to_num(b, nan=7.0))
    # the mask-over-the-whole-cache route needs contiguous caches
    ws = bd.alloc_workspace(pd.batch, wl.H, wl.top_k, flags=bd.FLAG_MASKED_ROUTE)
    out, lse, idx = pd.new_outputs()
    with pytest.raises(bd.DsaError) as e:
        bd.masked_attn(pd.batch, pd.q, pd.kv, torch.from_numpy(res[0][1]).cuda(), wl.top_k,
                       wl.scale, out, lse, ws)
    assert e.value.status == bd.ERR_UNSUPPORTED


def test_paged_input_step_appends_into_the_page():
    lens, nq = [300, 900], [2, 3]
    wl = synth.custom(lens, nq, 16, 64, seed=205, caps=[320, 900])
    pw = synth.paged(wl, 64, seed=212)
    g = np.random.Generator(np.random.PCG64(206))
    T, d_model, d_q = wl.Nq, 256, 128

    def bf(shape, std):
        return synth.bf16_bits((g.standard_normal(shape) * std).astype(np.float32))
    x, c_q = bf((T, d_model), 1.0), bf((T, d_q), 1.0)
    w_q_b, w_k, w_proj = bf((4096, d_q), 0.1), bf((128, d_model), 0.06), bf((32, d_model), 0.06)
    want_q, want_k, want_w = oracle.indexer_project(*_args(wl), x, c_q, w_q_b, w_k, w_proj,
                                                    wl.k_idx)
    b = bd.Batch.from_workload(pw)
    dev = {k: bd.bf16_tensor(v) for k, v in dict(x=x, c_q=c_q, w_q_b=w_q_b, w_k=w_k,
                                                 w_proj=w_proj, k=pw.paged.k_idx).items()}
    q_idx = torch.empty(T, 32, 128, dtype=torch.bfloat16, device="cuda")
    w = torch.empty(T, 32, device="cuda")
    ws = bd.indexer_project_workspace(b, d_model, d_q)
    bd.indexer_project(b, dev["x"], dev["c_q"], dev["w_q_b"], dev["w_k"], dev["w_proj"], q_idx,
                       dev["k"], w, ws)
    bd.check_device_status(ws)
    got_k = dev["k"].view(torch.int16).cpu().numpy().view(np.uint16)
    ps, bt = pw.paged.page_size, pw.paged.block_table
    # every position's row, through the block table, holds the oracle's cache row
    changed = 0
    for bi in range(wl.B):
        for s in range(int(wl.ctx_lens[bi])):
            row = int(bt[bi, s // ps]) * ps + s % ps
            want = want_k[int(wl.kv_offsets[bi]) + s]
            d = np.abs(got_k[row].astype(np.int32) - want.astype(np.int32))
            assert d.max() <= 1, (bi, s)
            changed += int(not np.array_equal(got_k[row], pw.paged.k_idx[row]))
    assert changed >= 1
    assert np.abs(w.cpu().numpy() - want_w).max() <= 1e-3
