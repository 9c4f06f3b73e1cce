"""CUDA path against the CPU oracle, through the C ABI (needs a B200).

Each step is checked alone (scores; selection on the oracle's own scores;
attention on the oracle's own index sets) and as the fused layer, on seeded
synthetic inputs: small ragged cases spanning several tiles with ragged
tails, the edge cases, and the specified workloads at full size (every query
of the decode workloads; a seeded sample of rows of the 16K prefill).
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


def _up4(x):
    return (int(x) + 3) // 4 * 4


def _args(wl):
    return (wl.q_offsets, wl.kv_offsets, wl.ctx_lens)


def gpu_scores(wl):
    dw = bd.DeviceWorkload(wl)
    ld = _up4(wl.ctx_lens.max())
    scores = torch.full((wl.Nq, ld), float("nan"), device="cuda")
    bd.indexer_score(dw.batch, dw.q_idx, dw.w, dw.k_idx, scores, ld, dw.ws)
    bd.check_device_status(dw.ws)
    return scores.cpu().numpy()


def gpu_topk(wl, scores_np, top_k):
    b = bd.Batch.from_workload(wl)
    ld = scores_np.shape[1]
    scores = torch.from_numpy(np.ascontiguousarray(scores_np, np.float32)).cuda()
    idx = torch.full((wl.Nq, top_k), -7, dtype=torch.int32, device="cuda")
    ws = bd.alloc_workspace(b, 1, top_k)
    bd.topk(b, scores, ld, top_k, idx, ws)
    bd.check_device_status(ws)
    return idx.cpu().numpy()


def gpu_attn(wl, idx_np):
    dw = bd.DeviceWorkload(wl)
    top_k = idx_np.shape[1]
    ws = bd.alloc_workspace(dw.batch, wl.H, top_k)
    idx = torch.from_numpy(np.ascontiguousarray(idx_np, np.int32)).cuda()
    out = torch.full((wl.Nq, wl.H, 512), float("nan"), device="cuda")
    lse = torch.full((wl.Nq, wl.H), float("nan"), device="cuda")
    bd.sparse_attn(dw.batch, dw.q, dw.kv, idx, top_k, wl.scale, out, lse, ws)
    bd.check_device_status(ws)
    return out.cpu().numpy(), lse.cpu().numpy()


def gpu_layer(wl):
    dw = bd.DeviceWorkload(wl)
    out, lse, idx = dw.forward()
    bd.check_device_status(dw.ws)
    return out.cpu().numpy(), lse.cpu().numpy(), idx.cpu().numpy()


# Small shapes: several 128-key tiles, ragged tails, every queries-per-group
# variant (1, 2, 4, 8 per sequence), unaligned cache offsets and spare rows.
SMALL = {
    "prefill_T1024": lambda: synth.prefill(1024, 16, 256, seed=100),
    "ragged_mixed": lambda: synth.custom([300, 129, 1000, 1, 128, 517], [3, 1, 7, 1, 2, 517], 16,
                                         64, seed=101, caps=[301, 140, 1000, 9, 128, 517]),
    "decode_ragged": lambda: synth.custom([5000, 777, 128, 129, 2], [1, 1, 1, 1, 1], 64, 128,
                                          seed=102),
    "two_queries": lambda: synth.custom([700, 900], [2, 2], 8, 100, seed=103),
    "four_queries": lambda: synth.custom([257, 1023], [4, 3], 8, 33, seed=104),
}


@pytest.mark.parametrize("name", sorted(SMALL))
def test_indexer_scores_match_oracle(name):
    wl = SMALL[name]()
    got = gpu_scores(wl)
    ref = oracle.indexer_scores(*_args(wl), wl.q_idx, wl.w, wl.k_idx, ld=got.shape[1])
    worst = parity.check_scores(got, ref, wl)
    # entries past each query's position are left untouched
    pos = wl.positions()
    for r in range(wl.Nq):
        assert np.isnan(got[r, pos[r] + 1:]).all(), r
    print(f"{name}: worst relative score error {worst:.2e}")


@pytest.mark.parametrize("name", sorted(SMALL))
def test_topk_exact_on_oracle_scores(name):
    wl = SMALL[name]()
    ref_scores = oracle.indexer_scores(*_args(wl), wl.q_idx, wl.w, wl.k_idx,
                                       ld=_up4(wl.ctx_lens.max()))
    want = oracle.topk(*_args(wl), ref_scores, wl.top_k)
    got = gpu_topk(wl, np.nan_to_num(ref_scores, nan=0.0), wl.top_k)
    assert np.array_equal(got, want)


def _score_rows(lens, seed, kind):
    """Long synthetic score rows (one query per sequence) with forced ties."""
    lens = np.asarray(lens)
    g = np.random.Generator(np.random.PCG64(seed))
    ld = _up4(lens.max())
    sc = np.zeros((lens.size, ld), np.float32)
    for r, L in enumerate(lens):
        if kind == "normal":
            sc[r, :L] = g.standard_normal(L, dtype=np.float32)
        elif kind == "coarse":            # few distinct values: ties everywhere
            sc[r, :L] = g.integers(-3, 4, size=L).astype(np.float32) * 0.5
        elif kind == "zeros":             # -0 and +0 mixed: one value
            sc[r, :L] = np.where(g.random(L) < 0.5, -0.0, 0.0).astype(np.float32)
        elif kind == "heavy":             # wide dynamic range, negatives
            sc[r, :L] = (g.standard_normal(L) * np.exp(g.standard_normal(L) * 8)).astype(
                np.float32)
        elif kind == "tied_cut":          # the k-th largest inside a group of 300 equal
            v = g.standard_normal(L).astype(np.float32)  # scores spread over the row
            if L > 2048:
                t = np.sort(v)[::-1][1950]
                v[np.arange(0, L, L // 300)[:300]] = t
            sc[r, :L] = v
    return sc


# Row sets that exercise every launch shape of the selection kernel: clusters
# of 8 CTAs (few long rows), 4, 2 and 1 (many short rows), and the
# single-CTA fallback for rows longer than eight shared-memory slices.
ROW_SETS = {
    "decode_4x128k": [131072] * 4,
    "mixed_long": [131072, 40000, 2049, 2048, 100],
    "twenty_50k": [50000] * 20,
    "five_5000": [5000, 4999, 4097, 3000, 2500],
    "many_3000": [3000] * 300,
    "one_400k": [400000],
}


@pytest.mark.parametrize("rows", sorted(ROW_SETS))
@pytest.mark.parametrize("kind", ["normal", "coarse", "zeros", "heavy", "tied_cut"])
def test_topk_long_rows(kind, rows):
    lens = ROW_SETS[rows]
    wl = synth.Workload("rows", np.arange(len(lens) + 1, dtype=np.int32),
                        np.concatenate([[0], np.cumsum(lens)]).astype(np.int64),
                        np.array(lens, np.int32), None, None, None, None, None, 2048, 1.0)
    sc = _score_rows(lens, 7, kind)
    want = oracle.topk(*_args(wl), sc, 2048)
    got = gpu_topk(wl, sc, 2048)
    assert np.array_equal(got, want)


ATTN = {
    "prefill_h16": lambda: synth.prefill(300, 16, 64, seed=110),
    "prefill_h20": lambda: synth.prefill(200, 20, 48, seed=111),
    "decode_h64_split": lambda: synth.custom([3000, 2100, 64], [1, 1, 1], 64, 2048, seed=112),
    "decode_h128": lambda: synth.custom([2500], [1], 128, 1024, seed=113),
    "mixed_h1": lambda: synth.custom([90, 40], [5, 40], 1, 32, seed=114),
    # 12 rows: too many one-tile slices for two waves, so the many-row kernel
    # runs with slices of the selected set and the merge
    "decode_12rows_split": lambda: synth.custom([2200 + 150 * i for i in range(12)], [1] * 12, 64,
                                                2048, seed=116),
    # 48 query rows of 2048 selected each: P without its lo part, split over
    # CTAs and merged
    "long_rows_hi_only": lambda: synth.custom([3000], [48], 64, 2048, seed=117),
    # 80 heads: a full 64-head block and one of 16, whose query rows past H
    # are zero in tensor memory; short rows (P with its lo part), then rows
    # of 1024 selected (P alone)
    "prefill_h80": lambda: synth.prefill(256, 80, 96, seed=118),
    "long_rows_h80_hi_only": lambda: synth.custom([1500], [40], 80, 1024, seed=119),
    # three sequences, 600 query rows through the many-row kernel: its L2
    # prefetch for the row one wave later crosses sequence boundaries
    "ragged_prefill_3seq": lambda: synth.custom([600, 900, 300], [200, 300, 100], 64, 256,
                                                seed=120),
}


@pytest.mark.parametrize("name", sorted(ATTN))
def test_sparse_attention_matches_oracle(name):
    wl = ATTN[name]()
    _, idx, _, _ = oracle.dsa_layer(*_args(wl), wl.q_idx, wl.w, wl.k_idx, wl.q, wl.kv, wl.top_k,
                                    wl.scale)
    ref_out, ref_lse = oracle.sparse_attn(*_args(wl), wl.q, wl.kv, idx, wl.scale)
    out, lse = gpu_attn(wl, idx)
    e = parity.check_attention(out, lse, ref_out, ref_lse)
    print(f"{name}: max |out err| {e[0]:.2e}, max |lse err| {e[1]:.2e}")


def test_sparse_attention_scattered_unused_slots():
    wl = synth.custom([500], [3], 16, 96, seed=115)
    g = np.random.Generator(np.random.PCG64(5))
    idx = np.full((3, 96), -1, np.int32)
    for r, p in enumerate(wl.positions()):
        chosen = np.sort(g.choice(p + 1, size=60, replace=False))
        slots = np.sort(g.choice(96, size=60, replace=False))
        idx[r, slots] = chosen
    idx[2, :] = -1  # a row with nothing selected: out = 0, lse = -inf
    ref_out, ref_lse = oracle.sparse_attn(*_args(wl), wl.q, wl.kv, idx, wl.scale)
    out, lse = gpu_attn(wl, idx)
    assert (out[2] == 0).all() and np.isneginf(lse[2]).all()
    parity.check_attention(out[:2], lse[:2], ref_out[:2], ref_lse[:2])


def _layer_check(wl, rows=None, full_equivalence=False):
    got_out, got_lse, got_idx = gpu_layer(wl)
    sample = None if rows is None else rows
    ld = _up4(wl.ctx_lens.max())
    ref_scores, ref_idx, ref_out, ref_lse = oracle.dsa_layer(
        *_args(wl), wl.q_idx, wl.w, wl.k_idx, wl.q, wl.kv, wl.top_k, wl.scale, sample=sample,
        ld=ld)
    swaps = parity.check_selection(got_idx, ref_idx, ref_scores, wl, rows)
    # attention checked on the GPU's own selection (equal to the oracle's up to ties)
    att_out, att_lse = oracle.sparse_attn(*_args(wl), wl.q, wl.kv, got_idx, wl.scale,
                                          sample=sample)
    e = parity.check_attention(got_out, got_lse, att_out, att_lse, rows)
    if swaps == 0:
        parity.check_attention(got_out, got_lse, ref_out, ref_lse, rows)
    if full_equivalence:
        full_out, full_lse = oracle.full_causal_attn(*_args(wl), wl.q, wl.kv, wl.scale,
                                                     sample=sample)
        parity.check_attention(got_out, got_lse, full_out, full_lse, rows)
    print(f"{wl.name}: boundary swaps {swaps}, max |out err| {e[0]:.2e}, lse {e[1]:.2e}")
    return got_out, got_idx


def test_layer_tiny_prefill_topk_below_context():
    out, _ = _layer_check(synth.tiny_prefill(256))
    # forced below the context, later queries differ from full causal attention
    wl = synth.tiny_prefill(256)
    full, _ = oracle.full_causal_attn(*_args(wl), wl.q, wl.kv, wl.scale,
                                      sample=np.arange(600, 1024))
    assert np.abs(out[600:] - full[600:]).max() > 1e-2


def test_layer_tiny_prefill_topk_covers_context_is_full_attention():
    _layer_check(synth.tiny_prefill(2048), full_equivalence=True)


@pytest.mark.parametrize("name", sorted(SMALL))
def test_layer_small_shapes(name):
    _layer_check(SMALL[name]())


def test_layer_edge_cases():
    # single token contexts, top_k = 1, one head, sequences without queries
    _layer_check(synth.custom([1, 1, 5, 9], [1, 1, 5, 0], 1, 1, seed=120))
    _layer_check(synth.custom([1, 130, 2], [1, 130, 2], 3, 2048, seed=121))


def test_empty_batch_launches_nothing():
    b = bd.Batch(np.zeros(1, np.int32), np.zeros(1, np.int64), np.zeros(0, np.int32))
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    fake = 1 << 16  # never dereferenced: there is nothing to compute
    st = bd.lib.dsa_layer_forward(b.ref, fake, 64, fake, fake, fake, fake, 2048, 0.04, fake,
                                  None, fake, ws.data_ptr(), 256, 0, None)
    assert st == bd.OK
    bd.check_device_status(ws)


def test_layer_decode_b8_32k_full():
    _layer_check(synth.decode_b8_32k())


def test_layer_decode_b4_128k_full():
    _layer_check(synth.decode_b4_128k())


def test_layer_prefill_16k_sampled_rows():
    wl = synth.prefill_16k()
    must = list(range(64)) + list(range(2040, 2057)) + [wl.Nq - 1]
    rows = parity.sample_rows(wl, 160, seed=2, must=must)
    _layer_check(wl, rows=rows)


def _hist_batch():
    """Decode rows long enough for the histogram-driven selection, with special rows:
    0 normal, 1 shorter than top_k, 2 small-integer inputs (exact ties at the
    threshold), 3 all-zero indexer queries (every score ties: the threshold bin
    overflows the candidate buffer), 4 normal and long."""
    wl = synth.custom([9000, 1500, 20000, 12000, 40000], [1] * 5, 16, 2048, seed=140)
    g = np.random.Generator(np.random.PCG64(141))
    k0 = int(wl.kv_offsets[2])
    wl.q_idx[2] = synth.bf16_bits(g.integers(-1, 2, size=(32, 128)).astype(np.float32))
    wl.k_idx[k0:k0 + 20000] = synth.bf16_bits(
        g.integers(-1, 2, size=(20000, 128)).astype(np.float32))
    wl.w[2] = g.integers(-2, 3, size=32).astype(np.float32)
    wl.q_idx[3] = 0
    return wl


def test_layer_histogram_selection_special_rows():
    wl = _hist_batch()
    got_out, got_lse, got_idx = gpu_layer(wl)
    ld = _up4(wl.ctx_lens.max())
    ref_scores, ref_idx, _, _ = oracle.dsa_layer(*_args(wl), wl.q_idx, wl.w, wl.k_idx, wl.q,
                                                 wl.kv, wl.top_k, wl.scale, ld=ld)
    # rows 1-3 have exactly representable scores: the selection must be identical
    for r in (1, 2, 3):
        assert np.array_equal(got_idx[r], ref_idx[r]), r
    assert np.array_equal(got_idx[3], np.arange(2048))  # all ties: lowest positions
    parity.check_selection(got_idx, ref_idx, ref_scores, wl)
    att_out, att_lse = oracle.sparse_attn(*_args(wl), wl.q, wl.kv, got_idx, wl.scale)
    parity.check_attention(got_out, got_lse, att_out, att_lse)


def test_repeated_calls_on_one_workspace_agree():
    """Histograms, counters and other workspace state are left ready for the next call."""
    wl = _hist_batch()
    dw = bd.DeviceWorkload(wl)
    first = [t.cpu().numpy() for t in dw.forward()]
    for _ in range(3):
        again = [t.cpu().numpy() for t in dw.forward()]
        for a, b in zip(first, again):
            assert np.array_equal(a, b)
    bd.check_device_status(dw.ws)
    _, idx, _, _ = oracle.dsa_layer(*_args(wl), wl.q_idx, wl.w, wl.k_idx, wl.q, wl.kv, 2048,
                                    wl.scale)
    ref_out, ref_lse = oracle.sparse_attn(*_args(wl), wl.q, wl.kv, idx, wl.scale)
    parity.check_attention(first[0], first[1], ref_out, ref_lse)


def test_standalone_calls_between_layer_calls_leave_it_unchanged():
    """Standalone calls may use the layer's workspace as scratch in between."""
    wl = _hist_batch()
    dw = bd.DeviceWorkload(wl)
    first = [t.cpu().numpy() for t in dw.forward()]
    ld = _up4(wl.ctx_lens.max())
    scores = torch.zeros(wl.Nq, ld, device="cuda")
    out, lse, idx = dw.new_outputs()
    bd.indexer_score(dw.batch, dw.q_idx, dw.w, dw.k_idx, scores, ld, dw.ws)
    bd.topk(dw.batch, scores, ld, wl.top_k, idx, dw.ws)
    bd.sparse_attn(dw.batch, dw.q, dw.kv, idx, wl.top_k, wl.scale, out, lse, dw.ws)
    again = [t.cpu().numpy() for t in dw.forward()]
    for a, b in zip(first, again):
        assert np.array_equal(a, b)
    assert np.array_equal(idx.cpu().numpy(), first[2])
    bd.check_device_status(dw.ws)


@pytest.mark.parametrize("make", [_hist_batch, lambda: synth.prefill(1024, 16, 256, seed=100),
                                  lambda: synth.custom([5000, 777, 128, 129, 2], [1] * 5, 64, 128,
                                                       seed=102)])
def test_workspace_control_block_is_zero_after_calls(make):
    """Calls leave the workspace's control block (the kernels' error word)
    zero, so the next call and dsa_check_device_status start clean."""
    wl = make()
    dw = bd.DeviceWorkload(wl)
    for _ in range(2):
        dw.forward()
        torch.cuda.synchronize()
        assert not dw.ws[:256].any().item()
    ld = _up4(wl.ctx_lens.max())
    scores = torch.zeros(wl.Nq, ld, device="cuda")
    bd.indexer_score(dw.batch, dw.q_idx, dw.w, dw.k_idx, scores, ld, dw.ws)
    torch.cuda.synchronize()
    assert not dw.ws[:256].any().item()


def test_ragged_stacked_24_layers_every_row():
    """The ragged serving batch (32 contexts log-uniform in [1024, 131072],
    some below top_k) as 24 stacked layers, each with its own caches and
    indexer inputs; layer l+1's main query is chained from layer l's output
    through the fixed projection.  Every row of every layer is checked against
    the oracle, teacher-forced: the oracle runs each layer on the same query
    the GPU chain produced.  The oracle's own chain (its outputs feeding its
    next layer) runs beside it, and the drift between the two chains' final
    outputs is reported."""
    proj = synth.glue_projection(4)
    q_gpu = q_ora = None
    swaps_total, worst = 0, 0.0
    for layer in range(24):
        wl = synth.ragged_layer(layer)
        if layer == 0:
            assert wl.ctx_lens.min() < wl.top_k  # the top_k >= context path is exercised
        else:
            wl.q = q_gpu
        got_out, got_lse, got_idx = gpu_layer(wl)
        ld = _up4(wl.ctx_lens.max())
        ref_scores, ref_idx, ref_out, ref_lse = oracle.dsa_layer(
            *_args(wl), wl.q_idx, wl.w, wl.k_idx, wl.q, wl.kv, wl.top_k, wl.scale, ld=ld)
        swaps = parity.check_selection(got_idx, ref_idx, ref_scores, wl)
        att_out, att_lse = oracle.sparse_attn(*_args(wl), wl.q, wl.kv, got_idx, wl.scale)
        e = parity.check_attention(got_out, got_lse, att_out, att_lse)
        if swaps == 0:
            parity.check_attention(got_out, got_lse, ref_out, ref_lse)
        swaps_total += swaps
        worst = max(worst, e[0])
        if layer == 0:
            ora_out = ref_out
        else:  # the oracle's own chain
            _, _, ora_out, _ = oracle.dsa_layer(*_args(wl), wl.q_idx, wl.w, wl.k_idx, q_ora,
                                                wl.kv, wl.top_k, wl.scale, ld=ld)
        q_gpu = synth.chain_query(got_out, proj)
        q_ora = synth.chain_query(ora_out, proj)
        assert q_gpu.shape == wl.q.shape
    drift = float(np.abs(got_out.astype(np.float64) - ora_out).max())
    rms = float(np.sqrt(np.mean(ora_out.astype(np.float64) ** 2)))
    assert np.isfinite(drift)
    print(f"ragged 24 layers: boundary swaps {swaps_total}, worst per-layer |out err| "
          f"{worst:.2e}; end-to-end drift after 24 layers: max |gpu - oracle chain| "
          f"{drift:.2e} (output rms {rms:.2e})")


def _concentrated_batch():
    """Decode rows whose selected positions are not spread evenly: in row 0 the
    top scores sit in one contiguous range of 3000 positions (so a few chunks
    of the row hold hundreds of selected positions each, several 96-row tiles),
    row 1 mixes that range with the rest, rows 2-5 are plain.  Six rows: the
    fused tail, which attends over balanced shares of such rows."""
    wl = synth.custom([20000, 30000, 9000, 50000, 12000, 25000], [1] * 6, 64, 2048, seed=170)
    g = np.random.Generator(np.random.PCG64(171))
    v = g.standard_normal(128).astype(np.float32)
    v /= np.linalg.norm(v)
    for r, (lo, hi, amp) in enumerate([(5000, 8000, 6.0), (100, 1200, 2.0)]):
        k0 = int(wl.kv_offsets[r])
        qi = synth.bf16_to_f32(wl.q_idx[r]).copy()
        qi[:] = 4.0 * v + 0.25 * qi
        wl.q_idx[r] = synth.bf16_bits(qi)
        wl.w[r] = np.abs(wl.w[r])
        kk = synth.bf16_to_f32(wl.k_idx[k0 + lo:k0 + hi]).copy()
        kk += amp * v
        wl.k_idx[k0 + lo:k0 + hi] = synth.bf16_bits(kk)
    return wl


def test_layer_decode_concentrated_selection():
    wl = _concentrated_batch()
    got_out, got_idx = _layer_check(wl)
    # row 0 really concentrates: most of its selection lies in the planted range
    sel = got_idx[0]
    assert ((sel >= 5000) & (sel < 8000)).sum() >= 1500


def test_layer_decode_12_rows():
    """12 decode rows: 12 chunks per row in the fused tail, so each CTA merges
    683 output units, more than it has threads (two passes)."""
    _layer_check(synth.custom([20000, 20000, 9000, 9000, 9000, 9000] + [30000] * 6, [1] * 12, 64,
                              2048, seed=165))


def test_layer_decode_14_rows():
    """14 decode rows: the separate selection, attention and merge kernels."""
    _layer_check(synth.custom([20000, 20000, 9000, 9000, 9000, 9000] + [30000] * 8, [1] * 14, 64,
                              2048, seed=165))
