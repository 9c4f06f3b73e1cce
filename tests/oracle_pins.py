"""Pins of the CPU oracle to facts fixed outside the oracle itself.

Each pin is a plain function that raises AssertionError when the oracle breaks
the fact it checks.  They are collected by ``test_oracle.py`` and, with a
planted mistake switched on inside the oracle, by its mutation test (every
planted mistake must trip at least one pin).

Sources of truth used here, none of which is the oracle's own code:
  * hand-worked examples under ``tests/golden/`` (the pages print none);
  * closed forms (one-hot weights give a squared norm; one selected row gives
    that row's V exactly; all-zero scores select the first positions);
  * library routines on CPU in float64 (torch.einsum, torch SDPA);
  * brute-force enumeration of subsets on tiny inputs;
  * invariants (positive rescaling of w, permutation of cache rows);
  * the pages' statement that with top_k larger than the context the layer
    equals full attention, and differs once top_k is forced below it
    (aiaulis.com paragraph 7; aiunderstanding.org "What happened";
    devotd.net section 4).
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np
import torch

import oracle
from dsa_lightning_indexer_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _one_seq(L, nq):
    return (np.array([0, nq], np.int32), np.array([0, L], np.int64), np.array([L], np.int32))


def _bf16(x):
    return synth.bf16_bits(np.asarray(x, dtype=np.float32))


def _f(b):
    return synth.bf16_to_f32(b).astype(np.float64)


def _ulp_close(a, b, ulps=1):
    a = np.asarray(a, np.float32)
    b = np.asarray(b, np.float32)
    sp = np.spacing(np.maximum(np.abs(a), np.abs(b)).astype(np.float32))
    return bool(np.all(np.abs(a.astype(np.float64) - b.astype(np.float64)) <= ulps * sp))


# ---------------------------------------------------------------- scores ----

def pin_score_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "indexer_worked_example.json")))
    qo, ko, cl = _one_seq(3, 1)
    q_idx = _bf16(np.array(g["q_idx"], np.float32)[None])
    w = np.array([g["w"]], np.float32)
    k_idx = _bf16(g["k_idx"])
    sc = oracle.indexer_scores(qo, ko, cl, q_idx, w, k_idx)
    assert np.array_equal(sc[0], np.array(g["scores"], np.float32)), sc
    for k, key in ((1, "idx_top1"), (2, "idx_top2"), (5, "idx_top5")):
        idx = oracle.topk(qo, ko, cl, sc, k)
        assert idx[0].tolist() == g[key], (k, idx)


def pin_score_onehot_is_squared_norm():
    """w one-hot on head h and q_idx[h] = k_idx[s*] give score(s*) = |k_s*|^2."""
    L = 40
    k_idx = synth.normal_bf16(11, 0, 0, (L, synth.DI))
    q_idx = synth.normal_bf16(11, 0, 1, (1, synth.HI, synth.DI))
    s_star, h = 17, 5
    q_idx[0, h] = k_idx[s_star]
    w = np.zeros((1, synth.HI), np.float32)
    w[0, h] = 1.0
    qo, ko, cl = _one_seq(L, 1)
    sc = oracle.indexer_scores(qo, ko, cl, q_idx, w, k_idx)
    kf = _f(k_idx[s_star])
    assert sc[0, s_star] == np.float32(np.dot(kf, kf)), (sc[0, s_star], np.dot(kf, kf))
    # every other position: ReLU of a dot product, times 1
    dots = _f(k_idx) @ _f(q_idx[0, h])
    assert _ulp_close(sc[0, :L], np.maximum(dots, 0.0).astype(np.float32))


def pin_scores_match_torch_einsum():
    """Scores equal a float64 torch.einsum restatement to within one fp32 rounding."""
    wl = synth.custom([50, 33], [7, 33], 4, 16, seed=12)
    sc = oracle.indexer_scores(wl.q_offsets, wl.kv_offsets, wl.ctx_lens, wl.q_idx, wl.w,
                               wl.k_idx)
    pos = wl.positions()
    qi = torch.from_numpy(_f(wl.q_idx))
    ki = torch.from_numpy(_f(wl.k_idx))
    w = torch.from_numpy(wl.w.astype(np.float64))
    for b in range(wl.B):
        r0, r1 = int(wl.q_offsets[b]), int(wl.q_offsets[b + 1])
        k0 = int(wl.kv_offsets[b])
        kb = ki[k0:k0 + int(wl.ctx_lens[b])]
        dots = torch.einsum("qhj,sj->qhs", qi[r0:r1], kb)
        ref = torch.einsum("qh,qhs->qs", w[r0:r1], torch.relu(dots)).numpy()
        for r in range(r0, r1):
            p = int(pos[r])
            assert _ulp_close(sc[r, :p + 1], ref[r - r0, :p + 1].astype(np.float32)), r
            assert np.isnan(sc[r, p + 1:]).all(), "scores past the query position must stay unset"


# ------------------------------------------------------------- selection ----

def _brute_force_select(scores, n_pos, n_sel):
    """The unique subset of size n_sel whose every member beats every non-member."""
    key = [(float(scores[s]), -s) for s in range(n_pos)]
    found = []
    for sub in itertools.combinations(range(n_pos), n_sel):
        inside = set(sub)
        worst_in = min(key[s] for s in inside) if inside else None
        best_out = max((key[s] for s in range(n_pos) if s not in inside), default=None)
        if worst_in is None or best_out is None or worst_in > best_out:
            found.append(list(sub))
    assert len(found) == 1, found
    return found[0]


def pin_select_brute_force_with_ties():
    """Tiny rows with many tied scores: the oracle's set equals the enumerated one."""
    g = np.random.Generator(np.random.PCG64(21))
    for trial in range(6):
        L = int(g.integers(1, 11))
        nq = int(g.integers(1, L + 1))
        top_k = int(g.integers(1, 9))
        q_idx = _bf16(g.integers(-1, 2, size=(nq, 2, 3)).astype(np.float32))
        k_idx = _bf16(g.integers(-1, 2, size=(L, 3)).astype(np.float32))
        w = g.integers(-2, 3, size=(nq, 2)).astype(np.float32)
        qo, ko, cl = _one_seq(L, nq)
        sc = oracle.indexer_scores(qo, ko, cl, q_idx, w, k_idx)
        idx = oracle.topk(qo, ko, cl, sc, top_k)
        for r in range(nq):
            p = L - nq + r
            n_sel = min(top_k, p + 1)
            want = _brute_force_select(sc[r], p + 1, n_sel)
            assert idx[r].tolist() == want + [-1] * (top_k - n_sel), (trial, r, idx[r], want)


def pin_select_properties_random():
    wl = synth.custom([300, 90, 7], [20, 90, 7], 4, 64, seed=22)
    sc = oracle.indexer_scores(wl.q_offsets, wl.kv_offsets, wl.ctx_lens, wl.q_idx, wl.w,
                               wl.k_idx)
    idx = oracle.topk(wl.q_offsets, wl.kv_offsets, wl.ctx_lens, sc, wl.top_k)
    for r, p in enumerate(wl.positions()):
        n_sel = min(wl.top_k, int(p) + 1)
        sel = idx[r, :n_sel]
        assert (idx[r, n_sel:] == -1).all()
        assert (np.diff(sel) > 0).all() and sel[0] >= 0 and sel[-1] <= p
        rest = np.setdiff1d(np.arange(p + 1), sel)
        if rest.size:
            worst_in = min((sc[r, s], -s) for s in sel)
            best_out = max((sc[r, s], -s) for s in rest)
            assert worst_in > best_out


def pin_select_all_zero_scores_take_first_positions():
    """q_idx = 0 makes every score 0; the tie rule then keeps positions 0..n_sel-1."""
    L, nq, top_k = 200, 5, 64
    qo, ko, cl = _one_seq(L, nq)
    q_idx = np.zeros((nq, synth.HI, synth.DI), np.uint16)
    w = synth.rng(23, 0, 1).standard_normal((nq, synth.HI)).astype(np.float32)
    k_idx = synth.normal_bf16(23, 0, 2, (L, synth.DI))
    sc = oracle.indexer_scores(qo, ko, cl, q_idx, w, k_idx)
    assert (sc[:, :L - nq + 1] == 0).all()
    idx = oracle.topk(qo, ko, cl, sc, top_k)
    assert (idx == np.arange(top_k, dtype=np.int32)[None]).all()
    # the same with negative weights only: ReLU(0) * w is zero of either sign
    sc2 = oracle.indexer_scores(qo, ko, cl, q_idx, -np.abs(w), k_idx)
    assert (np.signbit(sc2[:, :L - nq + 1]) == False).all()  # noqa: E712


def pin_select_invariant_under_positive_weight_scaling():
    wl = synth.custom([257], [9], 4, 40, seed=24)
    args = (wl.q_offsets, wl.kv_offsets, wl.ctx_lens)
    idx1 = oracle.topk(*args, oracle.indexer_scores(*args, wl.q_idx, wl.w, wl.k_idx), 40)
    idx2 = oracle.topk(*args, oracle.indexer_scores(*args, wl.q_idx, wl.w * np.float32(8.0),
                                                    wl.k_idx), 40)
    assert np.array_equal(idx1, idx2)


def pin_select_follows_cache_permutation():
    """Decode: permuting the cache rows permutes the selected positions."""
    L, top_k = 500, 37
    wl = synth.decode(1, L, 4, top_k, seed=25)
    args = (wl.q_offsets, wl.kv_offsets, wl.ctx_lens)
    sc = oracle.indexer_scores(*args, wl.q_idx, wl.w, wl.k_idx)
    assert np.unique(sc[0]).size == L
    idx = oracle.topk(*args, sc, top_k)
    perm = synth.rng(25, 0, 9).permutation(L)          # new row i holds old row perm[i]
    sc_p = oracle.indexer_scores(*args, wl.q_idx, wl.w, wl.k_idx[perm])
    idx_p = oracle.topk(*args, sc_p, top_k)
    assert np.array_equal(np.sort(perm[idx_p[0]]), idx[0])


# ------------------------------------------------------------- attention ----

def pin_attention_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "attention_worked_example.json")))
    qo, ko, cl = _one_seq(3, 1)
    q = _bf16(np.array(g["q"], np.float32)[None, None])
    kv = _bf16(g["kv"])
    out, lse = oracle.sparse_attn(qo, ko, cl, q, kv, np.array([[0, 1, 2, -1]], np.int32),
                                  g["scale"], Dv=g["Dv"])
    e = math.e
    assert abs(out[0, 0, 0] - 3 * e / (1 + 2 * e)) < 1e-7
    assert out[0, 0, 1] == 2.0
    assert abs(lse[0, 0] - math.log(1 + 2 * e)) < 1e-6


def _sdpa(q, kv, scale, mask):
    """float64 torch SDPA of queries [n, H, D] over rows kv [L, D] with a bool mask [n, L]."""
    qt = torch.from_numpy(_f(q)).permute(1, 0, 2)               # [H, n, D]
    kt = torch.from_numpy(_f(kv))[None].expand(qt.shape[0], -1, -1)
    vt = kt[..., :synth.DV]
    m = torch.from_numpy(mask)[None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=scale)
    logits = (qt @ kt.transpose(1, 2)) * scale
    lse = torch.logsumexp(logits.masked_fill(~m, -math.inf), dim=-1)
    return o.permute(1, 0, 2).numpy(), lse.permute(1, 0).numpy()


def pin_full_causal_matches_torch_sdpa():
    wl = synth.custom([70, 45], [70, 3], 3, 8, seed=31)
    out, lse = oracle.full_causal_attn(wl.q_offsets, wl.kv_offsets, wl.ctx_lens, wl.q, wl.kv,
                                       wl.scale)
    pos = wl.positions()
    for b in range(wl.B):
        r0, r1 = int(wl.q_offsets[b]), int(wl.q_offsets[b + 1])
        k0, L = int(wl.kv_offsets[b]), int(wl.ctx_lens[b])
        mask = np.arange(L)[None, :] <= pos[r0:r1, None]
        ro, rl = _sdpa(wl.q[r0:r1], wl.kv[k0:k0 + L], wl.scale, mask)
        assert np.abs(out[r0:r1] - ro).max() < 1e-6
        assert np.abs(lse[r0:r1] - rl).max() < 1e-5


def pin_sparse_matches_torch_sdpa_with_index_mask():
    wl = synth.custom([160], [12], 4, 24, seed=32)
    args = (wl.q_offsets, wl.kv_offsets, wl.ctx_lens)
    _, idx, out, lse = oracle.dsa_layer(*args, wl.q_idx, wl.w, wl.k_idx, wl.q, wl.kv, wl.top_k,
                                        wl.scale)
    mask = np.zeros((wl.Nq, 160), bool)
    for r in range(wl.Nq):
        mask[r, idx[r][idx[r] >= 0]] = True
    ro, rl = _sdpa(wl.q, wl.kv, wl.scale, mask)
    assert np.abs(out - ro).max() < 1e-6
    assert np.abs(lse - rl).max() < 1e-5


def pin_topk_at_least_context_is_full_attention():
    """top_k >= p+1 for every query: the layer equals full causal attention (SDPA)."""
    T, H = 96, 4
    wl = synth.prefill(T, H, 128, seed=33)
    args = (wl.q_offsets, wl.kv_offsets, wl.ctx_lens)
    _, idx, out, lse = oracle.dsa_layer(*args, wl.q_idx, wl.w, wl.k_idx, wl.q, wl.kv, 128,
                                        wl.scale)
    for r in range(T):
        assert idx[r, :r + 1].tolist() == list(range(r + 1))
    mask = np.arange(T)[None, :] <= np.arange(T)[:, None]
    ro, rl = _sdpa(wl.q, wl.kv, wl.scale, mask)
    assert np.abs(out - ro).max() < 1e-6
    assert np.abs(lse - rl).max() < 1e-5
    # at exactly top_k = p+1 for the last query as well
    _, idx2, out2, _ = oracle.dsa_layer(*args, wl.q_idx, wl.w, wl.k_idx, wl.q, wl.kv, T,
                                        wl.scale)
    assert np.array_equal(out2, out) and (idx2 == idx[:, :T]).all()


def pin_topk_below_context_differs():
    """top_k forced below the context changes the output of later queries."""
    T, H, k = 120, 4, 16
    wl = synth.prefill(T, H, k, seed=34)
    args = (wl.q_offsets, wl.kv_offsets, wl.ctx_lens)
    _, _, out, _ = oracle.dsa_layer(*args, wl.q_idx, wl.w, wl.k_idx, wl.q, wl.kv, k, wl.scale)
    full, _ = oracle.full_causal_attn(*args, wl.q, wl.kv, wl.scale)
    diff = np.abs(out - full).max(axis=(1, 2))
    assert (diff[:k] < 1e-6).all(), "queries with p+1 <= top_k see their whole context"
    assert (diff[k:] > 1e-3).sum() >= (T - k) // 2


def pin_single_row_returns_its_value():
    """p = 0, or top_k = 1: the output is that row's V exactly, lse its logit."""
    T, H = 30, 3
    wl = synth.prefill(T, H, 1, seed=35)
    args = (wl.q_offsets, wl.kv_offsets, wl.ctx_lens)
    _, idx, out, lse = oracle.dsa_layer(*args, wl.q_idx, wl.w, wl.k_idx, wl.q, wl.kv, 1,
                                        wl.scale)
    kvf = _f(wl.kv)
    assert idx[0, 0] == 0
    for r in range(T):
        s = int(idx[r, 0])
        assert 0 <= s <= r
        assert (out[r] == kvf[s, :synth.DV].astype(np.float32)[None]).all()
        logit = wl.scale * (_f(wl.q[r]) @ kvf[s])
        assert np.abs(lse[r] - logit).max() < 1e-5 * max(1.0, np.abs(logit).max())




# --------------------------------------------------- indexer input step ----

def pin_projection_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "indexer_projection_worked_example.json")))
    qo, ko, cl = _one_seq(3, 2)
    sentinel = _bf16(np.full((3, g["Di"]), 7.0, np.float32))
    q_idx, k_out, w = oracle.indexer_project(
        qo, ko, cl, _bf16(g["x"]), _bf16(g["c_q"]), _bf16(g["w_q_b"]), _bf16(g["w_k"]),
        _bf16(g["w_proj"]), sentinel)
    assert np.array_equal(_f(q_idx), np.array(g["q_idx"], np.float64))
    for row, vals in g["k_rows"].items():
        assert np.array_equal(_f(k_out[int(row)]), np.array(vals, np.float64))
    assert np.array_equal(k_out[0], sentinel[0])           # earlier token untouched
    assert np.array_equal(w.astype(np.float64), np.array(g["w"], np.float64))


def pin_projection_identity_weights_copy_their_inputs():
    # unit rows pick input entries exactly: q_idx = c_q, k = x[:, :Di], w = x[:, 5:5+Hi]
    Hi, Di, d_model = 3, 4, 16
    d_q = Hi * Di
    g = np.random.Generator(np.random.PCG64(21))
    qo = np.array([0, 2, 3], np.int32)
    ko = np.array([0, 6, 10], np.int64)
    cl = np.array([5, 4], np.int32)
    x = _bf16(g.standard_normal((3, d_model)))
    c_q = _bf16(g.standard_normal((3, d_q)))
    w_q_b = _bf16(np.eye(d_q))
    w_k = _bf16(np.eye(Di, d_model))
    w_proj = _bf16(np.eye(Hi, d_model, k=5))
    k0 = np.zeros((10, Di), np.uint16)
    q_idx, k_out, w = oracle.indexer_project(qo, ko, cl, x, c_q, w_q_b, w_k, w_proj, k0)
    assert np.array_equal(q_idx.reshape(3, d_q), c_q)
    # new tokens: sequence 0 positions 3, 4 (rows 3, 4); sequence 1 position 3 (row 6 + 3)
    for t, row in enumerate([3, 4, 9]):
        assert np.array_equal(k_out[row], x[t, :Di]), (t, row)
    assert np.array_equal(w, _f(x[:, 5:5 + Hi]).astype(np.float32))
    written = {3, 4, 9}
    for row in range(10):
        if row not in written:
            assert not k_out[row].any(), row


def pin_projection_matches_float64_matmul():
    # the general case is a matmul: compare with torch's float64 product, rounded
    # to bf16 through fp32 as the step stores it
    Hi, Di, d_model, d_q = 4, 8, 96, 40
    g = np.random.Generator(np.random.PCG64(22))
    qo = np.array([0, 3, 3, 5], np.int32)
    ko = np.array([0, 7, 9, 15], np.int64)
    cl = np.array([6, 2, 5], np.int32)
    Nq, rows = 5, 15
    x = _bf16(g.standard_normal((Nq, d_model)))
    c_q = _bf16(g.standard_normal((Nq, d_q)))
    w_q_b = _bf16(g.standard_normal((Hi * Di, d_q)) * 0.2)
    w_k = _bf16(g.standard_normal((Di, d_model)) * 0.1)
    w_proj = _bf16(g.standard_normal((Hi, d_model)) * 0.1)
    k0 = _bf16(g.standard_normal((rows, Di)))
    q_idx, k_out, w = oracle.indexer_project(qo, ko, cl, x, c_q, w_q_b, w_k, w_proj, k0)
    T = lambda a: torch.from_numpy(_f(a))  # noqa: E731
    want_q = (T(c_q) @ T(w_q_b).T).numpy().astype(np.float32)
    want_k = (T(x) @ T(w_k).T).numpy().astype(np.float32)
    want_w = (T(x) @ T(w_proj).T).numpy()
    assert np.array_equal(q_idx.reshape(Nq, -1), synth.bf16_bits(want_q))
    # new tokens' cache rows: the last nq_b positions of each sequence
    new_rows = [3, 4, 5, 12, 13]
    assert np.array_equal(k_out[new_rows], synth.bf16_bits(want_k))
    others = [r for r in range(rows) if r not in new_rows]
    assert np.array_equal(k_out[others], k0[others])
    assert np.allclose(w.astype(np.float64), want_w, rtol=1e-6, atol=1e-7)


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
