"""Comparison rules between the CUDA path and the CPU oracle.

Tolerances:
  * index scores: |gpu - ref| <= SCORE_RTOL * (|ref| + rms(ref row)).  Each
    head's dot product sums 128 exact bf16 products in fp32 on the tensor
    core (relative error below about 128 * 2^-24 = 8e-6 of the sum of the
    products' magnitudes), then 32 fp32 multiply-adds weight the heads; the
    reference is computed in double and rounded once, so 2e-5 of the score's
    magnitude plus the row's rms covers both;
  * selected sets: identical, except for positions whose oracle score lies
    within TIE_RTOL (relative) of the oracle's k-th score; such boundary swaps
    are counted and reported;
  * attention output: max |gpu - ref| <= OUT_ATOL (2e-3, bf16 inputs, fp32
    accumulation); log-sum-exp: <= LSE_ATOL.
"""
from __future__ import annotations

import numpy as np

SCORE_RTOL = 2e-5
TIE_RTOL = 1e-5
OUT_ATOL = 2e-3
LSE_ATOL = 1e-4


def positions(wl):
    return wl.positions()


def check_scores(gpu, ref, wl, rows=None):
    """Returns the worst |err| / (|ref| + rms) over the compared entries."""
    pos = positions(wl)
    rows = range(wl.Nq) if rows is None else rows
    worst = 0.0
    for r in rows:
        p = int(pos[r])
        g = gpu[r, :p + 1].astype(np.float64)
        o = ref[r, :p + 1].astype(np.float64)
        scale = np.abs(o) + np.sqrt(np.mean(o * o)) + 1e-30
        err = np.abs(g - o) / scale
        worst = max(worst, float(err.max()))
        assert err.max() <= SCORE_RTOL, (r, float(err.max()), int(err.argmax()))
    return worst


def check_index_structure(idx, wl, rows=None):
    pos = positions(wl)
    rows = range(wl.Nq) if rows is None else rows
    k = idx.shape[1]
    for r in rows:
        p = int(pos[r])
        n = min(k, p + 1)
        sel = idx[r, :n]
        assert (idx[r, n:] == -1).all(), r
        assert sel.min() >= 0 and sel.max() <= p, r
        assert n == 1 or (np.diff(sel) > 0).all(), r


def check_selection(gpu_idx, ref_idx, ref_scores, wl, rows=None):
    """Sets equal up to boundary ties of the oracle's scores; returns the swap count."""
    check_index_structure(gpu_idx, wl, rows)
    pos = positions(wl)
    rows = range(wl.Nq) if rows is None else rows
    k = gpu_idx.shape[1]
    swaps = 0
    for r in rows:
        p = int(pos[r])
        n = min(k, p + 1)
        a = gpu_idx[r, :n]
        b = ref_idx[r, :n]
        if np.array_equal(a, b):
            continue
        sc = ref_scores[r, :p + 1].astype(np.float64)
        theta = sc[b].min()
        diff = np.setxor1d(a, b)
        near = np.abs(sc[diff] - theta) <= TIE_RTOL * abs(theta)
        assert near.all(), (r, diff[~near][:8], sc[diff[~near][:8]], theta)
        swaps += diff.size // 2
    return swaps


def check_attention(gpu_out, gpu_lse, ref_out, ref_lse, rows=None):
    """Returns (max |out err|, max |lse err|)."""
    if rows is not None:
        gpu_out, ref_out = gpu_out[rows], ref_out[rows]
        gpu_lse, ref_lse = gpu_lse[rows], ref_lse[rows]
    e_out = float(np.abs(gpu_out.astype(np.float64) - ref_out).max())
    e_lse = float(np.abs(gpu_lse.astype(np.float64) - ref_lse).max())
    assert np.isfinite(gpu_out).all()
    assert e_out <= OUT_ATOL, e_out
    assert e_lse <= LSE_ATOL, e_lse
    return e_out, e_lse


def sample_rows(wl, n, seed=0, must=()):
    """A seeded sample of query rows: the listed ones plus uniform draws."""
    g = np.random.Generator(np.random.PCG64(seed))
    rows = set(int(r) for r in must if 0 <= r < wl.Nq)
    extra = g.choice(wl.Nq, size=min(n, wl.Nq), replace=False)
    for r in extra:
        if len(rows) >= n:
            break
        rows.add(int(r))
    return np.array(sorted(rows), dtype=np.int64)
