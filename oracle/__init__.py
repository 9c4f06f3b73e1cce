"""CPU oracle of the DSA layer — TEST INFRASTRUCTURE ONLY.

Plain double-precision C++ (``dsa_oracle.cpp``) behind a thin ctypes wrapper.
Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package; the product library never does, and the
two share no code.  What the functions compute, and which passage of the
source pages each step follows, is written in the header of ``dsa_oracle.cpp``.

Array conventions (numpy, C-contiguous):
  q_offsets  int32 [B+1]   query rows of sequence b: [q_offsets[b], q_offsets[b+1])
  kv_offsets int64 [B+1]   first cache row of sequence b
  ctx_lens   int32 [B]     context length L_b (rows 0..L_b-1 of the sequence)
  q_idx      uint16 [Nq, Hi, Di]  indexer queries, bf16 bit patterns
  w          float32 [Nq, Hi]     per-head indexer weights
  k_idx      uint16 [rows, Di]    indexer key cache, bf16
  q          uint16 [Nq, H, D]    attention queries, bf16
  kv         uint16 [rows, D]     shared latent key cache, bf16; V = first Dv
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.cpp")
_SO = os.path.join(_HERE, "_build", "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (OpenMP, no fast-math, no FP contraction)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        os.makedirs(os.path.dirname(_SO), exist_ok=True)
        tmp = _SO + f".{os.getpid()}.tmp"
        subprocess.check_call([
            "g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
            "-fPIC", "-shared", _SRC, "-o", tmp,
        ])
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.oracle_set_threads.argtypes = [i32]
        lib.oracle_max_threads.restype = i32
        lib.oracle_set_fault.argtypes = [i32]
        lib.oracle_indexer_scores.argtypes = [i32, P, P, P, i32, i32, P, P, P, P, i64, P, i64]
        lib.oracle_topk.argtypes = [i32, P, P, P, P, i64, i32, P, P, i64]
        lib.oracle_sparse_attn.argtypes = [i32, P, P, P, i32, i32, i32, P, P, P, i32, dbl,
                                           P, P, P, i64]
        lib.oracle_full_causal_attn.argtypes = [i32, P, P, P, i32, i32, i32, P, P, dbl, P, P,
                                                P, i64]
        lib.oracle_dsa_layer.argtypes = [i32, P, P, P, i32, i32, P, P, P, i32, i32, i32, P, P,
                                         i32, dbl, P, i64, P, P, P, P, i64]
        lib.oracle_indexer_project.argtypes = [i32, P, P, P, i32, i32, i64, i64, P, P, P, P, P,
                                               P, P, P, P, i64]
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _batch(q_offsets, kv_offsets, ctx_lens):
    qo = _c(q_offsets, np.int32)
    ko = _c(kv_offsets, np.int64)
    cl = _c(ctx_lens, np.int32)
    B = cl.shape[0]
    assert qo.shape == (B + 1,) and ko.shape == (B + 1,)
    nq = np.diff(qo)
    assert (nq >= 0).all() and (nq <= cl).all(), "each sequence needs nq_b <= L_b"
    assert (cl <= np.diff(ko)).all(), "context longer than the sequence's cache rows"
    return B, qo, ko, cl


def _sample(sample):
    if sample is None:
        return None, 0
    s = _c(sample, np.int64)
    return s, s.shape[0]


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def set_fault(f: int) -> None:
    """Plant a known mistake in the oracle (mutation tests only); 0 restores it."""
    _load().oracle_set_fault(int(f))


def indexer_scores(q_offsets, kv_offsets, ctx_lens, q_idx, w, k_idx, ld=None, sample=None):
    """Index scores [Nq, ld] float32; entries past each query's position stay NaN."""
    B, qo, ko, cl = _batch(q_offsets, kv_offsets, ctx_lens)
    q_idx = _c(q_idx, np.uint16)
    w = _c(w, np.float32)
    k_idx = _c(k_idx, np.uint16)
    Nq, Hi, Di = q_idx.shape
    assert w.shape == (Nq, Hi) and k_idx.shape[1] == Di
    ld = int(ld if ld is not None else max(int(cl.max()), 1))
    scores = np.full((Nq, ld), np.nan, dtype=np.float32)
    s, ns = _sample(sample)
    _load().oracle_indexer_scores(B, _ptr(qo), _ptr(ko), _ptr(cl), Hi, Di, _ptr(q_idx),
                                  _ptr(w), _ptr(k_idx), _ptr(scores), ld, _ptr(s), ns)
    return scores


def topk(q_offsets, kv_offsets, ctx_lens, scores, top_k, sample=None):
    """Selected positions [Nq, top_k] int32, ascending, -1 padded."""
    B, qo, ko, cl = _batch(q_offsets, kv_offsets, ctx_lens)
    scores = _c(scores, np.float32)
    Nq, ld = scores.shape
    assert ld >= int(cl.max())
    idx = np.full((Nq, top_k), -2, dtype=np.int32)
    s, ns = _sample(sample)
    _load().oracle_topk(B, _ptr(qo), _ptr(ko), _ptr(cl), _ptr(scores), ld, int(top_k),
                        _ptr(idx), _ptr(s), ns)
    return idx


def sparse_attn(q_offsets, kv_offsets, ctx_lens, q, kv, idx, scale, Dv=512, sample=None):
    """Attention over the listed positions: out [Nq, H, Dv] f32, lse [Nq, H] f32."""
    B, qo, ko, cl = _batch(q_offsets, kv_offsets, ctx_lens)
    q = _c(q, np.uint16)
    kv = _c(kv, np.uint16)
    idx = _c(idx, np.int32)
    Nq, H, D = q.shape
    top_k = idx.shape[1]
    out = np.full((Nq, H, Dv), np.nan, dtype=np.float32)
    lse = np.full((Nq, H), np.nan, dtype=np.float32)
    s, ns = _sample(sample)
    _load().oracle_sparse_attn(B, _ptr(qo), _ptr(ko), _ptr(cl), H, D, Dv, _ptr(q), _ptr(kv),
                               _ptr(idx), top_k, float(scale), _ptr(out), _ptr(lse),
                               _ptr(s), ns)
    return out, lse


def full_causal_attn(q_offsets, kv_offsets, ctx_lens, q, kv, scale, Dv=512, sample=None):
    """Full causal attention over positions 0..p (no indexer)."""
    B, qo, ko, cl = _batch(q_offsets, kv_offsets, ctx_lens)
    q = _c(q, np.uint16)
    kv = _c(kv, np.uint16)
    Nq, H, D = q.shape
    out = np.full((Nq, H, Dv), np.nan, dtype=np.float32)
    lse = np.full((Nq, H), np.nan, dtype=np.float32)
    s, ns = _sample(sample)
    _load().oracle_full_causal_attn(B, _ptr(qo), _ptr(ko), _ptr(cl), H, D, Dv, _ptr(q),
                                    _ptr(kv), float(scale), _ptr(out), _ptr(lse), _ptr(s), ns)
    return out, lse


def dsa_layer(q_offsets, kv_offsets, ctx_lens, q_idx, w, k_idx, q, kv, top_k, scale,
              Dv=512, sample=None, ld=None):
    """Whole layer: returns (scores, idx, out, lse) for every (sampled) query row."""
    B, qo, ko, cl = _batch(q_offsets, kv_offsets, ctx_lens)
    q_idx = _c(q_idx, np.uint16)
    w = _c(w, np.float32)
    k_idx = _c(k_idx, np.uint16)
    q = _c(q, np.uint16)
    kv = _c(kv, np.uint16)
    Nq, Hi, Di = q_idx.shape
    _, H, D = q.shape
    ld = int(ld if ld is not None else max(int(cl.max()), 1))
    scores = np.full((Nq, ld), np.nan, dtype=np.float32)
    idx = np.full((Nq, top_k), -2, dtype=np.int32)
    out = np.full((Nq, H, Dv), np.nan, dtype=np.float32)
    lse = np.full((Nq, H), np.nan, dtype=np.float32)
    s, ns = _sample(sample)
    _load().oracle_dsa_layer(B, _ptr(qo), _ptr(ko), _ptr(cl), Hi, Di, _ptr(q_idx), _ptr(w),
                             _ptr(k_idx), H, D, Dv, _ptr(q), _ptr(kv), int(top_k), float(scale),
                             _ptr(scores), ld, _ptr(idx), _ptr(out), _ptr(lse), _ptr(s), ns)
    return scores, idx, out, lse


def indexer_project(q_offsets, kv_offsets, ctx_lens, x, c_q, w_q_b, w_k, w_proj, k_idx,
                    sample=None):
    """The indexer's input step for every (sampled) query row: returns
    (q_idx [Nq, Hi, Di] bf16 bits, k_idx with the new tokens' rows written,
    w [Nq, Hi] float32).  x [Nq, d_model] and c_q [Nq, d_q] are bf16 bits;
    weights are [out, in] bf16 bits: w_q_b [Hi*Di, d_q], w_k [Di, d_model],
    w_proj [Hi, d_model].  k_idx is copied, not modified."""
    B, qo, ko, cl = _batch(q_offsets, kv_offsets, ctx_lens)
    x = _c(x, np.uint16)
    c_q = _c(c_q, np.uint16)
    w_q_b = _c(w_q_b, np.uint16)
    w_k = _c(w_k, np.uint16)
    w_proj = _c(w_proj, np.uint16)
    k_out = np.array(k_idx, dtype=np.uint16, copy=True, order="C")
    Nq, d_model = x.shape
    d_q = c_q.shape[1]
    Di = w_k.shape[0]
    Hi = w_proj.shape[0]
    assert c_q.shape[0] == Nq and w_q_b.shape == (Hi * Di, d_q)
    assert w_k.shape == (Di, d_model) and w_proj.shape == (Hi, d_model)
    assert k_out.shape[1] == Di
    q_idx = np.zeros((Nq, Hi, Di), dtype=np.uint16)
    w = np.full((Nq, Hi), np.nan, dtype=np.float32)
    s, ns = _sample(sample)
    _load().oracle_indexer_project(B, _ptr(qo), _ptr(ko), _ptr(cl), Hi, Di, int(d_model),
                                   int(d_q), _ptr(x), _ptr(c_q), _ptr(w_q_b), _ptr(w_k),
                                   _ptr(w_proj), _ptr(q_idx), _ptr(k_out), _ptr(w), _ptr(s), ns)
    return q_idx, k_out, w
