"""Context-parallel decode: one DSA layer over a context split across GPUs.

The indexer scan is O(context) (aiunderstanding.org "Why it matters"; devotd.net
section 2: the indexer scores every earlier token), so a context too long for
one GPU's memory or time is split into contiguous ranges of positions, one per
rank.  Every rank holds its range of both caches and runs, on its own GPU:

  1. the indexer and the top-k selection over its own positions (the C ABI's
     dsa_indexer_score and dsa_topk with DSA_FLAG_SCORE_HISTOGRAM);
  2. an all-gather of every rank's (score, position) candidates: top_k per
     query per rank;
  3. the exact global selection: the global top-k is always inside the union
     of the per-range top-k sets, and with the candidates concatenated in
     rank order they are in ascending global position, so dsa_topk's tie rule
     (lower index first) is exactly the global one;
  4. attention over the selected rows it owns (dsa_sparse_attn, with the
     log-sum-exp of each head);
  5. a log-sum-exp merge of the ranks' partial outputs: an all-reduce of the
     maxima, then of the weighted outputs and weights.

Steps 1 and 4 run in the library's kernels, steps 2 and 5 are collectives
(NCCL through torch.distributed), step 3 is dsa_topk again.  Decode only: one
query per sequence, at the last position of the context.  The collectives
move top_k * 8 bytes of candidates and H * 512 * 4 bytes of output per query
and rank.  Communication goes through a small interface so that the same code
also runs as N emulated ranks in one process (one GPU, ranks in turn; no rank
waits on another's kernels).
"""
from __future__ import annotations

import dataclasses
from typing import List

import numpy as np
import torch

from . import binding as bd


@dataclasses.dataclass
class Shard:
    """One rank's range [start, stop) of every sequence's positions, on its GPU.

    q [Nq, H, 576], q_idx [Nq, 32, 128], w [Nq, 32] are every query's (replicated);
    k_idx [rows, 128] and kv [rows, 576] hold this range's rows, sequence b's
    at local_offsets[b] (contiguous, at least one row per sequence even when
    its range is empty)."""
    start: np.ndarray          # int64 [B] first global position held
    stop: np.ndarray           # int64 [B] one past the last
    ctx_lens: np.ndarray       # int32 [B] global context lengths
    local_offsets: np.ndarray  # int64 [B+1]
    q: torch.Tensor
    q_idx: torch.Tensor
    w: torch.Tensor
    k_idx: torch.Tensor
    kv: torch.Tensor
    scale: float


def make_shards(ctx_lens, kv_offsets, q, q_idx, w, k_idx, kv, scale, n_ranks, devices):
    """Splits contiguous host caches (bf16 bit patterns, one query per sequence)
    into n_ranks shards of position ranges, rank r's on devices[r]."""
    ctx_lens = np.asarray(ctx_lens, np.int64)
    starts, stops = shard_ranges(ctx_lens, n_ranks)
    shards = []
    for r in range(n_ranks):
        dev = devices[r]
        lens = stops[r] - starts[r]
        caps = np.maximum(lens, 1)
        lo = np.concatenate([[0], np.cumsum(caps)]).astype(np.int64)
        kk = np.zeros((int(lo[-1]), k_idx.shape[1]), np.uint16)
        vv = np.zeros((int(lo[-1]), kv.shape[1]), np.uint16)
        for b in range(ctx_lens.size):
            src = int(kv_offsets[b] + starts[r, b])
            kk[lo[b]:lo[b] + lens[b]] = k_idx[src:src + lens[b]]
            vv[lo[b]:lo[b] + lens[b]] = kv[src:src + lens[b]]
        shards.append(Shard(starts[r], stops[r], ctx_lens.astype(np.int32), lo,
                            bd.bf16_tensor(q, dev), bd.bf16_tensor(q_idx, dev),
                            torch.from_numpy(np.ascontiguousarray(w)).to(dev),
                            bd.bf16_tensor(kk, dev), bd.bf16_tensor(vv, dev), float(scale)))
    return shards


def shard_ranges(ctx_lens, n_ranks, align=128):
    """Contiguous, nearly equal ranges of each sequence's positions per rank,
    boundaries on multiples of `align` (empty ranges allowed)."""
    ctx_lens = np.asarray(ctx_lens, np.int64)
    starts = np.zeros((n_ranks, ctx_lens.size), np.int64)
    stops = np.zeros_like(starts)
    for b, L in enumerate(ctx_lens):
        per = -(-int(L) // n_ranks)
        per = -(-per // align) * align
        for r in range(n_ranks):
            starts[r, b] = min(int(L), r * per)
            stops[r, b] = min(int(L), (r + 1) * per)
    return starts, stops


class LocalComm:
    """All ranks in one process: the collectives combine per-rank lists."""

    def __init__(self, n_ranks):
        self.n = n_ranks

    def all_gather_cat(self, per_rank: List[torch.Tensor], dim) -> List[torch.Tensor]:
        cat = torch.cat(per_rank, dim=dim)
        return [cat for _ in per_rank]

    def all_reduce(self, per_rank: List[torch.Tensor], op) -> List[torch.Tensor]:
        acc = per_rank[0].clone()
        for t in per_rank[1:]:
            acc = torch.maximum(acc, t) if op == "max" else acc + t
        return [acc for _ in per_rank]


class DistComm:
    """One rank per process: torch.distributed collectives (NCCL on GPUs)."""

    def __init__(self, dist):
        self.dist = dist
        self.n = dist.get_world_size()

    def all_gather_cat(self, per_rank, dim):
        (t,) = per_rank
        parts = [torch.empty_like(t) for _ in range(self.n)]
        self.dist.all_gather(parts, t.contiguous())
        return [torch.cat(parts, dim=dim)]

    def all_reduce(self, per_rank, op):
        (t,) = per_rank
        t = t.clone()
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX if op == "max" else self.dist.ReduceOp.SUM)
        return [t]


def _local_batch(sh: Shard):
    """The shard as a batch of its own: each sequence's range as a context of
    stop - start positions, its one query at the range's last position (so it
    sees the whole range: every range ends at or before the query)."""
    lens = (sh.stop - sh.start).astype(np.int32)
    nq = (lens > 0).astype(np.int32)
    qo = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    return bd.Batch(qo, sh.local_offsets, lens, sh.q.device), nq


def local_candidates(sh: Shard, top_k: int):
    """Steps 1: this range's top_k (score, global position) per query; padding
    (fewer positions than top_k) as (-inf, -1)."""
    dev = sh.q.device
    B = sh.ctx_lens.size
    batch, nq = _local_batch(sh)
    scores = torch.full((B, top_k), float("-inf"), device=dev)
    pos = torch.full((B, top_k), -1, dtype=torch.int64, device=dev)
    rows = np.nonzero(nq)[0]
    if rows.size:
        sel = torch.from_numpy(rows).to(dev)
        max_len = int((sh.stop - sh.start).max())
        ld = (max_len + 3) // 4 * 4
        ws = bd.alloc_workspace(batch, sh.q.shape[1], top_k, dev)
        sc = torch.empty(rows.size, ld, device=dev)
        idx = torch.empty(rows.size, top_k, dtype=torch.int32, device=dev)
        bd.indexer_score(batch, sh.q_idx[sel].contiguous(), sh.w[sel].contiguous(), sh.k_idx, sc,
                         ld, ws, flags=bd.FLAG_SCORE_HISTOGRAM)
        bd.topk(batch, sc, ld, top_k, idx, ws, flags=bd.FLAG_SCORE_HISTOGRAM)
        bd.check_device_status(ws)
        valid = idx >= 0
        li = idx.clamp(min=0).long()
        s_loc = torch.gather(sc, 1, li)
        start = torch.from_numpy(sh.start[rows]).to(dev)[:, None]
        scores[sel] = torch.where(valid, s_loc, torch.full_like(s_loc, float("-inf")))
        pos[sel] = torch.where(valid, li + start, torch.full_like(li, -1))
    return scores, pos


def select_global(cand_scores, cand_pos, top_k, ctx_lens):
    """Step 3: the exact top_k of every query over all ranks' candidates
    (ascending global positions, -1 padded), by dsa_topk on the candidate
    rows; padding candidates score -inf and are dropped if they come in."""
    dev = cand_scores.device
    Nq, n_cand = cand_scores.shape
    ld = (n_cand + 3) // 4 * 4
    sc = torch.full((Nq, ld), float("-inf"), device=dev)
    sc[:, :n_cand] = cand_scores
    qo = np.arange(Nq + 1, dtype=np.int32)
    ko = np.arange(Nq + 1, dtype=np.int64) * ld
    batch = bd.Batch(qo, ko, np.full(Nq, n_cand, np.int32), dev)
    ws = bd.alloc_workspace(batch, 1, top_k, dev)
    ci = torch.empty(Nq, top_k, dtype=torch.int32, device=dev)
    bd.topk(batch, sc, ld, top_k, ci, ws)
    bd.check_device_status(ws)
    picked = torch.where(ci >= 0, torch.gather(cand_pos, 1, ci.clamp(min=0).long()),
                         torch.full_like(ci, -1, dtype=torch.int64))
    # real positions keep their ascending order; padding moves to the end
    key = torch.where(picked >= 0, picked, torch.full_like(picked, 1 << 62))
    picked = torch.sort(key, dim=1).values
    n_sel = torch.clamp(torch.from_numpy(np.asarray(ctx_lens, np.int64)).to(dev), max=top_k)
    keep = torch.arange(top_k, device=dev)[None, :] < n_sel[:, None]
    return torch.where(keep, picked, torch.full_like(picked, -1)).to(torch.int32)


def local_attention(sh: Shard, idx_global, top_k):
    """Step 4: attention over the selected rows this rank holds; out is
    normalised over them and lse is their log-sum-exp (-inf: none)."""
    dev = sh.q.device
    B, H = sh.ctx_lens.size, sh.q.shape[1]
    start = torch.from_numpy(sh.start).to(dev)[:, None]
    stop = torch.from_numpy(sh.stop).to(dev)[:, None]
    g = idx_global.long()
    mine = (g >= start) & (g < stop)
    local = torch.where(mine, g - start, torch.full_like(g, -1)).to(torch.int32)
    # the attention call's batch: every sequence, one query seeing its range
    lens = np.maximum(sh.stop - sh.start, 1).astype(np.int32)
    out = torch.empty(B, H, 512, device=dev)
    lse = torch.empty(B, H, device=dev)
    batch = bd.Batch(np.arange(B + 1, dtype=np.int32), sh.local_offsets, lens, dev)
    ws = bd.alloc_workspace(batch, H, top_k, dev)
    bd.sparse_attn(batch, sh.q, sh.kv, local.contiguous(), top_k, sh.scale, out, lse, ws)
    bd.check_device_status(ws)
    return out, lse


def lse_merge(outs, lses, comm):
    """Step 5: O = sum_r e^(lse_r - M) O_r / sum_r e^(lse_r - M), M = max_r lse_r."""
    M = comm.all_reduce(lses, "max")
    wts, wouts = [], []
    for o, l, m in zip(outs, lses, M):
        m_safe = torch.where(torch.isfinite(m), m, torch.zeros_like(m))
        wgt = torch.where(torch.isfinite(l), torch.exp(l - m_safe), torch.zeros_like(l))
        wts.append(wgt)
        wouts.append(o * wgt[..., None])
    S = comm.all_reduce(wts, "sum")
    O = comm.all_reduce(wouts, "sum")
    res = []
    for s, o, m in zip(S, O, M):
        inv = torch.where(s > 0, 1.0 / s, torch.zeros_like(s))
        res.append((o * inv[..., None], torch.where(s > 0, m + torch.log(s),
                                                    torch.full_like(s, float("-inf")))))
    return res


def cp_decode(shards: List[Shard], comm, top_k):
    """One context-parallel decode step over `shards` (this process's ranks:
    all of them under LocalComm, one under DistComm).  Returns, per shard,
    (out [B, H, 512], lse [B, H], idx [B, top_k]), the same on every rank."""
    cands = [local_candidates(sh, top_k) for sh in shards]
    all_sc = comm.all_gather_cat([c[0] for c in cands], dim=1)
    all_pos = comm.all_gather_cat([c[1] for c in cands], dim=1)
    idxs = [select_global(s, p, top_k, sh.ctx_lens) for s, p, sh in zip(all_sc, all_pos, shards)]
    parts = [local_attention(sh, ix, top_k) for sh, ix in zip(shards, idxs)]
    merged = lse_merge([p[0] for p in parts], [p[1] for p in parts], comm)
    return [(o, l, ix) for (o, l), ix in zip(merged, idxs)]
