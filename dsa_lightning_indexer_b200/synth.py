"""Seeded synthetic inputs for the DSA layer.

This module only draws random inputs and lays them out; it holds none of the
layer's arithmetic.  Tests, the benchmark and the smoke check take their inputs
from here, and the same host arrays feed both the CUDA library and the CPU
oracle.

Normal tensors are drawn in float32 with numpy's PCG64, in consecutive blocks
of BLOCK elements (row-major order), block i from SeedSequence([seed, layer,
tensor_id, i]); the blocks are drawn in parallel threads, and the values do
not depend on the thread count.  Other draws (weights, lengths, directions)
come from one PCG64 seeded with SeedSequence([seed, layer, tensor_id]).
Values are rounded to bfloat16 with round-to-nearest-even; bf16 tensors are
held as their uint16 bit patterns.

The shapes follow the released Kimi-K3.1-Pro configuration (llama.cpp b12180
news, devotd.net configuration table): indexer of 32 heads x 128, no RoPE,
top_k 2048; the attention side is a shared key-only latent cache of width 576
whose first 512 entries are V.
"""
from __future__ import annotations

import dataclasses
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

HI = 32       # indexer heads
DI = 128      # indexer head dim
D = 576       # latent key width
DV = 512      # value width (leading part of the latent row)

# tensor ids inside SeedSequence([seed, layer, tensor_id])
T_QIDX, T_W, T_KIDX, T_Q, T_KV, T_DIRS, T_ASSIGN, T_LENS, T_PROJ = range(9)


BLOCK = 1 << 22  # elements per independently seeded block of a normal tensor


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit pattern (uint16), round to nearest even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if x.size >= (1 << 16):  # the same rounding, multi-threaded, for big tensors
        import torch
        return torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    u = x.view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """bfloat16 bit pattern (uint16) -> float32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(
        np.float32)


def rng(seed: int, layer: int, tensor_id: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, layer, tensor_id])))


def normal_f32(seed, layer, tid, shape, std=1.0) -> np.ndarray:
    """N(0, std^2) float32 draws of `shape`, in seeded blocks of BLOCK elements."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)
    nblk = max(1, (n + BLOCK - 1) // BLOCK)

    def fill(i):
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, layer, tid, i])))
        a, b = i * BLOCK, min(n, (i + 1) * BLOCK)
        g.standard_normal(size=b - a, dtype=np.float32, out=out[a:b])

    if nblk == 1:
        fill(0)
    else:
        with ThreadPoolExecutor(min(nblk, os.cpu_count() or 1)) as ex:
            list(ex.map(fill, range(nblk)))
    if std != 1.0:
        out *= np.float32(std)
    return out.reshape(shape)


def normal_bf16(seed, layer, tid, shape, std=1.0) -> np.ndarray:
    return bf16_bits(normal_f32(seed, layer, tid, shape, std))


@dataclasses.dataclass
class Workload:
    """One DSA-layer problem, host arrays only."""
    name: str
    q_offsets: np.ndarray   # int32 [B+1]
    kv_offsets: np.ndarray  # int64 [B+1]
    ctx_lens: np.ndarray    # int32 [B]
    q_idx: np.ndarray       # uint16 [Nq, 32, 128]
    w: np.ndarray           # float32 [Nq, 32]
    k_idx: np.ndarray       # uint16 [rows, 128]
    q: np.ndarray           # uint16 [Nq, H, 576]
    kv: np.ndarray          # uint16 [rows, 576]
    top_k: int
    scale: float            # float32-representable softmax scale

    @property
    def B(self) -> int:
        return int(self.ctx_lens.shape[0])

    @property
    def Nq(self) -> int:
        return int(self.q_offsets[-1])

    @property
    def H(self) -> int:
        return int(self.q.shape[1])

    @property
    def rows(self) -> int:
        return int(self.kv_offsets[-1])

    def positions(self) -> np.ndarray:
        """Position p of every query row (int64 [Nq])."""
        out = np.empty(self.Nq, dtype=np.int64)
        for b in range(self.B):
            a, e = int(self.q_offsets[b]), int(self.q_offsets[b + 1])
            out[a:e] = int(self.ctx_lens[b]) - (e - a) + np.arange(e - a)
        return out


def softmax_scale(d: int = D) -> float:
    return float(np.float32(1.0 / math.sqrt(d)))


def _assemble(name, seed, layer, nq_per_seq, lens, H, top_k, planted=False, caps=None):
    lens = np.asarray(lens, dtype=np.int64)
    B = lens.shape[0]
    nq = np.asarray(nq_per_seq, dtype=np.int64)
    caps = lens if caps is None else np.asarray(caps, dtype=np.int64)
    q_off = np.zeros(B + 1, dtype=np.int32)
    q_off[1:] = np.cumsum(nq)
    kv_off = np.zeros(B + 1, dtype=np.int64)
    kv_off[1:] = np.cumsum(caps)
    Nq, rows = int(q_off[-1]), int(kv_off[-1])
    q_idx = normal_bf16(seed, layer, T_QIDX, (Nq, HI, DI))
    w = rng(seed, layer, T_W).standard_normal(size=(Nq, HI), dtype=np.float32) * np.float32(
        1.0 / math.sqrt(HI))
    if planted:
        # K_idx[s] = N(0, I) + 3 * u_{c(s)}: 64 random unit directions, one per token.
        g = rng(seed, layer, T_DIRS)
        dirs = g.standard_normal(size=(64, DI), dtype=np.float32)
        dirs /= np.linalg.norm(dirs, axis=1, keepdims=True)
        assign = rng(seed, layer, T_ASSIGN).integers(0, 64, size=rows)
        base = normal_f32(seed, layer, T_KIDX, (rows, DI))
        base += np.float32(3.0) * dirs[assign]
        k_idx = bf16_bits(base)
    else:
        k_idx = normal_bf16(seed, layer, T_KIDX, (rows, DI))
    q = normal_bf16(seed, layer, T_Q, (Nq, H, D))
    kv = normal_bf16(seed, layer, T_KV, (rows, D))
    return Workload(name, q_off, kv_off, lens.astype(np.int32), q_idx, w.astype(np.float32),
                    k_idx, q, kv, int(top_k), softmax_scale())


def prefill(T, H, top_k, seed, planted=False, name=None, layer=0) -> Workload:
    """One causal sequence of T tokens, every token a query."""
    return _assemble(name or f"prefill_T{T}_H{H}_k{top_k}", seed, layer, [T], [T], H, top_k,
                     planted=planted)


def decode(B, L, H, top_k, seed, name=None, layer=0) -> Workload:
    """B sequences of L cached tokens (the new one included), one query each."""
    return _assemble(name or f"decode_B{B}_L{L}_H{H}_k{top_k}", seed, layer, [1] * B, [L] * B,
                     H, top_k)


def ragged_lengths(n, lo, hi, seed) -> np.ndarray:
    """Context lengths drawn log-uniform in [lo, hi]."""
    u = rng(seed, 0, T_LENS).uniform(math.log(lo), math.log(hi), size=n)
    return np.floor(np.exp(u)).astype(np.int64).clip(lo, hi)


def ragged_decode(lens, H, top_k, seed, layer=0, name=None) -> Workload:
    """Decode over sequences of the given lengths, contiguous caches with offsets."""
    lens = np.asarray(lens, dtype=np.int64)
    return _assemble(name or f"ragged_B{lens.shape[0]}_H{H}_k{top_k}", seed, layer,
                     [1] * lens.shape[0], lens, H, top_k)


def custom(lens, nq, H, top_k, seed, layer=0, caps=None, name="custom") -> Workload:
    """Any mix of sequence lengths and per-sequence query counts (test shapes)."""
    return _assemble(name, seed, layer, nq, lens, H, top_k, caps=caps)


@dataclasses.dataclass
class PagedCaches:
    """The caches of a workload laid out in pages: position s of sequence b
    is row block_table[b, s // page_size] * page_size + s % page_size."""
    page_size: int
    block_table: np.ndarray  # int32 [B, max_blocks]
    cache_rows: int
    k_idx: np.ndarray        # uint16 [cache_rows, 128]
    kv: np.ndarray           # uint16 [cache_rows, 576]


def paged(wl: Workload, page_size: int, seed: int, spare_pages: int = 3) -> Workload:
    """The same workload with its caches cut into pages of `page_size` rows,
    placed in a seeded random order among `spare_pages` unused pages (filled
    with other values); the contiguous arrays stay on the workload for the
    oracle.  Only the data layout changes."""
    B = wl.B
    caps = np.diff(wl.kv_offsets).astype(np.int64)
    n_pages = [int((c + page_size - 1) // page_size) for c in caps]
    total = sum(n_pages) + spare_pages
    order = rng(seed, 0, T_PROJ + 1).permutation(total)
    bt = np.full((B, max(1, max(n_pages))), -1, dtype=np.int32)
    k_pg = normal_bf16(seed, 1, T_KIDX, (total * page_size, DI))
    kv_pg = normal_bf16(seed, 1, T_KV, (total * page_size, D))
    at = 0
    for b in range(B):
        k0 = int(wl.kv_offsets[b])
        for j in range(n_pages[b]):
            page = int(order[at])
            at += 1
            bt[b, j] = page
            lo, hi = j * page_size, min(int(caps[b]), (j + 1) * page_size)
            dst = page * page_size
            k_pg[dst:dst + hi - lo] = wl.k_idx[k0 + lo:k0 + hi]
            kv_pg[dst:dst + hi - lo] = wl.kv[k0 + lo:k0 + hi]
    out = dataclasses.replace(wl, name=wl.name + f"_paged{page_size}")
    out.paged = PagedCaches(page_size, bt, total * page_size, k_pg, kv_pg)
    return out


def glue_projection(seed, n_in=DV, H=64) -> np.ndarray:
    """Fixed random bf16 projection [n_in, H*576] ~ N(0, 1/n_in) chaining stacked layers."""
    return normal_bf16(seed, 0, T_PROJ, (n_in, H * D), std=1.0 / math.sqrt(n_in))


def chain_query(out: np.ndarray, proj: np.ndarray) -> np.ndarray:
    """Next stacked layer's main query from this layer's output [Nq, H, 512]:
    the mean over heads, RMS-normalised and rounded to bf16, times the fixed
    projection [512, H*576], rounded to bf16 -> [Nq, H, 576] bit patterns."""
    m = np.asarray(out, dtype=np.float64).mean(axis=1)
    m = m / np.sqrt((m * m).mean(axis=1, keepdims=True) + 1e-6)
    x = bf16_to_f32(bf16_bits(m.astype(np.float32)))
    q = x @ bf16_to_f32(proj)
    return bf16_bits(q).reshape(out.shape[0], -1, D)


# The five workloads the layer is specified on.
def tiny_prefill(top_k: int) -> Workload:
    """Prefill, 1 sequence of 1024 tokens, 16 heads; run at top_k 256 and 2048. Seed 0."""
    return prefill(1024, 16, top_k, seed=0, name=f"prefill_T1024_H16_k{top_k}")


def decode_b8_32k() -> Workload:
    """Decode, 8 sequences x 32768 cached tokens, 64 heads, top_k 2048. Seed 1."""
    return decode(8, 32768, 64, 2048, seed=1, name="decode_B8_L32768")


def prefill_16k() -> Workload:
    """Prefill, 16384 tokens, 64 heads, top_k 2048, planted low-rank indexer keys. Seed 2."""
    return prefill(16384, 64, 2048, seed=2, planted=True, name="prefill_T16384_planted")


def decode_b4_128k() -> Workload:
    """Decode, 4 sequences x 131072 cached tokens, 64 heads, top_k 2048. Seed 3."""
    return decode(4, 131072, 64, 2048, seed=3, name="decode_B4_L131072")


def ragged_lengths_32() -> np.ndarray:
    """The 32 log-uniform context lengths in [1024, 131072] of the ragged workload. Seed 4."""
    return ragged_lengths(32, 1024, 131072, seed=4)


def ragged_layer(layer: int) -> Workload:
    """Layer `layer` (0..23) of the stacked ragged decode: own caches and indexer inputs."""
    return ragged_decode(ragged_lengths_32(), 64, 2048, seed=4, layer=layer,
                         name=f"ragged_B32_layer{layer}")
