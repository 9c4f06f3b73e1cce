"""The benchmark's roofline arithmetic, checked against figures worked out by
hand from the layer's definition (no GPU needed): algorithmic bytes of the
128K decode step and of one indexer launch, causal indexer flops of the 16K
prefill, and the kernel count of one layer call."""
import numpy as np
import pytest

import bench
from dsa_lightning_indexer_b200 import synth


def _layout(lens, nq, H, top_k):
    """A workload with the given sequence layout and zero-stride tensors (only
    shapes and offsets matter here)."""
    lens = np.asarray(lens, np.int64)
    nq = np.asarray(nq, np.int64)
    q_off = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    kv_off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    Nq, rows = int(q_off[-1]), int(kv_off[-1])
    z16 = np.uint16(0)
    return synth.Workload("layout", q_off, kv_off, lens.astype(np.int32),
                          np.broadcast_to(z16, (Nq, synth.HI, synth.DI)),
                          np.broadcast_to(np.float32(0), (Nq, synth.HI)),
                          np.broadcast_to(z16, (rows, synth.DI)),
                          np.broadcast_to(z16, (Nq, H, synth.D)),
                          np.broadcast_to(z16, (rows, synth.D)), top_k, synth.softmax_scale())


def test_decode_128k_bytes():
    wl = _layout([131072] * 4, [1] * 4, 64, 2048)
    # indexer: every cached key's 256 bytes, plus each query's 32x128 bf16 and 32 fp32 weights
    k1 = 4 * 131072 * 256 + 4 * (8192 + 128)
    assert bench.indexer_bytes(wl) == k1 == 134_251_008
    # layer: keys, 2048 gathered 1152-byte latent rows per query, and per query
    # q (64x576 bf16), q_idx, w, out (64x512 fp32), lse, idx
    per_q = 64 * 576 * 2 + 32 * 128 * 2 + 32 * 4 + 64 * 512 * 4 + 64 * 4 + 2048 * 4
    total = 4 * 131072 * 256 + 4 * 2048 * 1152 + 4 * per_q
    got = bench.decode_bytes(wl)
    assert got["total"] == total == 144_541_184
    assert got["total"] / 4 / 1e6 == pytest.approx(36.14, abs=0.01)  # MB per decode token


def test_short_contexts_gather_every_row():
    wl = _layout([1000, 3000], [1, 1], 64, 2048)
    assert bench.decode_bytes(wl)["kv"] == (1000 + 2048) * 1152


def test_prefill_16k_indexer_flops():
    wl = _layout([16384], [16384], 64, 2048)
    pairs = 16384 * 16385 // 2  # causal (query, key) pairs, own position included
    assert bench.indexer_causal_flops(wl) == 2 * 32 * 128 * pairs
    assert bench.indexer_causal_flops(wl) / 1e12 == pytest.approx(1.0996, abs=1e-4)


def test_kernels_per_layer_call():
    # decode 8 x 32K: histogram zeroing, indexer, the fused tail (selection,
    # attention, merge)
    assert bench.launches_per_layer(_layout([32768] * 8, [1] * 8, 64, 2048)) == 3
    # decode 4 x 128K: zeroing, indexer, top-k filter + emit, attention, merge of the slices
    assert bench.launches_per_layer(_layout([131072] * 4, [1] * 4, 64, 2048)) == 6
    # decode 14 x 32K: zeroing, indexer, the tail's selection, attention, merge
    assert bench.launches_per_layer(_layout([32768] * 14, [1] * 14, 64, 2048)) == 5
    # 32 ragged decode rows: zeroing, indexer, filter + emit, attention, merge of the slices
    assert bench.launches_per_layer(_layout([40000] * 32, [1] * 32, 64, 2048)) == 6
    # more than 64 heads: no fused tail
    assert bench.launches_per_layer(_layout([131072] * 4, [1] * 4, 128, 2048)) == 6
    # prefill 16K: indexer, one top-k kernel, attention
    assert bench.launches_per_layer(_layout([16384], [16384], 64, 2048)) == 3


def test_device_glue_matches_the_chaining_definition():
    """The bench's glue between stacked ragged layers (torch ops, run here on
    the CPU) against the workload's host definition of the chained query."""
    import torch
    g = np.random.Generator(np.random.PCG64(11))
    out = g.standard_normal((32, 64, 512)).astype(np.float32) * 0.3
    proj = synth.glue_projection(4)
    want = synth.bf16_to_f32(synth.chain_query(out, proj))
    q = torch.empty(32, 64, synth.D, dtype=torch.bfloat16)
    bench.glue_step(torch.from_numpy(out),
                    torch.from_numpy(proj.view(np.int16)).view(torch.bfloat16), q)
    got = q.float().numpy()
    assert got.shape == want.shape
    # fp32 sums in another order may round a few results to the neighbouring
    # bf16 value (or, for results that cancel to near zero, differ by ~1e-6 of
    # the unit-scale entries)
    close = np.abs(got - want) <= 2.0 ** -7 * np.abs(want) + 1e-4
    assert close.all()
    assert (got == want).mean() > 0.99


def test_prefill_oracle_sample_and_extrapolation():
    rows = bench.prefill_sample_rows(16384)
    assert rows.size == 512 and np.unique(rows).size == 512
    assert set(range(64)) | set(range(2040, 2057)) <= set(rows.tolist())
    assert np.array_equal(rows, bench.prefill_sample_rows(16384))  # seeded
    # on a small prefill: the extrapolation weights rows by their work, so a
    # sample of every row extrapolates to its own time
    wl = synth.prefill(200, 4, 32, seed=9)
    full = bench.prefill_oracle(wl, total=200)
    assert full["extrapolated_full_s"] == pytest.approx(full["per_row_ms"] * 200 / 1e3)
    part = bench.prefill_oracle(wl, total=40)
    assert part["kind"] == "oracle" and "EXTRAPOLATED" in part["sample"]
    assert part["value"] > 0


def test_profiled_traffic_follows_the_source_hashes(tmp_path):
    """The roofline's DRAM traffic comes from the committed ncu record only
    while the kernel's sources still hash to the prefixes recorded with it."""
    import hashlib
    import json
    import os
    rec = json.load(open(os.path.join(os.path.dirname(bench.__file__), "profiles",
                                      "indexer_score_b4_128k_traffic.json")))
    assert rec["traffic_bytes"] == rec["dram_bytes_read"] + rec["dram_bytes_write"]
    # the record is close to the launch's algorithmic bytes (no re-reads)
    assert 1.0 <= rec["traffic_bytes"] / rec["algorithmic_bytes"] < 1.01
    csrc = os.path.join(os.path.dirname(bench.__file__), "dsa_lightning_indexer_b200", "csrc")
    for name in rec["source_sha256_prefix"]:
        assert os.path.exists(os.path.join(csrc, name)), name
    good = dict(rec)
    good["source_sha256_prefix"] = {
        n: hashlib.sha256(open(os.path.join(csrc, n), "rb").read()).hexdigest()[:16]
        for n in rec["source_sha256_prefix"]}
    p = tmp_path / "good.json"
    p.write_text(json.dumps(good))
    assert bench.profiled_traffic(str(p)) == rec["traffic_bytes"]
    stale = dict(good)
    stale["source_sha256_prefix"] = {n: "0" * 16 for n in good["source_sha256_prefix"]}
    p2 = tmp_path / "stale.json"
    p2.write_text(json.dumps(stale))
    assert bench.profiled_traffic(str(p2)) is None
    assert bench.profiled_traffic(str(tmp_path / "missing.json")) is None


def test_prefill_16k_attention_useful_flops():
    wl = _layout([16384], [16384], 64, 2048)
    # rows p < 2048 select p + 1 keys, the rest 2048
    keys = 2048 * 2049 // 2 + (16384 - 2048) * 2048
    assert keys == 31458304
    assert bench.attention_useful_flops(wl) == 2 * 64 * (576 + 512) * keys
    assert bench.attention_useful_flops(wl) / 1e12 == pytest.approx(4.381, abs=1e-3)
