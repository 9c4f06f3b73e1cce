"""The C-ABI library: it loads, exports every symbol include/dsa.h declares,
and rejects invalid arguments on the host before any launch (no GPU needed)."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

from dsa_lightning_indexer_b200 import binding as bd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa.h")
FAKE = 0x10000  # aligned, never dereferenced: every case below fails validation first


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"DSA_API\s+[\w\s\*]+?\b(dsa_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    assert declared_symbols() == sorted([
        "dsa_workspace_size", "dsa_indexer_score", "dsa_topk", "dsa_sparse_attn",
        "dsa_layer_forward", "dsa_check_device_status", "dsa_status_string",
        "dsa_sparse_attn_noalloc", "dsa_indexer_project_workspace_size",
        "dsa_indexer_project", "dsa_masked_attn"])


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(bd.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert set(declared_symbols()) == set(bd.SIGNATURES)


def test_status_strings():
    names = ["DSA_OK", "DSA_ERR_INVALID_ARG", "DSA_ERR_UNSUPPORTED", "DSA_ERR_WORKSPACE",
             "DSA_ERR_CUDA", "DSA_ERR_DEVICE_TIMEOUT", "DSA_ERR_NOT_SM100", "DSA_ERR_BAD_INDEX"]
    assert [bd.status_string(i) for i in range(8)] == names
    assert bd.status_string(99) == "DSA_ERR_UNKNOWN"


class FakeBatch:
    """A dsa_batch whose device pointers are placeholders (never dereferenced)."""

    def __init__(self, q_off, kv_off, lens, null_device=False):
        self.hq = np.ascontiguousarray(q_off, np.int32)
        self.hk = np.ascontiguousarray(kv_off, np.int64)
        self.hl = np.ascontiguousarray(lens, np.int32)
        d = None if null_device else FAKE
        self.c = bd._CBatch(len(lens), int(self.hq[-1]), d, d, d, self.hq.ctypes.data,
                            self.hk.ctypes.data, self.hl.ctypes.data, 0, 0, None, None, 0)

    @property
    def ref(self):
        return ctypes.byref(self.c)


def _topk(b, top_k=16, scores=FAKE, ld=64, idx=FAKE, ws=FAKE, ws_bytes=1 << 20, flags=0):
    return bd.lib.dsa_topk(b.ref, scores, ld, top_k, idx, ws, ws_bytes, flags, None)


def _attn(b, H=16, top_k=16, q=FAKE, kv=FAKE, idx=FAKE, scale=0.04, out=FAKE, lse=None,
          ws=FAKE, ws_bytes=1 << 30):
    return bd.lib.dsa_sparse_attn(b.ref, q, H, kv, idx, top_k, scale, out, lse, ws, ws_bytes,
                                  None)


def test_batch_validation():
    good = FakeBatch([0, 1], [0, 64], [64])
    assert bd.lib.dsa_workspace_size(good.ref, 16, 16, 0) > 0
    bad = [
        FakeBatch([0, 1], [0, 64], [64], null_device=True),  # null device arrays
        FakeBatch([1, 1], [0, 64], [64]),                    # q_offsets[0] != 0
        FakeBatch([0, 5], [0, 64], [4]),                     # more queries than context
        FakeBatch([0, 1], [0, 64], [65]),                    # context beyond the cache rows
        FakeBatch([0, 1, 0], [0, 8, 16], [8, 8]),            # decreasing offsets
        FakeBatch([0, 1], [0, -3], [1]),                     # negative capacity
    ]
    for b in bad:
        assert bd.lib.dsa_workspace_size(b.ref, 16, 16, 0) == 0
        assert _topk(b) == bd.ERR_INVALID_ARG
        assert _attn(b) == bd.ERR_INVALID_ARG
    assert bd.lib.dsa_topk(None, FAKE, 64, 16, FAKE, FAKE, 1 << 20, 0, None) == bd.ERR_INVALID_ARG


def test_shape_and_pointer_validation():
    b = FakeBatch([0, 1], [0, 64], [64])
    assert _topk(b, top_k=0) == bd.ERR_INVALID_ARG
    assert _topk(b, top_k=2049) == bd.ERR_UNSUPPORTED
    assert _topk(b, scores=None) == bd.ERR_INVALID_ARG
    assert _topk(b, idx=FAKE + 4) == bd.ERR_UNSUPPORTED        # misaligned
    assert _topk(b, ld=63) == bd.ERR_INVALID_ARG               # ld below the context
    assert _topk(b, ld=66) == bd.ERR_INVALID_ARG               # ld not a multiple of 4
    assert _topk(b, ws=None) == bd.ERR_WORKSPACE
    assert _topk(b, ws_bytes=100) == bd.ERR_WORKSPACE
    assert _attn(b, H=0) == bd.ERR_INVALID_ARG
    assert _attn(b, H=129) == bd.ERR_UNSUPPORTED
    assert _attn(b, scale=float("nan")) == bd.ERR_INVALID_ARG
    assert _attn(b, lse=FAKE + 8) == bd.ERR_UNSUPPORTED
    assert _attn(b, ws_bytes=16) == bd.ERR_WORKSPACE
    st = bd.lib.dsa_indexer_score(b.ref, FAKE, FAKE, FAKE, FAKE, 60, FAKE, 1 << 20, 0, None)
    assert st == bd.ERR_INVALID_ARG
    st = bd.lib.dsa_layer_forward(b.ref, FAKE, 16, FAKE, FAKE, FAKE, FAKE, 16, 0.04, FAKE,
                                  None, None, FAKE, 1 << 30, 0, None)
    assert st == bd.ERR_INVALID_ARG                             # idx is required


def test_empty_batch_is_a_no_op():
    b = FakeBatch([0], [0], [])
    assert _topk(b) == bd.OK
    assert _attn(b) == bd.OK
    b0 = FakeBatch([0, 0], [0, 8], [8])                         # one sequence, no queries
    assert _topk(b0) == bd.OK


def test_workspace_grows_with_the_problem():
    # One row of 4M positions needs its 16 MB of scores on top of the control
    # block; one row of 128K fits in far less.
    small = FakeBatch([0, 1], [0, 131072], [131072])
    big = FakeBatch([0, 1], [0, 1 << 22], [1 << 22])
    assert bd.lib.dsa_workspace_size(big.ref, 64, 2048, 0) > (1 << 22) * 4
    assert bd.lib.dsa_workspace_size(big.ref, 64, 2048, 0) > bd.lib.dsa_workspace_size(
        small.ref, 64, 2048, 0)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_a_b200_is_refused():
    b = FakeBatch([0, 1], [0, 64], [64])
    assert _topk(b) == bd.ERR_NOT_SM100


def test_flag_validation():
    b = FakeBatch([0, 1], [0, 64], [64])
    hist, stall = bd.FLAG_SCORE_HISTOGRAM, bd.FLAG_TEST_STALL

    def score(batch, flags):
        return bd.lib.dsa_indexer_score(batch.ref, FAKE, FAKE, FAKE, FAKE, 64, FAKE, 1 << 20,
                                        flags, None)

    def layer(flags):
        return bd.lib.dsa_layer_forward(b.ref, FAKE, 16, FAKE, FAKE, FAKE, FAKE, 16, 0.04, FAKE,
                                        None, FAKE, FAKE, 1 << 30, flags, None)
    assert score(b, 0x2) == bd.ERR_INVALID_ARG                 # reserved bit
    assert score(b, stall) == bd.ERR_INVALID_ARG               # a layer-only flag
    assert _topk(b, flags=0x4) == bd.ERR_INVALID_ARG
    assert _topk(b, flags=stall) == bd.ERR_INVALID_ARG
    assert layer(hist) == bd.ERR_INVALID_ARG                   # the layer builds it itself
    assert layer(0x10) == bd.ERR_INVALID_ARG
    # workspace checks come before the device check: too small for the histograms
    assert bd.lib.dsa_indexer_score(b.ref, FAKE, FAKE, FAKE, FAKE, 64, FAKE, 300, hist,
                                    None) == bd.ERR_WORKSPACE


def test_workspace_covers_the_standalone_histogram_region():
    # a decode batch long enough for the histogram-driven selection
    b = FakeBatch([0, 1, 2], [0, 40000, 60000], [40000, 20000])
    size = bd.lib.dsa_workspace_size(b.ref, 16, 2048, 0)
    hist_zero = 2 * (4096 + 2048 + 4) * 4
    assert size >= 256 + hist_zero
    st = bd.lib.dsa_topk(b.ref, FAKE, 40000, 2048, FAKE, FAKE, 256 + hist_zero,
                         bd.FLAG_SCORE_HISTOGRAM, None)
    assert st == bd.ERR_WORKSPACE                              # needs the lists too
