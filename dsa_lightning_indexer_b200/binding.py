"""Thin Python binding of the C ABI in ``include/dsa.h`` (ctypes).

Argument marshalling only: every step of the layer runs in the CUDA kernels of
``libdsa_b200.so``.  Tensors are torch CUDA tensors (bf16 data may be given as
``torch.bfloat16`` or as its ``int16``/``uint16`` bit patterns); the current
torch stream is passed as the CUDA stream.  A non-OK status raises
``DsaError``.  There is no fallback: if the shared library cannot be loaded,
importing this module fails.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

from . import build as _build

_P = ctypes.c_void_p


class DsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {status_string(self.status)} ({self.status})")


# status codes (dsa_status)
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_DEVICE_TIMEOUT, \
    ERR_NOT_SM100, ERR_BAD_INDEX = range(8)

# flags
FLAG_SCORE_HISTOGRAM = 0x1
FLAG_TEST_STALL = 0x80000000
FLAG_MASKED_ROUTE = 0x2

INDEX_HEADS, INDEX_DIM, LATENT_DIM, VALUE_DIM, MAX_TOPK, MAX_HEADS = 32, 128, 576, 512, 2048, 128
CONTROL_BYTES = 256

# Every symbol the header declares, with its ctypes signature.
SIGNATURES = {
    "dsa_workspace_size": (ctypes.c_size_t, [_P, ctypes.c_int, ctypes.c_int, ctypes.c_uint32]),
    "dsa_indexer_score": (ctypes.c_int, [_P, _P, _P, _P, _P, ctypes.c_int64, _P, ctypes.c_size_t,
                                         ctypes.c_uint32, _P]),
    "dsa_topk": (ctypes.c_int, [_P, _P, ctypes.c_int64, ctypes.c_int, _P, _P, ctypes.c_size_t,
                                ctypes.c_uint32, _P]),
    "dsa_sparse_attn": (ctypes.c_int, [_P, _P, ctypes.c_int, _P, _P, ctypes.c_int,
                                       ctypes.c_float, _P, _P, _P, ctypes.c_size_t, _P]),
    "dsa_layer_forward": (ctypes.c_int, [_P, _P, ctypes.c_int, _P, _P, _P, _P, ctypes.c_int,
                                         ctypes.c_float, _P, _P, _P, _P, ctypes.c_size_t,
                                         ctypes.c_uint32, _P]),
    "dsa_masked_attn": (ctypes.c_int, [_P, _P, ctypes.c_int, _P, _P, ctypes.c_int,
                                       ctypes.c_float, _P, _P, _P, ctypes.c_size_t, _P]),
    "dsa_sparse_attn_noalloc": (ctypes.c_int, [_P, _P, ctypes.c_int, _P, _P, ctypes.c_int,
                                               ctypes.c_float, _P, _P, _P]),
    "dsa_indexer_project_workspace_size": (ctypes.c_size_t, [_P, ctypes.c_int64,
                                                             ctypes.c_int64]),
    "dsa_indexer_project": (ctypes.c_int, [_P, _P, ctypes.c_int64, _P, ctypes.c_int64, _P, _P,
                                           _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "dsa_check_device_status": (ctypes.c_int, [_P, ctypes.c_size_t, _P]),
    "dsa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
}


def _load():
    path = _build.build()  # no-op when the in-tree library is current
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()
LIB_PATH = _build.LIB


def status_string(status: int) -> str:
    return lib.dsa_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != OK:
        raise DsaError(status, where)


class _CBatch(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Nq", ctypes.c_int32),
                ("q_offsets", _P), ("kv_offsets", _P), ("ctx_lens", _P),
                ("h_q_offsets", _P), ("h_kv_offsets", _P), ("h_ctx_lens", _P),
                ("page_size", ctypes.c_int32), ("max_blocks", ctypes.c_int32),
                ("block_table", _P), ("h_block_table", _P), ("cache_rows", ctypes.c_int64)]


class Batch:
    """Sequence layout of one call: device arrays plus the host mirrors.

    Contiguous caches: kv_offsets [B+1].  Paged caches: give page_size (a
    power of two >= 64), block_table [B, max_blocks] int32 page numbers and
    cache_rows; kv_offsets may then be None."""

    def __init__(self, q_offsets, kv_offsets, ctx_lens, device="cuda", page_size=0,
                 block_table=None, cache_rows=0):
        self.h_q_offsets = np.ascontiguousarray(q_offsets, dtype=np.int32)
        self.h_kv_offsets = (None if kv_offsets is None
                             else np.ascontiguousarray(kv_offsets, dtype=np.int64))
        self.h_ctx_lens = np.ascontiguousarray(ctx_lens, dtype=np.int32)
        self.h_block_table = (None if block_table is None
                              else np.ascontiguousarray(block_table, dtype=np.int32))
        self.B = int(self.h_ctx_lens.shape[0])
        self.Nq = int(self.h_q_offsets[-1]) if self.h_q_offsets.size else 0
        to_dev = (lambda a: None if a is None or device is None
                  else torch.from_numpy(a).to(device))
        self.q_offsets = to_dev(self.h_q_offsets)
        self.kv_offsets = to_dev(self.h_kv_offsets)
        self.ctx_lens = to_dev(self.h_ctx_lens)
        self.block_table = to_dev(self.h_block_table)
        dp = (lambda t: t.data_ptr() if t is not None else None)
        hp = (lambda a: a.ctypes.data if a is not None else None)
        max_blocks = int(self.h_block_table.shape[1]) if self.h_block_table is not None else 0
        self.c = _CBatch(self.B, self.Nq, dp(self.q_offsets), dp(self.kv_offsets),
                         dp(self.ctx_lens), hp(self.h_q_offsets), hp(self.h_kv_offsets),
                         hp(self.h_ctx_lens), int(page_size), max_blocks,
                         dp(self.block_table), hp(self.h_block_table), int(cache_rows))

    @property
    def ref(self):
        return ctypes.byref(self.c)

    @property
    def max_len(self) -> int:
        return int(self.h_ctx_lens.max()) if self.B else 0

    @classmethod
    def from_workload(cls, wl, device="cuda"):
        pg = getattr(wl, "paged", None)
        if pg is not None:
            return cls(wl.q_offsets, None, wl.ctx_lens, device, page_size=pg.page_size,
                       block_table=pg.block_table, cache_rows=pg.cache_rows)
        return cls(wl.q_offsets, wl.kv_offsets, wl.ctx_lens, device)


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch tensor")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _bf16(t):
    if t.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
        raise TypeError(f"expected bf16 data (bfloat16 or 16-bit bit patterns), got {t.dtype}")
    return _ptr(t)


def _f32(t):
    if t is not None and t.dtype != torch.float32:
        raise TypeError(f"expected float32, got {t.dtype}")
    return _ptr(t)


def _i32(t):
    if t.dtype != torch.int32:
        raise TypeError(f"expected int32, got {t.dtype}")
    return _ptr(t)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def workspace_size(batch: Batch, H: int, top_k: int, flags: int = 0) -> int:
    return int(lib.dsa_workspace_size(batch.ref, int(H), int(top_k), int(flags)))


def alloc_workspace(batch: Batch, H: int, top_k: int, device="cuda", flags=0) -> torch.Tensor:
    """A zero-filled workspace large enough for every call on this batch
    (with FLAG_MASKED_ROUTE, for dsa_masked_attn too)."""
    n = workspace_size(batch, H, top_k, flags)
    if n == 0:
        raise DsaError(ERR_INVALID_ARG, "dsa_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def indexer_score(batch, q_idx, w, k_idx, scores, ld, ws, stream=None, flags=0):
    _check(lib.dsa_indexer_score(batch.ref, _bf16(q_idx), _f32(w), _bf16(k_idx), _f32(scores),
                                 int(ld), _ptr(ws), ws.numel(), int(flags), _stream(stream)),
           "dsa_indexer_score")


def topk(batch, scores, ld, top_k, idx, ws, stream=None, flags=0):
    _check(lib.dsa_topk(batch.ref, _f32(scores), int(ld), int(top_k), _i32(idx), _ptr(ws),
                        ws.numel(), int(flags), _stream(stream)), "dsa_topk")


def sparse_attn(batch, q, kv, idx, top_k, scale, out, lse, ws, stream=None):
    H = int(q.shape[1])
    _check(lib.dsa_sparse_attn(batch.ref, _bf16(q), H, _bf16(kv), _i32(idx), int(top_k),
                               float(scale), _f32(out), _f32(lse), _ptr(ws), ws.numel(),
                               _stream(stream)), "dsa_sparse_attn")


def masked_attn(batch, q, kv, idx, top_k, scale, out, lse, ws, stream=None):
    """Attention over the listed rows computed as a mask over the whole cache."""
    H = int(q.shape[1])
    _check(lib.dsa_masked_attn(batch.ref, _bf16(q), H, _bf16(kv), _i32(idx), int(top_k),
                               float(scale), _f32(out), _f32(lse), _ptr(ws), ws.numel(),
                               _stream(stream)), "dsa_masked_attn")


def sparse_attn_noalloc(batch, q, kv, idx, top_k, scale, out, lse, stream=None):
    """dsa_sparse_attn without a workspace (scratch in a static device array)."""
    H = int(q.shape[1])
    _check(lib.dsa_sparse_attn_noalloc(batch.ref, _bf16(q), H, _bf16(kv), _i32(idx), int(top_k),
                                       float(scale), _f32(out), _f32(lse), _stream(stream)),
           "dsa_sparse_attn_noalloc")


def layer_forward(batch, q, q_idx, w, k_idx, kv, top_k, scale, out, lse, idx, ws, stream=None,
                  flags=0):
    H = int(q.shape[1])
    _check(lib.dsa_layer_forward(batch.ref, _bf16(q), H, _bf16(q_idx), _f32(w), _bf16(k_idx),
                                 _bf16(kv), int(top_k), float(scale), _f32(out), _f32(lse),
                                 _i32(idx), _ptr(ws), ws.numel(), int(flags), _stream(stream)),
           "dsa_layer_forward")


def indexer_project_workspace(batch, d_model, d_q, device="cuda"):
    """A zero-filled workspace for dsa_indexer_project on this batch."""
    n = int(lib.dsa_indexer_project_workspace_size(batch.ref, int(d_model), int(d_q)))
    if n == 0:
        raise DsaError(ERR_INVALID_ARG, "dsa_indexer_project_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def indexer_project(batch, x, c_q, w_q_b, w_k, w_proj, q_idx, k_idx, w, ws, stream=None):
    """The indexer's input step: q_idx, w out; the new tokens' k rows into k_idx."""
    _check(lib.dsa_indexer_project(batch.ref, _bf16(x), int(x.shape[1]), _bf16(c_q),
                                   int(c_q.shape[1]), _bf16(w_q_b), _bf16(w_k), _bf16(w_proj),
                                   _bf16(q_idx), _bf16(k_idx), _f32(w), _ptr(ws), ws.numel(),
                                   _stream(stream)), "dsa_indexer_project")


def check_device_status(ws, stream=None):
    _check(lib.dsa_check_device_status(_ptr(ws), ws.numel(), _stream(stream)),
           "dsa_check_device_status")


# ---------------------------------------------------------------- helpers --

def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    """Host bf16 bit patterns (uint16) -> torch.bfloat16 tensor on `device`."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to(device).view(torch.bfloat16)


class DeviceWorkload:
    """A synthetic workload resident on the GPU, ready for the C ABI."""

    def __init__(self, wl, device="cuda"):
        self.wl = wl
        self.batch = Batch.from_workload(wl, device)
        pg = getattr(wl, "paged", None)
        self.q_idx = bf16_tensor(wl.q_idx, device)
        self.w = torch.from_numpy(wl.w).to(device)
        self.k_idx = bf16_tensor(wl.k_idx if pg is None else pg.k_idx, device)
        self.q = bf16_tensor(wl.q, device)
        self.kv = bf16_tensor(wl.kv if pg is None else pg.kv, device)
        self.top_k = wl.top_k
        self.scale = wl.scale
        self.H = wl.H
        self.ws = alloc_workspace(self.batch, self.H, self.top_k, device)

    def new_outputs(self):
        dev = self.q.device
        out = torch.empty(self.batch.Nq, self.H, VALUE_DIM, dtype=torch.float32, device=dev)
        lse = torch.empty(self.batch.Nq, self.H, dtype=torch.float32, device=dev)
        idx = torch.empty(self.batch.Nq, self.top_k, dtype=torch.int32, device=dev)
        return out, lse, idx

    def forward(self, out=None, lse=None, idx=None, stream=None, flags=0):
        if out is None:
            out, lse, idx = self.new_outputs()
        layer_forward(self.batch, self.q, self.q_idx, self.w, self.k_idx, self.kv,
                      self.top_k, self.scale, out, lse, idx, self.ws, stream, flags)
        return out, lse, idx


def loaded_library_path() -> str:
    return os.path.realpath(LIB_PATH)
