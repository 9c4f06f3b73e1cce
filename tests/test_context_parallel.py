"""Context-parallel decode: the collectives of the merge as two gloo ranks on
the CPU against the one-process emulation, and (needs a B200) the whole step
as 2 and 4 emulated ranks on one GPU against the single-GPU layer and the
oracle."""
import datetime
import multiprocessing as mp
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from dsa_lightning_indexer_b200 import synth
from tests import parity


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _parts(seed=0, n=2, B=3, H=4):
    g = torch.Generator().manual_seed(seed)
    outs = [torch.randn(B, H, 512, generator=g) for _ in range(n)]
    lses = [torch.randn(B, H, generator=g) * 3 for _ in range(n)]
    lses[1][0, 1] = float("-inf")  # a head with no selected rows on rank 1
    return outs, lses


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import torch.distributed as dist
    from dsa_lightning_indexer_b200.context_parallel import DistComm
    from dsa_lightning_indexer_b200 import context_parallel as cp
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=60))
        outs, lses = _parts()
        comm = DistComm(dist)
        ((o, l),) = cp.lse_merge([outs[rank]], [lses[rank]], comm)
        (cat,) = comm.all_gather_cat([torch.full((2, 3), float(rank))], dim=1)
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, o.numpy(), l.numpy(), cat.numpy(), None))
    except Exception as e:  # reported to the parent instead of hanging it
        q.put((rank, None, None, None, repr(e)))


def test_merge_collectives_on_two_gloo_ranks():
    pytest.importorskip("torch.distributed")
    try:
        from dsa_lightning_indexer_b200 import context_parallel as cp
    except Exception as e:  # the binding needs the built library, not a GPU
        pytest.skip(repr(e))
    outs, lses = _parts()
    ((want_o, want_l), _) = cp.lse_merge(outs, lses, cp.LocalComm(2))
    # the definition: a softmax over the union is the lse-weighted average
    M = torch.maximum(lses[0], lses[1])
    w0, w1 = torch.exp(lses[0] - M), torch.exp(lses[1] - M)
    ref = (outs[0] * w0[..., None] + outs[1] * w1[..., None]) / (w0 + w1)[..., None]
    assert torch.allclose(want_o, ref, atol=1e-6)
    assert torch.allclose(want_l, M + torch.log(w0 + w1), atol=1e-6)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        got = sorted((q.get(timeout=180) for _ in range(2)), key=lambda x: x[0])
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    for rank, o, l, cat, err in got:
        assert err is None, err
        assert np.allclose(o, want_o.numpy(), atol=1e-6) and np.allclose(l, want_l.numpy(), atol=1e-6)
        assert np.array_equal(cat, np.concatenate([np.zeros((2, 3)), np.ones((2, 3))], axis=1))


@pytest.mark.gpu
@pytest.mark.parametrize("n_ranks", [2, 4])
def test_context_parallel_decode_emulated_ranks(n_ranks):
    from dsa_lightning_indexer_b200 import binding as bd
    from dsa_lightning_indexer_b200 import context_parallel as cp
    wl = synth.custom([40000, 9000, 1500, 70000], [1] * 4, 64, 2048, seed=220)
    dw = bd.DeviceWorkload(wl)
    lay_out, lay_lse, lay_idx = (t.cpu().numpy() for t in dw.forward())
    bd.check_device_status(dw.ws)
    shards = cp.make_shards(wl.ctx_lens, wl.kv_offsets, wl.q, wl.q_idx, wl.w, wl.k_idx, wl.kv,
                            wl.scale, n_ranks, ["cuda"] * n_ranks)
    res = cp.cp_decode(shards, cp.LocalComm(n_ranks), wl.top_k)
    for out, lse, idx in res:  # every rank holds the same result
        assert np.array_equal(idx.cpu().numpy(), lay_idx)  # the exact global selection
        o, l = out.cpu().numpy(), lse.cpu().numpy()
        parity.check_attention(o, l, lay_out, lay_lse.astype(np.float64))
    att_out, att_lse = oracle.sparse_attn(wl.q_offsets, wl.kv_offsets, wl.ctx_lens, wl.q, wl.kv,
                                          lay_idx, wl.scale)
    parity.check_attention(res[0][0].cpu().numpy(), res[0][1].cpu().numpy(), att_out, att_lse)
