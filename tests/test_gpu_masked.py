"""The mask-over-the-whole-cache route (dsa_masked_attn) against the oracle
and the gather route (needs a B200).

The pages describe llama.cpp applying the selection as a mask over the whole
cache (aiaulis.com paragraph 4; devotd.net section 2); this library gathers
the selected rows instead and keeps the mask route as a measured comparison.
Both must compute the same attention over the listed rows.
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


def _args(wl):
    return (wl.q_offsets, wl.kv_offsets, wl.ctx_lens)


CASES = {
    # decode rows of several lengths, 64 heads, the layer's own selection
    "decode_h64": lambda: synth.custom([20000, 9000, 3000, 50000], [1] * 4, 64, 2048, seed=190),
    # ragged queries, 16 heads, rows shorter than top_k, spare cache rows
    "ragged_h16": lambda: synth.custom([700, 1500, 90], [3, 1, 90], 16, 256, seed=191,
                                       caps=[760, 1500, 100]),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_masked_route_matches_oracle_and_gather(name):
    wl = CASES[name]()
    _, idx, _, _ = oracle.dsa_layer(*_args(wl), wl.q_idx, wl.w, wl.k_idx, wl.q, wl.kv, wl.top_k,
                                    wl.scale)
    if name == "ragged_h16":  # some unused slots in the middle of a row
        idx[0, 10:20] = -1
    ref_out, ref_lse = oracle.sparse_attn(*_args(wl), wl.q, wl.kv, idx, wl.scale)
    dw = bd.DeviceWorkload(wl)
    ws = bd.alloc_workspace(dw.batch, wl.H, wl.top_k, flags=bd.FLAG_MASKED_ROUTE)
    d_idx = torch.from_numpy(idx).cuda()
    out = torch.full((wl.Nq, wl.H, 512), float("nan"), device="cuda")
    lse = torch.full((wl.Nq, wl.H), float("nan"), device="cuda")
    bd.masked_attn(dw.batch, dw.q, dw.kv, d_idx, wl.top_k, wl.scale, out, lse, ws)
    bd.check_device_status(ws)
    m_out, m_lse = out.cpu().numpy(), lse.cpu().numpy()
    e = parity.check_attention(m_out, m_lse, ref_out, ref_lse)
    bd.sparse_attn(dw.batch, dw.q, dw.kv, d_idx, wl.top_k, wl.scale, out, lse, ws)
    bd.check_device_status(ws)
    parity.check_attention(m_out, m_lse, out.cpu().numpy(), lse.cpu().numpy().astype(np.float64))
    print(f"{name}: masked route max |out err| {e[0]:.2e}, lse {e[1]:.2e}")


def test_masked_route_skips_out_of_range_indices():
    wl = synth.custom([700, 900], [1, 2], 16, 64, seed=192, caps=[760, 950])
    _, idx, _, _ = oracle.dsa_layer(*_args(wl), wl.q_idx, wl.w, wl.k_idx, wl.q, wl.kv, wl.top_k,
                                    wl.scale)
    expect = idx.copy()
    idx[0, 3], expect[0, 3] = 705, -1        # past p, inside the allocated rows
    idx[2, 7], expect[2, 7] = -9, -1         # below -1
    ref_out, ref_lse = oracle.sparse_attn(*_args(wl), wl.q, wl.kv, expect, wl.scale)
    dw = bd.DeviceWorkload(wl)
    ws = bd.alloc_workspace(dw.batch, wl.H, wl.top_k, flags=bd.FLAG_MASKED_ROUTE)
    out = torch.full((wl.Nq, wl.H, 512), float("nan"), device="cuda")
    lse = torch.full((wl.Nq, wl.H), float("nan"), device="cuda")
    bd.masked_attn(dw.batch, dw.q, dw.kv, torch.from_numpy(idx).cuda(), wl.top_k, wl.scale, out,
                   lse, ws)
    with pytest.raises(bd.DsaError) as e:
        bd.check_device_status(ws)
    assert e.value.status == bd.ERR_BAD_INDEX
    parity.check_attention(out.cpu().numpy(), lse.cpu().numpy(), ref_out, ref_lse)
