"""The indexer's input step (dsa_indexer_project) against the oracle (needs a B200).

q_idx and the new tokens' indexer keys are bf16 roundings of fp32 sums.  The
oracle rounds its double sums the same way, so the two agree except where
the fp32 sum's own error (a small multiple of 2^-24 times the sum of the
products' magnitudes, i.e. absolute, not relative to the result) moves a
result across a rounding boundary: one bf16 unit of the result, plus 1e-5
of the row's rms for results that cancel to near zero; more than 99% must
agree bit for bit.  w (fp32) within 2e-5 of (|ref| + rms of the row).  Rows
of the key cache other than the new tokens' must be left untouched.
"""
import numpy as np
import pytest
import torch

import oracle
from dsa_lightning_indexer_b200 import synth

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from dsa_lightning_indexer_b200 import binding as bd


def _case(lens, nq, caps, d_model, d_q, seed):
    lens, nq, caps = (np.asarray(a, np.int64) for a in (lens, nq, caps))
    qo = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    ko = np.concatenate([[0], np.cumsum(caps)]).astype(np.int64)
    T, rows = int(qo[-1]), int(ko[-1])
    g = np.random.Generator(np.random.PCG64(seed))

    def bf(shape, std):
        return synth.bf16_bits((g.standard_normal(shape) * std).astype(np.float32))
    return dict(qo=qo, ko=ko, cl=lens.astype(np.int32), x=bf((T, d_model), 1.0),
                c_q=bf((T, d_q), 1.0), w_q_b=bf((4096, d_q), d_q ** -0.5),
                w_k=bf((128, d_model), d_model ** -0.5), w_proj=bf((32, d_model), d_model ** -0.5),
                k_idx=bf((rows, 128), 1.0))


def _ulp_diff(a_bits, b_bits):
    """Distance in bf16 units in the last place (same-sign finite values)."""
    a = a_bits.astype(np.int32)
    b = b_bits.astype(np.int32)
    ka = np.where(a & 0x8000, 0x8000 - (a & 0x7FFF), 0x8000 + a)
    kb = np.where(b & 0x8000, 0x8000 - (b & 0x7FFF), 0x8000 + b)
    return np.abs(ka - kb)


CASES = {
    # decode: 4 new tokens at the assumed model widths, caches with spare rows
    "decode_4tok": lambda: _case([3000, 17, 1, 900], [1, 1, 1, 1], [3100, 40, 8, 900], 7168, 1536,
                                 180),
    # prefill-like: 1000 new tokens over three sequences, several token tiles
    "prefill_1000tok": lambda: _case([600, 300, 300], [600, 250, 150], [600, 320, 300], 512, 256,
                                     181),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_indexer_project_matches_oracle(name):
    c = CASES[name]()
    want_q, want_k, want_w = oracle.indexer_project(c["qo"], c["ko"], c["cl"], c["x"], c["c_q"],
                                                    c["w_q_b"], c["w_k"], c["w_proj"], c["k_idx"])
    b = bd.Batch(c["qo"], c["ko"], c["cl"])
    dev = {k: bd.bf16_tensor(c[k]) for k in ("x", "c_q", "w_q_b", "w_k", "w_proj", "k_idx")}
    T = int(c["qo"][-1])
    q_idx = torch.full((T, 32, 128), -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    w = torch.full((T, 32), float("nan"), device="cuda")
    ws = bd.indexer_project_workspace(b, c["x"].shape[1], c["c_q"].shape[1])
    for _ in range(2):  # twice on one workspace: the split-K tickets start clean each call
        bd.indexer_project(b, dev["x"], dev["c_q"], dev["w_q_b"], dev["w_k"], dev["w_proj"],
                           q_idx, dev["k_idx"], w, ws)
    bd.check_device_status(ws)
    got_q = q_idx.view(torch.int16).cpu().numpy().view(np.uint16)
    got_k = dev["k_idx"].view(torch.int16).cpu().numpy().view(np.uint16)
    got_w = w.cpu().numpy()
    dq = _ulp_diff(got_q, want_q)
    dk = _ulp_diff(got_k, want_k)
    assert (dq == 0).mean() > 0.99 and (dk == 0).mean() > 0.99
    for got, want in ((got_q.reshape(T, -1), want_q.reshape(T, -1)), (got_k, want_k)):
        g32, w32 = synth.bf16_to_f32(got).astype(np.float64), synth.bf16_to_f32(want).astype(
            np.float64)
        rms = np.sqrt((w32 ** 2).mean(axis=1, keepdims=True))
        bound = 2.0 ** -7 * np.abs(w32) + 1e-5 * rms
        assert (np.abs(g32 - w32) <= bound).all(), float((np.abs(g32 - w32) / bound).max())
    new_rows = set()
    for bi in range(len(c["cl"])):
        nq = int(c["qo"][bi + 1] - c["qo"][bi])
        for j in range(nq):
            new_rows.add(int(c["ko"][bi] + c["cl"][bi] - nq + j))
    others = np.array(sorted(set(range(got_k.shape[0])) - new_rows))
    assert np.array_equal(got_k[others], c["k_idx"][others])      # untouched
    ref = want_w.astype(np.float64)
    scale = np.abs(ref) + np.sqrt((ref ** 2).mean(axis=1, keepdims=True))
    assert (np.abs(got_w - ref) <= 2e-5 * scale).all()
    print(f"{name}: bf16 outputs off by one unit in the last place: q_idx "
          f"{(dq > 0).mean():.2e}, k {(dk[sorted(new_rows)] > 0).mean():.2e}")
