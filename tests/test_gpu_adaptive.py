"""GPU parity of idx_adaptive_topk (cutoff-margin adaptive budget) against the oracle.

The margin sigma, the quantile and the trigger are decisions taken from
floating point, so the exact checks apply the oracle's rule to the GPU's own
fp32 scores (exported by idx_debug_scores): sigma must match bit for bit, and
the trigger flags and index lists exactly.  End to end against the oracle's
double scores, index recall must reach 0.999; sigma may differ in the last
bits there, which can move rows lying exactly at tau.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle as O
from oracle import adaptive as A
from sparse_attention_indexer_05_b200 import _native as N
from sparse_attention_indexer_05_b200 import workloads as W
from tests._util import recall, to_dev

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def idx():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_indexer_05_b200 as m
    return m


def _run(idx, P, k, rho, q):
    dev = (to_dev(P.q), to_dev(P.k), to_dev(P.w), to_dev(P.cu_seqlens))
    ws = torch.empty(idx.adaptive_workspace_size(P.T, P.q.shape[1], P.q.shape[2], k, rho, len(P.cu_seqlens) - 1,
                                                 dev[0].dtype), dtype=torch.uint8, device="cuda")
    i, s, sg, tr = idx.adaptive_topk(*dev, k, rho, q, workspace=ws)
    assert idx.device_status(ws) == "IDX_OK"
    return dev, i.cpu().numpy(), s.cpu().numpy(), sg.cpu().numpy(), tr.cpu().numpy().astype(bool)


def _gpu_rows(idx, P, dev, k):
    """The GPU's fp32 scores of every row over its own prefix."""
    rows = torch.arange(P.T, dtype=torch.int32)
    full = idx.debug_scores(0, *dev, k, rows).cpu().numpy()
    out = []
    for b in range(len(P.cu_seqlens) - 1):
        for t in range(int(P.cu_seqlens[b + 1] - P.cu_seqlens[b])):
            out.append(full[P.cu_seqlens[b] + t, :t + 1].astype(np.float32))
    return out


def _exact_against_gpu_scores(idx, P, k, rho, q):
    dev, gi, gs, gsig, gtr = _run(idx, P, k, rho, q)
    rows = _gpu_rows(idx, P, dev, k)
    wi, wsig, wtr, tau = A.adaptive_select(rows, k, rho, q)
    assert np.array_equal(gsig.view(np.uint32)[~np.isnan(gsig)], wsig.view(np.uint32)[~np.isnan(wsig)])
    assert np.array_equal(np.isnan(gsig), np.isnan(wsig))
    assert np.array_equal(gtr, wtr)
    assert np.array_equal(gi, wi)
    # scores of the kept positions are the exported ones; -inf on padding
    for t, r in enumerate(rows):
        m = gi[t] >= 0
        assert np.array_equal(gs[t][m].view(np.uint32), r[gi[t][m]].view(np.uint32)), t
        assert np.all(np.isneginf(gs[t][~m])), t
    return gi, gsig, gtr


def test_adaptive_packed_bit_exact_and_recall(idx):
    P = W.prefill([3000, 1777, 129, 40, 64], H=64, d=128, topk=128, rho=0.95, planted=0.01, seed=3)
    k, rho, q = 128, 2, 0.4
    gi, gsig, gtr = _exact_against_gpu_scores(idx, P, k, rho, q)
    n_def = int((~np.isnan(gsig)).sum())
    assert gtr.sum() >= int(np.ceil(q * n_def))           # ties at tau may add rows
    wi, wsig, wtr, _ = A.adaptive_topk(P.q, P.k, P.w, P.cu_seqlens, k, rho, q)
    assert recall(gi, wi) >= 0.999
    assert np.mean(gtr == wtr) >= 0.99


def test_adaptive_exact_integer_inputs(idx):
    # exact arithmetic: the GPU's fp32 scores equal the oracle's double ones,
    # so everything must match the end-to-end oracle bit for bit (many ties)
    P = W.exact_ints([700, 333, 5], H=64, d=128, topk=32, seed=5)
    for rho, q in ((2, 0.4), (3, 0.0), (2, 1.0), (4, 0.25)):
        _, gi, _, gsig, gtr = _run(idx, P, 32, rho, q)
        wi, wsig, wtr, _ = A.adaptive_topk(P.q, P.k, P.w, P.cu_seqlens, 32, rho, q)
        assert np.array_equal(np.isnan(gsig), np.isnan(wsig))
        assert np.array_equal(gsig[~np.isnan(gsig)], wsig[~np.isnan(wsig)]), (rho, q)
        assert np.array_equal(gtr, wtr), (rho, q)
        assert np.array_equal(gi, wi), (rho, q)


def test_adaptive_fp32_cuda_core_path(idx):
    P = W.small_fp32(L=2048, H=4, d=64, topk=64, seed=2)
    _exact_against_gpu_scores(idx, P, 64, 2, 0.4)


def test_adaptive_short_rows_and_argument_checks(idx):
    # every row shorter than k + 1: sigma undefined everywhere, nothing triggers
    P = W.prefill([50, 20], H=64, d=128, topk=64, seed=6)
    _, gi, _, gsig, gtr = _run(idx, P, 64, 2, 0.4)
    assert np.isnan(gsig).all() and not gtr.any()
    assert np.array_equal(gi, O.dense_topk(P.q, P.k, P.w, P.cu_seqlens, 128))
    dev = (to_dev(P.q), to_dev(P.k), to_dev(P.w), to_dev(P.cu_seqlens))
    with pytest.raises(ValueError):
        idx.adaptive_topk(*dev, 64, 1, 0.4)
    with pytest.raises(N.IdxError) as e:   # the library rejects q outside [0, 1] before any launch
        idx.adaptive_topk(*dev, 64, 2, 1.5)
    assert e.value.code == 1


def test_adaptive_full_size_131072(idx):
    # the headline request: 131072 tokens, k = 2048, rho = 2, q = 0.4.
    # Properties at any size: trigger = (sigma <= the oracle's quantile of the
    # GPU sigmas); triggered rows equal the dense top-(rho k), the others the
    # dense top-k padded (both from the dense entry point), on sampled rows;
    # sigma of sampled rows from the dense top-(rho k) scores.
    P = W.cfg_long_single(seed=0)
    k, rho, q = 2048, 2, 0.4
    dev, gi, gs, gsig, gtr = _run(idx, P, k, rho, q)
    tau, r = A.quantile_threshold(gsig, q)
    assert np.array_equal(gtr, ~np.isnan(gsig) & (gsig <= tau))
    assert np.isnan(gsig[:k]).all() and not np.isnan(gsig[k:]).any()
    rng = np.random.default_rng(9)
    rows = np.unique(np.r_[0, k - 1, k, k + 1, P.T - 1, rng.integers(0, P.T, 40)])
    d2, d2s = idx.dense_topk(*dev, rho * k, return_scores=True)
    d1 = idx.dense_topk(*dev, k)
    d2, d2s, d1 = d2.cpu().numpy(), d2s.cpu().numpy(), d1.cpu().numpy()
    for t in rows:
        if gtr[t]:
            assert np.array_equal(gi[t], d2[t]), t
        else:
            want = np.full(rho * k, -1, np.int32)
            want[:k] = d1[t]
            assert np.array_equal(gi[t], want), t
        m = d2[t] >= 0
        s = A.cutoff_margin(d2s[t][m], k)
        assert (np.isnan(s) and np.isnan(gsig[t])) or s.view(np.uint32) == gsig[t].view(np.uint32), t
    # recall of sampled rows against the oracle (double scores)
    sample = rows[rows >= k][:12]
    want = O.dense_topk(P.q, P.k, P.w, P.cu_seqlens, rho * k, rows=sample)
    for j, t in enumerate(sample):
        if gtr[t]:
            assert recall(gi[t][None], want[j][None]) >= 0.999, t
