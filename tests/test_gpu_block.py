"""GPU parity of the block pre-filter mode of idx_pivot_topk.

For sampled members, every step is checked against the oracle:
  - the proxy's block scores (GPU, exported) match the oracle's scores of the
    proxy against the oracle's block mean keys, within tolerance;
  - the oracle's selection rule on those GPU block scores gives the blocks,
    and with the partial block the candidate layout of the GPU;
  - the member's re-scores over that candidate set match the oracle's, and
    re-selecting on them reproduces the GPU's output row exactly;
  - recall against the oracle's own block-mode rows is >= 0.999.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle as O
from sparse_attention_indexer_05_b200 import workloads as W
from tests._util import check_scores, recall, reselect, score_rows, to_dev

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
BN = 64


@pytest.fixture(scope="module")
def idx():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_indexer_05_b200 as m
    return m


def _block_keys(k, key0, nfull):
    return np.stack([O.block_mean(k, key0 + j * BN, BN) for j in range(nfull)]) if nfull else k[:0]


def _check_block_rows(idx, P, dev, got, rows, topk, g, c, ws):
    q, k, w, cu = dev
    cu_h = P.cu_seqlens
    want = O.pivot_topk(P.q, P.k, P.w, cu_h, topk, g, c, O.BLOCK, rows=rows, bn=BN)
    assert recall(got[rows], want) >= 0.999
    nb = c // BN
    base, first = 0, []
    for b in range(len(cu_h) - 1):
        first.append(base)
        base += (cu_h[b + 1] - cu_h[b] + g - 1) // g
    geo, plist = [], []
    for r in rows:
        b = int(np.searchsorted(cu_h, r, side="right") - 1)
        t = int(r - cu_h[b])
        n = int(cu_h[b + 1] - cu_h[b])
        lo = (t // g) * g
        hi = min(lo + g, n)
        geo.append((b, t, lo, hi))
        plist.append(first[b] + t // g)
    uniq, slot = np.unique(np.asarray(plist), return_inverse=True)
    bsc = idx.debug_scores(3, q, k, w, cu, topk, torch.from_numpy(uniq.astype(np.int32)), g=g, c=c,
                           workspace=ws).cpu().numpy()[slot]
    msc = idx.debug_scores(4, q, k, w, cu, topk, torch.from_numpy(rows.astype(np.int32)), g=g, c=c,
                           workspace=ws).cpu().numpy()
    kb_cache = {}
    jobs = []
    for (b, t, lo, hi) in geo:
        nfull = hi // BN
        if (b, nfull) not in kb_cache:
            kb_cache[(b, nfull)] = _block_keys(P.k, int(cu_h[b]), nfull)
        qb, wb = O.group_proxy(P.q, P.w, int(cu_h[b] + lo), hi - lo)
        jobs.append((qb[None], kb_cache[(b, nfull)], wb[None], 0, 0, nfull))
    live = [j for j in jobs if j[5] > 0]
    scored = iter(score_rows(live))
    ora = [next(scored) if j[5] > 0 else None for j in jobs]
    for i, r in enumerate(rows):
        b, t, lo, hi = geo[i]
        nfull = hi // BN
        if nfull:
            check_scores(bsc[i, :nfull], ora[i])
        partial = hi % BN != 0
        kr = nb - (1 if partial else 0)
        blocks = reselect(bsc[i, :nfull], kr) if kr > 0 and nfull else np.full(max(kr, 0), -1)
        slots = np.full(nb, -1, np.int64)
        slots[:len(blocks)] = blocks
        cand = np.full(c, -1, np.int64)
        for j, blk in enumerate(slots):
            if blk >= 0:
                cand[j * BN:(j + 1) * BN] = blk * BN + np.arange(BN)
        if partial:
            part0 = (hi // BN) * BN
            tail = part0 + np.arange(BN)
            cand[(nb - 1) * BN:] = np.where(tail <= hi - 1, tail, -1)
        keep = (cand >= 0) & (cand <= t)
        ms = msc[i]
        # member re-scores of the kept candidates against the oracle
        ora_m = O.score_row(P.q, P.k, P.w, int(r), int(cu_h[b]), hi)
        check_scores(ms[keep], ora_m[cand[keep]])
        assert np.array_equal(reselect(ms[keep], topk, cand[keep].astype(np.int32)), got[r]), r


def test_block_small_packed(idx):
    topk, g, c = 128, 4, 512
    P = W.prefill([3000, 1777, 129, 40, 64], H=64, d=128, topk=topk, rho=0.95, planted=0.01, seed=3)
    dev = (to_dev(P.q), to_dev(P.k), to_dev(P.w), to_dev(P.cu_seqlens))
    ws = torch.empty(idx.pivot_workspace_size(P.T, 64, 128, topk, 5, g, c, "block"), dtype=torch.uint8,
                     device="cuda")
    out = idx.pivot_topk(*dev, topk, g, c, "block", workspace=ws)
    assert idx.device_status(ws) == "IDX_OK"
    got = out.cpu().numpy()
    want = O.pivot_topk(P.q, P.k, P.w, P.cu_seqlens, topk, g, c, O.BLOCK, bn=BN)
    assert recall(got, want) >= 0.999
    # ragged tails, the first rows, rows around block edges, the short requests
    rows = np.unique(np.r_[0, 1, 62, 63, 64, 65, 127, 2999, 3000, 3063, 4776, 4777, 4800, 4905, 4906,
                           4945, 4946, 5009, np.random.default_rng(1).integers(0, P.T, 24)])
    _check_block_rows(idx, P, dev, got, rows, topk, g, c, ws)


def test_block_g1_and_minimum_budget(idx):
    # g = 1 (each query its own proxy) and c = 64: one block, or just the partial one
    topk = 32
    P = W.prefill([700, 333], H=64, d=128, topk=topk, rho=0.95, planted=0.02, seed=4)
    dev = (to_dev(P.q), to_dev(P.k), to_dev(P.w), to_dev(P.cu_seqlens))
    for g, c in ((1, 64), (1, 256), (3, 64)):
        ws = torch.empty(idx.pivot_workspace_size(P.T, 64, 128, topk, 2, g, c, "block"), dtype=torch.uint8,
                         device="cuda")
        got = idx.pivot_topk(*dev, topk, g, c, "block", workspace=ws).cpu().numpy()
        assert idx.device_status(ws) == "IDX_OK"
        want = O.pivot_topk(P.q, P.k, P.w, P.cu_seqlens, topk, g, c, O.BLOCK, bn=BN)
        assert recall(got, want) >= 0.999, (g, c)
        rows = np.unique(np.r_[0, 63, 64, 699, 700, 763, 1032, np.random.default_rng(g + c).integers(0, P.T, 8)])
        _check_block_rows(idx, P, dev, got, rows, topk, g, c, ws)


def test_block_fp32_cuda_core_path(idx):
    P = W.small_fp32(L=2048, H=4, d=64, topk=64, seed=2)
    dev = (to_dev(P.q), to_dev(P.k), to_dev(P.w), to_dev(P.cu_seqlens))
    topk, g, c = 64, 2, 256
    ws = torch.empty(idx.pivot_workspace_size(P.T, 4, 64, topk, 1, g, c, "block", torch.float32),
                     dtype=torch.uint8, device="cuda")
    got = idx.pivot_topk(*dev, topk, g, c, "block", workspace=ws).cpu().numpy()
    assert idx.device_status(ws) == "IDX_OK"
    want = O.pivot_topk(P.q, P.k, P.w, P.cu_seqlens, topk, g, c, O.BLOCK, bn=BN)
    assert recall(got, want) >= 0.999


def test_block_argument_checks(idx):
    P = W.prefill([256], H=64, d=128, topk=64, seed=5)
    dev = (to_dev(P.q), to_dev(P.k), to_dev(P.w), to_dev(P.cu_seqlens))
    assert idx.pivot_workspace_size(256, 64, 128, 64, 1, 4, 100, "block") == 0   # not a multiple of 64
    assert idx.pivot_workspace_size(256, 64, 128, 128, 1, 4, 64, "block") == 0   # c < topk
    with pytest.raises(ValueError):
        idx.pivot_topk(*dev, 64, 4, 96, "block")


def test_block_full_size_65536_g4_c4096(idx):
    P = W.cfg_pivot_64k(seed=0)
    dev = (to_dev(P.q), to_dev(P.k), to_dev(P.w), to_dev(P.cu_seqlens))
    topk, g, c = 2048, 4, 4096
    ws = torch.empty(idx.pivot_workspace_size(P.T, 64, 128, topk, 1, g, c, "block"), dtype=torch.uint8,
                     device="cuda")
    got = idx.pivot_topk(*dev, topk, g, c, "block", workspace=ws).cpu().numpy()
    assert idx.device_status(ws) == "IDX_OK"
    rng = np.random.default_rng(7)
    rows = np.unique(np.r_[0, 2047, 4095, 4096, 65535, rng.integers(0, P.T, 6)])
    _check_block_rows(idx, P, dev, got, rows, topk, g, c, ws)
