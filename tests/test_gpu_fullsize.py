"""GPU parity at the full workload sizes, on sampled rows the oracle computes
one by one, in the same launch configuration bench.py times:

  * dense over one 16384-token request is in test_gpu_parity.py;
  * PIVOT over one 65536-token request, g=4, c=4096, Reuse and Refine;
  * dense over one 131072-token request, and Refine g=16, c=4096 over the
    same tokens packed as 2 x 65536 (the bench step);
  * decode: 64 requests x 131072-token caches, G=2, dense and Refine c=4096.

For a small sample of rows (the oracle scores them one by one):
  - the GPU scores the selection used match the oracle's within tolerance;
  - recall against the oracle's row is >= 0.999.
For a larger sample (>= 256 rows per case, every decode row), where only the
GPU's own exported scores are needed:
  - the oracle's selection rule applied to those GPU scores reproduces the
    GPU row exactly (and is well formed).
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle as O
from sparse_attention_indexer_05_b200 import workloads as W
from tests._util import check_rows_wellformed, check_scores, recall, reselect, score_rows, to_dev

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def idx():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_indexer_05_b200 as m
    return m


def _sample(n, k, seed):
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 2047, 2048, n // 2, n - 2, n - 1]
    return np.unique(np.concatenate([fixed, rng.integers(0, n, k)])).astype(np.int64)


def _resel_rows(n, seed, k=256):
    """>= k distinct rows spread over [0, n), stratified by position."""
    rng = np.random.default_rng(seed)
    r = ((np.arange(k) + rng.random(k)) * (n / k)).astype(np.int64)
    return np.unique(np.concatenate([r, [0, 1, 2047, 2048, n - 1]]))


def _check_dense_rows(idx, P, dev, got, rows, topk, ws, resel_rows=None):
    q, k, w, cu = dev
    cu_h = P.cu_seqlens
    want = O.dense_topk(P.q, P.k, P.w, cu_h, topk, rows=rows)
    assert recall(got[rows], want) >= 0.999
    allr = np.unique(np.concatenate([rows, resel_rows])) if resel_rows is not None else rows
    sc = idx.debug_scores(0, q, k, w, cu, topk, torch.from_numpy(allr.astype(np.int32)), workspace=ws).cpu().numpy()
    at = {int(r): i for i, r in enumerate(allr)}
    geo = []
    for r in allr:
        b = int(np.searchsorted(cu_h, r, side="right") - 1)
        geo.append((int(r), int(cu_h[b]), int(r - cu_h[b])))
    ora = score_rows([(P.q, P.k, P.w, int(r), int(cu_h[np.searchsorted(cu_h, r, side="right") - 1]),
                       int(r - cu_h[np.searchsorted(cu_h, r, side="right") - 1]) + 1) for r in rows])
    for i, r in enumerate(rows):
        r = int(r)
        _, key0, t = geo[at[r]]
        check_scores(sc[at[r], :t + 1], ora[i])
    for r, key0, t in geo:
        assert np.array_equal(reselect(sc[at[r], :t + 1], topk), got[r]), r


def _check_pivot_rows(idx, P, dev, got, rows, topk, g, c, mode, ws, resel_rows=None):
    q, k, w, cu = dev
    cu_h = P.cu_seqlens
    om = O.REUSE if mode == "reuse" else O.REFINE
    want = O.pivot_topk(P.q, P.k, P.w, cu_h, topk, g, c, om, rows=rows)
    assert recall(got[rows], want) >= 0.999, mode
    if resel_rows is not None:
        _reselect_pivot_rows(idx, P, dev, got, resel_rows, topk, g, c, mode, ws)
    # proxy index of each sampled member: groups are request-local
    plist, geo = [], []
    base = 0
    req_first_proxy = []
    for b in range(len(cu_h) - 1):
        req_first_proxy.append(base)
        base += (cu_h[b + 1] - cu_h[b] + g - 1) // g
    for r in rows:
        b = int(np.searchsorted(cu_h, r, side="right") - 1)
        t = int(r - cu_h[b])
        n = int(cu_h[b + 1] - cu_h[b])
        lo = (t // g) * g
        plist.append(req_first_proxy[b] + t // g)
        geo.append((b, t, lo, min(lo + g, n)))
    # export each proxy once (members of one group share it)
    uniq, slot = np.unique(np.asarray(plist), return_inverse=True)
    psc = idx.debug_scores(1, q, k, w, cu, topk, torch.from_numpy(uniq.astype(np.int32)), g=g,
                           c=c if mode == "refine" else 0).cpu().numpy()[slot]
    msc = None
    if mode == "refine":
        msc = idx.debug_scores(2, q, k, w, cu, topk, torch.from_numpy(rows.astype(np.int32)), g=g, c=c,
                               workspace=ws).cpu().numpy()
    prox = [O.group_proxy(P.q, P.w, int(cu_h[b] + lo), hi - lo) for b, t, lo, hi in geo]
    ora = score_rows([(qb[None], P.k, wb[None], 0, int(cu_h[b]), hi)
                      for (qb, wb), (b, t, lo, hi) in zip(prox, geo)])
    for i, r in enumerate(rows):
        b, t, lo, hi = geo[i]
        ps = psc[i, :hi]
        check_scores(ps, ora[i])
        if mode == "reuse":
            assert np.array_equal(reselect(ps[:t + 1], topk), got[r]), (mode, r)
        else:
            C = reselect(ps, c)
            Cv = C[C >= 0]
            ms = msc[i, :len(Cv)]
            keep = Cv <= t
            assert np.array_equal(reselect(ms[keep], topk, Cv[keep]), got[r]), (mode, r)


def _reselect_pivot_rows(idx, P, dev, got, rows, topk, g, c, mode, ws):
    """The oracle's selection rule on the GPU's exported proxy and member
    scores reproduces every sampled row (no oracle scores needed)."""
    q, k, w, cu = dev
    cu_h = P.cu_seqlens
    first, base = [], 0
    for b in range(len(cu_h) - 1):
        first.append(base)
        base += (cu_h[b + 1] - cu_h[b] + g - 1) // g
    plist, geo = [], []
    for r in rows:
        b = int(np.searchsorted(cu_h, r, side="right") - 1)
        t = int(r - cu_h[b])
        n = int(cu_h[b + 1] - cu_h[b])
        lo = (t // g) * g
        plist.append(first[b] + t // g)
        geo.append((t, min(lo + g, n)))
    uniq, slot = np.unique(np.asarray(plist), return_inverse=True)
    psc = idx.debug_scores(1, q, k, w, cu, topk, torch.from_numpy(uniq.astype(np.int32)), g=g,
                           c=c if mode == "refine" else 0).cpu().numpy()
    msc = None
    if mode == "refine":
        msc = idx.debug_scores(2, q, k, w, cu, topk, torch.from_numpy(np.asarray(rows).astype(np.int32)), g=g,
                               c=c, workspace=ws).cpu().numpy()
    Cs = {}
    for i, r in enumerate(rows):
        t, hi = geo[i]
        ps = psc[slot[i], :hi]
        if mode == "reuse":
            assert np.array_equal(reselect(ps[:t + 1], topk), got[r]), (mode, r)
        else:
            if slot[i] not in Cs:
                C = reselect(ps, c)
                Cs[slot[i]] = C[C >= 0]
            Cv = Cs[slot[i]]
            keep = Cv <= t
            assert np.array_equal(reselect(msc[i, :len(Cv)][keep], topk, Cv[keep]), got[r]), (mode, r)


def test_pivot_65536_g4_c4096_reuse_and_refine(idx):
    P = W.cfg_pivot_64k(seed=0)
    dev = (to_dev(P.q), to_dev(P.k), to_dev(P.w), to_dev(P.cu_seqlens))
    topk, g, c = 2048, 4, 4096
    rows = _sample(P.T, 8, 1)
    for mode in ("reuse", "refine"):
        ws = torch.empty(idx.pivot_workspace_size(P.T, 64, 128, topk, 1, g, c, mode), dtype=torch.uint8,
                         device="cuda")
        out = idx.pivot_topk(*dev, topk, g, c, mode, workspace=ws)
        assert idx.device_status(ws) == "IDX_OK"
        got = out.cpu().numpy()
        check_rows_wellformed(got[rows], [int(r) for r in rows], topk)
        rr = _resel_rows(P.T, 11)
        check_rows_wellformed(got[rr], [int(r) for r in rr], topk)
        _check_pivot_rows(idx, P, dev, got, rows, topk, g, c, mode, ws, resel_rows=rr)


def test_long_131072_dense_and_packed_refine(idx):
    P = W.cfg_long_single(seed=0)
    topk, g, c = 2048, 16, 4096
    q, k, w = to_dev(P.q), to_dev(P.k), to_dev(P.w)
    cu1 = to_dev(np.array([0, 131072], np.int32))
    ws = torch.empty(idx.dense_workspace_size(P.T, 64, 128, topk, 1), dtype=torch.uint8, device="cuda")
    out = idx.dense_topk(q, k, w, cu1, topk, workspace=ws)
    assert idx.device_status(ws) == "IDX_OK"
    got = out.cpu().numpy()
    rows = _sample(P.T, 6, 2)
    check_rows_wellformed(got[rows], [int(r) for r in rows], topk)
    rr = _resel_rows(P.T, 12)
    check_rows_wellformed(got[rr], [int(r) for r in rr], topk)
    _check_dense_rows(idx, P, (q, k, w, cu1), got, rows, topk, ws, resel_rows=rr)
    del ws
    # the same tokens as two packed 65536-token requests, PIVOT Refine g=16
    P.cu_seqlens = np.array([0, 65536, 131072], np.int32)
    cu2 = to_dev(P.cu_seqlens)
    ws2 = torch.empty(idx.pivot_workspace_size(P.T, 64, 128, topk, 2, g, c, "refine"), dtype=torch.uint8,
                      device="cuda")
    out2 = idx.pivot_topk(q, k, w, cu2, topk, g, c, "refine", workspace=ws2)
    assert idx.device_status(ws2) == "IDX_OK"
    got2 = out2.cpu().numpy()
    rows2 = np.unique(np.concatenate([_sample(P.T, 4, 3), [65535, 65536, 65537]]))
    bounds = [int(r - (65536 if r >= 65536 else 0)) for r in rows2]
    check_rows_wellformed(got2[rows2], bounds, topk)
    rr2 = _resel_rows(P.T, 13)
    check_rows_wellformed(got2[rr2], [int(r - (65536 if r >= 65536 else 0)) for r in rr2], topk)
    _check_pivot_rows(idx, P, (q, k, w, cu2), got2, rows2, topk, g, c, "refine", ws2, resel_rows=rr2)


def test_decode_64x131072_dense_and_refine(idx):
    D = W.cfg_decode(seed=0)
    topk, c = 2048, 4096
    B, G, n = 64, 2, 131072
    dq, dkc, dw, dkv = to_dev(D.q), to_dev(D.kcache), to_dev(D.w), to_dev(D.kv_len)
    reqs = np.array([0, 17, 63])
    qf = D.q.reshape(B * G, 64, 128)
    wf = D.w.reshape(B * G, 64)
    kf = D.kcache.reshape(-1, 128)
    for mode, om in (("dense", O.DENSE), ("refine", O.REFINE)):
        ws = torch.empty(max(idx.decode_workspace_size(B, G, n, 64, 128, topk, c, m) for m in ("dense", mode)),
                         dtype=torch.uint8, device="cuda")
        out = idx.decode_topk(dq, dkc, dkv, dw, topk, c, mode, workspace=ws)
        assert idx.device_status(ws) == "IDX_OK"
        got = out.cpu().numpy()
        want = O.decode_topk(D.q, D.kcache, D.w, D.kv_len, topk, c, om, reqs=reqs)
        assert recall(got[reqs], want) >= 0.999, mode
        if mode == "dense":
            sc = idx.debug_decode_scores(0, dq, dkc, dkv, dw, topk, c, mode, workspace=ws).cpu().numpy()
            jobs = [(int(b), m) for b in reqs for m in range(G)]
            ora = score_rows([(qf, kf, wf, b * G + m, b * n, n - G + m + 1) for b, m in jobs])
            for (b, m), o in zip(jobs, ora):
                t = n - G + m
                check_scores(sc[b * G + m, :t + 1], o)
            for b in range(B):  # every row: the oracle's rule on the GPU's scores
                for m in range(G):
                    assert np.array_equal(reselect(sc[b * G + m, :n - G + m + 1], topk), got[b, m]), (b, m)
        else:
            ps = idx.debug_decode_scores(1, dq, dkc, dkv, dw, topk, c, mode, workspace=ws).cpu().numpy()
            ms = idx.debug_decode_scores(2, dq, dkc, dkv, dw, topk, c, mode, workspace=ws).cpu().numpy()
            prox = [O.group_proxy(qf, wf, int(b * G), G) for b in reqs]
            ora = score_rows([(qb[None], kf, wb[None], 0, int(b * n), n) for (qb, wb), b in zip(prox, reqs)])
            for b, o in zip(reqs, ora):
                check_scores(ps[b, :n], o)
            for b in range(B):  # every request: the oracle's rule on the GPU's scores
                C = reselect(ps[b, :n], c)
                for m in range(G):
                    t = n - G + m
                    keep = C <= t
                    assert np.array_equal(reselect(ms[b * G + m, :c][keep], topk, C[keep]), got[b, m]), (b, m)
