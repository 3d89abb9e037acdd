"""Row-range calls (idx_dense_topk_rows, idx_pivot_topk_rows), on one GPU:
  * one request split across ranks: the calls for every rank's zig-zag share
    must stitch together into exactly the full call's result, indices and
    scores bit for bit, and leave rows outside the range untouched.  The
    ranks run one after another here (independent calls, nothing waits on
    another rank), which is what each GPU of a split run does;
  * a long prefill in row chunks with a workspace sized for one chunk
    (*_workspace_size_rows): the same result, with the per-row scratch a
    fraction of the full call's.
"""
from __future__ import annotations

import numpy as np
import pytest

from sparse_attention_indexer_05_b200 import multirank as M
from sparse_attention_indexer_05_b200 import workloads as W
from tests._util import to_dev

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def idx():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_indexer_05_b200 as m
    return m


def _stitch(call, T, topk, ranges):
    oi = torch.full((T, topk), -7, dtype=torch.int32, device="cuda")
    os_ = torch.full((T, topk), 7.0, dtype=torch.float32, device="cuda")
    for lo, hi in ranges:
        call(oi, os_, (lo, hi))
    return oi.cpu().numpy(), os_.cpu().numpy()


@pytest.mark.parametrize("world", [2, 3])
def test_split_single_request_dense_reuse_refine(idx, world):
    topk = 64
    P = W.prefill([3000], H=64, d=128, topk=topk, rho=0.95, planted=0.01, seed=9)
    q, k, w, cu = to_dev(P.q), to_dev(P.k), to_dev(P.w), to_dev(P.cu_seqlens)
    T = P.T
    cases = [("dense", None, 1), ("reuse", 4, 4), ("refine", 16, 16)]
    for mode, g, align in cases:
        if mode == "dense":
            full_i, full_s = idx.dense_topk(q, k, w, cu, topk, return_scores=True)

            def call(oi, os_, rows):
                idx.dense_topk(q, k, w, cu, topk, out_idx=oi, out_score=os_, rows=rows)
        else:
            full_i, full_s = idx.pivot_topk(q, k, w, cu, topk, g, 128, mode, return_scores=True)

            def call(oi, os_, rows, g=g, mode=mode):
                idx.pivot_topk(q, k, w, cu, topk, g, 128, mode, out_idx=oi, out_score=os_, rows=rows)
        full_i, full_s = full_i.cpu().numpy(), full_s.cpu().numpy()
        # every rank's share, one rank after another, into one buffer
        ranges = [rg for r in range(world) for rg in M.zigzag_ranges(T, world, r, align)]
        gi, gs = _stitch(call, T, topk, ranges)
        assert np.array_equal(gi, full_i), mode
        assert np.array_equal(gs.view(np.uint32), full_s.view(np.uint32)), mode
        # one rank alone writes its rows and nothing else
        mine = M.zigzag_ranges(T, world, 1, align)
        gi, _ = _stitch(call, T, topk, mine)
        own = np.zeros(T, bool)
        for lo, hi in mine:
            own[lo:hi] = True
        assert np.array_equal(gi[own], full_i[own]), mode
        assert (gi[~own] == -7).all(), mode


def test_ranges_across_packed_requests_and_cut_groups(idx):
    topk, g, c = 32, 4, 64
    P = W.prefill([500, 77, 1200], H=64, d=128, topk=topk, rho=0.95, planted=0.01, seed=4)
    q, k, w, cu = to_dev(P.q), to_dev(P.k), to_dev(P.w), to_dev(P.cu_seqlens)
    T = P.T
    # ranges that cross request boundaries and cut groups in two
    ranges = [(0, 3), (3, 499), (499, 578), (578, 579), (579, 1000), (1000, T)]
    for mode in ("reuse", "refine"):
        full = idx.pivot_topk(q, k, w, cu, topk, g, c, mode).cpu().numpy()

        def call(oi, os_, rows, mode=mode):
            idx.pivot_topk(q, k, w, cu, topk, g, c, mode, out_idx=oi, out_score=os_, rows=rows)
        gi, _ = _stitch(call, T, topk, ranges)
        assert np.array_equal(gi, full), mode
    full = idx.dense_topk(q, k, w, cu, topk).cpu().numpy()
    gi, _ = _stitch(lambda oi, os_, rows: idx.dense_topk(q, k, w, cu, topk, out_idx=oi, out_score=os_, rows=rows),
                    T, topk, ranges)
    assert np.array_equal(gi, full)
    # the guardrail with a range
    full = idx.pivot_topk(q, k, w, cu, topk, g, c, "refine", dense_below=300).cpu().numpy()
    gi, _ = _stitch(lambda oi, os_, rows: idx.pivot_topk(q, k, w, cu, topk, g, c, "refine", out_idx=oi,
                                                         out_score=os_, rows=rows, dense_below=300),
                    T, topk, ranges)
    assert np.array_equal(gi, full)


def test_bad_ranges_are_rejected(idx):
    from sparse_attention_indexer_05_b200 import _native as N
    P = W.prefill([100], H=64, d=128, topk=8, seed=1)
    q, k, w, cu = to_dev(P.q), to_dev(P.k), to_dev(P.w), to_dev(P.cu_seqlens)
    for rows in ((-1, 10), (20, 10), (0, 101)):
        with pytest.raises(N.IdxError):
            idx.dense_topk(q, k, w, cu, 8, rows=rows)
        with pytest.raises(N.IdxError):
            idx.pivot_topk(q, k, w, cu, 8, 4, 16, "refine", rows=rows)


@pytest.mark.parametrize("mode,g,db", [("dense", 1, 0), ("reuse", 4, 0), ("refine", 16, 0), ("refine", 4, 700)])
def test_chunked_prefill_with_bounded_workspace(idx, mode, g, db):
    topk, c, chunk = 64, 128, 750
    P = W.prefill([3000, 333], H=64, d=128, topk=topk, rho=0.95, planted=0.01, seed=21)
    q, k, w, cu = to_dev(P.q), to_dev(P.k), to_dev(P.w), to_dev(P.cu_seqlens)
    T, S = P.T, 2
    if mode == "dense":
        full_ws = idx.dense_workspace_size(T, 64, 128, topk, S)
        ws_size = idx.dense_workspace_size(T, 64, 128, topk, S, max_rows=chunk)
        full_i, full_s = idx.dense_topk(q, k, w, cu, topk, return_scores=True)
    else:
        full_ws = idx.pivot_workspace_size(T, 64, 128, topk, S, g, c, mode, dense_below=db)
        ws_size = idx.pivot_workspace_size(T, 64, 128, topk, S, g, c, mode, dense_below=db, max_rows=chunk)
        full_i, full_s = idx.pivot_topk(q, k, w, cu, topk, g, c, mode, return_scores=True, dense_below=db)
    assert ws_size < full_ws
    ws = torch.empty(ws_size, dtype=torch.uint8, device="cuda")

    def call(oi, os_, rows):
        if mode == "dense":
            idx.dense_topk(q, k, w, cu, topk, out_idx=oi, out_score=os_, rows=rows, workspace=ws)
        else:
            idx.pivot_topk(q, k, w, cu, topk, g, c, mode, out_idx=oi, out_score=os_, rows=rows, workspace=ws,
                           dense_below=db)
    # chunks that do not line up with groups or requests
    ranges = [(lo, min(lo + chunk, T)) for lo in range(0, T, chunk)]
    gi, gs = _stitch(call, T, topk, ranges)
    assert np.array_equal(gi, full_i.cpu().numpy()), mode
    assert np.array_equal(gs.view(np.uint32), full_s.cpu().numpy().view(np.uint32)), mode
    # through the C ABI, a range longer than the workspace was sized for is
    # refused (IDX_ERR_WORKSPACE) before anything runs
    from sparse_attention_indexer_05_b200 import _native as N
    oi = torch.empty(T, topk, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    if mode == "dense":
        rc = N.lib().idx_dense_topk_rows(q.data_ptr(), k.data_ptr(), w.data_ptr(), cu.data_ptr(), S, T, 64, 128,
                                         topk, N.BF16, 0, 2 * chunk, oi.data_ptr(), None, ws.data_ptr(), ws.numel(),
                                         st)
    else:
        rc = N.lib().idx_pivot_topk_rows(q.data_ptr(), k.data_ptr(), w.data_ptr(), cu.data_ptr(), S, T, 64, 128,
                                         topk, N.BF16, g, c, N.MODE_REUSE if mode == "reuse" else N.MODE_REFINE, db,
                                         0, 2 * chunk, oi.data_ptr(), None, ws.data_ptr(), ws.numel(), st)
    assert rc == 3, N.STATUS.get(rc, rc)
