"""GPU parity of the block pre-filter with the Quest bound in prefill
(idx_pivot_topk with IDX_MODE_QUEST) against the oracle's ORA_QUEST mode:
  * rows are well formed (ascending, unique, inside the member's prefix)
    and hold as many positions as the oracle's rows (the candidate sets have
    the same blocks and partial block);
  * index recall against the oracle is >= 0.999 on the tensor-core re-score
    path (bf16, H=64, d=128) over packed ragged requests (one too short for
    a complete block) and on the CUDA-core path (fp32), g = 1, 4 and 16;
  * a request split into row ranges stitches into the full call bit for bit;
  * the guardrail is refused (IDX_ERR_UNSUPPORTED), like the block-mean rule.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle as O
from sparse_attention_indexer_05_b200 import multirank as M
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


def _check(got, want, cu):
    for b in range(len(cu) - 1):
        for t in range(int(cu[b + 1] - cu[b])):
            r = int(cu[b]) + t
            row = got[r]
            sel = row[row >= 0]
            assert len(sel) == int((want[r] >= 0).sum()), r
            assert (row[len(sel):] == -1).all(), r
            assert (np.diff(sel) > 0).all() and (sel <= t).all(), r


@pytest.mark.parametrize("g,c", [(1, 64), (4, 128), (16, 256)])
def test_quest_bf16_packed(idx, g, c):
    topk = 32
    P = W.prefill([1500, 40, 700, 129], H=64, d=128, topk=topk, rho=0.95, planted=0.01, seed=51)
    q, k, w, cu = to_dev(P.q), to_dev(P.k), to_dev(P.w), to_dev(P.cu_seqlens)
    ws = torch.empty(idx.pivot_workspace_size(P.T, 64, 128, topk, 4, g, c, "quest"), dtype=torch.uint8,
                     device="cuda")
    got = idx.pivot_topk(q, k, w, cu, topk, g, c, "quest", workspace=ws).cpu().numpy()
    assert idx.device_status(ws) == "IDX_OK"
    want = O.pivot_topk(P.q, P.k, P.w, P.cu_seqlens, topk, g, c, O.QUEST, bn=64)
    _check(got, want, P.cu_seqlens)
    assert recall(got, want) >= 0.999


def test_quest_fp32_cuda_cores(idx):
    topk, g, c = 16, 4, 128
    P = W.small_fp32(L=900, H=4, d=64, topk=topk, seed=52)
    P.cu_seqlens = np.array([0, 300, 900], np.int32)
    q, k, w, cu = to_dev(P.q), to_dev(P.k), to_dev(P.w), to_dev(P.cu_seqlens)
    got = idx.pivot_topk(q, k, w, cu, topk, g, c, "quest").cpu().numpy()
    want = O.pivot_topk(P.q, P.k, P.w, P.cu_seqlens, topk, g, c, O.QUEST, bn=64)
    _check(got, want, P.cu_seqlens)
    assert recall(got, want) >= 0.999


def test_quest_row_ranges_stitch_and_guardrail_refused(idx):
    from sparse_attention_indexer_05_b200 import _native as N
    topk, g, c = 64, 16, 512
    P = W.prefill([4096], H=64, d=128, topk=topk, rho=0.95, planted=0.01, seed=53)
    q, k, w, cu = to_dev(P.q), to_dev(P.k), to_dev(P.w), to_dev(P.cu_seqlens)
    full_i, full_s = idx.pivot_topk(q, k, w, cu, topk, g, c, "quest", return_scores=True)
    oi = torch.full((P.T, topk), -7, dtype=torch.int32, device="cuda")
    os_ = torch.full((P.T, topk), 7.0, dtype=torch.float32, device="cuda")
    for r in range(3):
        for lo, hi in M.zigzag_ranges(P.T, 3, r, g):
            idx.pivot_topk(q, k, w, cu, topk, g, c, "quest", out_idx=oi, out_score=os_, rows=(lo, hi))
    assert torch.equal(oi, full_i)
    assert torch.equal(os_.view(torch.int32), full_s.view(torch.int32))
    rows = np.arange(0, P.T, 37)
    want = O.pivot_topk(P.q, P.k, P.w, P.cu_seqlens, topk, g, c, O.QUEST, rows=rows, bn=64)
    assert recall(full_i.cpu().numpy()[rows], want) >= 0.999
    # through the C ABI: the guardrail is refused before anything runs
    ws = torch.empty(idx.pivot_workspace_size(P.T, 64, 128, topk, 1, g, c, "quest"), dtype=torch.uint8,
                     device="cuda")
    rc = N.lib().idx_pivot_topk(q.data_ptr(), k.data_ptr(), w.data_ptr(), cu.data_ptr(), 1, P.T, 64, 128, topk,
                                N.BF16, g, c, N.MODE_QUEST, 256, oi.data_ptr(), None, ws.data_ptr(), ws.numel(),
                                torch.cuda.current_stream().cuda_stream)
    assert rc == 2, N.STATUS.get(rc, rc)


def test_quest_full_size_packed_2x65536_g16(idx):
    # the bench's block leg: 2 x 65536 tokens, g = 16, c = 4096, sampled rows
    # (the first and last of each request, the group edges around them, and
    # random rows) against the oracle, and every row well formed
    topk, g, c = 2048, 16, 4096
    P = W.cfg_long_packed(seed=0)
    q, k, w, cu = to_dev(P.q), to_dev(P.k), to_dev(P.w), to_dev(P.cu_seqlens)
    ws = torch.empty(idx.pivot_workspace_size(P.T, 64, 128, topk, 2, g, c, "quest"), dtype=torch.uint8,
                     device="cuda")
    got = idx.pivot_topk(q, k, w, cu, topk, g, c, "quest", workspace=ws).cpu().numpy()
    assert idx.device_status(ws) == "IDX_OK"
    rng = np.random.default_rng(54)
    rows = np.unique(np.concatenate([[0, 15, 16, 4095, 4096, 65535, 65536, 65551, 131071],
                                     rng.integers(0, P.T, 16)])).astype(np.int64)
    want = O.pivot_topk(P.q, P.k, P.w, P.cu_seqlens, topk, g, c, O.QUEST, rows=rows, bn=64)
    assert recall(got[rows], want) >= 0.999
    for r, wr in zip(rows, want):
        t = int(r - (65536 if r >= 65536 else 0))
        row = got[r]
        sel = row[row >= 0]
        assert len(sel) == int((wr >= 0).sum()), r
        assert (np.diff(sel) > 0).all() and (sel <= t).all(), r
