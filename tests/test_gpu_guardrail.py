"""GPU parity of the guardrail (idx_pivot_topk with dense_below > 0).

The rule (PIVOT page, Results, indexer speed: PIVOT falls back to a dense
scan for short groups): a group whose last member's prefix holds at most
dense_below keys takes the dense top-k of each member.  Checked through the
C ABI on packed ragged requests, on the tensor-core path (bf16, H=64,
d=128) and on the CUDA-core path (fp32):
  * rows of short groups equal idx_dense_topk's rows, indices and scores bit
    for bit; every other row equals the unguarded call's row bit for bit
    (the group structure after the short groups is unchanged);
  * the result matches the oracle's guarded rule (recall >= 0.999, exact on
    exact-integer inputs, where every score is exact);
  * rows are well formed and the device status is IDX_OK.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle as O
from sparse_attention_indexer_05_b200 import workloads as W
from tests._util import check_rows_wellformed, recall, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def idx():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_indexer_05_b200 as m
    return m


def _dense_rows(n, g, db):
    if db <= 0 or g == 1:
        return 0
    return n if n <= db else (db // g) * g


def _run(idx, P, topk, g, c, mode, db):
    q, k, w, cu = to_dev(P.q), to_dev(P.k), to_dev(P.w), to_dev(P.cu_seqlens)
    S = len(P.cu_seqlens) - 1
    ws = torch.empty(idx.pivot_workspace_size(P.T, P.H, P.d, topk, S, g, c, mode, q.dtype, db),
                     dtype=torch.uint8, device="cuda")
    o, s = idx.pivot_topk(q, k, w, cu, topk, g, c, mode, workspace=ws, return_scores=True, dense_below=db)
    assert idx.device_status(ws) == "IDX_OK"
    return o.cpu().numpy(), s.cpu().numpy()


def _check_structure(idx, P, topk, g, c, mode, dbs):
    q, k, w, cu = to_dev(P.q), to_dev(P.k), to_dev(P.w), to_dev(P.cu_seqlens)
    cu_h = P.cu_seqlens
    dense_i, dense_s = idx.dense_topk(q, k, w, cu, topk, return_scores=True)
    dense_i, dense_s = dense_i.cpu().numpy(), dense_s.cpu().numpy()
    plain_i, plain_s = _run(idx, P, topk, g, c, mode, 0)
    bounds = [t for b in range(len(cu_h) - 1) for t in range(cu_h[b + 1] - cu_h[b])]
    for db in dbs:
        gi, gs = _run(idx, P, topk, g, c, mode, db)
        check_rows_wellformed(gi, bounds, topk)
        for b in range(len(cu_h) - 1):
            n = int(cu_h[b + 1] - cu_h[b])
            nd = _dense_rows(n, g, db)
            r0, r1 = int(cu_h[b]), int(cu_h[b]) + nd
            assert np.array_equal(gi[r0:r1], dense_i[r0:r1]), (mode, g, db, b)
            assert np.array_equal(gs[r0:r1], dense_s[r0:r1]), (mode, g, db, b)
            assert np.array_equal(gi[r1:cu_h[b + 1]], plain_i[r1:cu_h[b + 1]]), (mode, g, db, b)
            assert np.array_equal(gs[r1:cu_h[b + 1]], plain_s[r1:cu_h[b + 1]]), (mode, g, db, b)
        om = O.REUSE if mode == "reuse" else O.REFINE
        want = O.pivot_topk(P.q, P.k, P.w, cu_h, topk, g, c, om, dense_below=db)
        assert recall(gi, want) >= 0.999, (mode, g, db, recall(gi, want))


@pytest.mark.parametrize("mode", ["reuse", "refine"])
@pytest.mark.parametrize("g", [4, 16])
def test_guardrail_bf16_tensor_cores(idx, mode, g):
    topk, c = 64, 128
    P = W.prefill([700, 45, 1300, 3], H=64, d=128, topk=topk, rho=0.95, planted=0.01, seed=31)
    # 0 < db < every length; a threshold between group boundaries; one that
    # covers whole requests; one that covers every request
    _check_structure(idx, P, topk, g, c, mode, [1, 130, 257, 701, 1 << 20])


@pytest.mark.parametrize("mode", ["reuse", "refine"])
def test_guardrail_fp32_cuda_cores(idx, mode):
    topk, c, g = 16, 40, 4
    P = W.small_fp32(L=600, H=4, d=64, topk=topk, seed=5)
    P.cu_seqlens = np.array([0, 250, 600], np.int32)
    _check_structure(idx, P, topk, g, c, mode, [97, 300])


def test_guardrail_exact_integers_match_oracle(idx):
    topk, c, g = 8, 16, 4
    P = W.exact_ints([90, 37, 64], H=64, d=128, topk=topk, seed=3)
    for mode, om in (("reuse", O.REUSE), ("refine", O.REFINE)):
        for db in (20, 40, 64):
            gi, _ = _run(idx, P, topk, g, c, mode, db)
            want = O.pivot_topk(P.q, P.k, P.w, P.cu_seqlens, topk, g, c, om, dense_below=db)
            assert np.array_equal(gi, want), (mode, db)
