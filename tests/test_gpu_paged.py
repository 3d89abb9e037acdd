"""GPU parity of the paged-cache decode entry point.

The keys of each request are scattered over a shuffled page pool through a
block table (the paged layout of serving engines); the result must be the
contiguous-cache decode's, bit for bit (same kernels, same tile contents),
wherever both take the tensor-core scan, and must match the oracle run on
the contiguous cache.  Unused pages, the unused tail of each request's last
page and block-table entries past the request hold large garbage or
out-of-range page ids: a wrong page read would change the top-k.
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


def paginate(kc: np.ndarray, kv_len, page: int, seed: int, extra: int = 3):
    """Scatter kc [B, n_max, d] (bf16 bits) into a shuffled pool [num_pages, page, d]
    and a block table [B, ceil(n_max / page)]."""
    B, n_max, d = kc.shape
    rng = np.random.default_rng(seed)
    need = [(int(n) + page - 1) // page for n in kv_len]
    max_pages = (n_max + page - 1) // page
    num_pages = sum(need) + extra
    perm = rng.permutation(num_pages)
    pool = np.zeros((num_pages, page, d), np.uint16)
    garbage = W.bf16_bits(rng.standard_normal((page, d), dtype=np.float32) * np.float32(1000.0))
    bt = np.where(rng.random((B, max_pages)) < 0.5, -1, num_pages + 7).astype(np.int32)
    i = 0
    for b in range(B):
        n = int(kv_len[b])
        for j in range(need[b]):
            p = int(perm[i])
            i += 1
            bt[b, j] = p
            lo, hi = j * page, min(j * page + page, n)
            pool[p, :hi - lo] = kc[b, lo:hi]
            pool[p, hi - lo:] = garbage[hi - lo:]
    for p in perm[i:]:
        pool[int(p)] = garbage
    return pool, bt


def _run_both(idx, D, page, mode, topk, c, seed):
    B, G = D.q.shape[:2]
    n_max = D.kcache.shape[1]
    q, kc, w, kv = to_dev(D.q), to_dev(D.kcache), to_dev(D.w), to_dev(D.kv_len)
    pool, bt = paginate(D.kcache, D.kv_len, page, seed)
    dpool, dbt = to_dev(pool), to_dev(bt)
    ws = torch.empty(idx.decode_workspace_size(B, G, max(n_max, bt.shape[1] * page), 64, 128, topk, c, mode,
                                               q.dtype), dtype=torch.uint8, device="cuda")
    ref_i, ref_s = idx.decode_topk(q, kc, kv, w, topk, c, mode, workspace=ws, return_scores=True)
    assert idx.device_status(ws) == "IDX_OK"
    got_i, got_s = idx.decode_paged_topk(q, dpool, dbt, kv, w, topk, c, mode, workspace=ws, return_scores=True)
    assert idx.device_status(ws) == "IDX_OK"
    return ref_i.cpu().numpy(), ref_s.cpu().numpy(), got_i.cpu().numpy(), got_s.cpu().numpy()


@pytest.mark.parametrize("page", [8, 16, 64, 128, 256])
def test_paged_equals_contiguous(idx, page):
    topk, c = 128, 256
    D = W.decode(B=5, n=3000, G=2, H=64, d=128, topk=topk, c=c, seed=2,
                 kv_len=[3000, 2500, 129, 2, 1777], n_max=3000)
    bounds = [int(n) - 2 + m for n in D.kv_len for m in range(2)]
    for mode in ("dense", "reuse", "refine"):
        ri, rs, gi, gs = _run_both(idx, D, page, mode, topk, c, seed=page)
        check_rows_wellformed(gi, bounds, topk)
        assert np.array_equal(gi, ri), (page, mode)
        assert np.array_equal(gs.view(np.uint32), rs.view(np.uint32)), (page, mode)


@pytest.mark.parametrize("page", [1, 4, 8, 64])
def test_small_pages_against_oracle(idx, page):
    # pages under 8 keys take the CUDA-core scan, 8 and more the tensor-core
    # scan (64: the serving page size the bench uses): compare with the oracle
    topk, c = 64, 128
    D = W.decode(B=3, n=700, G=2, H=64, d=128, topk=topk, c=c, seed=5, kv_len=[700, 300, 3], n_max=700)
    bounds = [int(n) - 2 + m for n in D.kv_len for m in range(2)]
    for mode, om in (("dense", O.DENSE), ("reuse", O.REUSE), ("refine", O.REFINE)):
        _, _, gi, _ = _run_both(idx, D, page, mode, topk, c, seed=page)
        check_rows_wellformed(gi, bounds, topk)
        want = O.decode_topk(D.q, D.kcache, D.w, D.kv_len, topk, c, om)
        assert recall(gi, want) >= 0.999, (page, mode)


def test_paged_full_size_64x131072(idx):
    # 64 requests x 131072 keys in 64-key pages (two TMA boxes per key tile) and
    # 256-key pages; ragged lengths on a few requests
    D = W.cfg_decode(seed=0)
    D.kv_len[[3, 40]] = [131072 - 37, 70001]
    topk, c = 2048, 4096
    for page in (64, 256):
        for mode in ("dense", "refine"):
            ri, rs, gi, gs = _run_both(idx, D, page, mode, topk, c, seed=page)
            assert np.array_equal(gi, ri), (page, mode)
            assert np.array_equal(gs.view(np.uint32), rs.view(np.uint32)), (page, mode)
    reqs = np.array([3, 40])
    want = O.decode_topk(D.q, D.kcache, D.w, D.kv_len, topk, c, O.REFINE, reqs=reqs)
    assert recall(gi[reqs], want) >= 0.999
