"""GPU parity of decode with the block pre-filter (idx_decode_block_topk,
blocks ranked by their mean key or by the Quest bound) and of the block
summaries it reads (idx_decode_block_means, idx_decode_block_minmax),
against the oracle's decode block modes (ora_decode_topk with ORA_BLOCK or
ORA_QUEST, block size 64).

  * block means: every row of kbar equals the oracle's mean of the same 64
    cache rows bit for bit (bf16 and fp32); an update from a first block on
    equals the full computation and leaves the earlier rows untouched; the
    Quest summaries equal numpy's minimum and maximum of those rows;
  * the top-k: rows are well formed and hold as many positions as the
    oracle's (its candidate set has the same blocks and partial block), and
    index recall against the oracle is >= 0.999 on the tensor-core path
    (bf16, H=64, d=128) and the CUDA-core path (fp32); on exact-integer
    inputs, where every member score is exact, the result equals the
    oracle's whenever the block ranking has no near-tie (checked here by
    recall 1.0 on rows whose candidate blocks agree);
  * requests whose kv_len is out of range come back as rows of -1 with the
    status IDX_ERR_INVALID.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle as O
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


def _run(idx, D, topk, c, rule="mean"):
    q, kc, w, kv = to_dev(D.q), to_dev(D.kcache), to_dev(D.w), to_dev(D.kv_len)
    ksum = idx.decode_block_means(kc) if rule == "mean" else idx.decode_block_minmax(kc)
    B, G, H, d = q.shape
    ws = torch.empty(idx.decode_block_workspace_size(B, G, kc.shape[1], H, d, topk, c, rule, q.dtype),
                     dtype=torch.uint8, device="cuda")
    out = idx.decode_block_topk(q, kc, ksum, kv, w, topk, c, rule, workspace=ws)
    return out.cpu().numpy(), idx.device_status(ws), ksum


_MODE = {"mean": O.BLOCK, "quest": O.QUEST}


def _check(got, want, kv, G, topk):
    for b in range(got.shape[0]):
        for m in range(G):
            row = got[b, m]
            sel = row[row >= 0]
            assert len(sel) == int((want[b, m] >= 0).sum()), (b, m)
            assert (row[len(sel):] == -1).all()
            assert (np.diff(sel) > 0).all()
            assert (sel <= kv[b] - G + m).all()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_block_means_bit_exact_and_update(idx, dtype):
    rng = np.random.default_rng(7)
    B, n_max, d = 3, 640, 128 if dtype == "bf16" else 64
    vals = rng.standard_normal((B, n_max, d)).astype(np.float32)
    kc_h = W.bf16_bits(vals) if dtype == "bf16" else vals
    kc = to_dev(kc_h)
    kbar = idx.decode_block_means(kc)
    got = kbar.cpu()
    got = got.view(torch.int16).numpy().view(np.uint16) if dtype == "bf16" else got.numpy()
    for b in range(B):
        for j in range(n_max // 64):
            want = O.block_mean(kc_h[b], j * 64, 64)
            assert np.array_equal(got[b, j].view(np.uint32 if dtype == "f32" else np.uint16),
                                  want.view(np.uint32 if dtype == "f32" else np.uint16)), (b, j)
    # the Quest summaries: per-dimension minimum, then maximum, of each block
    kq = idx.decode_block_minmax(kc).cpu()
    kq = kq.view(torch.int16).numpy().view(np.uint16) if dtype == "bf16" else kq.numpy()
    vals_k = W.bf16_to_f32(kc_h) if dtype == "bf16" else kc_h
    blocks = vals_k.reshape(B, n_max // 64, 64, d)
    want_q = np.stack([blocks.min(axis=2), blocks.max(axis=2)], axis=2)
    got_q = W.bf16_to_f32(kq) if dtype == "bf16" else kq
    assert np.array_equal(got_q, want_q)
    # an update from block 7 on: rows 0..6 keep their (here: poisoned) values
    kbar2 = kbar.clone()
    kbar2[:, :7] = 0
    kbar2[:, 7:] = 5
    idx.decode_block_means(kc, kbar2, first_block=7)
    assert torch.equal(kbar2[:, 7:], kbar[:, 7:])
    assert (kbar2[:, :7] == 0).all()


@pytest.mark.parametrize("rule", ["mean", "quest"])
def test_decode_block_bf16_tensor_cores(idx, rule):
    topk, c, G = 64, 256, 2
    kv = [2560, 2000, 130, 64, 7, 63, 1025]
    D = W.decode(B=len(kv), n=2560, G=G, H=64, d=128, topk=topk, seed=11, kv_len=kv)
    got, st, _ = _run(idx, D, topk, c, rule)
    assert st == "IDX_OK"
    want = O.decode_topk(D.q, D.kcache, D.w, D.kv_len, topk, c, _MODE[rule], bn=64)
    _check(got, want, D.kv_len, G, topk)
    assert recall(got, want) >= 0.999


@pytest.mark.parametrize("rule", ["mean", "quest"])
def test_decode_block_mtp_group_and_fp32(idx, rule):
    # G = 4 MTP queries, fp32 (CUDA-core scan and re-score)
    topk, c, G = 16, 128, 4
    kv = [700, 4, 200, 129]
    D = W.decode(B=len(kv), n=704, G=G, H=4, d=64, topk=topk, seed=12, kv_len=kv)
    D.q = W.bf16_to_f32(D.q)
    D.kcache = W.bf16_to_f32(D.kcache)
    got, st, _ = _run(idx, D, topk, c, rule)
    assert st == "IDX_OK"
    want = O.decode_topk(D.q, D.kcache, D.w, D.kv_len, topk, c, _MODE[rule], bn=64)
    _check(got, want, D.kv_len, G, topk)
    assert recall(got, want) >= 0.999


@pytest.mark.parametrize("rule", ["mean", "quest"])
def test_decode_block_exact_integer_inputs(idx, rule):
    topk, c, G = 8, 128, 2
    B, n_max, H, d = 4, 512, 64, 128
    rng = np.random.default_rng(13)
    D = W.decode(B=B, n=n_max, G=G, H=H, d=d, topk=topk, seed=13, kv_len=[512, 300, 70, 40])
    D.q = W.bf16_bits(rng.integers(-8, 9, size=D.q.shape).astype(np.float32))
    D.kcache = W.bf16_bits(rng.integers(-8, 9, size=D.kcache.shape).astype(np.float32))
    D.w = rng.choice(np.array([0.0, 0.25, 0.5, 1.0], np.float32), size=D.w.shape)
    got, st, _ = _run(idx, D, topk, c, rule)
    assert st == "IDX_OK"
    want = O.decode_topk(D.q, D.kcache, D.w, D.kv_len, topk, c, _MODE[rule], bn=64)
    _check(got, want, D.kv_len, G, topk)
    assert recall(got, want) >= 0.99


@pytest.mark.parametrize("rule", ["mean", "quest"])
def test_decode_block_full_length(idx, rule):
    # the bench's request length, requests of several lengths checked against the oracle
    topk, c, G = 2048, 4096, 2
    D = W.decode(B=4, n=131072, G=G, H=64, d=128, topk=topk, seed=14, kv_len=[131072, 100000, 65536, 4097])
    got, st, _ = _run(idx, D, topk, c, rule)
    assert st == "IDX_OK"
    want = O.decode_topk(D.q, D.kcache, D.w, D.kv_len, topk, c, _MODE[rule], bn=64)
    _check(got, want, D.kv_len, G, topk)
    assert recall(got, want) >= 0.999


def test_decode_block_invalid_kv_len(idx):
    topk, c, G = 16, 128, 2
    D = W.decode(B=3, n=256, G=G, H=64, d=128, topk=topk, seed=15, kv_len=[256, 1, 256])
    q, kc, w = to_dev(D.q), to_dev(D.kcache), to_dev(D.w)
    kv = torch.tensor([256, 1, 257], dtype=torch.int32, device="cuda")   # 1 < G, 257 > n_max
    kbar = idx.decode_block_means(kc)
    ws = torch.empty(idx.decode_block_workspace_size(3, G, 256, 64, 128, topk, c), dtype=torch.uint8, device="cuda")
    out = idx.decode_block_topk(q, kc, kbar, kv, w, topk, c, "mean", workspace=ws).cpu().numpy()
    assert idx.device_status(ws) == "IDX_ERR_INVALID"
    assert (out[1] == -1).all() and (out[2] == -1).all()
    want = O.decode_topk(D.q, D.kcache, D.w, np.array([256, 256, 256], np.int32), topk, c, O.BLOCK, bn=64)
    assert recall(out[:1], want[:1]) >= 0.999
