"""GPU parity of the token-sparse attention (idx_sparse_attn) against the oracle.

Tolerance, from the arithmetic: P is rounded to bf16 before the value
product (relative error <= 2^-9 per weight, so at most 2^-9 * max_j |v_j|
per output element), the output itself is rounded to bf16 (2^-9 * |o|), and
the logits are fp32 sums of 576 products (relative error about 576 * 2^-24
of sum |q_i k_i|).  The test allows twice these bounds.
"""
from __future__ import annotations

import math

import numpy as np
import pytest

import oracle as O
from sparse_attention_indexer_05_b200 import workloads as W
from tests._util import to_dev

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
DQK, DV = 576, 512


@pytest.fixture(scope="module")
def idx():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_indexer_05_b200 as m
    return m


def _bf16_to_np(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _check(q, kv, ix, cu_q, cu_kv, scale, out, lse, rows):
    o_ora, l_ora = O.sparse_attn(q, kv, ix, cu_q, cu_kv, DV, scale, rows=rows)
    og = W.bf16_to_f32(_bf16_to_np(out)).astype(np.float64)
    lg = lse.cpu().numpy().astype(np.float64)
    kvf = W.bf16_to_f32(kv).astype(np.float64)
    qf = W.bf16_to_f32(q).astype(np.float64)
    H = q.shape[1]
    for i, r in enumerate(rows):
        b = int(np.searchsorted(cu_q, r, side="right") - 1)
        sel = ix[r][ix[r] >= 0]
        if len(sel) == 0:
            assert np.all(og[r] == 0.0) and np.all(np.isneginf(lg[r])), r
            continue
        V = kvf[cu_kv[b] + sel]
        vmax = np.abs(V[:, :DV]).max(axis=0)
        tol = 2.0 ** -8 * (vmax[None, :] + np.abs(o_ora[i])) + 1e-6
        bad = np.abs(og[r] - o_ora[i]) > tol
        assert not bad.any(), (r, int(bad.sum()), float(np.max(np.abs(og[r] - o_ora[i]) - tol)))
        mag = scale * (np.abs(qf[r]) @ np.abs(V).T).max(axis=1)  # per head: max_j sum |q_i k_i|
        ltol = 2 * (576 * 2.0 ** -24 * mag + 1e-6 * (1 + np.abs(l_ora[i])))
        assert np.all(np.abs(lg[r] - l_ora[i]) <= ltol), (r, float(np.max(np.abs(lg[r] - l_ora[i]) - ltol)))


def _rand(shape, rng, scale=1.0):
    return W.bf16_bits((rng.standard_normal(shape, dtype=np.float32) * np.float32(scale)))


def test_attn_packed_random_indices(idx):
    # two requests (25 and 15 query rows over 300 and 3000 kv rows); random
    # index sets with -1 anywhere, a duplicate, a row with no entry, ragged topk
    rng = np.random.default_rng(11)
    H, topk = 128, 80
    cu_q = np.array([0, 25, 40], np.int32)
    cu_kv = np.array([0, 300, 3300], np.int32)
    q = _rand((40, H, DQK), rng)
    kv = _rand((3300, DQK), rng)
    ix = np.full((40, topk), -1, np.int32)
    for r in range(40):
        n = 300 if r < 25 else 3000
        m = int(rng.integers(1, topk + 1))
        ix[r, :m] = rng.choice(n, size=m, replace=False)
        rng.shuffle(ix[r])
    ix[3, :2] = [17, 17]
    ix[7, :] = -1
    scale = 1.0 / math.sqrt(192.0)
    dq, dkv, dix, dcq, dck = to_dev(q), to_dev(kv), to_dev(ix), to_dev(cu_q), to_dev(cu_kv)
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    out, lse = idx.sparse_attn(dq, dkv, dix, dcq, dck, scale, workspace=ws, return_lse=True)
    assert idx.device_status(ws) == "IDX_OK"
    _check(q, kv, ix, cu_q, cu_kv, scale, out, lse, np.arange(40))


def test_attn_fewer_heads_large_logits(idx):
    # H = 64 (rows 64..127 of the MMA unused) and logits spread over hundreds:
    # the running maximum moves many times (O rescaled in TMEM)
    rng = np.random.default_rng(12)
    H, topk, R, N = 64, 256, 6, 4096
    q = _rand((R, H, DQK), rng, 2.0)
    kv = _rand((N, DQK), rng, 2.0)
    # ascending logits along the list so the max keeps growing chunk after chunk
    ix = np.sort(rng.choice(N, size=(R, topk)), axis=1).astype(np.int32)
    cu = np.array([0, R], np.int32)
    cukv = np.array([0, N], np.int32)
    kvf = W.bf16_to_f32(kv)
    order = np.argsort(kvf @ W.bf16_to_f32(q)[0, 0])  # keys ordered by head 0 logit of row 0
    ix[0] = order[-topk:].astype(np.int32)
    scale = 0.5
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    out, lse = idx.sparse_attn(to_dev(q), to_dev(kv), to_dev(ix), to_dev(cu), to_dev(cukv), scale, workspace=ws,
                               return_lse=True)
    assert idx.device_status(ws) == "IDX_OK"
    _check(q, kv, ix, cu, cukv, scale, out, lse, np.arange(R))


def test_attn_on_indexer_output_and_decode_layout(idx):
    # the dense indexer's own top-k (ascending positions, -1 padded short rows)
    P = W.prefill([1500], H=64, d=128, topk=128, rho=0.95, planted=0.01, seed=6)
    dq_i, dk_i, dw_i, dcu = to_dev(P.q), to_dev(P.k), to_dev(P.w), to_dev(P.cu_seqlens)
    sel = idx.dense_topk(dq_i, dk_i, dw_i, dcu, 128)
    rng = np.random.default_rng(13)
    q = _rand((1500, 128, DQK), rng)
    kv = _rand((1500, DQK), rng)
    scale = 1.0 / math.sqrt(192.0)
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    out, lse = idx.sparse_attn(to_dev(q), to_dev(kv), sel, dcu, dcu, scale, workspace=ws, return_lse=True)
    assert idx.device_status(ws) == "IDX_OK"
    rows = np.r_[0, 1, 127, 128, 129, 777, 1499]
    _check(q, kv, sel.cpu().numpy(), P.cu_seqlens, P.cu_seqlens, scale, out, lse, rows)
    # decode layout: B requests x G query rows over a [B, n_max] cache
    B, G, n_max = 3, 2, 1000
    qd = _rand((B * G, 128, DQK), rng)
    kc = _rand((B * n_max, DQK), rng)
    kvl = [1000, 613, 64]
    ixd = np.full((B * G, 96), -1, np.int32)
    for b in range(B):
        for m in range(G):
            t = kvl[b] - G + m
            ixd[b * G + m, :min(96, t + 1)] = np.sort(rng.choice(t + 1, size=min(96, t + 1), replace=False))
    cq = np.arange(0, B * G + 1, G, dtype=np.int32)
    ck = np.arange(0, B * n_max + 1, n_max, dtype=np.int32)
    out, lse = idx.sparse_attn(to_dev(qd), to_dev(kc), to_dev(ixd), to_dev(cq), to_dev(ck), scale, workspace=ws,
                               return_lse=True)
    assert idx.device_status(ws) == "IDX_OK"
    _check(qd, kc, ixd, cq, ck, scale, out, lse, np.arange(B * G))


def test_attn_flags_out_of_range_positions(idx):
    rng = np.random.default_rng(14)
    q = _rand((2, 128, DQK), rng)
    kv = _rand((100, DQK), rng)
    ix = np.array([[3, 5, 150, -1], [7, 8, 9, 10]], np.int32)  # 150 >= kv length 100
    cu = np.array([0, 2], np.int32)
    ck = np.array([0, 100], np.int32)
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    out, lse = idx.sparse_attn(to_dev(q), to_dev(kv), to_dev(ix), to_dev(cu), to_dev(ck), 0.1, workspace=ws,
                               return_lse=True)
    assert idx.device_status(ws) == "IDX_ERR_INVALID"
    ix_ok = ix.copy()
    ix_ok[0, 2] = -1  # the flagged entry is skipped
    _check(q, kv, ix_ok, cu, ck, 0.1, out, lse, np.arange(2))


def test_attn_full_topk_2048_sampled(idx):
    # 1024 query rows with k = 2048 positions each over a 65536-row latent cache
    rng = np.random.default_rng(15)
    R, N, topk = 1024, 65536, 2048
    g = torch.Generator(device="cuda")
    g.manual_seed(15)
    dq = torch.randn(R, 128, DQK, generator=g, device="cuda").to(torch.bfloat16)
    dkv = torch.randn(N, DQK, generator=g, device="cuda").to(torch.bfloat16)
    ix = np.sort(np.stack([rng.choice(N, size=topk, replace=False) for _ in range(R)]), axis=1).astype(np.int32)
    cu = np.array([0, R], np.int32)
    ck = np.array([0, N], np.int32)
    scale = 1.0 / math.sqrt(192.0)
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    out, lse = idx.sparse_attn(dq, dkv, to_dev(ix), to_dev(cu), to_dev(ck), scale, workspace=ws, return_lse=True)
    assert idx.device_status(ws) == "IDX_OK"
    q = _bf16_to_np(dq)
    kv = _bf16_to_np(dkv)
    _check(q, kv, ix, cu, ck, scale, out, lse, np.array([0, 511, 1023]))
