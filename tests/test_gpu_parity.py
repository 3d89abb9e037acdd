"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

For every case: (1) scores the GPU selection used, exported through the
debug hook, agree with the oracle's double-precision scores within
1e-3 * max(|I|, 1e-3 * row max); (2) re-applying the oracle's selection
rule to those GPU scores reproduces the GPU's indices exactly; (3) recall
against the oracle's indices is >= 0.999; (4) every row is well formed
(ascending, unique, causal, -1 padded); (5) the device status is IDX_OK.
Exact-integer inputs additionally require bit-equal scores and indices.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle as O
from sparse_attention_indexer_05_b200 import workloads as W
from tests._util import check_rows_wellformed, check_scores, recall, reselect, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def idx():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_indexer_05_b200 as m
    return m


def _dev_inputs(P):
    return to_dev(P.q), to_dev(P.k), to_dev(P.w), to_dev(P.cu_seqlens)


def _bounds_dense(cu):
    return [t for b in range(len(cu) - 1) for t in range(cu[b + 1] - cu[b])]


def _dense_case(idx, P, topk, rows_for_scores=None, full_oracle=True):
    q, k, w, cu = _dev_inputs(P)
    ws = torch.empty(idx.dense_workspace_size(P.T, P.H, P.d, topk, len(P.cu_seqlens) - 1, q.dtype),
                     dtype=torch.uint8, device="cuda")
    out, osc = idx.dense_topk(q, k, w, cu, topk, workspace=ws, return_scores=True)
    assert idx.device_status(ws) == "IDX_OK"
    got = out.cpu().numpy()
    gsc = osc.cpu().numpy()
    cu_h = P.cu_seqlens
    bounds = _bounds_dense(cu_h)
    check_rows_wellformed(got, bounds, topk)
    rows = np.arange(P.T) if full_oracle else np.asarray(rows_for_scores)
    want = O.dense_topk(P.q, P.k, P.w, cu_h, topk, rows=rows)
    assert recall(got[rows], want) >= 0.999
    srows = np.arange(P.T) if rows_for_scores is None else np.asarray(rows_for_scores)
    sc = idx.debug_scores(0, q, k, w, cu, topk, torch.from_numpy(srows.astype(np.int32)), workspace=ws)
    sc = sc.cpu().numpy()
    for i, r in enumerate(srows):
        b = int(np.searchsorted(cu_h, r, side="right") - 1)
        t = int(r - cu_h[b])
        g = sc[i, :t + 1]
        assert np.isfinite(g).all()
        check_scores(g, O.score_row(P.q, P.k, P.w, int(r), int(cu_h[b]), t + 1))
        assert np.array_equal(reselect(g, topk), got[r]), f"re-selection differs at row {r}"
        sel = got[r][got[r] >= 0]
        assert np.array_equal(gsc[r][:len(sel)], g[sel])            # out_score = the scores used
        assert np.all(np.isneginf(gsc[r][len(sel):]))
    return got


def test_fp32_small_all_rows(idx):
    P = W.small_fp32()
    _dense_case(idx, P, 64)


def test_bf16_dense_ragged_requests(idx):
    P = W.prefill([1500, 1037, 1, 130], H=64, d=128, topk=128, rho=0.95, planted=0.01, seed=3)
    _dense_case(idx, P, 128)


def test_bf16_dense_full_16k_sampled(idx):
    P = W.cfg_dense_16k(seed=0)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 2046, 2047, 2048, 2049, 16383, 16382],
                                     np.random.default_rng(0).integers(0, 16384, 22)]))
    _dense_case(idx, P, 2048, rows_for_scores=rows, full_oracle=False)


def test_exact_integer_inputs_bit_exact(idx):
    P = W.exact_ints([700, 333], H=64, d=128, topk=32, seed=5)
    q, k, w, cu = _dev_inputs(P)
    out = idx.dense_topk(q, k, w, cu, 32).cpu().numpy()
    want = O.dense_topk(P.q, P.k, P.w, P.cu_seqlens, 32)
    assert np.array_equal(out, want)
    rows = np.array([0, 5, 699, 700, 1032])
    sc = idx.debug_scores(0, q, k, w, cu, 32, torch.from_numpy(rows.astype(np.int32))).cpu().numpy()
    for i, r in enumerate(rows):
        b = int(np.searchsorted(P.cu_seqlens, r, side="right") - 1)
        t = int(r - P.cu_seqlens[b])
        ora = O.score_row(P.q, P.k, P.w, int(r), int(P.cu_seqlens[b]), t + 1)
        assert np.array_equal(sc[i, :t + 1].astype(np.float64), ora)
    for mode in ("reuse", "refine"):
        o = idx.pivot_topk(q, k, w, cu, 32, 4, 64, mode).cpu().numpy()
        wnt = O.pivot_topk(P.q, P.k, P.w, P.cu_seqlens, 32, 4, 64, O.REUSE if mode == "reuse" else O.REFINE)
        assert np.array_equal(o, wnt), mode


@pytest.mark.parametrize("g,c", [(4, 256), (16, 256), (1, 128), (3, 200)])
def test_bf16_pivot(idx, g, c):
    topk = 128
    P = W.prefill([1100, 777, 5], H=64, d=128, topk=topk, rho=0.95, planted=0.01, seed=7)
    q, k, w, cu = _dev_inputs(P)
    cu_h = P.cu_seqlens
    S = len(cu_h) - 1
    bounds = _bounds_dense(cu_h)
    for mode, om in (("reuse", O.REUSE), ("refine", O.REFINE)):
        ws = torch.empty(idx.pivot_workspace_size(P.T, P.H, P.d, topk, S, g, c, mode, q.dtype),
                         dtype=torch.uint8, device="cuda")
        out = idx.pivot_topk(q, k, w, cu, topk, g, c, mode, workspace=ws)
        assert idx.device_status(ws) == "IDX_OK"
        got = out.cpu().numpy()
        check_rows_wellformed(got, bounds, topk)
        want = O.pivot_topk(P.q, P.k, P.w, cu_h, topk, g, c, om)
        assert recall(got, want) >= 0.999, (mode, recall(got, want))
        # proxies in request order: proxy p of request b covers [i*g, min((i+1)*g, n))
        prox = []
        for b in range(S):
            n = cu_h[b + 1] - cu_h[b]
            for i in range((n + g - 1) // g):
                prox.append((b, i * g, min((i + 1) * g, n)))
        pr = np.arange(len(prox), dtype=np.int32)
        psc = idx.debug_scores(1, q, k, w, cu, topk, torch.from_numpy(pr), g=g,
                               c=c if mode == "refine" else 0).cpu().numpy()
        msc = None
        if mode == "refine":
            msc = idx.debug_scores(2, q, k, w, cu, topk, torch.arange(P.T, dtype=torch.int32), g=g, c=c,
                                   workspace=ws).cpu().numpy()
        for p, (b, lo, hi) in enumerate(prox):
            t_last = hi - 1
            ps = psc[p, :t_last + 1]
            qb, wb = O.group_proxy(P.q, P.w, int(cu_h[b] + lo), hi - lo)
            check_scores(ps, O.score_row(qb[None], P.k, wb[None], 0, int(cu_h[b]), t_last + 1))
            C = reselect(ps, c) if mode == "refine" else None
            for t in range(lo, hi):
                r = cu_h[b] + t
                if mode == "reuse":
                    assert np.array_equal(reselect(ps[:t + 1], topk), got[r]), (mode, r)
                else:
                    Cv = C[C >= 0]
                    ms = msc[r, :len(Cv)]
                    keep = Cv <= t
                    assert np.array_equal(reselect(ms[keep], topk, Cv[keep]), got[r]), (mode, r)


def test_decode_modes(idx):
    topk, c = 128, 256
    D = W.decode(B=5, n=3000, G=2, H=64, d=128, topk=topk, c=c, seed=2,
                 kv_len=[3000, 2500, 129, 2, 1777], n_max=3000)
    q, kc, w, kv = to_dev(D.q), to_dev(D.kcache), to_dev(D.w), to_dev(D.kv_len)
    for mode, om in (("dense", O.DENSE), ("reuse", O.REUSE), ("refine", O.REFINE)):
        ws = torch.empty(max(idx.decode_workspace_size(5, 2, 3000, 64, 128, topk, c, m, q.dtype)
                             for m in ("dense", mode)), dtype=torch.uint8, device="cuda")
        out = idx.decode_topk(q, kc, kv, w, topk, c, mode, workspace=ws)
        assert idx.device_status(ws) == "IDX_OK"
        got = out.cpu().numpy()
        bounds = [int(n) - 2 + m for n in D.kv_len for m in range(2)]
        check_rows_wellformed(got, bounds, topk)
        want = O.decode_topk(D.q, D.kcache, D.w, D.kv_len, topk, c, om)
        assert recall(got, want) >= 0.999, mode
        if mode == "dense":
            sc = idx.debug_decode_scores(0, q, kc, kv, w, topk, c, mode, workspace=ws).cpu().numpy()
            for b in range(5):
                for m in range(2):
                    t = int(D.kv_len[b]) - 2 + m
                    g = sc[b * 2 + m, :t + 1]
                    check_scores(g, O.score_row(D.q.reshape(10, 64, 128), D.kcache.reshape(-1, 128),
                                                D.w.reshape(10, 64), b * 2 + m, b * 3000, t + 1))
                    assert np.array_equal(reselect(g, topk), got[b, m])
        else:
            ps = idx.debug_decode_scores(1, q, kc, kv, w, topk, c, mode, workspace=ws).cpu().numpy()
            ms = idx.debug_decode_scores(2, q, kc, kv, w, topk, c, mode, workspace=ws).cpu().numpy() \
                if mode == "refine" else None
            for b in range(5):
                n = int(D.kv_len[b])
                prs = ps[b, :n]
                qb, wb = O.group_proxy(D.q.reshape(10, 64, 128), D.w.reshape(10, 64), b * 2, 2)
                check_scores(prs, O.score_row(qb[None], D.kcache.reshape(-1, 128), wb[None], 0, b * 3000, n))
                for m in range(2):
                    t = n - 2 + m
                    if mode == "reuse":
                        assert np.array_equal(reselect(prs[:t + 1], topk), got[b, m])
                    else:
                        C = reselect(prs, c)
                        Cv = C[C >= 0]
                        mm = ms[b * 2 + m, :len(Cv)]
                        keep = Cv <= t
                        assert np.array_equal(reselect(mm[keep], topk, Cv[keep]), got[b, m])


def test_decode_rows_longer_than_the_select_cache(idx):
    """n_max = 140000: each of the 8 CTAs of a row's cluster holds 17504
    positions, more than it keeps in shared memory, so the decode select reads
    its segment from global memory on every pass.  Dense and Reuse indices
    equal the oracle's rule re-applied to the GPU's own scores."""
    topk, c, n_max = 2048, 4096, 140000
    D = W.decode(B=2, n=n_max, G=2, H=64, d=128, topk=topk, c=c, seed=5, kv_len=[140000, 70001], n_max=n_max)
    q, kc, w, kv = to_dev(D.q), to_dev(D.kcache), to_dev(D.w), to_dev(D.kv_len)
    for mode in ("dense", "reuse"):
        ws = torch.empty(max(idx.decode_workspace_size(2, 2, n_max, 64, 128, topk, c, m, q.dtype)
                             for m in ("dense", mode)), dtype=torch.uint8, device="cuda")
        got = idx.decode_topk(q, kc, kv, w, topk, c, mode, workspace=ws).cpu().numpy()
        assert idx.device_status(ws) == "IDX_OK"
        bounds = [int(n) - 2 + m for n in D.kv_len for m in range(2)]
        check_rows_wellformed(got, bounds, topk)
        stage = 0 if mode == "dense" else 1
        sc = idx.debug_decode_scores(stage, q, kc, kv, w, topk, c, mode, workspace=ws).cpu().numpy()
        for b in range(2):
            for m in range(2):
                t = int(D.kv_len[b]) - 2 + m
                row = sc[b * 2 + m, :t + 1] if mode == "dense" else sc[b, :t + 1]
                assert np.array_equal(reselect(row, topk), got[b, m]), (mode, b, m)


def test_decode_exact_integer_inputs(idx):
    """Integer q and cache in [-2, 2] (exact in bf16) and dyadic w: every decode
    score is an exact fp32 integer, ties are frequent, and the selected indices
    must equal the oracle's bit for bit.  n_max = 5000 and the ragged kv_len
    leave segments of the decode select that end inside a 32-position run; the
    tensor-core scan (H = 64, d = 128) and the CUDA-core scan (H = 4, d = 16)."""
    for H, d in ((64, 128), (4, 16)):
        B, G, n_max, topk, c = 3, 2, 5000, 512, 1024
        rng = np.random.default_rng(11)
        q = W.bf16_bits(rng.integers(-2, 3, size=(B, G, H, d)).astype(np.float32))
        kc = W.bf16_bits(rng.integers(-2, 3, size=(B, n_max, d)).astype(np.float32))
        w = rng.choice(np.array([0.0, 0.25, 0.5, 1.0], np.float32), size=(B, G, H)).astype(np.float32)
        kv_len = np.array([5000, 4097, 1500], np.int32)
        qd, kd, wd, kvd = to_dev(q), to_dev(kc), to_dev(w), to_dev(kv_len)
        for mode, om in (("dense", O.DENSE), ("reuse", O.REUSE), ("refine", O.REFINE)):
            ws = torch.empty(idx.decode_workspace_size(B, G, n_max, H, d, topk, c, mode, qd.dtype),
                             dtype=torch.uint8, device="cuda")
            out = idx.decode_topk(qd, kd, kvd, wd, topk, c, mode, workspace=ws)
            assert idx.device_status(ws) == "IDX_OK"
            got = out.cpu().numpy().reshape(B * G, topk)
            want = O.decode_topk(q, kc, w, kv_len, topk, c, om).reshape(B * G, topk)
            assert np.array_equal(got, want), (H, d, mode)


def test_edges_short_prefixes_and_empty_request(idx):
    # topk larger than every prefix; an empty request in the middle; T = 1 case
    P = W.prefill([300, 0, 150], H=64, d=128, topk=512, rho=0.9, planted=0.0, seed=9)
    q, k, w, cu = _dev_inputs(P)
    out = idx.dense_topk(q, k, w, cu, 512).cpu().numpy()
    for r in range(P.T):
        b = int(np.searchsorted(P.cu_seqlens, r, side="right") - 1)
        t = r - P.cu_seqlens[b]
        assert np.array_equal(out[r][:t + 1], np.arange(t + 1)) and (out[r][t + 1:] == -1).all()
    P1 = W.prefill([1], H=64, d=128, topk=4, seed=1)
    q1, k1, w1, cu1 = _dev_inputs(P1)
    assert idx.dense_topk(q1, k1, w1, cu1, 4).cpu().numpy().tolist() == [[0, -1, -1, -1]]
    o1 = idx.pivot_topk(q1, k1, w1, cu1, 4, 4, 8, "refine").cpu().numpy().tolist()
    assert o1 == [[0, -1, -1, -1]]


def test_monotone_scores_force_compaction(idx):
    """Scores rising with position append every key, so the candidate buffer
    fills and is compacted repeatedly; the result must still be exact."""
    L, H, d, topk = 4096, 64, 128, 64
    u = np.ones(d, np.float32) / np.sqrt(d)
    ramp = (np.arange(L, dtype=np.float32) / L)[:, None]
    noise = np.random.default_rng(1).standard_normal((L, d)).astype(np.float32) * 0.01
    kf = ramp * u * 8 + noise
    qf = np.broadcast_to(u * 2, (L, H, d)).astype(np.float32)
    P = W.Prefill("ramp", W.bf16_bits(qf), W.bf16_bits(kf), np.full((L, H), 1.0 / H, np.float32),
                  np.array([0, L], np.int32), topk)
    for order in (1, -1):
        if order == -1:
            P.k = W.bf16_bits(kf[::-1].copy())
        q, k, w, cu = _dev_inputs(P)
        rows = np.array([0, 63, 64, 1000, 2047, 4095])
        _dense_case(idx, P, topk, rows_for_scores=rows, full_oracle=False)


def test_invalid_cu_seqlens_flagged_on_device(idx):
    P = W.prefill([64, 64], H=64, d=128, topk=8, seed=1)
    q, k, w, _ = _dev_inputs(P)
    bad = torch.tensor([0, 64, 100], dtype=torch.int32, device="cuda")   # last != T
    ws = torch.empty(idx.dense_workspace_size(128, 64, 128, 8, 2, q.dtype), dtype=torch.uint8, device="cuda")
    out = idx.dense_topk(q, k, w, bad, 8, workspace=ws).cpu().numpy()
    assert idx.device_status(ws) == "IDX_ERR_INVALID"
    assert (out == -1).all()
    kvbad = torch.tensor([1, 64], dtype=torch.int32, device="cuda")       # kv_len < G
    D = W.decode(B=2, n=64, G=2, H=64, d=128, topk=8, c=16, seed=1)
    ws2 = torch.empty(idx.decode_workspace_size(2, 2, 64, 64, 128, 8, 16, "dense", q.dtype), dtype=torch.uint8,
                      device="cuda")
    o2 = idx.decode_topk(to_dev(D.q), to_dev(D.kcache), kvbad, to_dev(D.w), 8, 16, "dense",
                         workspace=ws2).cpu().numpy()
    assert idx.device_status(ws2) == "IDX_ERR_INVALID"
    assert (o2[0] == -1).all() and (o2[1] >= 0).any()
