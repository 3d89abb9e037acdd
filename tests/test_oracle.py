"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each pin below checks the oracle against something other than its own code:
a hand-worked example (tests/golden/hand_example.json), exact rational
brute force on tiny inputs, a textbook special case reduced to a library
sort, closed forms and invariants that follow from the definitions on the
PIVOT page, and a statistical closed form for Gaussian inputs.  A mutation
test then plants plausible mistakes in a copy of the oracle (on the CPU) and
checks that some pin catches each of them.
"""
from __future__ import annotations

import json
import math
import os
import subprocess
from fractions import Fraction

import numpy as np
import pytest

import oracle as O
from oracle import build as obuild
from sparse_attention_indexer_05_b200 import workloads as W

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden", "hand_example.json")


def _bf(x):
    return W.bf16_bits(np.asarray(x, np.float32))


def _hand():
    with open(GOLDEN) as f:
        G = json.load(f)
    q = _bf(G["q"])
    k = _bf(G["k"])
    w = np.asarray(G["w"], np.float32)
    return G, q, k, w


# ------------------------------------------------------------------ pins

def pin_hand_scores():
    G, q, k, w = _hand()
    for t, want in enumerate(G["scores"]):
        got = O.score_row(q, k, w, t, 0, t + 1)
        assert np.array_equal(got, np.asarray(want, np.float64)), (t, got, want)
    for t0, want in G["proxy_scores"].items():
        t0 = int(t0)
        qb, wb = O.group_proxy(q, w, t0, 2)
        got = O.score_row(qb[None], k, wb[None], 0, 0, t0 + 2)
        assert np.array_equal(got, np.asarray(want, np.float64)), (t0, got, want)


def pin_hand_topk():
    G, q, k, w = _hand()
    cu = np.array([0, 4], np.int32)
    for kk, want in G["dense"].items():
        got = O.dense_topk(q, k, w, cu, int(kk))
        assert got.tolist() == want, ("dense", kk, got.tolist(), want)
    for kk, want in G["reuse_g2"].items():
        got = O.pivot_topk(q, k, w, cu, int(kk), 2, int(kk), O.REUSE)
        assert got.tolist() == want, ("reuse", kk, got.tolist(), want)
    for tag, want in G["refine_g2"].items():
        kk, c = (int(x[1:]) for x in tag.split("_"))
        got = O.pivot_topk(q, k, w, cu, kk, 2, c, O.REFINE)
        assert got.tolist() == want, ("refine", tag, got.tolist(), want)


def pin_hand_guardrail():
    """The guardrail on the hand example: dense rows for short groups, PIVOT rows otherwise."""
    G, q, k, w = _hand()
    cu = np.array([0, 4], np.int32)
    Gd = G["guarded_g2"]
    for db, want in Gd["reuse_k1"].items():
        got = O.pivot_topk(q, k, w, cu, 1, 2, 1, O.REUSE, dense_below=int(db))
        assert got.tolist() == want, ("reuse k1", db, got.tolist(), want)
    for db, want in Gd["refine_k1_c1"].items():
        got = O.pivot_topk(q, k, w, cu, 1, 2, 1, O.REFINE, dense_below=int(db))
        assert got.tolist() == want, ("refine k1 c1", db, got.tolist(), want)
    for db, want in Gd["reuse_k2"].items():
        got = O.pivot_topk(q, k, w, cu, 2, 2, 2, O.REUSE, dense_below=int(db))
        assert got.tolist() == want, ("reuse k2", db, got.tolist(), want)


def pin_guardrail_reductions():
    """dense_below >= every request length gives dense for every mode and g;
    dense_below below the first group's prefix gives plain PIVOT; in between,
    exactly the groups whose prefix fits take the dense rows."""
    P = W.prefill([37, 20, 5], H=4, d=32, topk=5, rho=0.9, planted=0.1, seed=17)
    cu = P.cu_seqlens
    dense = O.dense_topk(P.q, P.k, P.w, cu, 5)
    for mode, c in ((O.REUSE, 5), (O.REFINE, 8)):
        for g in (2, 3, 8):
            plain = O.pivot_topk(P.q, P.k, P.w, cu, 5, g, c, mode)
            assert np.array_equal(O.pivot_topk(P.q, P.k, P.w, cu, 5, g, c, mode, dense_below=37), dense)
            assert np.array_equal(O.pivot_topk(P.q, P.k, P.w, cu, 5, g, c, mode, dense_below=0), plain)
            for db in (1, 9, 16):
                got = O.pivot_topk(P.q, P.k, P.w, cu, 5, g, c, mode, dense_below=db)
                for b in range(3):
                    n = cu[b + 1] - cu[b]
                    for t in range(n):
                        t_last = min((t // g + 1) * g, n) - 1
                        want = dense if t_last + 1 <= db else plain
                        assert np.array_equal(got[cu[b] + t], want[cu[b] + t]), (mode, g, db, b, t)


def pin_hand_decode():
    G, q, k, w = _hand()
    qd = q[2:4][None]          # the decode queries are rows 2 and 3
    wd = w[2:4][None]
    kc = k[None]
    kv = np.array([4], np.int32)
    D = G["decode_G2_kv4"]
    assert O.decode_topk(qd, kc, wd, kv, 2)[0].tolist() == D["dense_k2"]
    assert O.decode_topk(qd, kc, wd, kv, 1)[0].tolist() == D["dense_k1"]
    assert O.decode_topk(qd, kc, wd, kv, 1, 1, O.REUSE)[0].tolist() == D["reuse_k1"]
    assert O.decode_topk(qd, kc, wd, kv, 1, 1, O.REFINE)[0].tolist() == D["refine_k1_c1"]
    assert O.decode_topk(qd, kc, wd, kv, 2, 3, O.REFINE)[0].tolist() == D["refine_k2_c3"]


def _frac_scores(qf, kf, wf, t, key0, n):
    """Exact rational I[t, key0+s], s < n (brute force)."""
    H, d = qf.shape[1], qf.shape[2]
    out = []
    for s in range(n):
        tot = Fraction(0)
        for j in range(H):
            dot = sum(Fraction(float(qf[t, j, i])) * Fraction(float(kf[key0 + s, i])) for i in range(d))
            if dot > 0:
                tot += Fraction(float(wf[t, j])) * dot
        out.append(tot)
    return out


def _brute_select(scores, k, pos=None):
    pos = list(range(len(scores))) if pos is None else list(pos)
    order = sorted(range(len(scores)), key=lambda i: (-scores[i], pos[i]))
    sel = sorted(pos[i] for i in order[:k])
    return sel + [-1] * (k - len(sel))


def _tiny_case(seed, lengths=(7, 5), H=3, d=5):
    rng = np.random.default_rng(seed)
    T = sum(lengths)
    q = _bf(rng.standard_normal((T, H, d)))
    k = _bf(rng.standard_normal((T, d)))
    w = rng.random((T, H)).astype(np.float32)
    if seed % 2:
        w -= np.float32(0.3)          # some negative head weights
    cu = np.zeros(len(lengths) + 1, np.int32)
    cu[1:] = np.cumsum(lengths)
    return q, k, w, cu


def pin_bruteforce_dense():
    for seed in range(3):
        q, k, w, cu = _tiny_case(seed)
        qf, kf = W.bf16_to_f32(q), W.bf16_to_f32(k)
        for kk in (1, 3, 6):
            got = O.dense_topk(q, k, w, cu, kk)
            for b in range(len(cu) - 1):
                for t in range(cu[b + 1] - cu[b]):
                    r = cu[b] + t
                    ex = _frac_scores(qf, kf, w, r, cu[b], t + 1)
                    sc = O.score_row(q, k, w, r, cu[b], t + 1)
                    for a, e in zip(sc, ex):
                        assert abs(a - float(e)) <= 1e-12 * (1 + abs(float(e))), (r, a, e)
                    assert got[r].tolist() == _brute_select(ex, kk), (seed, kk, r)


def pin_bruteforce_pivot():
    for seed in range(2):
        q, k, w, cu = _tiny_case(seed + 10, lengths=(9, 6))
        kf = W.bf16_to_f32(k)
        qf = W.bf16_to_f32(q)
        for g, kk, c in ((2, 2, 3), (3, 2, 2), (4, 3, 5)):
            reuse = O.pivot_topk(q, k, w, cu, kk, g, c, O.REUSE)
            refine = O.pivot_topk(q, k, w, cu, kk, g, c, O.REFINE)
            for b in range(len(cu) - 1):
                n = cu[b + 1] - cu[b]
                for lo in range(0, n, g):
                    hi = min(lo + g, n)
                    qb, wb = O.group_proxy(q, w, cu[b] + lo, hi - lo)
                    ps = _frac_scores(W.bf16_to_f32(qb)[None], kf[cu[b]:], wb[None], 0, 0, hi)
                    order = sorted(range(hi), key=lambda s: (-ps[s], s))
                    C = order[:min(c, hi)]
                    for t in range(lo, hi):
                        r = cu[b] + t
                        assert reuse[r].tolist() == _brute_select(ps[:t + 1], kk), (seed, g, r)
                        Ct = [s for s in C if s <= t]
                        ms = [_frac_scores(qf, kf, w, r, cu[b] + s, 1)[0] for s in Ct]
                        assert refine[r].tolist() == _brute_select(ms, kk, Ct), (seed, g, r)


def pin_exact_integer_inputs():
    P = W.exact_ints([40, 25], H=4, d=16, topk=8, seed=3)
    qf, kf = W.bf16_to_f32(P.q).astype(np.int64), W.bf16_to_f32(P.k).astype(np.int64)
    got = O.dense_topk(P.q, P.k, P.w, P.cu_seqlens, 8)
    n_ties = 0
    for b in range(2):
        c0, c1 = P.cu_seqlens[b], P.cu_seqlens[b + 1]
        for t in range(c1 - c0):
            r = c0 + t
            dots = kf[c0:r + 1] @ qf[r].T                     # [t+1, H] exact integers
            ex = [sum(Fraction(float(P.w[r, j])) * int(max(dots[s, j], 0)) for j in range(4))
                  for s in range(t + 1)]
            sc = O.score_row(P.q, P.k, P.w, r, c0, t + 1)
            assert [Fraction(x) for x in sc] == ex
            n_ties += len(ex) - len(set(ex))
            assert got[r].tolist() == _brute_select(ex, 8)
    assert n_ties > 50  # the case really exercises the tie rule


def pin_textbook_single_head():
    """H = 1, w = 1: the top-k of ReLU(q . k_s), a library sort."""
    rng = np.random.default_rng(5)
    L, d = 50, 8
    q = _bf(rng.standard_normal((L, 1, d)))
    k = _bf(rng.standard_normal((L, d)))
    w = np.ones((L, 1), np.float32)
    cu = np.array([0, L], np.int32)
    got = O.dense_topk(q, k, w, cu, 7)
    qf = W.bf16_to_f32(q).astype(np.float64)[:, 0]
    kf = W.bf16_to_f32(k).astype(np.float64)
    S = np.maximum(qf @ kf.T, 0.0)
    for t in range(L):
        s = S[t, :t + 1]
        order = np.lexsort((np.arange(t + 1), -s))[:7]
        want = np.sort(order).tolist() + [-1] * (7 - min(7, t + 1))
        assert got[t].tolist() == want, t


def pin_pivot_special_cases():
    P = W.prefill([37, 20], H=4, d=32, topk=5, rho=0.9, planted=0.1, seed=7)
    dense = O.dense_topk(P.q, P.k, P.w, P.cu_seqlens, 5)
    for mode in (O.REUSE, O.REFINE):
        g1 = O.pivot_topk(P.q, P.k, P.w, P.cu_seqlens, 5, 1, 5, mode)
        assert np.array_equal(g1, dense), ("g=1 must equal dense", mode)
    for g in (2, 3, 8):
        full = O.pivot_topk(P.q, P.k, P.w, P.cu_seqlens, 5, g, 64, O.REFINE)
        assert np.array_equal(full, dense), ("Refine with c >= prefix must equal dense", g)


def pin_invariants():
    P = W.prefill([70, 33], H=4, d=32, topk=16, rho=0.9, planted=0.05, seed=11)
    cu = P.cu_seqlens
    outs = {kk: O.dense_topk(P.q, P.k, P.w, cu, kk) for kk in (8, 16, 17)}
    for b in range(2):
        for t in range(cu[b + 1] - cu[b]):
            r = cu[b] + t
            sc = O.score_row(P.q, P.k, P.w, r, cu[b], t + 1)
            assert (sc >= 0).all()                                  # w >= 0
            for kk, o in outs.items():
                row = o[r]
                sel = row[row >= 0]
                assert len(sel) == min(kk, t + 1)                   # short prefix: every index
                assert (row[len(sel):] == -1).all()
                assert (sel <= t).all() and (sel >= 0).all()       # causal
                assert len(set(sel.tolist())) == len(sel)           # no duplicates
                assert (np.diff(sel) > 0).all()                     # ascending
            a, b_, c_ = (set(outs[kk][r][outs[kk][r] >= 0].tolist()) for kk in (8, 16, 17))
            assert a <= b_ <= c_                                     # nested in k
    for mode in (O.REUSE, O.REFINE):
        o = O.pivot_topk(P.q, P.k, P.w, cu, 16, 4, 24, mode)
        for b in range(2):
            for t in range(cu[b + 1] - cu[b]):
                row = o[cu[b] + t]
                sel = row[row >= 0]
                assert len(sel) == min(16, t + 1) and (sel <= t).all() and (np.diff(sel) > 0).all()


def pin_reuse_within_proxy_ranking():
    """Reuse member i lies inside the proxy top-(k + |G| - 1) of the group."""
    P = W.prefill([45], H=4, d=32, topk=6, rho=0.9, planted=0.1, seed=13)
    g, kk = 4, 6
    reuse = O.pivot_topk(P.q, P.k, P.w, P.cu_seqlens, kk, g, kk, O.REUSE)
    for lo in range(0, 45, g):
        hi = min(lo + g, 45)
        qb, wb = O.group_proxy(P.q, P.w, lo, hi - lo)
        ps = O.score_row(qb[None], P.k, wb[None], 0, 0, hi)
        top = set(O.select(ps, kk + hi - lo - 1).tolist()) - {-1}
        for t in range(lo, hi):
            row = reuse[t]
            assert set(row[row >= 0].tolist()) <= top


def pin_proxy_exact_mean():
    """For power-of-two groups whose fp32 sum is exact, the proxy is the exact
    mean rounded once to bf16 (nearest, ties to even)."""
    rng = np.random.default_rng(17)
    for cnt in (1, 2, 4, 8, 16):
        # values with 8 significant bits and exponents within a narrow band
        vals = rng.integers(-255, 256, size=(cnt, 2, 8)).astype(np.float32) / np.float32(64)
        q = _bf(vals)
        assert np.array_equal(W.bf16_to_f32(q), vals)
        w = rng.integers(0, 64, size=(cnt, 2)).astype(np.float32) / np.float32(64)
        qb, wb = O.group_proxy(q, w, 0, cnt)
        for j in range(2):
            assert Fraction(float(wb[j])) == sum(Fraction(float(x)) for x in w[:, j]) / cnt
            for i in range(8):
                exact = sum(Fraction(float(v)) for v in vals[:, j, i]) / cnt
                assert Fraction(float(W.bf16_to_f32(qb[j:j + 1, i:i + 1])[0, 0])) == _round_bf16(exact)
    # identical members: the proxy is the member itself
    q = np.repeat(_bf(rng.standard_normal((1, 3, 8))), 5, axis=0)
    w = np.repeat(rng.random((1, 3)).astype(np.float32), 5, axis=0)
    qb, wb = O.group_proxy(q, w, 0, 5)
    assert np.array_equal(qb, q[0])


def _round_bf16(x: Fraction) -> Fraction:
    """Round a rational to the nearest bf16 value, ties to even (8-bit significand)."""
    if x == 0:
        return Fraction(0)
    sgn = -1 if x < 0 else 1
    a = abs(x)
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (e - 7)
    m = a / ulp
    lo = math.floor(m)
    rem = m - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return sgn * lo * ulp


def pin_decode_matches_prefill():
    """Decode (dense, Reuse, Refine) equals the prefill forms on the same data."""
    rng = np.random.default_rng(19)
    B, G, H, d, n_max = 3, 2, 4, 16, 40
    kv = np.array([40, 24, 2], np.int32)
    kc = _bf(rng.standard_normal((B, n_max, d)))
    qd = _bf(rng.standard_normal((B, G, H, d)))
    wd = rng.random((B, G, H)).astype(np.float32)
    for mode, c, kv in ((O.DENSE, 0, np.array([40, 23, 3], np.int32)), (O.REUSE, 6, kv),
                        (O.REFINE, 6, kv), (O.BLOCK, 8, kv)):
        got = O.decode_topk(qd, kc, wd, kv, 5, c, mode, bn=4)
        for b in range(B):
            n = kv[b]
            # prefill request of length n whose last G rows are the decode queries;
            # n - G is a multiple of G here so the last group is exactly them
            q = np.zeros((n, H, d), np.uint16)
            w = np.zeros((n, H), np.float32)
            q[n - G:] = qd[b]
            w[n - G:] = wd[b]
            cu = np.array([0, n], np.int32)
            rows = np.arange(n - G, n)
            if mode == O.DENSE:
                want = O.dense_topk(q, kc[b, :n], w, cu, 5, rows=rows)
            else:
                assert (n - G) % G == 0
                want = O.pivot_topk(q, kc[b, :n], w, cu, 5, G, c, mode, rows=rows, bn=4)
            assert np.array_equal(got[b], want), (mode, b)


def pin_block_mean_exact():
    """The mean key of a block whose fp32 sum is exact is the exact mean rounded
    once to bf16 (nearest, ties to even); only rows r0 .. r0+bn-1 count."""
    rng = np.random.default_rng(29)
    for bn in (1, 2, 4, 64):
        vals = rng.integers(-255, 256, size=(bn + 3, 8)).astype(np.float32) / np.float32(64)
        k = _bf(vals)
        got = O.block_mean(k, 2, bn)
        for i in range(8):
            exact = sum(Fraction(float(v)) for v in vals[2:2 + bn, i]) / bn
            assert Fraction(float(W.bf16_to_f32(got[i:i + 1])[0])) == _round_bf16(exact), (bn, i)
    # (1 + 2^-8) / 2 lies halfway between two bf16 values: even wins -> 0.5;
    # (1 + 3 * 2^-8) / 2 likewise -> 0.5 + 2^-7
    k = _bf(np.array([[1.0, 1.0], [2.0 ** -8, 3 * 2.0 ** -8]], np.float32))
    got = W.bf16_to_f32(O.block_mean(k, 0, 2))
    assert got.tolist() == [0.5, 0.5 + 2.0 ** -7]


def pin_block_reductions():
    """Block pre-filter: block size 1 is Refine; a budget covering the prefix is dense."""
    P = W.prefill([37, 20], H=4, d=32, topk=5, rho=0.9, planted=0.1, seed=31)
    cu = P.cu_seqlens
    for g, c in ((2, 8), (4, 6), (3, 5)):
        a = O.pivot_topk(P.q, P.k, P.w, cu, 5, g, c, O.BLOCK, bn=1)
        b = O.pivot_topk(P.q, P.k, P.w, cu, 5, g, c, O.REFINE)
        assert np.array_equal(a, b), ("block size 1 must equal Refine", g, c)
    dense = O.dense_topk(P.q, P.k, P.w, cu, 5)
    for g, bn in ((2, 4), (4, 8), (3, 16)):
        a = O.pivot_topk(P.q, P.k, P.w, cu, 5, g, 64, O.BLOCK, bn=bn)
        assert np.array_equal(a, dense), ("a budget covering the prefix must equal dense", g, bn)


def pin_block_constant_keys_equal_refine():
    """Keys constant inside each block: a block's mean is its key, so the block
    ranking is the token ranking; with groups ending on block boundaries the
    block pre-filter keeps exactly Refine's candidate set (c a multiple of bn)."""
    rng = np.random.default_rng(37)
    L, H, d, bn = 48, 4, 16, 4
    kb = rng.integers(-8, 9, size=(L // bn, d)).astype(np.float32)
    k = _bf(np.repeat(kb, bn, axis=0))
    q = _bf(rng.integers(-8, 9, size=(L, H, d)).astype(np.float32))
    w = (rng.integers(0, 5, size=(L, H)) / 4).astype(np.float32)
    cu = np.array([0, L], np.int32)
    for c in (8, 12, 20):
        a = O.pivot_topk(q, k, w, cu, 6, 4, c, O.BLOCK, bn=bn)
        b = O.pivot_topk(q, k, w, cu, 6, 4, c, O.REFINE)
        assert np.array_equal(a, b), c


def pin_block_partial_closed_form():
    """A budget of one block and a group ending inside a block: the candidate
    set is the partial block, so member t gets positions part0 .. t."""
    P = W.prefill([30], H=4, d=16, topk=8, rho=0.9, planted=0.1, seed=41)
    bn, g = 8, 3
    got = O.pivot_topk(P.q, P.k, P.w, P.cu_seqlens, 8, g, bn, O.BLOCK, bn=bn)
    checked = 0
    for t in range(30):
        t_last = min((t // g) * g + g, 30) - 1
        if (t_last + 1) % bn == 0:
            continue
        part0 = ((t_last + 1) // bn) * bn
        want = list(range(part0, t + 1))
        assert got[t].tolist() == want + [-1] * (8 - len(want)), t
        checked += 1
    assert checked > 20


def pin_attn_single_entry():
    """One listed position: the output is that key's value part exactly and lse
    its scaled logit (integer inputs: every product and sum is exact)."""
    rng = np.random.default_rng(43)
    R, Ha, Dqk, Dv = 3, 4, 24, 16
    qi = rng.integers(-4, 5, size=(R, Ha, Dqk))
    ki = rng.integers(-4, 5, size=(10, Dqk))
    q, kv = _bf(qi.astype(np.float32)), _bf(ki.astype(np.float32))
    idx = np.full((R, 4), -1, np.int32)
    idx[:, 2] = [3, 0, 9]
    o, lse = O.sparse_attn(q, kv, idx, [0, R], [0, 10], Dv, 0.125)
    for r in range(R):
        j = idx[r, 2]
        assert np.array_equal(o[r], np.repeat(ki[j, :Dv][None].astype(np.float64), Ha, 0)), r
        for h in range(Ha):
            assert lse[r, h] == 0.125 * int((qi[r, h] * ki[j]).sum()), (r, h)


def pin_attn_equal_logits_mean():
    """q = 0: every logit is 0, so o is the plain mean of the listed value rows
    (a position listed twice counts twice) and lse = log(number listed)."""
    rng = np.random.default_rng(47)
    R, Ha, Dqk, Dv, N = 4, 2, 32, 24, 20
    kv = _bf(rng.standard_normal((N, Dqk)).astype(np.float32))
    q = np.zeros((R, Ha, Dqk), np.uint16)
    idx = np.array([[0, 5, 5, -1, 19], [-1, -1, 7, -1, -1], [1, 2, 3, 4, 6], [19, -1, 0, 0, 0]], np.int32)
    o, lse = O.sparse_attn(q, kv, idx, [0, R], [0, N], Dv, 0.7)
    vf = W.bf16_to_f32(kv).astype(np.float64)[:, :Dv]
    for r in range(R):
        sel = idx[r][idx[r] >= 0]
        want = vf[sel].mean(axis=0)
        for h in range(Ha):
            assert np.allclose(o[r, h], want, rtol=1e-14, atol=1e-15), r
            assert abs(lse[r, h] - math.log(len(sel))) < 1e-15, r


def pin_attn_library_sdpa():
    """Two packed requests of random bf16 inputs: the library's scaled
    dot-product attention (torch, float64, CPU) over the gathered rows."""
    import torch
    rng = np.random.default_rng(53)
    Ha, Dqk, Dv, topk = 4, 48, 32, 12
    cu_q = np.array([0, 5, 9], np.int32)
    cu_kv = np.array([0, 30, 47], np.int32)
    q = _bf(rng.standard_normal((9, Ha, Dqk)).astype(np.float32))
    kv = _bf(rng.standard_normal((47, Dqk)).astype(np.float32))
    idx = np.full((9, topk), -1, np.int32)
    for r in range(9):
        b = 0 if r < 5 else 1
        n = cu_kv[b + 1] - cu_kv[b]
        m = rng.integers(1, topk + 1)
        idx[r, :m] = rng.choice(n, size=m, replace=False)
    scale = 0.3
    o, lse = O.sparse_attn(q, kv, idx, cu_q, cu_kv, Dv, scale)
    qf = torch.from_numpy(W.bf16_to_f32(q).astype(np.float64))
    kf = torch.from_numpy(W.bf16_to_f32(kv).astype(np.float64))
    for r in range(9):
        b = 0 if r < 5 else 1
        rows = torch.from_numpy((cu_kv[b] + idx[r][idx[r] >= 0]).astype(np.int64))
        K = kf[rows]
        want = torch.nn.functional.scaled_dot_product_attention(qf[r][None], K[None], K[None, :, :Dv], scale=scale)[0]
        assert np.allclose(o[r], want.numpy(), rtol=1e-12, atol=1e-13), r
        wl = torch.logsumexp(scale * qf[r] @ K.T, dim=-1)
        assert np.allclose(lse[r], wl.numpy(), rtol=1e-13, atol=1e-13), r


def pin_attn_large_logits():
    """Logit gaps far beyond exp's range: the dominant key's value comes out
    exactly and lse equals its logit."""
    Dqk, Dv = 24, 16
    kv = np.zeros((6, Dqk), np.float32)
    kv[4] = 8.0
    kv[:, :Dv] += np.arange(Dv, dtype=np.float32)[None] / 4
    kv[4, :Dv] = np.arange(Dv, dtype=np.float32) - 3
    q = np.full((1, 1, Dqk), 8.0, np.float32)
    q16, kv16 = _bf(q), _bf(kv)
    o, lse = O.sparse_attn(q16, kv16, np.array([[0, 4, 1, 5]], np.int32), [0, 1], [0, 6], Dv, 1.0)
    assert np.array_equal(o[0, 0], kv[4, :Dv].astype(np.float64))
    assert lse[0, 0] == float((q[0, 0].astype(np.float64) * kv[4]).sum())


def pin_gaussian_mean_score():
    """i.i.d. Gaussian q, k: E[I] = sum_j w_j * sigma / sqrt(2 pi), sigma^2 = d var_q var_k."""
    P = W.small_fp32(L=512, H=4, d=64, topk=8, seed=23)
    rows = np.arange(256, 512, 8)
    tot, cnt = 0.0, 0
    pred = 0.0
    sigma = math.sqrt(64 * (1 / 64) * (1 / 64))
    for r in rows:
        sc = O.score_row(P.q, P.k, P.w, int(r), 0, int(r) + 1)
        tot += sc.sum()
        cnt += len(sc)
        pred += float(P.w[r].astype(np.float64).sum()) * sigma / math.sqrt(2 * math.pi) * len(sc)
    assert abs(tot / pred - 1.0) < 0.05, tot / pred


def pin_decode_block_full_budget_is_dense():
    """Decode block mode whose budget covers every block of the cache (and the
    partial one) gives every query its whole prefix as candidates: the dense
    decode top-k; a budget of one block with kv_len inside a block gives the
    partial block's positions up to each query."""
    rng = np.random.default_rng(41)
    B, G, H, d, n_max, bn = 4, 2, 4, 16, 256, 64
    kc = _bf(rng.standard_normal((B, n_max, d)))
    qd = _bf(rng.standard_normal((B, G, H, d)))
    wd = rng.random((B, G, H)).astype(np.float32)
    kv = np.array([256, 130, 64, 7], np.int32)
    dense = O.decode_topk(qd, kc, wd, kv, 9, 0, O.DENSE)
    blk = O.decode_topk(qd, kc, wd, kv, 9, n_max + bn, O.BLOCK, bn=bn)
    assert np.array_equal(blk, dense)
    kv1 = np.array([200, 130, 71, 7], np.int32)
    one = O.decode_topk(qd, kc, wd, kv1, 9, bn, O.BLOCK, bn=bn)
    for b in range(B):
        part0 = (kv1[b] // bn) * bn
        for m in range(G):
            t = kv1[b] - G + m
            want = list(range(part0, t + 1))[:9] if t >= part0 else []
            got = [x for x in one[b, m].tolist() if x >= 0]
            if t + 1 - part0 <= 9:
                assert got == want, (b, m, got, want)
            else:
                assert len(got) == 9 and all(part0 <= x <= t for x in got)


def pin_quest_hand_blocks():
    """Quest bound, worked by hand (one head, w = 1, d = 1, blocks of 2, one
    member at t = 4 that is its own proxy, c = 4 tokens = one complete block
    plus the partial block {4}):
      keys -10, 10, 3, 3, 1 and q = +1: block A = {-10, 10} has bound
      max(1*10, 1*-10) = 10, block B = {3, 3} has 3: A is kept, candidates
      {0, 1, 4} score 0, 10, 1, so the top-1 is position 1.  (The block
      means rank B first, 3 > 0, giving position 2; so would a bound taken
      from the minimum.)  With q = +2 and top-2: scores 0, 20, 2 -> {1, 4}.
      keys -10, 10, -5, -5, 1 and q = -1: A's bound is max(-10, 10) = 10,
      B's is max(5, 5) = 5: A is kept, candidates score 10, 0, 0, so the
      top-1 is position 0.  (A bound from the maximum alone gives A -10 ->
      0 and B 5, keeping B and giving position 2.)"""
    w = np.ones((5, 1), np.float32)
    cu = np.array([0, 5], np.int32)
    k1 = _bf(np.array([[-10.0], [10.0], [3.0], [3.0], [1.0]], np.float32))
    k2 = _bf(np.array([[-10.0], [10.0], [-5.0], [-5.0], [1.0]], np.float32))
    for k, qv, topk, want in ((k1, 1.0, 1, [1]), (k1, 2.0, 2, [1, 4]), (k2, -1.0, 1, [0])):
        q = _bf(np.full((5, 1, 1), qv, np.float32))
        got = O.pivot_topk(q, k, w, cu, topk, 1, 4, O.QUEST, rows=np.array([4]), bn=2)
        assert got[0].tolist() == want, (qv, got)
    q = _bf(np.full((5, 1, 1), 1.0, np.float32))
    assert O.pivot_topk(q, k1, w, cu, 1, 1, 4, O.BLOCK, rows=np.array([4]), bn=2)[0].tolist() == [2]


def pin_quest_reductions():
    """Quest: keys constant inside each block make the bound the exact dot
    product, so Quest ranks blocks as the block means do; a budget covering
    the prefix is dense; and decode Quest equals prefill Quest."""
    rng = np.random.default_rng(43)
    T, H, d, bn = 96, 3, 8, 4
    base = rng.standard_normal((T // bn, d)).astype(np.float32)
    k = _bf(np.repeat(base, bn, axis=0))
    q = _bf(rng.standard_normal((T, H, d)))
    w = rng.random((T, H)).astype(np.float32)
    cu = np.array([0, 60, T], np.int32)
    for g, c in ((4, 8), (3, 12)):
        a = O.pivot_topk(q, k, w, cu, 5, g, c, O.QUEST, bn=bn)
        b = O.pivot_topk(q, k, w, cu, 5, g, c, O.BLOCK, bn=bn)
        assert np.array_equal(a, b), (g, c)
    k2 = _bf(rng.standard_normal((T, d)))
    a = O.pivot_topk(q, k2, w, cu, 5, 4, 128, O.QUEST, bn=bn)
    assert np.array_equal(a, O.dense_topk(q, k2, w, cu, 5))
    B, G, n_max = 2, 2, 40
    kc = _bf(rng.standard_normal((B, n_max, d)))
    qd = _bf(rng.standard_normal((B, G, H, d)))
    wd = rng.random((B, G, H)).astype(np.float32)
    kv = np.array([40, 22], np.int32)
    got = O.decode_topk(qd, kc, wd, kv, 5, 8, O.QUEST, bn=4)
    for b in range(B):
        n = kv[b]
        qq = np.zeros((n, H, d), np.uint16)
        ww = np.zeros((n, H), np.float32)
        qq[n - G:] = qd[b]
        ww[n - G:] = wd[b]
        want = O.pivot_topk(qq, kc[b, :n], ww, np.array([0, n], np.int32), 5, G, 8, O.QUEST,
                            rows=np.arange(n - G, n), bn=4)
        assert np.array_equal(got[b], want), b


ALL_PINS = [pin_hand_scores, pin_hand_topk, pin_hand_guardrail, pin_guardrail_reductions, pin_hand_decode, pin_bruteforce_dense,
            pin_bruteforce_pivot, pin_exact_integer_inputs, pin_textbook_single_head,
            pin_pivot_special_cases, pin_invariants, pin_reuse_within_proxy_ranking,
            pin_proxy_exact_mean, pin_decode_matches_prefill, pin_gaussian_mean_score,
            pin_block_mean_exact, pin_block_reductions, pin_block_constant_keys_equal_refine,
            pin_block_partial_closed_form, pin_attn_single_entry, pin_attn_equal_logits_mean,
            pin_attn_library_sdpa, pin_attn_large_logits, pin_decode_block_full_budget_is_dense,
            pin_quest_hand_blocks, pin_quest_reductions]


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_pin(pin):
    pin()


# ------------------------------------------------------------- mutations

MUTANTS = {
    "relu_dropped": ("if (dot > 0.0) total +=", "total +="),
    "tie_to_higher_index": ("return (x->pos > y->pos) - (x->pos < y->pos);",
                            "return (x->pos < y->pos) - (x->pos > y->pos);"),
    "key_dims_reversed": ("load_elem(k, dtype, k_row + i)", "load_elem(k, dtype, k_row + (d - 1 - i))"),
    "request_offset_dropped": ("J->k, (size_t)(J->cu[b] + s) * J->d", "J->k, (size_t)(s) * J->d"),
    "proxy_sum_not_mean": ("float mean = sum / (float)cnt;", "float mean = sum;"),
    "proxy_w_endpoint": ("wbar[j] = ws / (float)cnt;", "wbar[j] = w[(size_t)m0 * H + j];"),
    "proxy_q_endpoint": ("load_elem(q, dtype, (size_t)(m0 + m) * H * d", "load_elem(q, dtype, (size_t)(m0) * H * d"),
    "refine_member_mask_dropped": ("if (s > t) continue; /* the member's causal mask */", ""),
    "reuse_member_prefix_ignored": ("select_topk(pc, t + 1, topk, out);", "select_topk(pc, n, topk, out);"),
    "candidate_budget_is_k": ("int nc = n < c ? n : c;", "int nc = n < topk ? n : topk;"),
    "decode_positions_all_last": ("int t = n - G + m;", "int t = n - 1;"),
    "pad_with_zero": ("for (int i = m; i < k; ++i) out[i] = -1;", "for (int i = m; i < k; ++i) out[i] = 0;"),
    "output_not_sorted": ("qsort(out, (size_t)m, sizeof(int), int_asc);", ""),
    "head_weight_dropped": ("total += (double)w_row[j] * dot;", "total += dot;"),
    "block_mean_not_divided": ("float mean = sum / (float)bn;", "float mean = sum;"),
    "block_partial_dropped": ("for (int s = part0; s < n && s <= t; ++s) {", "for (int s = n; s < n; ++s) {"),
    "block_budget_ignores_partial": ("int want = c / bn - (part0 < n ? 1 : 0);", "int want = c / bn;"),
    "block_partial_scored": ("int nfull = n / bn;", "int nfull = (n + bn - 1) / bn;"),
    "block_rank_by_position": ("qsort(pc, (size_t)nfull, sizeof(cand_t), by_score_desc_pos_asc);", ""),
    "block_member_mask_dropped": ("                if (s > t) continue;\n                mc[m].score", "                mc[m].score"),
    "block_keys_from_block_start_only": ("int s = pc[i].pos * bn + r;", "int s = pc[i].pos * bn;"),
    "attn_no_max_shift": ("double p = exp(z[j] - m);", "double p = exp(z[j]);"),
    "attn_value_from_tail": ("o[c] += p * load_elem(J->kv, J->dtype, kr + c);",
                             "o[c] += p * load_elem(J->kv, J->dtype, kr + (J->Dqk - J->Dv) + c);"),
    "attn_scale_dropped": ("z[j] = J->scale * dot;", "z[j] = dot;"),
    "attn_request_lookup_dropped": ("int b = find_request(J->cu_q, J->S, r);", "int b = 0;"),
    "attn_normaliser_dropped": ("for (int c = 0; c < J->Dv; ++c) o[c] /= l;", ""),
    "guard_strict_bound": ("if (J->dense_below > 0 && hi <= J->dense_below) {",
                           "if (J->dense_below > 0 && hi < J->dense_below) {"),
    "guard_by_first_member": ("if (J->dense_below > 0 && hi <= J->dense_below) {",
                              "if (J->dense_below > 0 && lo + 1 <= J->dense_below) {"),
    "guard_by_own_position": ("if (J->dense_below > 0 && hi <= J->dense_below) {",
                              "if (J->dense_below > 0 && t + 1 <= J->dense_below) {"),
    "quest_bound_from_minimum": ("bound += a > b ? a : b;", "bound += a < b ? a : b;"),
    "quest_bound_max_only": ("bound += a > b ? a : b;", "bound += a;"),
    "quest_relu_dropped": ("if (bound > 0.0) total += (double)wbar[j] * bound;", "total += (double)wbar[j] * bound;"),
    "quest_scored_by_mean": ("            if (mode == ORA_QUEST) {\n", "            if (0) {\n"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    with open(obuild.SRC) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation anchor not unique/absent: {old!r}"
    mpath = tmp_path / "mutant.c"
    mpath.write_text(src.replace(old, new))
    so = str(tmp_path / f"liboracle_{name}.so")
    obuild.build(str(mpath), so, extra=("-w",))
    failed = []
    with O.use(so):
        for pin in ALL_PINS:
            try:
                pin()
            except (AssertionError, ValueError):
                failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name}"
