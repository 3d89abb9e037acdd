"""Pins of the oracle's adaptive-budget rule (cutoff margin, quantile trigger,
padded expansion) against facts fixed outside its code.

- hand-worked examples (tests/golden/adaptive_hand.json; exact fractions, the
  fp32 result must be their round-to-nearest);
- the quantile against numpy's inverse-CDF quantile (a library routine);
- the ranking against the C oracle's selection;
- the page's cost accounting: rho k on a q fraction of rows, k elsewhere;
- special cases that reduce to the dense top-k of the C oracle: q = 1 is the
  dense top-(rho k), q = 0 is the dense top-k padded;
- planted mistakes (an off-by-one order statistic, a floor quantile, a strict
  trigger, the wrong tie-break) each fail one of the pins above.
"""
from __future__ import annotations

import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle as O
from oracle import adaptive as A
from sparse_attention_indexer_05_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "adaptive_hand.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _frac(s):
    return None if s is None else (s if s == "nan" else Fraction(s))


def _is_rn(value, exact) -> bool:
    """value (fp32) is the round-to-nearest of the exact fraction (or both NaN)."""
    if exact == "nan":
        return bool(np.isnan(value))
    if np.isnan(value):
        return False
    v = np.float32(value)
    up = np.nextafter(v, np.float32(np.inf))
    dn = np.nextafter(v, np.float32(-np.inf))
    err = abs(Fraction(float(v)) - exact)
    return err <= abs(Fraction(float(up)) - exact) and err <= abs(Fraction(float(dn)) - exact)


def _check_margins(mod=A):
    for case in _golden()["margin"]:
        got = mod.cutoff_margin(np.asarray(case["scores"], np.float32), case["k"])
        assert _is_rn(got, _frac(case["sigma"])), (case, got)


def _check_quantiles(mod=A):
    for case in _golden()["quantile"]:
        sig = np.array([np.nan if s == "nan" else float(Fraction(s)) for s in case["sigma"]], np.float32)
        tau, _ = mod.quantile_threshold(sig, case["q"])
        if case["tau"] is None:
            assert tau is None, case
        else:
            assert tau is not None and _is_rn(tau, Fraction(case["tau"])), (case, tau)
        trig = np.zeros(len(sig), bool) if tau is None else (~np.isnan(sig) & (sig <= tau))
        assert trig.tolist() == case["trigger"], case


def _check_selects(mod=A):
    for case in _golden()["select"]:
        rows = [np.asarray(r, np.float32) for r in case["rows"]]
        idx, sigma, trig, tau = mod.adaptive_select(rows, case["k"], case["rho"], case["q"])
        for s, want in zip(sigma, case["sigma"]):
            assert _is_rn(s, _frac(want)), (case["note"], s, want)
        assert (tau is None) == (case["tau"] is None)
        if tau is not None:
            assert _is_rn(tau, Fraction(case["tau"]))
        assert trig.tolist() == case["trigger"], case["note"]
        assert idx.tolist() == case["idx"], (case["note"], idx.tolist())


def test_margin_hand_examples():
    _check_margins()


def test_quantile_hand_examples():
    _check_quantiles()


def test_select_hand_examples():
    _check_selects()


def test_quantile_is_numpys_inverse_cdf():
    rng = np.random.default_rng(0)
    for n in (1, 2, 7, 100, 1001):
        for q in (0.1, 0.25, 0.4, 0.5, 0.9, 1.0):
            s = rng.random(n).astype(np.float32)
            s[rng.random(n) < 0.2] = np.nan
            s[:n // 3] = np.round(s[:n // 3], 1)  # some ties
            d = s[~np.isnan(s)]
            tau, r = A.quantile_threshold(s, q)
            if len(d) == 0 or r == 0:
                assert tau is None
                continue
            want = np.quantile(d.astype(np.float64), q, method="inverted_cdf")
            assert float(tau) == float(want), (n, q)


def test_ranking_matches_c_oracle_select():
    rng = np.random.default_rng(1)
    for n in (1, 5, 64, 300):
        s = np.round(rng.standard_normal(n), 1).astype(np.float32)  # many ties
        for m in (1, 3, 17, n):
            want = O.select(s.astype(np.float64), m)
            got = np.full(m, -1, np.int32)
            sel = np.sort(A.ranked(s)[:m])
            got[:len(sel)] = sel
            assert np.array_equal(got, want), (n, m)


def test_cost_accounting():
    # every row has >= rho k positions and a distinct sigma, and q T is an
    # integer: exactly q T rows keep rho k, the others k, so the mean kept
    # count is k (1 + q (rho - 1))
    rng = np.random.default_rng(2)
    k, rho, q, T = 5, 3, 0.4, 50
    rows = [rng.standard_normal(40).astype(np.float32) for _ in range(T)]
    idx, sigma, trig, tau = A.adaptive_select(rows, k, rho, q)
    assert len(np.unique(sigma)) == T
    assert trig.sum() == round(q * T)
    kept = (idx >= 0).sum(axis=1)
    assert kept.mean() == pytest.approx(k * (1 + q * (rho - 1)))
    assert set(kept.tolist()) == {k, rho * k}


def test_special_cases_reduce_to_dense():
    # exact-arithmetic inputs: fp32 scores equal the double ones, so the
    # ranking cannot differ from the C oracle's through rounding
    P = W.exact_ints([40, 25, 3], H=4, d=16, topk=4, seed=3)
    k, rho = 4, 2
    idx1, sig1, trig1, _ = A.adaptive_topk(P.q, P.k, P.w, P.cu_seqlens, k, rho, 1.0)
    assert np.array_equal(idx1, O.dense_topk(P.q, P.k, P.w, P.cu_seqlens, rho * k))
    assert np.array_equal(trig1, ~np.isnan(sig1))
    idx0, _, trig0, _ = A.adaptive_topk(P.q, P.k, P.w, P.cu_seqlens, k, rho, 0.0)
    want0 = np.full((P.T, rho * k), -1, np.int32)
    want0[:, :k] = O.dense_topk(P.q, P.k, P.w, P.cu_seqlens, k)
    assert np.array_equal(idx0, want0)
    assert not trig0.any()
    # rows with at most k positions: undefined sigma, whole prefix kept
    for b, n in enumerate(np.diff(P.cu_seqlens)):
        for t in range(min(k, int(n))):
            assert np.isnan(sig1[P.cu_seqlens[b] + t])


def test_nested_and_bounded():
    P = W.prefill([300, 129], H=8, d=32, topk=16, seed=4)
    idx, sigma, trig, _ = A.adaptive_topk(P.q, P.k, P.w, P.cu_seqlens, 16, 3, 0.4)
    dense = O.dense_topk(P.q, P.k, P.w, P.cu_seqlens, 48)
    d = sigma[~np.isnan(sigma)]
    assert ((d >= 0) & (d <= 1)).all()
    for t in range(P.T):
        got = idx[t][idx[t] >= 0]
        assert set(got) <= set(dense[t][dense[t] >= 0]) or not trig[t]
        assert len(got) == len(np.unique(got))


# ----------------------------------------------------------------- mutants
class _Mut:
    """A copy of the rule with one planted mistake."""

    def __init__(self, name):
        self.name = name
        self.ranked = A.ranked

    def cutoff_margin(self, scores, k):
        if self.name == "margin_off_by_one":
            s = np.sort(np.asarray(scores, np.float32))[::-1]
            if len(s) < k + 2:
                return np.float32(np.nan)
            den = np.float32(s[0] - s[k + 1])
            return np.float32(np.float32(s[k] - s[k + 1]) / den) if den > 0 else np.float32(0)
        if self.name == "margin_wrong_denominator":
            s = np.sort(np.asarray(scores, np.float32))[::-1]
            if len(s) < k + 1:
                return np.float32(np.nan)
            den = np.float32(s[0] - s[k - 1])
            return np.float32(np.float32(s[k - 1] - s[k]) / den) if den > 0 else np.float32(0)
        return A.cutoff_margin(scores, k)

    def quantile_threshold(self, sigma, qfrac):
        if self.name == "floor_quantile":
            s = np.asarray(sigma, np.float32)
            d = np.sort(s[~np.isnan(s)])
            r = int(np.floor(float(qfrac) * len(d)))
            return (None, 0) if r <= 0 else (np.float32(d[r - 1]), r)
        return A.quantile_threshold(sigma, qfrac)

    def adaptive_select(self, rows, k, rho, qfrac):
        T = len(rows)
        sigma = np.array([self.cutoff_margin(r, k) for r in rows], np.float32)
        tau, _ = self.quantile_threshold(sigma, qfrac)
        trig = np.zeros(T, bool)
        if tau is not None:
            trig = ~np.isnan(sigma) & ((sigma < tau) if self.name == "strict_trigger" else (sigma <= tau))
        out = np.full((T, rho * k), -1, np.int32)
        for t, row in enumerate(rows):
            r = np.asarray(row, np.float32)
            if self.name == "upper_index_wins":
                p = np.arange(len(r))
                order = p[np.lexsort((-p, -r.astype(np.float64)))]
            else:
                order = A.ranked(r)
            sel = np.sort(order[:rho * k if trig[t] else k])
            out[t, :len(sel)] = sel
        return out, sigma, trig, tau


@pytest.mark.parametrize("name", ["margin_off_by_one", "margin_wrong_denominator", "floor_quantile",
                                  "strict_trigger", "upper_index_wins"])
def test_pins_catch_planted_mistake(name):
    m = _Mut(name)
    caught = False
    for check in (_check_margins, _check_quantiles, _check_selects):
        try:
            check(m)
        except AssertionError:
            caught = True
    assert caught, name
