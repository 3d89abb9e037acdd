"""Adaptive top-k budget from the cutoff margin: the plain restatement.

TEST INFRASTRUCTURE ONLY (part of the oracle package; see ``oracle/__init__``).

Follows "Uncertainty-gated selection for block-sparse attention", Section 3
(Method), steps 3-5, and its Appendix A, steps (A.5)-(A.9), applied to the lightning
indexer's per-query scores instead of per-tile block scores:

* (A.5) sort the row's candidates by (score desc, position asc) and keep the
  first k+1: s_(0) >= s_(1) >= ... >= s_(k);
* (A.6) the normalised cutoff margin
      sigma = (s_(k-1) - s_(k)) / (s_(0) - s_(k))   in [0, 1];
* (A.7) the head mean of sigma: the indexer's score already sums over heads,
  so each query row carries one sigma and the mean is that value;
* (A.8) tau = the q-quantile of sigma over every row of the call (one
  "layer"), trigger = sigma <= tau;
* (A.9) a triggered row keeps its top-(rho k); any other row keeps its top-k
  and pads the remaining rho k - k slots with the sentinel (-1 here).

Readings where the pages leave a step open (each listed with the others in
the design notes):
* sigma is formed in fp32 from the fp32 scores, as the kernel does: the
  trigger is an integer decision taken from floating point, so both sides take
  it in the kernel's precision.  0/0 (the first k+1 scores all equal) counts as
  sigma = 0: the cut falls inside a tie, the most ambiguous case;
* a row with at most k candidates has no (k+1)-th score: sigma is undefined
  (NaN), the row never triggers and already holds its whole prefix;
* the quantile is the empirical (inverse-CDF) one over the rows with a
  defined sigma: tau is the ceil(q n)-th smallest of those n values, q n
  formed as an fp64 product (an fp32 q such as 0.4f would make
  ceil(0.4f * 50) = 21); with ceil(q n) = 0 nothing triggers.  Ties at tau
  all trigger;
* selected positions are listed in ascending order, as everywhere else.

No blocking, no streaming: every row is fully sorted.
"""
from __future__ import annotations

import math

import numpy as np


def cutoff_margin(scores, k: int) -> np.float32:
    """sigma of one row from its fp32 scores (any order); NaN with <= k entries."""
    s = np.sort(np.asarray(scores, np.float32))[::-1]
    if len(s) < k + 1:
        return np.float32(np.nan)
    num = np.float32(s[k - 1] - s[k])
    den = np.float32(s[0] - s[k])
    if den > 0:
        return np.float32(num / den)
    return np.float32(0.0)


def quantile_threshold(sigma, qfrac: float):
    """(tau, r): the r-th smallest defined sigma, r = ceil(q n); tau None when r = 0."""
    s = np.asarray(sigma, np.float32)
    d = np.sort(s[~np.isnan(s)])
    r = int(math.ceil(float(qfrac) * len(d)))
    r = min(r, len(d))
    if r <= 0:
        return None, 0
    return np.float32(d[r - 1]), r


def ranked(scores, pos=None) -> np.ndarray:
    """Positions ordered by (score desc, position asc)."""
    s = np.asarray(scores, np.float64)
    p = np.arange(len(s)) if pos is None else np.asarray(pos)
    return p[np.lexsort((p, -s))]


def adaptive_select(score_rows, k: int, rho: int, qfrac: float):
    """The rule on given fp32 score rows (row t: scores of positions 0..n_t-1).

    Returns (idx [T, rho k] int32, sigma [T] float32, trigger [T] bool, tau)."""
    T = len(score_rows)
    width = rho * k
    sigma = np.array([cutoff_margin(r, k) for r in score_rows], np.float32)
    tau, _ = quantile_threshold(sigma, qfrac)
    trigger = np.zeros(T, bool)
    if tau is not None:
        trigger = ~np.isnan(sigma) & (sigma <= tau)
    out = np.full((T, width), -1, np.int32)
    for t, row in enumerate(score_rows):
        keep = width if trigger[t] else k
        sel = np.sort(ranked(np.asarray(row, np.float32))[:keep])
        out[t, :len(sel)] = sel
    return out, sigma, trigger, tau


def adaptive_topk(q, k, w, cu_seqlens, topk: int, rho: int, qfrac: float, threads=None):
    """End to end: the oracle's double scores of every row, rounded to fp32,
    then the rule above.  Small inputs only (every row is scored in full)."""
    from concurrent.futures import ThreadPoolExecutor
    import os

    from . import score_row

    cu = np.asarray(cu_seqlens, np.int64)
    jobs = []
    for b in range(len(cu) - 1):
        for t in range(int(cu[b + 1] - cu[b])):
            jobs.append((int(cu[b]) + t, int(cu[b]), t + 1))
    with ThreadPoolExecutor(max_workers=threads or os.cpu_count() or 1) as ex:
        rows = list(ex.map(lambda j: score_row(q, k, w, *j).astype(np.float32), jobs))
    return adaptive_select(rows, topk, rho, qfrac)
