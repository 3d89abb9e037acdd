"""Helpers shared by the GPU parity tests (numpy <-> torch, comparisons)."""
from __future__ import annotations

import numpy as np

import oracle as O


def to_dev(a: np.ndarray, dev="cuda"):
    import torch
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def recall(got: np.ndarray, want: np.ndarray) -> float:
    got = got.reshape(-1, got.shape[-1])
    want = want.reshape(-1, want.shape[-1])
    inter = tot = 0
    for a, b in zip(got, want):
        sb = set(b[b >= 0].tolist())
        inter += len(set(a[a >= 0].tolist()) & sb)
        tot += len(sb)
    return inter / max(tot, 1)


def check_rows_wellformed(idx: np.ndarray, bounds, k: int):
    """ascending, unique, inside [0, bound], count = min(k, bound+1), -1 padded."""
    for row, bnd in zip(idx.reshape(-1, k), bounds):
        sel = row[row >= 0]
        n = min(k, bnd + 1)
        assert len(sel) == n, (len(sel), n)
        assert (row[n:] == -1).all()
        assert (sel <= bnd).all()
        assert (np.diff(sel) > 0).all()


def check_scores(gpu: np.ndarray, ora: np.ndarray, rtol=1e-3):
    """|I_gpu - I_ora| <= rtol * max(|I_ora|, 1e-3 * row max): the tolerance of
    bf16/fp32 inputs with fp32 accumulation against the double oracle."""
    gpu = np.asarray(gpu, np.float64)
    ora = np.asarray(ora, np.float64)
    assert np.isfinite(gpu).all(), "non-finite GPU score (an entry was not written)"
    m = np.abs(ora).max() if ora.size else 0.0
    tol = rtol * np.maximum(np.abs(ora), 1e-3 * m)
    bad = np.abs(gpu - ora) > tol
    assert not bad.any(), f"{bad.sum()} scores off, worst {np.max(np.abs(gpu - ora) - tol)}"


def score_rows(jobs, threads=16):
    """Oracle score rows for a list of (q, k, w, q_row, key0, n) jobs, in parallel
    (the oracle call releases the interpreter lock)."""
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=threads) as ex:
        return list(ex.map(lambda j: O.score_row(*j), jobs))


def reselect(scores_f32: np.ndarray, k: int, pos=None) -> np.ndarray:
    """The oracle's selection rule applied to scores the GPU exported."""
    return O.select(np.asarray(scores_f32, np.float32).astype(np.float64), k, pos)
