"""Seeded synthetic inputs for the indexer + top-k workloads.

This module only draws inputs; it holds none of the indexer's arithmetic.
The CUDA path and the CPU oracle both receive what it returns.

Recipes (one numpy PCG64 stream per tensor, derived from (seed, tensor id)):
  * keys: k[s] ~ N(0, 1) per element.  A fixed fraction of positions
    (exactly floor(frac * L), chosen uniformly without replacement) are
    "planted": their component along a seeded unit vector u is replaced by
    4 * sqrt(d), i.e. k[s] <- z - (z . u) u + 4 sqrt(d) u.  This gives the
    long-tailed score profile the PIVOT page describes (observation O3).
  * queries: AR(1) along positions, independently per (head, dim):
    q[0] = e[0], q[t] = rho q[t-1] + sqrt(1 - rho^2) e[t], e ~ N(0, 1).
    Neighbouring queries are then similar (observation O1).
  * w[t, j] ~ Uniform(0, 1) / H.
  * bf16 tensors are rounded to nearest even from fp32 and returned as
    uint16 bit patterns; fp32 tensors as float32.
  * the small fp32 case draws q and k i.i.d. N(0, std = 1/sqrt(d)) and
    w ~ Uniform(0, 1).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

# tensor ids for the per-tensor random streams
_Q, _K, _W, _PLANT_POS, _PLANT_DIR, _DEC_Q, _DEC_W = range(7)


def rng_for(seed: int, tensor_id: int, sub: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tensor_id, sub])))


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def keys(L: int, d: int, planted_frac: float, seed: int, sub: int = 0, scale: float = 4.0,
         bf16: bool = True) -> np.ndarray:
    """[L, d] keys; planted positions carry a u-component of scale*sqrt(d)."""
    z = rng_for(seed, _K, sub).standard_normal((L, d), dtype=np.float32)
    n_plant = int(np.floor(planted_frac * L))
    if n_plant > 0:
        pos = rng_for(seed, _PLANT_POS, sub).choice(L, size=n_plant, replace=False)
        u = rng_for(seed, _PLANT_DIR, 0).standard_normal(d).astype(np.float64)
        u /= np.linalg.norm(u)
        zp = z[pos].astype(np.float64)
        zp = zp - np.outer(zp @ u, u) + scale * np.sqrt(d) * u
        z[pos] = zp.astype(np.float32)
    return bf16_bits(z) if bf16 else z


def queries_ar1(L: int, H: int, d: int, rho: float, seed: int, sub: int = 0, bf16: bool = True,
                col_block: int = 512, threads: int = 8) -> np.ndarray:
    """[L, H, d] AR(1) queries along positions.  The H*d columns are drawn in
    blocks of `col_block`, each block from its own stream (seed, sub, block),
    so blocks are generated in parallel; within a block the recurrence runs
    along positions."""
    from concurrent.futures import ThreadPoolExecutor
    from scipy.signal import lfilter

    HD = H * d
    out = np.empty((L, HD), np.uint16 if bf16 else np.float32)
    if L == 0:
        return out.reshape(0, H, d)
    s = float(np.sqrt(1.0 - rho * rho))

    def block(c0):
        c1 = min(HD, c0 + col_block)
        # drawn as [columns, positions] so the recurrence runs along contiguous memory
        e = rng_for(seed, _Q, sub * 1000003 + c0 // col_block).standard_normal((c1 - c0, L), dtype=np.float32)
        e[:, 0] /= np.float32(s)  # so that q[0] = e[0]
        y = lfilter(np.array([s], np.float32), np.array([1.0, -rho], np.float32), e, axis=1)
        y = np.ascontiguousarray(y.T, dtype=np.float32)
        out[:, c0:c1] = bf16_bits(y) if bf16 else y

    with ThreadPoolExecutor(max_workers=max(1, threads)) as ex:
        list(ex.map(block, range(0, HD, col_block)))
    return out.reshape(L, H, d)


def weights(L: int, H: int, seed: int, sub: int = 0, scale: Optional[float] = None) -> np.ndarray:
    sc = (1.0 / H) if scale is None else scale
    return (rng_for(seed, _W, sub).random((L, H), dtype=np.float32) * np.float32(sc)).astype(np.float32)


@dataclass
class Prefill:
    """A packed prefill batch: q [T,H,d], k [T,d], w [T,H], cu_seqlens [R+1]."""
    name: str
    q: np.ndarray
    k: np.ndarray
    w: np.ndarray
    cu_seqlens: np.ndarray
    topk: int
    g: int = 4
    c: int = 4096
    meta: dict = field(default_factory=dict)

    @property
    def T(self):
        return self.q.shape[0]

    @property
    def H(self):
        return self.q.shape[1]

    @property
    def d(self):
        return self.q.shape[2]

    @property
    def bf16(self):
        return self.q.dtype == np.uint16


@dataclass
class Decode:
    """One decode step: q [B,G,H,d], kcache [B,n_max,d], w [B,G,H], kv_len [B]."""
    name: str
    q: np.ndarray
    kcache: np.ndarray
    w: np.ndarray
    kv_len: np.ndarray
    topk: int
    c: int = 4096
    meta: dict = field(default_factory=dict)


def prefill(lengths, H=64, d=128, topk=2048, rho=0.95, planted=0.01, seed=0, g=4, c=4096,
            name="prefill") -> Prefill:
    """Packed requests of the given lengths; each request has its own key and
    query streams (sub-stream = request index)."""
    lengths = [int(x) for x in lengths]
    cu = np.zeros(len(lengths) + 1, np.int32)
    cu[1:] = np.cumsum(lengths)
    qs, ks, ws = [], [], []
    for i, n in enumerate(lengths):
        qs.append(queries_ar1(n, H, d, rho, seed, sub=i))
        ks.append(keys(n, d, planted, seed, sub=i))
        ws.append(weights(n, H, seed, sub=i))
    q = np.concatenate(qs) if len(qs) > 1 else qs[0]
    k = np.concatenate(ks) if len(ks) > 1 else ks[0]
    w = np.concatenate(ws) if len(ws) > 1 else ws[0]
    return Prefill(name, q, k, w, cu, topk, g, c,
                   dict(lengths=lengths, rho=rho, planted=planted, seed=seed))


def small_fp32(L=2048, H=4, d=64, topk=64, seed=0) -> Prefill:
    """The fp32 dense case: q, k i.i.d. N(0, std 1/sqrt(d)); w ~ U(0,1)."""
    sd = np.float32(1.0 / np.sqrt(d))
    q = rng_for(seed, _Q).standard_normal((L, H, d), dtype=np.float32) * sd
    k = rng_for(seed, _K).standard_normal((L, d), dtype=np.float32) * sd
    w = rng_for(seed, _W).random((L, H), dtype=np.float32)
    cu = np.array([0, L], np.int32)
    return Prefill("fp32_L2048_H4_d64_k64", q.astype(np.float32), k.astype(np.float32), w, cu, topk,
                   meta=dict(lengths=[L], seed=seed))


def decode(B=64, n=131072, G=2, H=64, d=128, topk=2048, c=4096, rho=0.95, planted=0.01, seed=0,
           kv_len=None, n_max=None, name="decode") -> Decode:
    """Decode step over a contiguous cache [B, n_max, d]; request b's keys use
    the key recipe with sub-stream b; queries are AR(1) across the G positions."""
    from concurrent.futures import ThreadPoolExecutor

    n_max = int(n_max or n)
    kc = np.zeros((B, n_max, d), np.uint16)

    def fill(b):
        kc[b] = keys(n_max, d, planted, seed, sub=1000 + b)

    with ThreadPoolExecutor(max_workers=8) as ex:
        list(ex.map(fill, range(B)))
    e = rng_for(seed, _DEC_Q).standard_normal((B, G, H, d), dtype=np.float32)
    s = np.float32(np.sqrt(1.0 - rho * rho))
    qf = np.empty_like(e)
    qf[:, 0] = e[:, 0]
    for m in range(1, G):
        qf[:, m] = np.float32(rho) * qf[:, m - 1] + s * e[:, m]
    q = bf16_bits(qf)
    w = (rng_for(seed, _DEC_W).random((B, G, H), dtype=np.float32) * np.float32(1.0 / H)).astype(np.float32)
    if kv_len is None:
        kv_len = np.full(B, n, np.int32)
    return Decode(name, q, kc, w, np.asarray(kv_len, np.int32), topk, c,
                  dict(n=n, G=G, rho=rho, planted=planted, seed=seed))


def exact_ints(lengths, H=4, d=16, topk=8, seed=0, lo=-8, hi=8) -> Prefill:
    """Integer q, k in [lo, hi] (exact in bf16) and dyadic w in {0, 1/4, 1/2, 1}:
    every product and partial sum is exact in fp32 and in double, and ties are
    frequent, which exercises the lower-index tie rule."""
    lengths = [int(x) for x in lengths]
    T = sum(lengths)
    cu = np.zeros(len(lengths) + 1, np.int32)
    cu[1:] = np.cumsum(lengths)
    q = rng_for(seed, _Q).integers(lo, hi + 1, size=(T, H, d)).astype(np.float32)
    k = rng_for(seed, _K).integers(lo, hi + 1, size=(T, d)).astype(np.float32)
    w = rng_for(seed, _W).choice(np.array([0.0, 0.25, 0.5, 1.0], np.float32), size=(T, H))
    return Prefill("exact_ints", bf16_bits(q), bf16_bits(k), w.astype(np.float32), cu, topk,
                   meta=dict(lengths=lengths, seed=seed))


# ---------------------------------------------------------------- configs
# The five workload shapes (sizes as stated in their recipes).

def cfg_fp32_small(seed=0):
    return small_fp32(seed=seed)


def cfg_dense_16k(seed=0, L=16384):
    return prefill([L], rho=0.95, planted=0.01, seed=seed, name=f"dense_L{L}_H64_d128_k2048")


def cfg_pivot_64k(seed=0, L=65536):
    return prefill([L], rho=0.95, planted=0.01, seed=seed, g=4, c=4096,
                   name=f"pivot_g4_c4096_L{L}_H64_d128_k2048")


def cfg_long_single(seed=0, L=131072):
    return prefill([L], rho=0.98, planted=0.005, seed=seed, g=16, c=4096,
                   name=f"dense_L{L}_H64_d128_k2048")


def cfg_long_packed(seed=0, n=65536):
    return prefill([n, n], rho=0.98, planted=0.005, seed=seed, g=16, c=4096,
                   name=f"packed_2x{n}_refine_g16_c4096_H64_d128_k2048")


def cfg_decode(seed=0, B=64, n=131072):
    return decode(B=B, n=n, G=2, seed=seed, name=f"decode_B{B}_n{n}_G2_H64_d128_k2048_c4096")
