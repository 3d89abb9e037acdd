#!/usr/bin/env python
"""Benchmark of the lightning indexer + top-k on B200.

One step = one pass of the whole hot path over the long-prefill batch
(131072 tokens, H=64, d=128, k=2048, bf16 q/k, fp32 w): the dense
indexer + top-k over the batch as ONE 131072-token request, and PIVOT
Refine (g=16, c=4096) over the same tokens as TWO packed 65536-token
requests (proxy build, proxy scan, candidate select, member re-score,
member select).  `value` = query rows ranked per second (2 * 131072 per
step, whole job).  The decode step (B=64 requests x 131072-token caches,
G=2 MTP queries, dense and Refine c=4096, and dense over the same cache
scattered into 64-key pages behind a block table) is timed after it and
reported under "decode" as HBM GB/s of the cache scan.  The block
pre-filter variant of Refine (candidates from 64-key block means) runs on
the same packed batch under "block_prefilter", outside the step, and the
token-sparse attention (absorbed-MLA shapes: 128 heads, 576/512 dims) over
the dense selections of the last 16384 query rows under "sparse_attn".
The dense pass with the cutoff-margin adaptive budget (rho = 2, q = 0.4:
rows whose margin is in the bottom 40% keep 4096 positions, the others
2048) runs on the single request under "adaptive".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun): every rank runs its own batch (seed = rank): weak
scaling with no collective on the data path; the time is the max over
ranks of the device time.  --impl reference runs the CPU oracle (the
plain double-precision restatement) on the host cores on a bounded sample
of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

L_TOK, H, D, TOPK, G_REF, C_REF = 131072, 64, 128, 2048, 16, 4096
DEC_B, DEC_N, DEC_G = 64, 131072, 2
METRIC = "indexer+top-k queries/s and TFLOP/s (% bf16 TC peak); decode HBM GB/s @ L=128K"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=5)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-decode", action="store_true")
    p.add_argument("--no-block", action="store_true")
    p.add_argument("--no-attn", action="store_true")
    p.add_argument("--no-adaptive", action="store_true")
    p.add_argument("--attn-rows", type=int, default=16384)
    p.add_argument("--cpu-rows", type=int, default=512, help="oracle sample rows (dense + refine) per CPU step")
    p.add_argument("--no-configs", action="store_true",
                   help="skip the 16384-token dense and 65536-token PIVOT (g=4, c=4096) legs")
    p.add_argument("--crossover", action="store_true",
                   help="only time dense, Reuse and Refine on single requests of 1K..64K tokens (g=4, 16)")
    p.add_argument("--split", action="store_true",
                   help="N>1: split the one request across the ranks (zig-zag rows, strong scaling) instead of "
                        "giving each rank its own batch; times the main step only")
    p.add_argument("--skip-study", action="store_true",
                   help="CPU only: fraction of (row block, key tile) pairs a per-tile score bound could skip")
    p.add_argument("--dense-below", type=int, default=0,
                   help="--crossover: also time PIVOT with this guardrail threshold (0 = without; -1 = the "
                        "per-mode thresholds of GUARD_BELOW)")
    p.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline")
    p.add_argument("--tokens", type=int, default=L_TOK,
                   help="batch length (profiling runs use a smaller case; the bench line uses 131072)")
    p.add_argument("--only", default="all", choices=["all", "dense", "refine", "attn"],
                   help="profiling runs: time one half of the step only, or only the sparse attention leg "
                        "(its selections then come from an untimed dense call)")
    return p.parse_args()


def dense_flops_single(L=L_TOK):
    return 2.0 * H * D * L * (L + 1) / 2.0


def causal_flops(lengths):
    return sum(2.0 * H * D * n * (n + 1) / 2.0 for n in lengths)


def proxy_pairs(n, g):
    # sum over proxies of (t_last + 1), request of n tokens
    tot = 0
    for i in range((n + g - 1) // g):
        tot += min((i + 1) * g, n)
    return tot


SCORE_SOURCES = ["score_tc.cu", "tc.cuh", "common.cuh", "plan.cuh"]
# the parts of internal.h the score kernel reads: its constants, the plan
# layout and its argument struct (other declarations there do not change it)
SCORE_DECLS = [r"constexpr int (RB|KT|kMaxLen|kBlockShift|kBlockN) = [^;]*;",
               r"struct PlanLayout \{.*?\n\};", r"enum Sink \{[^}]*\};", r"struct ScoreArgs \{.*?\n\};"]


def score_sources_sha():
    """sha256 over the sources of the dense score kernel (to tell whether a
    recorded ncu traffic figure still describes the kernel that runs): its
    source files whole, and from internal.h the declarations it uses."""
    import hashlib
    import re
    csrc = os.path.join(ROOT, "sparse_attention_indexer_05_b200", "csrc")
    h = hashlib.sha256()
    for f in SCORE_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    with open(os.path.join(csrc, "internal.h")) as fh:
        text = fh.read()
    for pat in SCORE_DECLS:
        found = re.findall(pat, text, flags=re.S) if "struct" in pat or "enum" in pat else \
            [m.group(0) for m in re.finditer(pat, text)]
        if not found:
            raise RuntimeError(f"declaration not found in internal.h: {pat}")
        for m in found:
            h.update((m if isinstance(m, str) else m[0]).encode())
    return h.hexdigest()


def recorded_traffic(L):
    """DRAM bytes (read + write) of one dense score launch from the committed
    ncu capture, or None when the kernel changed since or the size differs."""
    path = os.path.join(ROOT, "profiles", "score_tc_dense_L131072_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    if rec.get("sources_sha256") != score_sources_sha() or rec.get("tokens") != L:
        return None
    return rec["dram_bytes_read"] + rec["dram_bytes_write"]


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            m = json.load(f)
        return m.get("bf16_tflops", 1590.0), m.get("bf16_tflops_sustained", 1400.0), m.get("hbm_gbs", 6650.0), "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = float(parts[2])
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def trace_report(lib):
    import ctypes
    buf = ctypes.create_string_buffer(1 << 16)
    n = lib.idx_trace_report(buf, len(buf))
    out = {}
    for line in buf.value.decode().splitlines():
        name, cnt, ms = line.split()
        out[name] = (int(cnt), float(ms))
    return n, out


def to_dev(a, dev):
    import torch
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def pinned(a):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16) if a.dtype == np.uint16 else np.ascontiguousarray(a))
    return t.pin_memory()



def timed_calls(fn, warmup, steps, lib, barrier, max_over_ranks):
    """Run fn warmup times, then time `steps` calls with CUDA events on the
    current stream (library tracer on); returns (ms per call, max over ranks,
    and the per-kernel split {name: (launches, ms per call)})."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    lib.idx_trace_enable(1)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    lib.idx_trace_enable(0)
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1) / steps)
    _, tr = trace_report(lib)
    return ms, {n: (c, t / steps) for n, (c, t) in tr.items()}


def kernel_ms(split, suffix, prefix=None):
    return sum(t for n, (c, t) in split.items()
               if n.endswith(suffix) and (prefix is None or n.startswith(prefix + "/")))


def run_configs(args, dev, lib, barrier, max_over_ranks, rank, bf16_sus):
    """The 16384-token dense case and the 65536-token PIVOT case (g=4,
    c=4096: dense, Reuse and Refine on the same inputs), each with the
    score kernel's rate against the sustained bf16 peak."""
    import torch

    import sparse_attention_indexer_05_b200 as idx
    from sparse_attention_indexer_05_b200 import multirank as M
    from sparse_attention_indexer_05_b200 import workloads as W
    out = {}

    def dense_leg(P, label):
        T = P.T
        q, k, w = to_dev(P.q, dev), to_dev(P.k, dev), to_dev(P.w, dev)
        cu = to_dev(P.cu_seqlens, dev)
        S = len(P.cu_seqlens) - 1
        o = torch.empty(T, TOPK, dtype=torch.int32, device=dev)
        ws = torch.empty(idx.dense_workspace_size(T, H, D, TOPK, S), dtype=torch.uint8, device=dev)
        ms, sp = timed_calls(lambda: idx.dense_topk(q, k, w, cu, TOPK, out_idx=o, workspace=ws), args.warmup,
                             args.steps, lib, barrier, max_over_ranks)
        assert idx.device_status(ws) == "IDX_OK"
        sms = kernel_ms(sp, "score_tc", "dense")
        fl = causal_flops(P.meta["lengths"])
        tf = fl / (sms / 1000.0) / 1e12 if sms > 0 else None
        del ws
        return {"workload": label, "ms_per_call": ms, "queries_per_s": T / (ms / 1000.0),
                "score_tc": {"ms": sms, "flops": fl, "tflops": tf, "frac_bf16_sustained": (tf / bf16_sus) if tf else None},
                "kernels_ms": {n: t for n, (c, t) in sp.items()}}, (q, k, w, cu, o)

    # the small fp32 case (L = 2048, H = 4, d = 64, k = 64): the CUDA-core path
    P1 = W.cfg_fp32_small(seed=M.rank_seed(rank))
    q1, k1, w1, c1 = (to_dev(P1.q, dev), to_dev(P1.k, dev), to_dev(P1.w, dev), to_dev(P1.cu_seqlens, dev))
    o1s = torch.empty(P1.T, P1.topk, dtype=torch.int32, device=dev)
    ws1s = torch.empty(idx.dense_workspace_size(P1.T, P1.H, P1.d, P1.topk, 1, torch.float32), dtype=torch.uint8,
                       device=dev)
    ms1, sp1 = timed_calls(lambda: idx.dense_topk(q1, k1, w1, c1, P1.topk, out_idx=o1s, workspace=ws1s), args.warmup,
                           max(args.steps, 20), lib, barrier, max_over_ranks)
    assert idx.device_status(ws1s) == "IDX_OK"
    fl1 = 2.0 * P1.H * P1.d * P1.T * (P1.T + 1) / 2.0
    s1 = kernel_ms(sp1, "score_simt", "dense")
    out["dense_fp32_2048"] = {"workload": "dense_L2048_H4_d64_k64_fp32 (CUDA-core path)", "ms_per_call": ms1,
                              "queries_per_s": P1.T / (ms1 / 1000.0), "score_simt_ms": s1,
                              "score_simt_tflops_fp32": fl1 / (s1 / 1000.0) / 1e12 if s1 > 0 else None,
                              "kernels_ms": {n: t for n, (c, t) in sp1.items()}}
    del P1, q1, k1, w1, c1, o1s, ws1s
    # dense L = 16384 (rho 0.95, 1% planted keys)
    P2 = W.cfg_dense_16k(seed=M.rank_seed(rank))
    out["dense_16384"], _ = dense_leg(P2, "dense_L16384_H64_d128_k2048")
    del P2
    # PIVOT L = 65536, g = 4, c = 4096 against dense on the same inputs
    P3 = W.cfg_pivot_64k(seed=M.rank_seed(rank))
    res, (q, k, w, cu, o) = dense_leg(P3, "dense_L65536_H64_d128_k2048")
    leg = {"dense": res}
    T = P3.T
    for mode in ("reuse", "refine"):
        ws = torch.empty(idx.pivot_workspace_size(T, H, D, TOPK, 1, 4, 4096, mode), dtype=torch.uint8, device=dev)
        ms, sp = timed_calls(lambda: idx.pivot_topk(q, k, w, cu, TOPK, 4, 4096, mode, out_idx=o, workspace=ws),
                             args.warmup, args.steps, lib, barrier, max_over_ranks)
        assert idx.device_status(ws) == "IDX_OK"
        sms = kernel_ms(sp, "score_tc", mode)
        fl = 2.0 * H * D * proxy_pairs(T, 4)
        tf = fl / (sms / 1000.0) / 1e12 if sms > 0 else None
        leg[mode] = {"ms_per_call": ms, "queries_per_s": T / (ms / 1000.0),
                     "speedup_vs_dense": res["ms_per_call"] / ms,
                     "proxy_scan": {"ms": sms, "flops": fl, "tflops": tf,
                                    "frac_bf16_sustained": (tf / bf16_sus) if tf else None},
                     "kernels_ms": {n: t for n, (c, t) in sp.items()}}
        del ws
    leg["workload"] = "pivot_L65536_g4_c4096_H64_d128_k2048 (dense, Reuse and Refine on the same inputs)"
    out["pivot_65536_g4_c4096"] = leg
    del q, k, w, cu, o, P3
    torch.cuda.empty_cache()
    return out



def run_skip_study(args):
    """Could the score kernel skip whole key tiles?  For sampled row blocks
    (8 consecutive queries, the kernel's unit) of the 16384-, 65536- and
    131072-token workloads, walk the key tiles (128 keys) in the kernel's
    ascending order and keep each row's exact running k-th best score tau
    (the best threshold any one-pass filter can hold; the kernel's is lower).
    A tile can be skipped only if, for all 8 rows, an upper bound on every
    score in the tile is below tau.  Two bounds are measured:
      box:  per head, max over the tile of q . k <= sum_i max(q_i kmin_i,
            q_i kmax_i) from the tile's per-dimension key range; then
            sum_j w_j max(0, bound_j);
      max:  the tile's true largest score per row (the tightest bound there
            is; no kernel can compute it without doing the work it would
            skip).
    Scores are computed here in fp32 from the bf16 inputs (a study, not a
    parity reference)."""
    from sparse_attention_indexer_05_b200 import workloads as W
    rng = np.random.default_rng(11)
    out = {}
    cases = [("dense_L16384_rho0.95_planted1%", lambda: W.cfg_dense_16k(seed=0)),
             ("pivot_L65536_rho0.95_planted1%", lambda: W.cfg_pivot_64k(seed=0)),
             ("long_L131072_rho0.98_planted0.5%", lambda: W.cfg_long_single(seed=0))]
    for name, make in cases:
        P = make()
        L = P.T
        q = W.bf16_to_f32(P.q)
        kk = W.bf16_to_f32(P.k)
        w = P.w.astype(np.float32)
        nblk = 24
        starts = np.sort(rng.choice(np.arange(TOPK // 8 + 1, L // 8), size=nblk, replace=False)) * 8
        pairs = skip_box = skip_max = row_pairs = row_skip_max = 0
        ratios = []
        for t0 in starts:
            rows = np.arange(t0, t0 + 8)
            t_hi = int(rows[-1])
            ntiles = t_hi // 128 + 1
            Kp = kk[:(ntiles * 128)]
            sc = np.zeros((8, ntiles * 128), np.float32)
            for c0 in range(0, ntiles * 128, 16384):
                dots = np.einsum("rhd,sd->rhs", q[rows], Kp[c0:c0 + 16384], optimize=True)
                sc[:, c0:c0 + 16384] = np.einsum("rh,rhs->rs", w[rows], np.maximum(dots, 0.0))
            pos = np.arange(ntiles * 128)
            sc = np.where(pos[None, :] <= rows[:, None], sc, -np.inf)
            kt = Kp.reshape(ntiles, 128, D)
            kmin, kmax = kt.min(axis=1), kt.max(axis=1)           # [ntiles, D]
            qr = q[rows]                                          # [8, H, D]
            hb = np.maximum(np.einsum("rhd,td->rht", np.maximum(qr, 0), kmax) +
                            np.einsum("rhd,td->rht", np.minimum(qr, 0), kmin), 0.0)
            box = np.einsum("rh,rht->rt", w[rows], hb)            # [8, ntiles]
            tmax = sc.reshape(8, ntiles, 128).max(axis=2)         # [8, ntiles]
            # exact running k-th best before each tile (the top-k kept as a set)
            tau = np.full((8, ntiles), -np.inf, np.float32)
            for r in range(8):
                top = sc[r, :TOPK].copy()
                for j in range(TOPK // 128, ntiles):
                    tau[r, j] = np.partition(top, 0)[0] if np.isfinite(top).all() else -np.inf
                    both = np.concatenate([top, sc[r, j * 128:(j + 1) * 128]])
                    top = np.partition(both, len(both) - TOPK)[len(both) - TOPK:]
            j0 = TOPK // 128
            pairs += ntiles - j0
            skip_box += int(np.all(box[:, j0:] < tau[:, j0:], axis=0).sum())
            skip_max += int(np.all(tmax[:, j0:] < tau[:, j0:], axis=0).sum())
            row_pairs += tmax[:, j0:].size
            row_skip_max += int((tmax[:, j0:] < tau[:, j0:]).sum())
            ok = np.isfinite(tmax[:, j0:]) & (tmax[:, j0:] > 0)
            ratios.append((box[:, j0:][ok] / tmax[:, j0:][ok]))
        out[name] = {"row_blocks": nblk, "tile_pairs": pairs, "skippable_box_bound": skip_box / pairs,
                     "skippable_exact_tile_max": skip_max / pairs,
                     "row_tile_pairs_below_tau_exact_tile_max": row_skip_max / row_pairs,
                     "box_bound_over_true_tile_max_median": float(np.median(np.concatenate(ratios)))}
        print(json.dumps({name: out[name]}), flush=True)
        del P, q, kk
    print(json.dumps({"skip_study": out, "unit": "fraction of causal (row block of 8, key tile of 128) pairs "
                      "after the first k keys", "topk": TOPK}))
    return 0

# Guardrail thresholds (dense_below) for this build on B200, from the
# crossover sweep (bench.py --crossover): the prefix length below which a
# group's PIVOT work costs more than its members' dense work.  Reuse only pays
# its fixed per-call costs at short lengths; Refine pays the candidate
# select, the key pack and the re-score per member.
GUARD_BELOW = {("reuse", 4): 2048, ("reuse", 16): 2048, ("refine", 4): 24576, ("refine", 16): 16384}


def run_crossover(args):
    """Dense against PIVOT Reuse and Refine (c = 4096) on one request of
    L tokens, L = 1K .. 64K, g = 4 and 16: the inputs of the 65536-token
    recipe cut to their first L tokens (a prefix of a request is a request)."""
    import torch

    import sparse_attention_indexer_05_b200 as idx
    from sparse_attention_indexer_05_b200 import _native as N
    from sparse_attention_indexer_05_b200 import workloads as W
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    lib = N.lib()
    P = W.cfg_pivot_64k(seed=0)
    qa, ka, wa = to_dev(P.q, dev), to_dev(P.k, dev), to_dev(P.w, dev)
    guard = args.dense_below
    rows = []
    for L in (1024, 2048, 4096, 8192, 12288, 16384, 24576, 32768, 49152, 65536):
        q, k, w = qa[:L].contiguous(), ka[:L].contiguous(), wa[:L].contiguous()
        cu = torch.tensor([0, L], dtype=torch.int32, device=dev)
        o = torch.empty(L, TOPK, dtype=torch.int32, device=dev)
        ws = torch.empty(idx.dense_workspace_size(L, H, D, TOPK, 1), dtype=torch.uint8, device=dev)
        dms, _ = timed_calls(lambda: idx.dense_topk(q, k, w, cu, TOPK, out_idx=o, workspace=ws), 2, 5, lib,
                             lambda: None, float)
        row = {"L": L, "dense_ms": dms}
        del ws
        for g in (4, 16):
            for mode in ("reuse", "refine"):
                gd = GUARD_BELOW[(mode, g)] if guard < 0 else guard
                for db in ((0, gd) if gd else (0,)):
                    kw = {"dense_below": db} if db else {}
                    ws = torch.empty(idx.pivot_workspace_size(L, H, D, TOPK, 1, g, 4096, mode, **kw),
                                     dtype=torch.uint8, device=dev)
                    ms, _ = timed_calls(lambda: idx.pivot_topk(q, k, w, cu, TOPK, g, 4096, mode, out_idx=o,
                                                               workspace=ws, **kw),
                                        2, 5, lib, lambda: None, float)
                    key = f"{mode}_g{g}" + (f"_guard{db}" if db else "")
                    row[key + "_ms"] = ms
                    row[key + "_speedup"] = dms / ms
                    del ws
        rows.append(row)
        print(json.dumps(row), flush=True)
    print(json.dumps({"crossover": rows, "c": 4096, "topk": TOPK,
                      "workload": "prefixes of the 65536-token recipe (rho 0.95, 1% planted keys), one request"}))
    return 0

# ---------------------------------------------------------------- CPU oracle
def oracle_sample(P, nrows, seed=0):
    """Time the oracle on `nrows` rows of the step (half dense on the single
    request, half Refine on the packed requests); returns (rows/s, seconds,
    threads, description)."""
    import oracle as O
    rng = np.random.default_rng(seed)
    nd = max(1, nrows // 2)
    nr = max(1, nrows - nd)
    # stratified by position so the sample's mean prefix matches the batch's
    dense_rows = np.sort((np.arange(nd) + rng.random(nd)) * (L_TOK / nd)).astype(np.int64)
    ref_rows = np.sort((np.arange(nr) + rng.random(nr)) * (L_TOK / nr)).astype(np.int64)
    cu1 = np.array([0, L_TOK], np.int32)
    cu2 = np.array([0, L_TOK // 2, L_TOK], np.int32)
    threads = os.cpu_count() or 1
    t0 = time.perf_counter()
    O.dense_topk(P.q, P.k, P.w, cu1, TOPK, rows=dense_rows, threads=threads)
    O.pivot_topk(P.q, P.k, P.w, cu2, TOPK, G_REF, C_REF, O.REFINE, rows=ref_rows, threads=threads)
    dt = time.perf_counter() - t0
    desc = (f"{nd} dense rows (single 131072-token request) + {nr} Refine g=16 c=4096 member rows "
            f"(2x65536 packed), stratified by position, seed {seed}; the rate is extrapolated to the "
            f"step's {2 * L_TOK} rows (a stratified sample has the batch's mean prefix)")
    return (nd + nr) / dt, dt, threads, desc


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from sparse_attention_indexer_05_b200 import workloads as W
    P = W.cfg_long_single(seed=0)
    times, rows = [], 0
    for i in range(args.warmup + args.steps):
        v, dt, threads, desc = oracle_sample(P, max(2, args.cpu_rows // 3), seed=i)
        if i >= args.warmup:
            times.append(dt)
            rows += max(2, args.cpu_rows // 3)
    val = rows / sum(times)
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "queries/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * sum(times) / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": "long_prefill_131072_dense+refine_g16_c4096", "tokens": L_TOK, "H": H, "d": D,
                   "topk": TOPK},
        "cpu_baseline": {"value": val, "unit": "queries/s", "cores": threads, "kind": "oracle",
                         "sample": f"per step: {desc}"},
        "e2e": {"value": val, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# --------------------------------------------------------------- GPU bench
def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.crossover:
        return run_crossover(args)
    if args.skip_study:
        return run_skip_study(args)
    import torch

    import sparse_attention_indexer_05_b200 as idx
    from sparse_attention_indexer_05_b200 import _native as N
    from sparse_attention_indexer_05_b200 import multirank as M
    from sparse_attention_indexer_05_b200 import workloads as W

    rank, world, local = M.init("nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    lib = N.lib()

    def barrier():
        M.barrier(dev)

    def max_over_ranks(x):
        return M.max_over_ranks(x, dev)

    L = args.tokens
    split = args.split and world > 1
    # split: every rank holds the same request (seed 0) and ranks only its rows
    P = W.cfg_long_single(seed=0 if split else M.rank_seed(rank), L=L)
    cu1_h = np.array([0, L], np.int32)
    cu2_h = np.array([0, L // 2, L], np.int32)
    q, k, w = to_dev(P.q, dev), to_dev(P.k, dev), to_dev(P.w, dev)
    cu1, cu2 = to_dev(cu1_h, dev), to_dev(cu2_h, dev)
    do_dense = args.only in ("all", "dense")
    do_refine = args.only in ("all", "refine")
    attn_only = args.only == "attn"
    ws1 = torch.empty(idx.dense_workspace_size(L, H, D, TOPK, 1) if do_dense else 256, dtype=torch.uint8,
                      device=dev)
    ws2 = torch.empty(idx.pivot_workspace_size(L, H, D, TOPK, 2, G_REF, C_REF, "refine") if do_refine else 256,
                      dtype=torch.uint8, device=dev)
    o1 = torch.empty(L, TOPK, dtype=torch.int32, device=dev)
    o2 = torch.empty(L, TOPK, dtype=torch.int32, device=dev)

    if split:
        # the rows this rank owns: zig-zag chunks of the dense request, and of
        # each packed request with whole groups
        r1 = M.zigzag_ranges(L, world, rank, align=8)
        r2 = [(lo + off, hi + off) for off in (0, L // 2)
              for lo, hi in M.zigzag_ranges(L // 2, world, rank, align=G_REF)]
    else:
        r1, r2 = [(0, L)], [(0, L)]

    def step(qq=q, kk=k, ww=w, c1=cu1, c2=cu2, oo1=o1, oo2=o2, st=None):
        if do_dense:
            for rg in r1:
                idx.dense_topk(qq, kk, ww, c1, TOPK, out_idx=oo1, workspace=ws1, stream=st, rows=rg)
        if do_refine:
            for rg in r2:
                idx.pivot_topk(qq, kk, ww, c2, TOPK, G_REF, C_REF, "refine", out_idx=oo2, workspace=ws2, stream=st,
                               rows=rg)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert (not do_dense or idx.device_status(ws1) == "IDX_OK") and \
        (not do_refine or idx.device_status(ws2) == "IDX_OK")

    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = Clocks(local)
    barrier()
    torch.cuda.synchronize()
    lib.idx_trace_enable(1)
    clocks.start()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    lib.idx_trace_enable(0)
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps)
    nlaunch, tr = trace_report(lib)
    rows_per_step = L * (int(do_dense) + int(do_refine))
    # whole job: every rank ranks its own batch, or the ranks share one
    rows_job = rows_per_step if split else world * rows_per_step
    value = rows_job / (ms / 1000.0)
    if split:  # the extra legs time independent work; the split run times the step only
        args.no_block = args.no_attn = args.no_adaptive = args.no_decode = args.no_configs = True

    bf16_peak, bf16_sus, hbm_peak, peak_src = peaks()
    n_dense, ms_dense = tr.get("dense/score_tc", (0, 0.0))
    dense_ms = ms_dense / max(1, n_dense)
    achieved = dense_flops_single(L) / (dense_ms / 1000.0) / 1e12 if dense_ms > 0 else None
    roof = {"kernel": "score_tc (dense pass)", "bound": "tensor", "achieved": achieved,
            "peak": bf16_sus, "unit": "TFLOP/s", "frac": (achieved / bf16_sus) if achieved else None,
            "traffic": recorded_traffic(L), "peak_kind": f"{peak_src} bf16 sustained (kernel timed inside a long step)",
            "flops_per_launch": dense_flops_single(L), "ms_per_launch": dense_ms}

    per_kernel = {name: {"launches": c, "ms_total": t, "ms_per_step": t / args.steps} for name, (c, t) in tr.items()}

    # ----------- Refine g=16 against dense on the same 2 x 65536 packing
    packed = None
    if args.only == "all" and not args.no_configs:
        wsp = torch.empty(idx.dense_workspace_size(L, H, D, TOPK, 2), dtype=torch.uint8, device=dev)
        pd_ms, pd_sp = timed_calls(lambda: idx.dense_topk(q, k, w, cu2, TOPK, out_idx=o1, workspace=wsp),
                                   args.warmup, args.steps, lib, barrier, max_over_ranks)
        assert idx.device_status(wsp) == "IDX_OK"
        del wsp
        pr_ms, pr_sp = timed_calls(lambda: idx.pivot_topk(q, k, w, cu2, TOPK, G_REF, C_REF, "refine", out_idx=o2,
                                                          workspace=ws2), args.warmup, args.steps, lib, barrier,
                                   max_over_ranks)
        packed = {"workload": f"packed_2x{L // 2}_g{G_REF}_c{C_REF} (dense and Refine on the same inputs)",
                  "dense_ms": pd_ms, "refine_ms": pr_ms, "speedup_refine_vs_dense": pd_ms / pr_ms,
                  "dense_score_tc_ms": kernel_ms(pd_sp, "score_tc"),
                  "refine_kernels_ms": {n: t for n, (c, t) in pr_sp.items()}}

    # --- the dense call as row chunks with a workspace sized for one chunk
    chunked = None
    if args.only == "all" and not args.no_configs and L == L_TOK:
        CH = 16384
        full_ws = idx.dense_workspace_size(L, H, D, TOPK, 1)
        ch_ws = idx.dense_workspace_size(L, H, D, TOPK, 1, max_rows=CH)
        wsc = torch.empty(ch_ws, dtype=torch.uint8, device=dev)
        oref = torch.empty_like(o1)
        fu_ms, _ = timed_calls(lambda: idx.dense_topk(q, k, w, cu1, TOPK, out_idx=oref, workspace=ws1),
                               args.warmup, args.steps, lib, barrier, max_over_ranks)
        oc = torch.full_like(o1, -7)

        def chunked_call():
            for lo in range(0, L, CH):
                idx.dense_topk(q, k, w, cu1, TOPK, out_idx=oc, workspace=wsc, rows=(lo, min(lo + CH, L)))
        ch_ms, ch_sp = timed_calls(chunked_call, args.warmup, args.steps, lib, barrier, max_over_ranks)
        assert idx.device_status(wsc) == "IDX_OK"
        chunked = {"workload": f"dense_{L}_as_{L // CH}_row_chunks_of_{CH}",
                   "ms_per_call": ch_ms, "full_call_ms": fu_ms,
                   "workspace_bytes": ch_ws, "full_call_workspace_bytes": full_ws,
                   "identical_to_full_call": bool(torch.equal(oc, oref)),
                   "kernels_ms": {n: t for n, (c, t) in ch_sp.items()}}
        del wsc, oref, oc

    # ---------------------------------------------------------------- e2e
    # Every step copies its inputs in from pinned host memory and reads its
    # results back, as a serving loop does: the copies of step i+1's inputs
    # and step i-1's results run on their own streams while step i computes
    # (two input sets and two output sets on the device).
    e2e = None
    if not args.no_e2e:
        hq, hk, hw, h1, h2 = pinned(P.q), pinned(P.k), pinned(P.w), pinned(cu1_h), pinned(cu2_h)
        hos = [(torch.empty(o1.shape, dtype=torch.int32).pin_memory(),
                torch.empty(o2.shape, dtype=torch.int32).pin_memory()) for _ in range(2)]
        sets = [(torch.empty_like(q), torch.empty_like(k), torch.empty_like(w), torch.empty_like(cu1),
                 torch.empty_like(cu2)) for _ in range(2)]
        outs = [(torch.empty_like(o1), torch.empty_like(o2)) for _ in range(2)]
        s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_cmp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_run(nsteps):
            for i in range(nsteps):
                b = i % 2
                dq, dk, dw, dc1, dc2 = sets[b]
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(ev_cmp[b])  # step i-2 finished reading input set b
                    dq.view(torch.int16).copy_(hq, non_blocking=True)
                    dk.view(torch.int16).copy_(hk, non_blocking=True)
                    dw.copy_(hw, non_blocking=True)
                    dc1.copy_(h1, non_blocking=True)
                    dc2.copy_(h2, non_blocking=True)
                    ev_in[b].record(s_in)
                with torch.cuda.stream(s_cmp):
                    s_cmp.wait_event(ev_in[b])
                    if i >= 2:
                        s_cmp.wait_event(ev_out[b])  # step i-2's results were read back
                    step(dq, dk, dw, dc1, dc2, outs[b][0], outs[b][1], st=s_cmp)
                    ev_cmp[b].record(s_cmp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_cmp[b])
                    hos[b][0].copy_(outs[b][0], non_blocking=True)
                    hos[b][1].copy_(outs[b][1], non_blocking=True)
                    ev_out[b].record(s_out)

        e2e_run(2)
        torch.cuda.synchronize()
        barrier()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(s_in)
        e2e_run(args.steps)
        s_out.wait_event(ev_cmp[(args.steps - 1) % 2])
        t1.record(s_out)  # after the last read-back, which follows every earlier step
        torch.cuda.synchronize()
        barrier()
        ems = max_over_ranks(t0.elapsed_time(t1) / args.steps)
        h2d = hq.numel() * 2 + hk.numel() * 2 + hw.numel() * 4 + h1.numel() * 4 + h2.numel() * 4
        d2h = (hos[0][0].numel() + hos[0][1].numel()) * 4
        e2e = {"value": rows_job / (ems / 1000.0), "unit": "queries/s", "ms_per_step": ems,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "overlap": "inputs of step i+1 and results of step i-1 copied while step i computes"}
        del sets, outs

    # ------------------------------------------- block pre-filter (Refine)
    blk = None
    if do_refine and not args.no_block:
        ws3 = torch.empty(idx.pivot_workspace_size(L, H, D, TOPK, 2, G_REF, C_REF, "block"), dtype=torch.uint8,
                          device=dev)
        o3 = torch.empty(L, TOPK, dtype=torch.int32, device=dev)

        def bstep():
            idx.pivot_topk(q, k, w, cu2, TOPK, G_REF, C_REF, "block", out_idx=o3, workspace=ws3)

        for _ in range(args.warmup):
            bstep()
        torch.cuda.synchronize()
        assert idx.device_status(ws3) == "IDX_OK"
        barrier()
        lib.idx_trace_enable(1)
        e0.record(stream)
        for _ in range(args.steps):
            bstep()
        e1.record(stream)
        torch.cuda.synchronize()
        lib.idx_trace_enable(0)
        barrier()
        bms = max_over_ranks(e0.elapsed_time(e1) / args.steps)
        _, trb = trace_report(lib)
        # overlap with the token-scan Refine output on sampled rows (o2 holds the last Refine step)
        srows = torch.from_numpy(np.random.default_rng(5).integers(0, L, 256)).to(dev)
        a, b_ = o2[srows].cpu().numpy(), o3[srows].cpu().numpy()
        ov = float(np.mean([len(set(x[x >= 0]) & set(y[y >= 0])) / max(1, (x >= 0).sum()) for x, y in zip(a, b_)]))
        blk = {"workload": f"block_prefilter_refine_2x{L // 2}_g{G_REF}_c{C_REF}_bn64", "ms_per_step": bms,
               "queries_per_s": world * L / (bms / 1000.0), "overlap_with_refine_topk": ov,
               "kernels": {n: {"launches": c, "ms_per_step": t / args.steps} for n, (c, t) in trb.items()}}
        del ws3
        # the same with the blocks ranked by the Quest bound (CUDA-core block scan)
        ws4 = torch.empty(idx.pivot_workspace_size(L, H, D, TOPK, 2, G_REF, C_REF, "quest"), dtype=torch.uint8,
                          device=dev)

        def qstep():
            idx.pivot_topk(q, k, w, cu2, TOPK, G_REF, C_REF, "quest", out_idx=o3, workspace=ws4)

        for _ in range(args.warmup):
            qstep()
        torch.cuda.synchronize()
        assert idx.device_status(ws4) == "IDX_OK"
        barrier()
        lib.idx_trace_enable(1)
        e0.record(stream)
        for _ in range(args.steps):
            qstep()
        e1.record(stream)
        torch.cuda.synchronize()
        lib.idx_trace_enable(0)
        barrier()
        qms = max_over_ranks(e0.elapsed_time(e1) / args.steps)
        _, trq = trace_report(lib)
        a, b_ = o2[srows].cpu().numpy(), o3[srows].cpu().numpy()
        ovq = float(np.mean([len(set(x[x >= 0]) & set(y[y >= 0])) / max(1, (x >= 0).sum()) for x, y in zip(a, b_)]))
        blk["quest"] = {"ms_per_step": qms, "queries_per_s": world * L / (qms / 1000.0),
                        "overlap_with_refine_topk": ovq,
                        "kernels": {n: {"launches": c, "ms_per_step": t / args.steps} for n, (c, t) in trq.items()}}
        del ws4, o3

    # ------------------------------- token-sparse attention on the selections
    att = None
    if attn_only:  # the selections the attention leg consumes, from one untimed dense call
        wsx = torch.empty(idx.dense_workspace_size(L, H, D, TOPK, 1), dtype=torch.uint8, device=dev)
        idx.dense_topk(q, k, w, cu1, TOPK, out_idx=o1, workspace=wsx)
        torch.cuda.synchronize()
        del wsx
        torch.cuda.empty_cache()  # the attention leg alone holds only its own inputs
    if (do_dense or attn_only) and not args.no_attn:
        Ra = min(args.attn_rows, L)
        gen = torch.Generator(device=dev)
        gen.manual_seed(4321 + rank)
        qa = torch.randn(Ra, 128, 576, generator=gen, device=dev).to(torch.bfloat16)
        kva = torch.randn(L, 576, generator=gen, device=dev).to(torch.bfloat16)
        sel = o1[L - Ra:]  # the dense indexer's selections of the last Ra query rows
        cq = torch.tensor([0, Ra], dtype=torch.int32, device=dev)
        ck = torch.tensor([0, L], dtype=torch.int32, device=dev)
        oa = torch.empty(Ra, 128, 512, dtype=torch.bfloat16, device=dev)
        wsa = torch.empty(256, dtype=torch.uint8, device=dev)
        sc = 1.0 / math.sqrt(192.0)

        def astep():
            idx.sparse_attn(qa, kva, sel, cq, ck, sc, out=oa, workspace=wsa)

        for _ in range(args.warmup):
            astep()
        torch.cuda.synchronize()
        assert idx.device_status(wsa) == "IDX_OK"
        nvalid = int((sel >= 0).sum().item())
        barrier()
        lib.idx_trace_enable(1)
        e0.record(stream)
        for _ in range(args.steps):
            astep()
        e1.record(stream)
        torch.cuda.synchronize()
        lib.idx_trace_enable(0)
        barrier()
        ams = max_over_ranks(e0.elapsed_time(e1) / args.steps)
        _, tra = trace_report(lib)
        kms = sum(t for n, (c, t) in tra.items() if n.endswith("attn_tc")) / args.steps
        useful = 2.0 * 128 * nvalid * (576 + 512)  # logits + weighted values, per listed key and head
        issued = 2.0 * 128 * (Ra * 2048) * (576 + 512)  # every slot of the 2048 is computed (-1 slots too)
        tf = useful / (kms / 1000.0) / 1e12 if kms > 0 else None
        att = {"workload": f"sparse_mla_attn_rows{Ra}_H128_dqk576_dv512_k2048_kv{L}",
               "indices": "dense indexer top-2048 of the last rows of the 131072-token request",
               "ms_per_step": ams, "kernel_ms": kms, "rows_per_s": world * Ra / (ams / 1000.0),
               "useful_flops": useful, "issued_flops": issued, "tflops_useful": tf,
               "frac_bf16_sustained": (tf / bf16_sus) if tf else None,
               "kernels": {n: {"launches": c, "ms_per_step": t / args.steps} for n, (c, t) in tra.items()}}
        del qa, kva, oa

    # -------------------- adaptive budget from the cutoff margin (dense)
    ada = None
    if do_dense and not args.no_adaptive:
        RHO_A, Q_A = 2, 0.4  # the working values of the uncertainty-gated selection page (Sec. 3.4, 3.5)
        wsad = torch.empty(idx.adaptive_workspace_size(L, H, D, TOPK, RHO_A, 1), dtype=torch.uint8, device=dev)
        ai = torch.empty(L, RHO_A * TOPK, dtype=torch.int32, device=dev)
        asc = torch.empty(L, RHO_A * TOPK, dtype=torch.float32, device=dev)
        asg = torch.empty(L, dtype=torch.float32, device=dev)
        atr = torch.empty(L, dtype=torch.uint8, device=dev)

        def adstep():
            idx.adaptive_topk(q, k, w, cu1, TOPK, RHO_A, Q_A, out_idx=ai, out_score=asc, out_sigma=asg,
                              out_trigger=atr, workspace=wsad)

        for _ in range(args.warmup):
            adstep()
        torch.cuda.synchronize()
        assert idx.device_status(wsad) == "IDX_OK"
        barrier()
        lib.idx_trace_enable(1)
        e0.record(stream)
        for _ in range(args.steps):
            adstep()
        e1.record(stream)
        torch.cuda.synchronize()
        lib.idx_trace_enable(0)
        barrier()
        adms = max_over_ranks(e0.elapsed_time(e1) / args.steps)
        _, trd = trace_report(lib)
        dense_ms = sum(v["ms_per_step"] for n, v in per_kernel.items() if n.startswith("dense/"))
        ndef = int((~torch.isnan(asg)).sum().item())
        ada = {"workload": f"adaptive_dense_{L}_k{TOPK}_rho{RHO_A}_q{Q_A}",
               "ms_per_step": adms, "queries_per_s": world * L / (adms / 1000.0),
               "ratio_to_dense_topk": adms / dense_ms if dense_ms > 0 else None,
               "rows_with_margin": ndef, "triggered_rows": int(atr.sum().item()),
               "mean_kept_per_row": float((ai >= 0).sum().item()) / L,
               "page_accounting_kept": TOPK * (1 + Q_A * (RHO_A - 1)),
               "kernels": {n: {"launches": c, "ms_per_step": t / args.steps} for n, (c, t) in trd.items()}}
        del wsad, ai, asc, asg, atr

    # ---------------------------- the 16384 dense and 65536 PIVOT configs
    cfgs = None
    if args.only == "all" and not args.no_configs and L == L_TOK:
        cfgs = run_configs(args, dev, lib, barrier, max_over_ranks, rank, bf16_sus)

    # ------------------------------------------------------------- decode
    dec = None
    if not args.no_decode:
        Dd = W.cfg_decode(seed=M.rank_seed(rank))
        dq_, dkc, dw_, dkv = to_dev(Dd.q, dev), to_dev(Dd.kcache, dev), to_dev(Dd.w, dev), to_dev(Dd.kv_len, dev)
        wsd = torch.empty(max(idx.decode_workspace_size(DEC_B, DEC_G, DEC_N, H, D, TOPK, C_REF, m)
                              for m in ("dense", "refine")), dtype=torch.uint8, device=dev)
        od = torch.empty(DEC_B, DEC_G, TOPK, dtype=torch.int32, device=dev)
        dec = {"workload": "decode_B64_n131072_G2_H64_d128_k2048", "kcache_bytes": Dd.kcache.nbytes}
        # the same cache scattered over a shuffled pool of 64-key pages (block-table layout)
        PAGE = 64
        npg = DEC_N // PAGE
        gen = torch.Generator(device=dev)
        gen.manual_seed(1234 + rank)
        perm = torch.randperm(DEC_B * npg, device=dev, generator=gen)
        dpool = torch.empty(DEC_B * npg, PAGE, D, dtype=dkc.dtype, device=dev)
        dpool[perm] = dkc.reshape(DEC_B * npg, PAGE, D)
        dbt = perm.to(torch.int32).reshape(DEC_B, npg)
        runs = {"dense": lambda m: idx.decode_topk(dq_, dkc, dkv, dw_, TOPK, C_REF, m, out_idx=od, workspace=wsd),
                "refine": lambda m: idx.decode_topk(dq_, dkc, dkv, dw_, TOPK, C_REF, m, out_idx=od, workspace=wsd),
                "paged64_dense": lambda m: idx.decode_paged_topk(dq_, dpool, dbt, dkv, dw_, TOPK, C_REF, "dense",
                                                                  out_idx=od, workspace=wsd)}
        for mode, fn in runs.items():
            for _ in range(args.warmup):
                fn(mode)
            torch.cuda.synchronize()
            assert idx.device_status(wsd) == "IDX_OK"
            lib.idx_trace_enable(1)
            e0.record(stream)
            for _ in range(args.steps):
                fn(mode)
            e1.record(stream)
            torch.cuda.synchronize()
            lib.idx_trace_enable(0)
            _, trd = trace_report(lib)
            step_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps)
            scan = [(n, c, t) for n, (c, t) in trd.items() if "decode_" in n.split("/")[-1]]
            scan_ms = sum(t for _, _, t in scan) / args.steps
            gbs = Dd.kcache.nbytes / (scan_ms / 1000.0) / 1e9 if scan_ms > 0 else None
            dec[mode] = {"ms_per_step": step_ms, "scan_kernel_ms": scan_ms,
                         "scan_GBps": gbs, "scan_frac_hbm": (gbs / hbm_peak) if gbs else None,
                         "kernels": {n: {"launches": c, "ms_per_step": t / args.steps} for n, (c, t) in trd.items()}}
        # the block pre-filter: the proxy scans the cache's block summaries
        # (kept by the caller beside the cache, so built once here, outside the
        # timing: block means, or per-block key min/max for the Quest rule),
        # then the chosen blocks' keys are re-scored
        for rule in ("mean", "quest"):
            ksum = idx.decode_block_means(dkc) if rule == "mean" else idx.decode_block_minmax(dkc)
            wsb = torch.empty(idx.decode_block_workspace_size(DEC_B, DEC_G, DEC_N, H, D, TOPK, C_REF, rule),
                              dtype=torch.uint8, device=dev)
            for _ in range(args.warmup):
                idx.decode_block_topk(dq_, dkc, ksum, dkv, dw_, TOPK, C_REF, rule, out_idx=od, workspace=wsb)
            torch.cuda.synchronize()
            assert idx.device_status(wsb) == "IDX_OK"
            lib.idx_trace_enable(1)
            e0.record(stream)
            for _ in range(args.steps):
                idx.decode_block_topk(dq_, dkc, ksum, dkv, dw_, TOPK, C_REF, rule, out_idx=od, workspace=wsb)
            e1.record(stream)
            torch.cuda.synchronize()
            lib.idx_trace_enable(0)
            _, trd = trace_report(lib)
            step_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps)
            # bytes the step must read: the block summaries of every request and
            # the c candidate keys of each (plus the queries)
            ks_bytes = ksum.numel() * ksum.element_size()
            cand_bytes = DEC_B * C_REF * D * dkc.element_size()
            dec["block_" + rule] = {
                "ms_per_step": step_ms, "block_summary_bytes": ks_bytes, "candidate_key_bytes": cand_bytes,
                "speedup_vs_dense": (dec["dense"]["ms_per_step"] / step_ms) if step_ms > 0 else None,
                "kernels": {n: {"launches": c, "ms_per_step": t / args.steps} for n, (c, t) in trd.items()}}
            del ksum, wsb
        # the same steps captured once in a CUDA graph and replayed (a serving
        # loop's form: no per-launch host work between the kernels)
        graph = {}
        kbar_g = idx.decode_block_means(dkc)
        wsb_g = torch.empty(idx.decode_block_workspace_size(DEC_B, DEC_G, DEC_N, H, D, TOPK, C_REF),
                            dtype=torch.uint8, device=dev)
        gsteps = {"dense": lambda: idx.decode_topk(dq_, dkc, dkv, dw_, TOPK, C_REF, "dense", out_idx=od,
                                                   workspace=wsd),
                  "refine": lambda: idx.decode_topk(dq_, dkc, dkv, dw_, TOPK, C_REF, "refine", out_idx=od,
                                                    workspace=wsd),
                  "block_mean": lambda: idx.decode_block_topk(dq_, dkc, kbar_g, dkv, dw_, TOPK, C_REF, "mean",
                                                              out_idx=od, workspace=wsb_g)}
        for name, fn in gsteps.items():
            gs = torch.cuda.Stream(dev)
            gs.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(gs):
                fn()
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=gs):
                fn()
            for _ in range(args.warmup):
                g.replay()
            torch.cuda.synchronize()
            e0.record(stream)
            for _ in range(args.steps):
                g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            graph[name] = max_over_ranks(e0.elapsed_time(e1) / args.steps)
            del g
        dec["graph_ms_per_step"] = graph
        del kbar_g, wsb_g
        dec["hbm_peak_GBps"] = hbm_peak
        del dpool, dbt, perm

    # -------------------------------------------------------- CPU baseline
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu and L == L_TOK:
        v, dt, threads, desc = oracle_sample(P, args.cpu_rows)
        cpu = {"value": v, "unit": "queries/s", "cores": threads, "kind": "oracle", "sample": desc,
               "seconds": dt}

    line = {
        "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "strong" if split else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"long_prefill_{L}_" + {"all": "dense+refine", "dense": "dense",
                                                          "refine": "refine", "attn": "none"}[args.only] + "_g16_c4096",
                   "tokens": L, "H": H, "d": D,
                   "topk": TOPK, "dense_requests": [L], "refine_requests": [L // 2, L // 2],
                   "g": G_REF, "c": C_REF,
                   "parallelism": (f"split{world} (one request, zig-zag rows per rank)" if split
                                   else f"dp{world} (independent batches)"),
                   "l2": "inputs larger than L2 (q is 2 GiB)"},
        "tflops_dense": achieved, "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "clocks": clk,
        "gpu_launches": nlaunch, "kernels": per_kernel, "block_prefilter": blk, "sparse_attn": att,
        "adaptive": ada, "decode": dec, "configs": cfgs,
        "packed_refine_vs_dense": packed, "dense_row_chunks": chunked,
    }
    if rank == 0:
        print(json.dumps(line))
    M.finish()
    return 0


if __name__ == "__main__":
    sys.exit(main())
