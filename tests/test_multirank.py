"""The N>1 host path on CPU: two gloo ranks, each with its own batch, the
barrier and the max-over-ranks reduction of the timing, and rank-0 checks
that the ranks' results are those of their own seeds.  Then one request
split across ranks: the zig-zag partition's properties (disjoint, covering,
groups whole, causal work balanced), and two gloo ranks that each rank the
rows they own (the oracle here, on the CPU) and together give the whole
request's result."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import oracle as O
    from sparse_attention_indexer_05_b200 import multirank as M
    from sparse_attention_indexer_05_b200 import workloads as W
    r, w, _ = M.init("gloo", timeout_s=60)
    P = W.prefill([40, 23], H=4, d=16, topk=6, seed=M.rank_seed(r))
    res = O.dense_topk(P.q, P.k, P.w, P.cu_seqlens, 6, threads=1)
    M.barrier()
    t = M.max_over_ranks(1.5 + r)           # stand-in per-rank time
    gathered = [None] * w
    torch.distributed.all_gather_object(gathered, res.tolist())
    if r == 0:
        out.put((t, gathered))
    M.finish()


def test_two_gloo_ranks_weak_scaling():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(i, 2, port, q)) for i in range(2)]
    for p in procs:
        p.start()
    t, gathered = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert t == 2.5                       # the max over ranks
    import oracle as O
    from sparse_attention_indexer_05_b200 import workloads as W
    for r in range(2):
        P = W.prefill([40, 23], H=4, d=16, topk=6, seed=r)
        assert gathered[r] == O.dense_topk(P.q, P.k, P.w, P.cu_seqlens, 6, threads=1).tolist()
    assert gathered[0] != gathered[1]     # each rank ranks its own batch


def test_zigzag_partition_properties():
    from sparse_attention_indexer_05_b200 import multirank as M
    for n in (131072, 65536, 16384, 1000, 37):
        for world in (1, 2, 3, 4, 8):
            for align in (1, 4, 16):
                parts = [M.zigzag_ranges(n, world, r, align) for r in range(world)]
                rows = np.zeros(n, np.int32)
                for ranges in parts:
                    for lo, hi in ranges:
                        assert 0 <= lo < hi <= n
                        rows[lo:hi] += 1
                        # groups [m*align, (m+1)*align) never straddle two ranks
                        assert lo % align == 0 and (hi % align == 0 or hi == n)
                assert (rows == 1).all(), (n, world, align)           # disjoint and covering
                if n >= 16384:
                    work = [M.causal_pairs(p) for p in parts]
                    assert max(work) <= 1.05 * min(work), (n, world, align, work)
    assert M.causal_pairs([(0, 4)]) == 1 + 2 + 3 + 4


def _split_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import oracle as O
    from sparse_attention_indexer_05_b200 import multirank as M
    from sparse_attention_indexer_05_b200 import workloads as W
    r, w, _ = M.init("gloo", timeout_s=60)
    P = W.prefill([301], H=4, d=16, topk=6, seed=5)       # one request, the same on every rank
    g = 4
    mine = {}
    for lo, hi in M.zigzag_ranges(P.T, w, r, align=g):
        rows = np.arange(lo, hi)
        mine[(lo, hi)] = (O.dense_topk(P.q, P.k, P.w, P.cu_seqlens, 6, rows=rows, threads=1).tolist(),
                          O.pivot_topk(P.q, P.k, P.w, P.cu_seqlens, 6, g, 12, O.REFINE, rows=rows,
                                       threads=1).tolist())
    gathered = [None] * w
    torch.distributed.all_gather_object(gathered, mine)
    if r == 0:
        out.put(gathered)
    M.finish()


def test_two_gloo_ranks_split_one_request():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(i, 2, port, q)) for i in range(2)]
    for p in procs:
        p.start()
    gathered = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import oracle as O
    from sparse_attention_indexer_05_b200 import workloads as W
    P = W.prefill([301], H=4, d=16, topk=6, seed=5)
    dense = O.dense_topk(P.q, P.k, P.w, P.cu_seqlens, 6, threads=1)
    refine = O.pivot_topk(P.q, P.k, P.w, P.cu_seqlens, 6, 4, 12, O.REFINE, threads=1)
    got_d = np.full_like(dense, -7)
    got_r = np.full_like(refine, -7)
    for part in gathered:
        for (lo, hi), (d_, r_) in part.items():
            got_d[lo:hi] = d_
            got_r[lo:hi] = r_
    assert np.array_equal(got_d, dense)
    assert np.array_equal(got_r, refine)
