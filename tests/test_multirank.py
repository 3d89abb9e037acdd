"""The N>1 host path on CPU: two gloo ranks, each with its own batch, the
barrier and the max-over-ranks reduction of the timing, and rank-0 checks
that the ranks' results are those of their own seeds."""
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
