"""Decode steps captured in a CUDA graph.  The entry points enqueue only
stream-ordered work (kernels, memsets) and allocate nothing, so a serving
loop can capture one decode step with its buffers and replay it after
writing the next step's queries, weights and lengths into those buffers.
Replays must give exactly what eager calls give on the same inputs: dense
decode, Refine decode, and the block pre-filter (block means and Quest)."""
from __future__ import annotations

import numpy as np
import pytest

from sparse_attention_indexer_05_b200 import workloads as W
from tests._util import to_dev

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def idx():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_indexer_05_b200 as m
    return m


def _inputs(seed, kv):
    D = W.decode(B=len(kv), n=4096, G=2, H=64, d=128, topk=128, seed=seed, kv_len=kv)
    return to_dev(D.q), to_dev(D.kcache), to_dev(D.w), to_dev(D.kv_len)


@pytest.mark.parametrize("mode", ["dense", "refine", "block_mean", "block_quest"])
def test_graph_replay_equals_eager(idx, mode):
    topk, c = 128, 512
    q, kc, w, kv = _inputs(1, [4096, 3000, 700, 64])
    B, G, H, d = q.shape
    n_max = kc.shape[1]
    od = torch.empty(B, G, topk, dtype=torch.int32, device="cuda")
    if mode.startswith("block"):
        rule = mode.split("_")[1]
        ksum = idx.decode_block_means(kc) if rule == "mean" else idx.decode_block_minmax(kc)
        ws = torch.empty(idx.decode_block_workspace_size(B, G, n_max, H, d, topk, c, rule), dtype=torch.uint8,
                         device="cuda")

        def step():
            idx.decode_block_topk(q, kc, ksum, kv, w, topk, c, rule, out_idx=od, workspace=ws)
    else:
        ws = torch.empty(idx.decode_workspace_size(B, G, n_max, H, d, topk, c, mode), dtype=torch.uint8,
                         device="cuda")

        def step():
            idx.decode_topk(q, kc, kv, w, topk, c, mode, out_idx=od, workspace=ws)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()  # first call outside the capture (one-time host setup)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step()
    torch.cuda.synchronize()
    for seed, lens in ((2, [4000, 2048, 65, 3000]), (3, [128, 4096, 1000, 2])):
        q2, _, w2, kv2 = _inputs(seed, lens)
        q.copy_(q2)
        w.copy_(w2)
        kv.copy_(kv2)
        g.replay()
        torch.cuda.synchronize()
        got = od.clone()
        assert idx.device_status(ws) == "IDX_OK"
        step()  # eager, same inputs
        torch.cuda.synchronize()
        assert torch.equal(got, od), (mode, seed)
    del g
