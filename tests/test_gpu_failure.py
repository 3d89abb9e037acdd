"""Failure detection without a GPU fault: a bounded device wait that runs
out reports IDX_ERR_TIMEOUT through the workspace status word, and the
context keeps working afterwards."""
import time

import numpy as np
import pytest

import oracle as O
from sparse_attention_indexer_05_b200 import workloads as W
from tests._util import to_dev

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def test_bounded_wait_times_out_and_context_survives():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_indexer_05_b200 as idx
    from sparse_attention_indexer_05_b200 import _native as N
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    t0 = time.time()
    assert N.lib().idx_debug_wait_probe(ws.data_ptr(), 200, torch.cuda.current_stream().cuda_stream) == 0
    assert idx.device_status(ws) == "IDX_ERR_TIMEOUT"
    assert time.time() - t0 < 5.0
    # the context is still usable: a normal call succeeds and is correct
    P = W.prefill([300], H=64, d=128, topk=32, seed=4)
    q, k, w, cu = to_dev(P.q), to_dev(P.k), to_dev(P.w), to_dev(P.cu_seqlens)
    ws2 = torch.empty(idx.dense_workspace_size(P.T, 64, 128, 32, 1), dtype=torch.uint8, device="cuda")
    out = idx.dense_topk(q, k, w, cu, 32, workspace=ws2).cpu().numpy()
    assert idx.device_status(ws2) == "IDX_OK"
    want = O.dense_topk(P.q, P.k, P.w, P.cu_seqlens, 32)
    inter = sum(len(set(a[a >= 0]) & set(b[b >= 0])) for a, b in zip(out, want))
    assert inter / (want >= 0).sum() >= 0.999
