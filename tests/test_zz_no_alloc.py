"""The decode entry point that allocates nothing (idx_decode_topk_noalloc).

It is for callers that cannot allocate device memory (a plugin that only
receives input and output buffers, a serving loop that must not allocate):
its scratch is a fixed device array inside the library.  The test calls it
through the C ABI twice in a row, on different inputs, and checks each
result against the workspace-taking idx_decode_topk (dense mode): the same
indices, and scores within the tolerance of the other parity tests; and
against the oracle's dense decode top-k (well-formed rows, recall >= 0.999,
the bar of the other bf16 decode parity tests).  It
also checks that a call too large for the fixed scratch is refused, that
arguments the workspace entry point rejects are rejected with the same
code, and that the device status word of the fixed scratch is reported by
idx_decode_noalloc_status.  This file is collected last so that a failure
here leaves every other test run.
"""
import numpy as np
import pytest

import oracle as O
from sparse_attention_indexer_05_b200 import workloads as W
from tests._util import check_rows_wellformed, recall, to_dev

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def _close(a, b, rtol=1e-3):
    fa, fb = np.isfinite(a), np.isfinite(b)
    assert np.array_equal(fa, fb)
    assert np.array_equal(a[~fa], b[~fb])              # -inf pads
    m = np.abs(b[fb]).max() if fb.any() else 0.0
    assert (np.abs(a[fa] - b[fb]) <= rtol * np.maximum(np.abs(b[fb]), 1e-3 * m)).all()


def test_noalloc_decode_matches_workspace_entry_point_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_attention_indexer_05_b200 as idx
    from sparse_attention_indexer_05_b200 import _native as N
    f = N.lib().idx_decode_topk_noalloc
    topk = 128
    for seed, kv in ((1, [2500, 1999, 130]), (2, [2500, 2, 2400])):
        D = W.decode(B=3, n=2500, G=2, H=64, d=128, topk=topk, seed=seed, kv_len=kv)
        q, kc, w, kvl = to_dev(D.q), to_dev(D.kcache), to_dev(D.w), to_dev(D.kv_len)
        ref_idx, ref_sc = idx.decode_topk(q, kc, kvl, w, topk, 0, "dense", return_scores=True)
        out_idx = torch.full((3, 2, topk), 7, dtype=torch.int32, device="cuda")
        out_sc = torch.zeros((3, 2, topk), dtype=torch.float32, device="cuda")
        rc = f(q.data_ptr(), kc.data_ptr(), kvl.data_ptr(), w.data_ptr(), 3, 2, 2500, 64, 128, topk, N.BF16,
               out_idx.data_ptr(), out_sc.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert rc == 0, N.STATUS.get(rc, rc)
        torch.cuda.synchronize()
        assert torch.equal(out_idx, ref_idx)
        _close(out_sc.cpu().numpy(), ref_sc.cpu().numpy())
        got = out_idx.cpu().numpy()
        check_rows_wellformed(got, [int(n) - 2 + m for n in kv for m in range(2)], topk)
        want = O.decode_topk(D.q, D.kcache, D.w, D.kv_len, topk, 0, O.DENSE)
        assert recall(got, want) >= 0.999, seed


def test_noalloc_refuses_calls_beyond_its_scratch():
    from sparse_attention_indexer_05_b200 import _native as N
    f = N.lib().idx_decode_topk_noalloc
    fake = 256  # never dereferenced: the size check fails before any launch
    rc = f(fake, fake, fake, fake, 64, 2, 131072, 64, 128, 2048, N.BF16, fake, None, None)
    assert rc == 2  # IDX_ERR_UNSUPPORTED


def test_noalloc_rejects_what_the_workspace_entry_point_rejects():
    from sparse_attention_indexer_05_b200 import _native as N
    L = N.lib()
    fake = 256  # never dereferenced: the argument checks fail before any launch
    cases = [
        (0, 2, 4096),     # no request
        (4, 9, 4096),     # more MTP queries than one row block holds
        (4, 2, 1),        # cache shorter than the query group
        (4, 2, 1 << 21),  # cache longer than the supported maximum
    ]
    for B, G, n in cases:
        a = L.idx_decode_topk_noalloc(fake, fake, fake, fake, B, G, n, 64, 128, 64, N.BF16, fake, None, None)
        b = L.idx_decode_topk(fake, fake, fake, fake, B, G, n, 64, 128, 64, 0, N.MODE_DENSE, N.BF16, fake, None,
                              fake, 1 << 40, None)
        assert a == b and a != 0, (B, G, n, a, b)


def test_noalloc_status_word_is_reported():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_indexer_05_b200 import _native as N
    L = N.lib()
    topk = 64
    D = W.decode(B=2, n=600, G=2, H=64, d=128, topk=topk, seed=3, kv_len=[600, 300])
    q, kc, w = to_dev(D.q), to_dev(D.kcache), to_dev(D.w)
    out_idx = torch.empty((2, 2, topk), dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream

    def call(kv):
        kvl = torch.tensor(kv, dtype=torch.int32, device="cuda")
        rc = L.idx_decode_topk_noalloc(q.data_ptr(), kc.data_ptr(), kvl.data_ptr(), w.data_ptr(), 2, 2, 600, 64,
                                       128, topk, N.BF16, out_idx.data_ptr(), None, st)
        assert rc == 0, N.STATUS.get(rc, rc)
        return L.idx_decode_noalloc_status(st)

    assert call([600, 300]) == 0
    # request 1 claims more keys than the cache holds: caught on the device,
    # its rows come back as -1 and the status word says IDX_ERR_INVALID
    assert call([600, 601]) == 1
    assert (out_idx[1] == -1).all()
    # the next call clears the status word again
    assert call([600, 300]) == 0
