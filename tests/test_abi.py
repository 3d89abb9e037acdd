"""The C ABI library loads, exports every declared entry point, and rejects
bad arguments on the host (no GPU needed: nothing is launched)."""
import ctypes
import os
import re

import pytest

from sparse_attention_indexer_05_b200 import _native as N
from sparse_attention_indexer_05_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return N.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "idx.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(idx_[a-z_]+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) == 29
    for n in names:
        assert hasattr(lib, n), n
        assert n in N.SIGNATURES, n


def test_status_strings(lib):
    for code, name in N.STATUS.items():
        assert lib.idx_status_string(code).decode() == name


def test_workspace_sizes(lib):
    assert lib.idx_dense_workspace_size(16384, 64, 128, 2048, 1, 0) > 16384 * 2048 * 8
    assert lib.idx_dense_workspace_size(0, 64, 128, 2048, 1, 0) == 0
    assert lib.idx_dense_workspace_size(100, 64, 12, 8, 1, 0) == 0        # d % 8 != 0
    assert lib.idx_pivot_workspace_size(65536, 64, 128, 2048, 1, 0, 4, 4096, 2, 0) > 0
    assert lib.idx_pivot_workspace_size(65536, 64, 128, 2048, 1, 0, 4, 1024, 2, 0) == 0   # c < k
    assert lib.idx_pivot_workspace_size(65536, 64, 128, 2048, 1, 0, 0, 4096, 2, 0) == 0   # g < 1
    assert lib.idx_pivot_workspace_size(65536, 64, 128, 2048, 1, 0, 4, 4096, 0, 0) == 0   # dense mode
    # the guardrail: members of short groups are scored rows of their own, so
    # the workspace grows with the threshold, up to one row per token
    plain = lib.idx_pivot_workspace_size(65536, 64, 128, 2048, 1, 0, 4, 4096, 2, 0)
    guard = lib.idx_pivot_workspace_size(65536, 64, 128, 2048, 1, 0, 4, 4096, 2, 8192)
    assert guard > plain
    assert lib.idx_pivot_workspace_size(65536, 64, 128, 2048, 1, 0, 4, 4096, 2, 1 << 20) >= guard
    assert lib.idx_pivot_workspace_size(65536, 64, 128, 2048, 1, 0, 4, 4096, 2, -1) == 0  # negative threshold
    assert lib.idx_pivot_workspace_size(65536, 64, 128, 2048, 1, 0, 4, 4096, 3, 64) == 0  # block mode
    # the Quest rule: block mode's rules, and the proxy's q+/q- in shared memory
    assert lib.idx_pivot_workspace_size(65536, 64, 128, 2048, 1, 0, 16, 4096, 4, 0) > 0
    assert lib.idx_pivot_workspace_size(65536, 64, 128, 2048, 1, 0, 16, 4096 + 32, 4, 0) == 0
    assert lib.idx_pivot_workspace_size(65536, 64, 128, 2048, 1, 0, 16, 4096, 4, 64) == 0
    assert lib.idx_pivot_workspace_size(65536, 256, 256, 2048, 1, 0, 16, 4096, 4, 0) == 0
    assert lib.idx_pivot_workspace_size(65536, 64, 128, 2048, 1, 0, 16, 4096, 5, 0) == 0   # no mode 5
    # row-range calls: the per-row scratch covers the call's rows only
    full = lib.idx_dense_workspace_size(131072, 64, 128, 2048, 1, 0)
    assert lib.idx_dense_workspace_size_rows(131072, 64, 128, 2048, 1, 0, 0) == full
    assert lib.idx_dense_workspace_size_rows(131072, 64, 128, 2048, 1, 0, 131072) == full
    assert lib.idx_dense_workspace_size_rows(131072, 64, 128, 2048, 1, 0, 16384) < full / 7
    assert lib.idx_dense_workspace_size_rows(131072, 64, 128, 2048, 1, 0, -1) == 0
    pf = lib.idx_pivot_workspace_size(131072, 64, 128, 2048, 2, 0, 16, 4096, 2, 0)
    assert lib.idx_pivot_workspace_size_rows(131072, 64, 128, 2048, 2, 0, 16, 4096, 2, 0, 16384) < pf / 5
    assert lib.idx_decode_workspace_size(64, 2, 131072, 64, 128, 2048, 4096, 2, 0) > 64 * 131072 * 4
    assert lib.idx_decode_workspace_size(64, 2, 1, 64, 128, 2048, 4096, 2, 0) == 0     # n_max < G


def test_adaptive_workspace_and_argument_checks(lib):
    assert lib.idx_adaptive_workspace_size(4096, 64, 128, 256, 2, 1, 0) > lib.idx_dense_workspace_size(
        4096, 64, 128, 512, 1, 0)
    assert lib.idx_adaptive_workspace_size(4096, 64, 128, 256, 1, 1, 0) == 0     # rho < 2
    assert lib.idx_adaptive_workspace_size(4096, 64, 128, 1 << 30, 4, 1, 0) == 0  # rho*topk overflows
    assert lib.idx_adaptive_workspace_size(4096, 64, 128, 4097, 2, 1, 0) == 0     # rho*topk above 8192
    fake = ctypes.c_void_p(256)  # never dereferenced: the checks fail first
    f = lib.idx_adaptive_topk
    assert f(fake, fake, fake, fake, 1, 10, 4, 64, 8, 1, 0.4, 0, fake, None, None, None, fake, 1 << 30, None) == 1
    assert f(fake, fake, fake, fake, 1, 10, 4, 64, 8, 2, 1.5, 0, fake, None, None, None, fake, 1 << 30, None) == 1
    assert f(fake, fake, fake, fake, 1, 10, 4, 64, 8, 2, float("nan"), 0, fake, None, None, None, fake, 1 << 30,
             None) == 1
    assert f(None, fake, fake, fake, 1, 10, 4, 64, 8, 2, 0.4, 0, fake, None, None, None, fake, 1 << 30, None) == 1
    assert f(fake, fake, fake, fake, 1, 10, 4, 64, 8, 2, 0.4, 0, fake, None, None, None, fake, 16, None) == 3
    assert f(fake, fake, fake, fake, 1, 10, 4, 64, 4097, 2, 0.4, 0, fake, None, None, None, fake, 1 << 30,
             None) == 2


def test_invalid_arguments_return_before_launch(lib):
    fake = ctypes.c_void_p(256)  # never dereferenced: the checks fail first
    # null q
    assert lib.idx_dense_topk(None, fake, fake, fake, 1, 10, 4, 64, 8, 0, fake, None, fake, 1 << 30, None) == 1
    # bad head dim
    assert lib.idx_dense_topk(fake, fake, fake, fake, 1, 10, 4, 60, 8, 0, fake, None, fake, 1 << 30, None) == 1
    # workspace too small
    assert lib.idx_dense_topk(fake, fake, fake, fake, 1, 10, 4, 64, 8, 0, fake, None, fake, 16, None) == 3
    # misaligned workspace
    assert lib.idx_dense_topk(fake, fake, fake, fake, 1, 10, 4, 64, 8, 0, fake, None, ctypes.c_void_p(264),
                              1 << 30, None) == 3
    # refine with c < k
    assert lib.idx_pivot_topk(fake, fake, fake, fake, 1, 10, 4, 64, 8, 0, 4, 4, 2, 0, fake, None, fake, 1 << 30,
                              None) == 1
    # unknown mode
    assert lib.idx_pivot_topk(fake, fake, fake, fake, 1, 10, 4, 64, 8, 0, 4, 16, 7, 0, fake, None, fake, 1 << 30,
                              None) == 1
    # negative guardrail threshold
    assert lib.idx_pivot_topk(fake, fake, fake, fake, 1, 10, 4, 64, 8, 0, 4, 16, 2, -1, fake, None, fake, 1 << 30,
                              None) == 1
    # the guardrail is not offered for the block pre-filter
    assert lib.idx_pivot_topk(fake, fake, fake, fake, 1, 10, 4, 64, 8, 0, 4, 64, 3, 64, fake, None, fake, 1 << 30,
                              None) == 2
    # decode: more MTP queries than a row block holds
    assert lib.idx_decode_topk(fake, fake, fake, fake, 2, 9, 64, 4, 64, 8, 0, 0, 0, fake, None, fake, 1 << 30,
                               None) == 2
    # decode: refine with c < k
    assert lib.idx_decode_topk(fake, fake, fake, fake, 2, 2, 64, 4, 64, 8, 4, 2, 0, fake, None, fake, 1 << 30,
                               None) == 1
    # paged decode: no block table / a page size that neither divides 128 nor is a multiple of it /
    # a logical cache longer than 2^20
    assert lib.idx_decode_paged_topk(fake, fake, None, fake, fake, 2, 2, 4, 16, 8, 4, 64, 8, 0, 0, 0, fake, None,
                                     fake, 1 << 30, None) == 1
    assert lib.idx_decode_paged_topk(fake, fake, fake, fake, fake, 2, 2, 4, 48, 8, 4, 64, 8, 0, 0, 0, fake, None,
                                     fake, 1 << 30, None) == 2
    assert lib.idx_decode_paged_topk(fake, fake, fake, fake, fake, 2, 2, 8193, 128, 8, 4, 64, 8, 0, 0, 0, fake,
                                     None, fake, 1 << 30, None) == 2
    # shape that fits neither kernel family
    assert lib.idx_dense_topk(fake, fake, fake, fake, 1, 10, 256, 256, 8, 1, fake, None, fake, 1 << 40,
                              None) == 2


def test_binding_refuses_cpu_tensors():
    torch = pytest.importorskip("torch")
    import sparse_attention_indexer_05_b200 as idx
    B.build()
    q = torch.zeros(4, 2, 8, dtype=torch.bfloat16)
    with pytest.raises((ValueError, RuntimeError)):
        idx.dense_topk(q, torch.zeros(4, 8, dtype=torch.bfloat16), torch.zeros(4, 2),
                       torch.tensor([0, 4], dtype=torch.int32), 2)


def test_sparse_attn_argument_checks(lib):
    """Host-side checks of idx_sparse_attn return before any launch."""
    fake = ctypes.c_void_p(256)  # never dereferenced: the checks fail first
    assert lib.idx_sparse_attn_workspace_size() == 256

    def call(q=fake, kv=fake, H=128, Dqk=576, Dv=512, scale=0.07, ws=fake, ws_bytes=256):
        return lib.idx_sparse_attn(q, kv, fake, fake, fake, 1, 4, 100, H, Dqk, Dv, 64, scale, 0, fake, None,
                                   ws, ws_bytes, None)

    assert call(kv=None) == 1                      # null latent rows
    assert call(Dv=600) == 1                       # value wider than the key
    assert call(scale=float("nan")) == 1           # non-finite scale
    assert call(Dqk=512) == 2                      # shape without a kernel
    assert call(H=256) == 2                        # more heads than the MMA's M
    assert call(ws_bytes=16) == 3                  # workspace too small
    assert call(ws=ctypes.c_void_p(264)) == 3      # misaligned workspace


def test_decode_block_workspace_and_argument_checks(lib):
    size = lib.idx_decode_block_workspace_size
    for rule in (0, 1):
        ok = size(64, 2, 131072, 64, 128, 2048, 4096, rule, 0)
        assert ok > 0
        # the block-score spill is a 64th of the token-score one
        assert ok < lib.idx_decode_workspace_size(64, 2, 131072, 64, 128, 2048, 4096, 2, 0)
        assert size(64, 2, 131072 - 1, 64, 128, 2048, 4096, rule, 0) == 0    # n_max not a multiple of 64
        assert size(64, 2, 131072, 64, 128, 2048, 4096 + 32, rule, 0) == 0   # c not a multiple of 64
        assert size(64, 2, 131072, 64, 128, 2048, 1024, rule, 0) == 0        # c < topk
        assert size(64, 9, 131072, 64, 128, 2048, 4096, rule, 0) == 0        # G above one row block
    assert size(64, 2, 131072, 64, 128, 2048, 4096, 2, 0) == 0               # no rule 2
    assert size(64, 2, 131072, 256, 256, 2048, 4096, 1, 0) == 0              # Quest proxy above shared memory
    fake = 256  # never dereferenced: the checks fail before any launch
    f = lib.idx_decode_block_topk
    args = [fake, fake, fake, 0, fake, fake, 4, 2, 4096, 64, 128, 64, 128, 0, fake, None, fake, 1 << 40, None]
    for i in (0, 1, 2, 4, 5, 14):  # q, kcache, ksum, kv_len, w, out_idx
        a = list(args)
        a[i] = None
        assert f(*a) == 1, i
    for i, v, code in ((12, 96, 1),    # c not a multiple of 64
                       (8, 4000, 1),   # n_max not a multiple of 64
                       (3, 2, 1),      # no rule 2
                       (7, 9, 2),      # G > 8
                       (17, 16, 3)):   # workspace too small
        a = list(args)
        a[i] = v
        assert f(*a) == code, (i, v)
    for m in (lib.idx_decode_block_means, lib.idx_decode_block_minmax):
        assert m(None, 4, 4096, 128, 0, 0, fake, None) == 1
        assert m(fake, 4, 4000, 128, 0, 0, fake, None) == 1   # n_max not a multiple of 64
        assert m(fake, 4, 4096, 12, 0, 0, fake, None) == 1    # d % 8 != 0
        assert m(fake, 4, 4096, 128, 0, -1, fake, None) == 1  # negative first block
