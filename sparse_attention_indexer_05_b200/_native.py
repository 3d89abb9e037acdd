"""ctypes view of libidx.so (declarations of include/idx.h)."""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libidx.so")

STATUS = {0: "IDX_OK", 1: "IDX_ERR_INVALID", 2: "IDX_ERR_UNSUPPORTED", 3: "IDX_ERR_WORKSPACE",
          4: "IDX_ERR_CUDA", 5: "IDX_ERR_TIMEOUT", 6: "IDX_ERR_OVERFLOW"}
BF16, F32 = 0, 1
MODE_DENSE, MODE_REUSE, MODE_REFINE, MODE_BLOCK, MODE_QUEST = 0, 1, 2, 3, 4

# every entry point of include/idx.h: name -> (restype, argtypes)
_vp, _fp, _ip = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
_i, _sz, _ll = ctypes.c_int, ctypes.c_size_t, ctypes.c_longlong
SIGNATURES = {
    "idx_dense_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "idx_dense_topk": (_i, [_vp, _vp, _fp, _ip, _i, _i, _i, _i, _i, _i, _ip, _fp, _vp, _sz, _vp]),
    "idx_adaptive_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "idx_adaptive_topk": (_i, [_vp, _vp, _fp, _ip, _i, _i, _i, _i, _i, _i, ctypes.c_double, _i, _ip, _fp, _fp,
                               _vp, _vp, _sz, _vp]),
    "idx_pivot_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i, _i, _i, _i]),
    "idx_pivot_topk": (_i, [_vp, _vp, _fp, _ip, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _ip, _fp, _vp, _sz,
                            _vp]),
    "idx_dense_workspace_size_rows": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "idx_pivot_workspace_size_rows": (_sz, [_i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i]),
    "idx_dense_topk_rows": (_i, [_vp, _vp, _fp, _ip, _i, _i, _i, _i, _i, _i, _i, _i, _ip, _fp, _vp, _sz, _vp]),
    "idx_pivot_topk_rows": (_i, [_vp, _vp, _fp, _ip, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _ip, _fp,
                                 _vp, _sz, _vp]),
    "idx_decode_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i, _i, _i]),
    "idx_decode_topk": (_i, [_vp, _vp, _ip, _fp, _i, _i, _i, _i, _i, _i, _i, _i, _i, _ip, _fp, _vp, _sz,
                             _vp]),
    "idx_decode_paged_topk": (_i, [_vp, _vp, _ip, _ip, _fp, _i, _i, _i, _i, _ll, _i, _i, _i, _i, _i, _i, _ip,
                                   _fp, _vp, _sz, _vp]),
    "idx_sparse_attn_workspace_size": (_sz, []),
    "idx_sparse_attn": (_i, [_vp, _vp, _ip, _ip, _ip, _i, _i, _ll, _i, _i, _i, _i, ctypes.c_float, _i, _vp, _fp,
                             _vp, _sz, _vp]),
    "idx_device_status": (_i, [_vp, _vp]),
    "idx_status_string": (ctypes.c_char_p, [_i]),
    "idx_debug_scores": (_i, [_i, _vp, _vp, _fp, _ip, _i, _i, _i, _i, _i, _i, _i, _i, _ip, _i, _fp, _ll,
                              _vp, _sz, _vp]),
    "idx_debug_decode_scores": (_i, [_i, _vp, _vp, _ip, _fp, _i, _i, _i, _i, _i, _i, _i, _i, _i, _fp, _ll,
                                     _vp, _sz, _vp]),
    "idx_uses_tensor_cores": (_i, [_i, _i, _i]),
    "idx_trace_enable": (_i, [_i]),
    "idx_debug_wait_probe": (_i, [_vp, ctypes.c_uint, _vp]),
    "idx_decode_block_means": (_i, [_vp, _i, _i, _i, _i, _i, _vp, _vp]),
    "idx_decode_block_minmax": (_i, [_vp, _i, _i, _i, _i, _i, _vp, _vp]),
    "idx_decode_block_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i, _i, _i]),
    "idx_decode_block_topk": (_i, [_vp, _vp, _vp, _i, _ip, _fp, _i, _i, _i, _i, _i, _i, _i, _i, _ip, _fp, _vp,
                                   _sz, _vp]),
    "idx_decode_topk_noalloc": (_i, [_vp, _vp, _ip, _fp, _i, _i, _i, _i, _i, _i, _i, _ip, _fp, _vp]),
    "idx_decode_noalloc_status": (_i, [_vp]),
    "idx_trace_report": (_ll, [ctypes.c_char_p, _sz]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load libidx.so; raise if it has not been built (there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m sparse_attention_indexer_05_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


class IdxError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS.get(code, code)}")
        self.code = code


def check(code: int, what: str):
    if code != 0:
        raise IdxError(code, what)
