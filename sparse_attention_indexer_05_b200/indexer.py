"""Python binding of libidx: the lightning indexer + per-query top-k.

Argument marshalling only: tensors are checked and their device pointers
passed to the C ABI (include/idx.h); every step of the computation runs in
the library's CUDA kernels.  torch provides device memory and streams.

Entry points (names follow the C ABI):
    dense_topk(q, k, w, cu_seqlens, topk)               -> idx [T, topk]
    pivot_topk(q, k, w, cu_seqlens, topk, g, c, mode)   -> idx [T, topk]
    decode_topk(q, kcache, kv_len, w, topk, c, mode)    -> idx [B, G, topk]
    decode_paged_topk(q, kpool, block_table, kv_len, w, topk, c, mode)  -> idx [B, G, topk]
    sparse_attn(q, kv, idx, cu_q, cu_kv, scale)         -> out [R, H, 512]
Each accepts out_idx / out_score / workspace to reuse buffers, and
return_scores=True to also get the selected scores.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import _native as N

MODES = {"dense": N.MODE_DENSE, "reuse": N.MODE_REUSE, "refine": N.MODE_REFINE, "block": N.MODE_BLOCK,
         "quest": N.MODE_QUEST}


def _mode(m) -> int:
    if isinstance(m, str):
        return MODES[m.lower()]
    return int(m)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return N.BF16
    if t.dtype == torch.float32:
        return N.F32
    raise TypeError(f"q/k must be bfloat16 or float32, got {t.dtype}")


def _dev(t: torch.Tensor, name: str, dtype=None) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _stream(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ws(workspace: Optional[torch.Tensor], need: int, device) -> torch.Tensor:
    if need == 0:
        raise ValueError("invalid arguments (workspace size 0)")
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    return workspace


def dense_workspace_size(T, H, d, topk, num_seqs, dtype=torch.bfloat16, max_rows=0) -> int:
    """Workspace bytes; max_rows > 0: for calls whose rows= range spans at most max_rows rows."""
    dt = N.BF16 if dtype == torch.bfloat16 else N.F32
    return int(N.lib().idx_dense_workspace_size_rows(T, H, d, topk, num_seqs, dt, int(max_rows)))


def adaptive_workspace_size(T, H, d, topk, rho, num_seqs, dtype=torch.bfloat16) -> int:
    dt = N.BF16 if dtype == torch.bfloat16 else N.F32
    return int(N.lib().idx_adaptive_workspace_size(T, H, d, topk, rho, num_seqs, dt))


def pivot_workspace_size(T, H, d, topk, num_seqs, g, c, mode, dtype=torch.bfloat16, dense_below=0,
                         max_rows=0) -> int:
    """Workspace bytes; max_rows > 0: for calls whose rows= range spans at most max_rows rows."""
    dt = N.BF16 if dtype == torch.bfloat16 else N.F32
    return int(N.lib().idx_pivot_workspace_size_rows(T, H, d, topk, num_seqs, dt, g, c, _mode(mode),
                                                     int(dense_below), int(max_rows)))


def decode_workspace_size(B, G, n_max, H, d, topk, c, mode, dtype=torch.bfloat16) -> int:
    dt = N.BF16 if dtype == torch.bfloat16 else N.F32
    return int(N.lib().idx_decode_workspace_size(B, G, n_max, H, d, topk, c, _mode(mode), dt))


def _outs(rows_shape, topk, device, out_idx, out_score, return_scores):
    if out_idx is None:
        out_idx = torch.empty(*rows_shape, topk, dtype=torch.int32, device=device)
    if out_score is None and return_scores:
        out_score = torch.empty(*rows_shape, topk, dtype=torch.float32, device=device)
    return out_idx, out_score


def dense_topk(q, k, w, cu_seqlens, topk: int, out_idx=None, out_score=None, workspace=None, stream=None,
               return_scores=False, rows=None):
    """Dense indexer + top-k; q [T,H,d], k [T,d], w [T,H] fp32, cu_seqlens int32 [S+1].
    rows=(lo, hi): compute output rows lo..hi-1 only (the others are left as they are)."""
    T, H, d = q.shape
    S = cu_seqlens.numel() - 1
    dt = _dtype_code(q)
    lo, hi = (0, T) if rows is None else (int(rows[0]), int(rows[1]))
    ws = _ws(workspace, dense_workspace_size(T, H, d, topk, S, q.dtype, max(1, hi - lo)), q.device)
    out_idx, out_score = _outs((T,), topk, q.device, out_idx, out_score, return_scores)
    N.check(N.lib().idx_dense_topk_rows(
        _dev(q, "q"), _dev(k, "k", q.dtype), _dev(w, "w", torch.float32), _dev(cu_seqlens, "cu_seqlens", torch.int32),
        S, T, H, d, topk, dt, lo, hi, _dev(out_idx, "out_idx", torch.int32),
        _dev(out_score, "out_score", torch.float32) if out_score is not None else None,
        ws.data_ptr(), ws.numel(), _stream(stream)), "idx_dense_topk_rows")
    return (out_idx, out_score) if return_scores else out_idx


def adaptive_topk(q, k, w, cu_seqlens, topk: int, rho: int = 2, qfrac: float = 0.4, out_idx=None, out_score=None,
                  out_sigma=None, out_trigger=None, workspace=None, stream=None):
    """Dense top-k with the cutoff-margin budget: rows whose margin sigma is in
    the bottom qfrac of the call keep rho*topk positions, the others topk
    (padded with -1).  Returns (idx [T, rho*topk], scores, sigma [T], trigger [T] uint8)."""
    T, H, d = q.shape
    S = cu_seqlens.numel() - 1
    dt = _dtype_code(q)
    width = rho * topk
    ws = _ws(workspace, adaptive_workspace_size(T, H, d, topk, rho, S, q.dtype), q.device)
    if out_idx is None:
        out_idx = torch.empty(T, width, dtype=torch.int32, device=q.device)
    if out_score is None:
        out_score = torch.empty(T, width, dtype=torch.float32, device=q.device)
    if out_sigma is None:
        out_sigma = torch.empty(T, dtype=torch.float32, device=q.device)
    if out_trigger is None:
        out_trigger = torch.empty(T, dtype=torch.uint8, device=q.device)
    N.check(N.lib().idx_adaptive_topk(
        _dev(q, "q"), _dev(k, "k", q.dtype), _dev(w, "w", torch.float32), _dev(cu_seqlens, "cu_seqlens", torch.int32),
        S, T, H, d, topk, rho, float(qfrac), dt, _dev(out_idx, "out_idx", torch.int32),
        _dev(out_score, "out_score", torch.float32), _dev(out_sigma, "out_sigma", torch.float32),
        _dev(out_trigger, "out_trigger", torch.uint8), ws.data_ptr(), ws.numel(), _stream(stream)),
        "idx_adaptive_topk")
    return out_idx, out_score, out_sigma, out_trigger


def pivot_topk(q, k, w, cu_seqlens, topk: int, g: int, c: int, mode="refine", out_idx=None, out_score=None,
               workspace=None, stream=None, return_scores=False, dense_below: int = 0, rows=None):
    """PIVOT Reuse / Refine indexer + top-k over groups of g queries.
    dense_below > 0: groups whose last member's prefix holds at most that many
    keys take the dense top-k (the guardrail).  rows=(lo, hi): output rows
    lo..hi-1 only."""
    T, H, d = q.shape
    S = cu_seqlens.numel() - 1
    dt = _dtype_code(q)
    m = _mode(mode)
    lo, hi = (0, T) if rows is None else (int(rows[0]), int(rows[1]))
    ws = _ws(workspace, pivot_workspace_size(T, H, d, topk, S, g, c, m, q.dtype, dense_below, max(1, hi - lo)),
             q.device)
    out_idx, out_score = _outs((T,), topk, q.device, out_idx, out_score, return_scores)
    N.check(N.lib().idx_pivot_topk_rows(
        _dev(q, "q"), _dev(k, "k", q.dtype), _dev(w, "w", torch.float32), _dev(cu_seqlens, "cu_seqlens", torch.int32),
        S, T, H, d, topk, dt, g, c, m, int(dense_below), lo, hi, _dev(out_idx, "out_idx", torch.int32),
        _dev(out_score, "out_score", torch.float32) if out_score is not None else None,
        ws.data_ptr(), ws.numel(), _stream(stream)), "idx_pivot_topk_rows")
    return (out_idx, out_score) if return_scores else out_idx


def decode_topk(q, kcache, kv_len, w, topk: int, c: int = 0, mode="dense", out_idx=None, out_score=None,
                workspace=None, stream=None, return_scores=False):
    """One decode step: q [B,G,H,d], kcache [B,n_max,d], kv_len int32 [B], w [B,G,H]."""
    B, G, H, d = q.shape
    n_max = kcache.shape[1]
    dt = _dtype_code(q)
    m = _mode(mode)
    ws = _ws(workspace, decode_workspace_size(B, G, n_max, H, d, topk, c, m, q.dtype), q.device)
    out_idx, out_score = _outs((B, G), topk, q.device, out_idx, out_score, return_scores)
    N.check(N.lib().idx_decode_topk(
        _dev(q, "q"), _dev(kcache, "kcache", q.dtype), _dev(kv_len, "kv_len", torch.int32),
        _dev(w, "w", torch.float32), B, G, n_max, H, d, topk, c, m, dt, _dev(out_idx, "out_idx", torch.int32),
        _dev(out_score, "out_score", torch.float32) if out_score is not None else None,
        ws.data_ptr(), ws.numel(), _stream(stream)), "idx_decode_topk")
    return (out_idx, out_score) if return_scores else out_idx


def decode_paged_topk(q, kpool, block_table, kv_len, w, topk: int, c: int = 0, mode="dense", out_idx=None,
                      out_score=None, workspace=None, stream=None, return_scores=False):
    """One decode step over a paged cache: q [B,G,H,d], kpool [num_pages,page,d],
    block_table int32 [B,max_pages], kv_len int32 [B], w [B,G,H]."""
    B, G, H, d = q.shape
    num_pages, page = kpool.shape[0], kpool.shape[1]
    max_pages = block_table.shape[1]
    if block_table.shape[0] != B:
        raise ValueError("block_table must have one row per request")
    dt = _dtype_code(q)
    m = _mode(mode)
    ws = _ws(workspace, decode_workspace_size(B, G, max_pages * page, H, d, topk, c, m, q.dtype), q.device)
    out_idx, out_score = _outs((B, G), topk, q.device, out_idx, out_score, return_scores)
    N.check(N.lib().idx_decode_paged_topk(
        _dev(q, "q"), _dev(kpool, "kpool", q.dtype), _dev(block_table, "block_table", torch.int32),
        _dev(kv_len, "kv_len", torch.int32), _dev(w, "w", torch.float32), B, G, max_pages, page, num_pages, H, d,
        topk, c, m, dt, _dev(out_idx, "out_idx", torch.int32),
        _dev(out_score, "out_score", torch.float32) if out_score is not None else None,
        ws.data_ptr(), ws.numel(), _stream(stream)), "idx_decode_paged_topk")
    return (out_idx, out_score) if return_scores else out_idx


def decode_block_means(kcache, kbar=None, first_block: int = 0, stream=None):
    """Block means [B, n_max/64, d] of a decode cache kcache [B, n_max, d]
    (n_max a multiple of 64); blocks >= first_block are (re)written."""
    B, n_max, d = kcache.shape
    if kbar is None:
        kbar = torch.empty(B, n_max // 64, d, dtype=kcache.dtype, device=kcache.device)
    N.check(N.lib().idx_decode_block_means(_dev(kcache, "kcache"), B, n_max, d, _dtype_code(kcache), first_block,
                                           _dev(kbar, "kbar", kcache.dtype), _stream(stream)),
            "idx_decode_block_means")
    return kbar


def decode_block_minmax(kcache, kminmax=None, first_block: int = 0, stream=None):
    """Per-block key minimum and maximum [B, n_max/64, 2, d] of a decode cache
    kcache [B, n_max, d] (the Quest rule's block summaries); blocks >=
    first_block are (re)written."""
    B, n_max, d = kcache.shape
    if kminmax is None:
        kminmax = torch.empty(B, n_max // 64, 2, d, dtype=kcache.dtype, device=kcache.device)
    N.check(N.lib().idx_decode_block_minmax(_dev(kcache, "kcache"), B, n_max, d, _dtype_code(kcache), first_block,
                                            _dev(kminmax, "kminmax", kcache.dtype), _stream(stream)),
            "idx_decode_block_minmax")
    return kminmax


_RULES = {"mean": 0, "quest": 1}


def decode_block_workspace_size(B, G, n_max, H, d, topk, c, rule="mean", dtype=torch.bfloat16) -> int:
    dt = N.BF16 if dtype == torch.bfloat16 else N.F32
    return int(N.lib().idx_decode_block_workspace_size(B, G, n_max, H, d, topk, c, _RULES[rule], dt))


def decode_block_topk(q, kcache, ksum, kv_len, w, topk: int, c: int, rule="mean", out_idx=None, out_score=None,
                      workspace=None, stream=None, return_scores=False):
    """One decode step with the block pre-filter: q [B,G,H,d], kcache [B,n_max,d],
    kv_len int32 [B], w [B,G,H]; ksum = block means [B,n_max/64,d] for
    rule="mean" (decode_block_means) or block min/max [B,n_max/64,2,d] for
    rule="quest" (decode_block_minmax)."""
    B, G, H, d = q.shape
    n_max = kcache.shape[1]
    dt = _dtype_code(q)
    ws = _ws(workspace, decode_block_workspace_size(B, G, n_max, H, d, topk, c, rule, q.dtype), q.device)
    out_idx, out_score = _outs((B, G), topk, q.device, out_idx, out_score, return_scores)
    N.check(N.lib().idx_decode_block_topk(
        _dev(q, "q"), _dev(kcache, "kcache", q.dtype), _dev(ksum, "ksum", q.dtype), _RULES[rule],
        _dev(kv_len, "kv_len", torch.int32), _dev(w, "w", torch.float32), B, G, n_max, H, d, topk, c, dt,
        _dev(out_idx, "out_idx", torch.int32),
        _dev(out_score, "out_score", torch.float32) if out_score is not None else None,
        ws.data_ptr(), ws.numel(), _stream(stream)), "idx_decode_block_topk")
    return (out_idx, out_score) if return_scores else out_idx


def sparse_attn(q, kv, idx, cu_q, cu_kv, scale: float, out=None, lse=None, workspace=None, stream=None,
                return_lse=False):
    """Token-sparse attention over the selected positions: q [R,H,576] bf16,
    kv [Nkv,576] bf16 (value = first 512 dims), idx int32 [R,topk] (-1 = none),
    cu_q / cu_kv int32 request boundaries over query rows and kv rows."""
    R, H, Dqk = q.shape
    Nkv = kv.shape[0]
    Dv = 512
    topk = idx.shape[1]
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty(R, H, Dv, dtype=q.dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty(R, H, dtype=torch.float32, device=q.device)
    ws = _ws(workspace, int(N.lib().idx_sparse_attn_workspace_size()), q.device)
    N.check(N.lib().idx_sparse_attn(
        _dev(q, "q"), _dev(kv, "kv", q.dtype), _dev(idx, "idx", torch.int32), _dev(cu_q, "cu_q", torch.int32),
        _dev(cu_kv, "cu_kv", torch.int32), cu_q.numel() - 1, R, Nkv, H, Dqk, Dv, topk, float(scale), dt,
        _dev(out, "out", q.dtype), _dev(lse, "lse", torch.float32) if lse is not None else None,
        ws.data_ptr(), ws.numel(), _stream(stream)), "idx_sparse_attn")
    return (out, lse) if return_lse else out


def device_status(workspace: torch.Tensor, stream=None) -> str:
    """Synchronise the stream and return the status name recorded in the workspace."""
    code = N.lib().idx_device_status(workspace.data_ptr(), _stream(stream))
    return N.STATUS.get(code, str(code))


def uses_tensor_cores(H: int, d: int, dtype=torch.bfloat16) -> bool:
    dt = N.BF16 if dtype == torch.bfloat16 else N.F32
    return bool(N.lib().idx_uses_tensor_cores(H, d, dt))


def debug_scores(stage: int, q, k, w, cu_seqlens, topk, rows, g=1, c=0, workspace=None, ld=None, stream=None):
    """Scores the selection used (test hook): stage 0 dense rows, 1 proxies, 2 Refine members,
    3 block-mode proxies against block mean keys, 4 block-mode members.
    `workspace` must be the one the matching top-k call used (required for stages 2 and 4)."""
    T, H, d = q.shape
    S = cu_seqlens.numel() - 1
    dt = _dtype_code(q)
    rows = rows.to(device=q.device, dtype=torch.int32).contiguous()
    width = ld or (c if stage in (2, 4) else (max(T // 64, 1) if stage == 3 else T))
    out = torch.full((rows.numel(), width), float("nan"), dtype=torch.float32, device=q.device)
    if workspace is None:
        if stage == 0:
            need = dense_workspace_size(T, H, d, topk, S, q.dtype)
        elif stage >= 3:
            need = pivot_workspace_size(T, H, d, topk, S, g, c, "block", q.dtype)
        else:
            need = pivot_workspace_size(T, H, d, topk, S, g, c if c > 0 else topk, "refine" if c > 0 else "reuse",
                                        q.dtype)
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    N.check(N.lib().idx_debug_scores(
        stage, _dev(q, "q"), _dev(k, "k", q.dtype), _dev(w, "w", torch.float32),
        _dev(cu_seqlens, "cu_seqlens", torch.int32), S, T, H, d, dt, g, c, topk, rows.data_ptr(), rows.numel(),
        out.data_ptr(), width, workspace.data_ptr(), workspace.numel(), _stream(stream)), "idx_debug_scores")
    return out


def debug_decode_scores(stage: int, q, kcache, kv_len, w, topk, c=0, mode="dense", workspace=None, stream=None):
    """Decode scores the selection used (test hook): stage 0 dense queries, 1 proxies, 2 Refine members."""
    B, G, H, d = q.shape
    n_max = kcache.shape[1]
    dt = _dtype_code(q)
    m = _mode(mode)
    rows = B if stage == 1 else B * G
    width = c if stage == 2 else n_max
    out = torch.full((rows, width), float("nan"), dtype=torch.float32, device=q.device)
    if workspace is None:
        need = max(decode_workspace_size(B, G, n_max, H, d, topk, c, mm, q.dtype)
                   for mm in ((0, m) if m != 0 else (0,)))
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    N.check(N.lib().idx_debug_decode_scores(
        stage, _dev(q, "q"), _dev(kcache, "kcache", q.dtype), _dev(kv_len, "kv_len", torch.int32),
        _dev(w, "w", torch.float32), B, G, n_max, H, d, topk, c, m, dt, out.data_ptr(), width,
        workspace.data_ptr(), workspace.numel(), _stream(stream)), "idx_debug_decode_scores")
    return out
