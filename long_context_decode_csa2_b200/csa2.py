"""Thin Python binding of the CSA2 C ABI (``include/csa2.h``).

Argument marshalling only: every function below forwards torch CUDA tensors
as raw device pointers to the function of the same name in ``libcsa2.so`` and
raises on a non-zero status.  All computation happens in the library's CUDA
kernels; there is no fallback of any kind.  Workspaces come from
``workspace(nbytes)`` (zero-filled, 256-byte aligned torch allocations).
"""
from __future__ import annotations

import ctypes as C
import os

import torch

from . import _build

MAIN_DIM, Q_HEADS, IDX_HEADS, IDX_DIM, BLOCK, WINDOW = 512, 16, 4, 128, 8, 128
DEV_FLAGS = {1: "INDEX_RANGE", 2: "ROW_LAYOUT", 4: "FP16_RANGE", 8: "LENGTH"}

_lib = None


class Csa2Error(RuntimeError):
    def __init__(self, status, fn, msg):
        super().__init__(f"{fn}: status {status} ({msg})")
        self.status = status


class MXFP4Cache(C.Structure):
    _fields_ = [("codes", C.c_void_p), ("scales", C.c_void_p), ("rows", C.c_int64)]


class PageTable:
    """Paged cache layout: ``pages`` [B, max_pages] int32 CUDA tensor of page
    ids, ``page_rows`` rows per page (a power of two, >= 512).  Pass it where a
    call takes ``seq_row_off``; the ``*_paged`` entry point is used then."""

    def __init__(self, pages: torch.Tensor, page_rows: int):
        assert pages.dtype == torch.int32 and pages.dim() == 2
        self.pages, self.page_rows = pages, int(page_rows)

    @property
    def max_pages(self):
        return self.pages.shape[1]


def lib():
    """Load (building first if the sources are newer) the CUDA library."""
    global _lib
    if _lib is None:
        path = _build.LIB
        if _build.stale():
            path = _build.build()
        if not os.path.exists(path):
            raise RuntimeError("libcsa2.so is missing and could not be built")
        L = C.CDLL(path)
        P, I, I64, F, Z = C.c_void_p, C.c_int, C.c_int64, C.c_float, C.c_size_t
        Cache = MXFP4Cache
        sig = {
            "csa2_index_full_workspace_bytes": (Z, [I, I, I, I]),
            "csa2_index_full": (I, [Cache, P, P, P, P, P, I, I, I, I, P, P, P, P, Z, P]),
            "csa2_index_reindex_workspace_bytes": (Z, [I, I, I]),
            "csa2_index_reindex": (I, [Cache, P, P, P, P, P, P, I, I, I, P, P, Z, P]),
            "csa2_sparse_attn_decode_workspace_bytes": (Z, [I, I]),
            "csa2_sparse_attn_decode": (I, [P, Cache, P, P, P, I, P, P, P, F, P, P, I, P, Z, P]),
            "csa2_compress_append_workspace_bytes": (Z, [I]),
            "csa2_compress_append": (I, [Cache, Cache, P, P, P, P, P, P, P, P, I, I, I64, I64, P, Z, P]),
            "csa2_compress_stream_workspace_bytes": (Z, [I]),
            "csa2_compress_stream": (I, [Cache, Cache, P, P, P, P, P, P, P, P, P, P, P, P, I, I64, I64, P, Z, P]),
            "csa2_index_multi_workspace_bytes": (Z, [I, I, I64, I, I]),
            "csa2_index_multi": (I, [Cache, P, P, P, P, P, P, I, I, I64, I, I, P, P, P, P, Z, P]),
            "csa2_index_full_pool": (I, [Cache, P, P, P, P, P, I, I, I, I, P, P, P, Z, P]),
            "csa2_index_full_topk": (I, [Cache, P, P, P, P, P, I, I, I, I, P, P, P, P, Z, P]),
            "csa2_index_full_paged": (I, [Cache, P, P, P, P, I, I, P, I, I, I, I, P, P, P, P, Z, P]),
            "csa2_index_reindex_paged": (I, [Cache, P, P, P, P, I, I, P, P, I, I, I, P, P, Z, P]),
            "csa2_sparse_attn_decode_paged": (I, [P, Cache, P, I, I, P, P, I, P, P, P, F, P, P, I, P, Z, P]),
            "csa2_compress_stream_paged": (I, [Cache, Cache, P, P, P, P, P, P, I, I, P, P, P, P, P, P, I, I64, I64, P,
                                               Z, P]),
            "csa2_score_positions_workspace_bytes": (Z, [I]),
            "csa2_score_positions": (I, [Cache, P, P, P, P, P, P, I, I, I, P, P, Z, P]),
            "csa2_topk_merge_workspace_bytes": (Z, [I, I, I]),
            "csa2_topk_merge": (I, [P, P, P, I, I, I, I, P, P, P, P, P, Z, P]),
            "csa2_attn_combine": (I, [P, P, I, I, P, P, P]),
            "csa2_index_prefill_workspace_bytes": (Z, [I, I64, I, I]),
            "csa2_index_prefill": (I, [Cache, P, P, P, P, I, I64, I64, I, I, I, P, P, P, Z, P]),
            "csa2_sparse_attn_prefill_workspace_bytes": (Z, [I, I]),
            "csa2_sparse_attn_prefill": (I, [P, P, I, Cache, I64, I64, I, P, I, P, I64, F, F, P, P, P, Z, P]),
            "csa2_sparse_attn_decode_noalloc": (I, [P, Cache, P, P, P, I, P, P, P, F, P, P, P, I, P]),
            "csa2_device_status": (I, [P, P, C.POINTER(C.c_uint32)]),
            "csa2_status_string": (C.c_char_p, [I]),
            "csa2_last_error": (C.c_char_p, []),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch tensor")
    if not t.is_cuda:
        raise ValueError("CSA2 arguments must be CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("CSA2 arguments must be contiguous")
    return t.data_ptr()


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _check(rc, fn):
    if rc != 0:
        L = lib()
        raise Csa2Error(rc, fn, L.csa2_last_error().decode() or L.csa2_status_string(rc).decode())


def cache(codes: torch.Tensor, scales: torch.Tensor) -> MXFP4Cache:
    """Describe an MXFP4 cache: codes uint8 [rows, n/2], scales uint8 [rows, n/32].

    The returned struct keeps references to both tensors, so the memory stays
    alive as long as the struct does."""
    assert codes.dtype == torch.uint8 and scales.dtype == torch.uint8 and codes.shape[0] == scales.shape[0]
    c = MXFP4Cache(_ptr(codes), _ptr(scales), codes.shape[0])
    c._keep = (codes, scales)
    return c


def workspace(nbytes: int, device=None) -> torch.Tensor:
    """Zero-filled device scratch (torch allocations are 256-byte aligned)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


def _ws(ws):
    return _ptr(ws), ws.numel()


def device_status(ws: torch.Tensor, stream=None) -> int:
    """Synchronise, return and clear the workspace's device status flags."""
    flags = C.c_uint32(0)
    rc = lib().csa2_device_status(_ptr(ws), _stream(stream), C.byref(flags))
    if rc not in (0, -5):
        _check(rc, "csa2_device_status")
    return int(flags.value)


# ----------------------------------------------------------------------------
# one wrapper per C entry point
# ----------------------------------------------------------------------------

def csa2_index_full_workspace_bytes(B, max_len, pool_blocks, k):
    return lib().csa2_index_full_workspace_bytes(B, max_len, pool_blocks, k)


def csa2_index_full(idx_k, q_codes, q_scales, w, seq_row_off, seq_len, max_len, pool_blocks, k, pool_out, topk_out,
                    ws, scores_out=None, stream=None):
    B = seq_len.shape[0]
    wp, wn = _ws(ws)
    if isinstance(seq_row_off, PageTable):
        pt = seq_row_off
        rc = lib().csa2_index_full_paged(idx_k, _ptr(q_codes), _ptr(q_scales), _ptr(w), _ptr(pt.pages), pt.page_rows,
                                         pt.max_pages, _ptr(seq_len), B, max_len, pool_blocks, k, _ptr(pool_out),
                                         _ptr(topk_out), _ptr(scores_out), wp, wn, _stream(stream))
        _check(rc, "csa2_index_full_paged")
        return
    rc = lib().csa2_index_full(idx_k, _ptr(q_codes), _ptr(q_scales), _ptr(w), _ptr(seq_row_off), _ptr(seq_len), B,
                               max_len, pool_blocks, k, _ptr(pool_out), _ptr(topk_out), _ptr(scores_out), wp, wn,
                               _stream(stream))
    _check(rc, "csa2_index_full")


def csa2_index_full_pool(idx_k, q_codes, q_scales, w, seq_row_off, seq_len, max_len, pool_blocks, k, pool_out, ws,
                         scores_out=None, stream=None):
    B = seq_len.shape[0]
    wp, wn = _ws(ws)
    rc = lib().csa2_index_full_pool(idx_k, _ptr(q_codes), _ptr(q_scales), _ptr(w), _ptr(seq_row_off), _ptr(seq_len),
                                    B, max_len, pool_blocks, k, _ptr(pool_out), _ptr(scores_out), wp, wn,
                                    _stream(stream))
    _check(rc, "csa2_index_full_pool")


def csa2_index_full_topk(idx_k, q_codes, q_scales, w, seq_row_off, seq_len, max_len, pool_blocks, k, pool, topk_out,
                         ws, scores_out=None, stream=None):
    B = seq_len.shape[0]
    wp, wn = _ws(ws)
    rc = lib().csa2_index_full_topk(idx_k, _ptr(q_codes), _ptr(q_scales), _ptr(w), _ptr(seq_row_off), _ptr(seq_len),
                                    B, max_len, pool_blocks, k, _ptr(pool), _ptr(topk_out), _ptr(scores_out), wp, wn,
                                    _stream(stream))
    _check(rc, "csa2_index_full_topk")


def csa2_index_reindex_workspace_bytes(B, pool_blocks, k):
    return lib().csa2_index_reindex_workspace_bytes(B, pool_blocks, k)


def csa2_index_reindex(idx_k, q_codes, q_scales, w, seq_row_off, seq_len, pool, k, topk_out, ws, stream=None):
    B, P = pool.shape
    wp, wn = _ws(ws)
    if isinstance(seq_row_off, PageTable):
        pt = seq_row_off
        rc = lib().csa2_index_reindex_paged(idx_k, _ptr(q_codes), _ptr(q_scales), _ptr(w), _ptr(pt.pages),
                                            pt.page_rows, pt.max_pages, _ptr(seq_len), _ptr(pool), B, P, k,
                                            _ptr(topk_out), wp, wn, _stream(stream))
        _check(rc, "csa2_index_reindex_paged")
        return
    rc = lib().csa2_index_reindex(idx_k, _ptr(q_codes), _ptr(q_scales), _ptr(w), _ptr(seq_row_off), _ptr(seq_len),
                                  _ptr(pool), B, P, k, _ptr(topk_out), wp, wn, _stream(stream))
    _check(rc, "csa2_index_reindex")


def csa2_sparse_attn_decode_workspace_bytes(B, k):
    return lib().csa2_sparse_attn_decode_workspace_bytes(B, k)


def csa2_sparse_attn_decode(q, main_kv, seq_row_off, seq_len, topk, win, win_scale, win_len, sm_scale, out, ws,
                            lse=None, stream=None):
    B, k = topk.shape
    wp, wn = _ws(ws)
    if isinstance(seq_row_off, PageTable):
        pt = seq_row_off
        rc = lib().csa2_sparse_attn_decode_paged(_ptr(q), main_kv, _ptr(pt.pages), pt.page_rows, pt.max_pages,
                                                 _ptr(seq_len), _ptr(topk), k, _ptr(win), _ptr(win_scale),
                                                 _ptr(win_len), float(sm_scale), _ptr(out), _ptr(lse), B, wp, wn,
                                                 _stream(stream))
        _check(rc, "csa2_sparse_attn_decode_paged")
        return
    rc = lib().csa2_sparse_attn_decode(_ptr(q), main_kv, _ptr(seq_row_off), _ptr(seq_len), _ptr(topk), k, _ptr(win),
                                       _ptr(win_scale), _ptr(win_len), float(sm_scale), _ptr(out), _ptr(lse), B, wp,
                                       wn, _stream(stream))
    _check(rc, "csa2_sparse_attn_decode")


def csa2_compress_append_workspace_bytes(B):
    return lib().csa2_compress_append_workspace_bytes(B)


def csa2_compress_append(main_kv, idx_k, raw, logits, tok_off, seq_row_off, seq_len_in, seq_len_out, ratio, max_new,
                         ws, w_idx=None, idx_raw=None, stream=None):
    B = seq_len_in.shape[0]
    wp, wn = _ws(ws)
    rc = lib().csa2_compress_append(main_kv, idx_k, _ptr(raw), _ptr(logits), _ptr(w_idx), _ptr(idx_raw),
                                    _ptr(tok_off), _ptr(seq_row_off), _ptr(seq_len_in), _ptr(seq_len_out), B, ratio,
                                    raw.shape[0], int(max_new), wp, wn, _stream(stream))
    _check(rc, "csa2_compress_append")


def csa2_compress_stream_workspace_bytes(B):
    return lib().csa2_compress_stream_workspace_bytes(B)


def csa2_compress_stream(main_kv, idx_k, raw, logits, tok_off, seq_row_off, seq_len_in, seq_len_out, pend_n, pend_raw,
                         pend_logit, max_new, ws, w_idx=None, idx_raw=None, pend_idx=None, stream=None):
    """seq_len_out may be seq_len_in (in place) or None; raw may be None when no token is appended."""
    B = seq_len_in.shape[0]
    wp, wn = _ws(ws)
    n_tok = raw.shape[0] if raw is not None else 0
    if isinstance(seq_row_off, PageTable):
        pt = seq_row_off
        rc = lib().csa2_compress_stream_paged(main_kv, idx_k, _ptr(raw), _ptr(logits), _ptr(w_idx), _ptr(idx_raw),
                                              _ptr(tok_off), _ptr(pt.pages), pt.page_rows, pt.max_pages,
                                              _ptr(seq_len_in), _ptr(seq_len_out), _ptr(pend_n), _ptr(pend_raw),
                                              _ptr(pend_logit), _ptr(pend_idx), B, n_tok, int(max_new), wp, wn,
                                              _stream(stream))
        _check(rc, "csa2_compress_stream_paged")
        return
    rc = lib().csa2_compress_stream(main_kv, idx_k, _ptr(raw), _ptr(logits), _ptr(w_idx), _ptr(idx_raw),
                                    _ptr(tok_off), _ptr(seq_row_off), _ptr(seq_len_in), _ptr(seq_len_out),
                                    _ptr(pend_n), _ptr(pend_raw), _ptr(pend_logit), _ptr(pend_idx), B, n_tok,
                                    int(max_new), wp, wn, _stream(stream))
    _check(rc, "csa2_compress_stream")


def csa2_index_multi_workspace_bytes(B, Q, max_vis, pool_blocks, k):
    return lib().csa2_index_multi_workspace_bytes(B, Q, max_vis, pool_blocks, k)


def csa2_index_multi(idx_k, q_codes, q_scales, w, seq_row_off, q_off, q_vis, max_vis, pool_blocks, k, pool_out,
                     topk_out, ws, q_row_off_out=None, stream=None):
    B, Q = seq_row_off.shape[0], q_vis.shape[0]
    wp, wn = _ws(ws)
    rc = lib().csa2_index_multi(idx_k, _ptr(q_codes), _ptr(q_scales), _ptr(w), _ptr(seq_row_off), _ptr(q_off),
                                _ptr(q_vis), B, Q, int(max_vis), pool_blocks, k, _ptr(pool_out), _ptr(topk_out),
                                _ptr(q_row_off_out), wp, wn, _stream(stream))
    _check(rc, "csa2_index_multi")


def csa2_score_positions_workspace_bytes(B):
    return lib().csa2_score_positions_workspace_bytes(B)


def csa2_score_positions(idx_k, q_codes, q_scales, w, seq_row_off, seq_len, ids, block, keys_out, ws, stream=None):
    """keys_out [B, n] uint32 (int32 tensors carry the bits) <- rank keys of ids [B, n] (block 1 or 8)."""
    B, n = ids.shape
    wp, wn = _ws(ws)
    rc = lib().csa2_score_positions(idx_k, _ptr(q_codes), _ptr(q_scales), _ptr(w), _ptr(seq_row_off), _ptr(seq_len),
                                    _ptr(ids), B, n, int(block), _ptr(keys_out), wp, wn, _stream(stream))
    _check(rc, "csa2_score_positions")


def csa2_topk_merge_workspace_bytes(G, B, n):
    return lib().csa2_topk_merge_workspace_bytes(G, B, n)


def csa2_topk_merge(keys, ids, src_off, k, out, ws, lo=None, hi=None, out_local=None, stream=None):
    """keys / ids [G, B, n] from the shards -> out [B, k] (and out_local [B, k] for [lo, hi))."""
    G, B, n = ids.shape
    wp, wn = _ws(ws)
    rc = lib().csa2_topk_merge(_ptr(keys), _ptr(ids), _ptr(src_off), G, B, n, k, _ptr(lo), _ptr(hi), _ptr(out),
                               _ptr(out_local), wp, wn, _stream(stream))
    _check(rc, "csa2_topk_merge")


def csa2_attn_combine(out_parts, lse_parts, out, lse=None, stream=None):
    """out_parts [G, B, 16, 512], lse_parts [G, B, 16] -> out [B, 16, 512], lse [B, 16]."""
    G, B = lse_parts.shape[0], lse_parts.shape[1]
    rc = lib().csa2_attn_combine(_ptr(out_parts), _ptr(lse_parts), G, B, _ptr(out), _ptr(lse), _stream(stream))
    _check(rc, "csa2_attn_combine")


def csa2_index_prefill_workspace_bytes(T, n_entries, pool_blocks, k):
    return lib().csa2_index_prefill_workspace_bytes(T, n_entries, pool_blocks, k)


def csa2_index_prefill(idx_k, q_codes, q_scales, w, q_pos, row0, n_entries, ratio, pool_blocks, k, pool_out,
                       topk_out, ws, stream=None):
    T = q_pos.shape[0]
    wp, wn = _ws(ws)
    rc = lib().csa2_index_prefill(idx_k, _ptr(q_codes), _ptr(q_scales), _ptr(w), _ptr(q_pos), T, row0, n_entries,
                                  ratio, pool_blocks, k, _ptr(pool_out), _ptr(topk_out), wp, wn, _stream(stream))
    _check(rc, "csa2_index_prefill")


def csa2_sparse_attn_prefill_workspace_bytes(T, k):
    return lib().csa2_sparse_attn_prefill_workspace_bytes(T, k)


def csa2_sparse_attn_prefill(q, q_pos, main_kv, row0, n_entries, ratio, topk, raw_win, win_scale, sm_scale, out, ws,
                             lse=None, stream=None):
    T, k = topk.shape
    wp, wn = _ws(ws)
    rc = lib().csa2_sparse_attn_prefill(_ptr(q), _ptr(q_pos), T, main_kv, row0, n_entries, ratio, _ptr(topk), k,
                                        _ptr(raw_win), raw_win.shape[0], float(win_scale), float(sm_scale), _ptr(out),
                                        _ptr(lse), wp, wn, _stream(stream))
    _check(rc, "csa2_sparse_attn_prefill")


def csa2_sparse_attn_decode_noalloc(q, main_kv, seq_row_off, seq_len, topk, win, win_scale, win_len, sm_scale, out,
                                    lse=None, flags_out=None, stream=None):
    """csa2_sparse_attn_decode without a workspace (fixed library scratch; B <= 64, k <= 512).

    For callers that may not allocate device memory while they run.  All calls
    on one device share the scratch, so calls that overlap on the GPU race."""
    B, k = topk.shape
    rc = lib().csa2_sparse_attn_decode_noalloc(_ptr(q), main_kv, _ptr(seq_row_off), _ptr(seq_len), _ptr(topk), k,
                                               _ptr(win), _ptr(win_scale), _ptr(win_len), float(sm_scale), _ptr(out),
                                               _ptr(lse), _ptr(flags_out), B, _stream(stream))
    _check(rc, "csa2_sparse_attn_decode_noalloc")
