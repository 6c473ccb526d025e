"""Thin Python binding of the CSA2 C ABI (``include/csa2.h``).

Argument marshalling only: every function below checks each tensor's element
type and size against the C declaration (the library sees only pointers),
forwards the torch CUDA tensors as raw device pointers to the function of the
same name in ``libcsa2.so`` and raises on a non-zero status.  All computation
happens in the library's CUDA kernels; there is no fallback of any kind.  Workspaces come from
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


# Element types of the C ABI's pointer arguments and the torch dtypes that
# may carry them (same width, same kind of number).
_KINDS = {
    "u8": (torch.uint8, torch.int8, torch.float8_e4m3fn),   # E2M1 codes, E8M0 scales, E4M3 bytes
    "bf16": (torch.bfloat16, torch.int16, torch.uint16),    # bf16 bit patterns
    "i32": (torch.int32, torch.uint32),                     # int32 ids / lengths, uint32 keys and flags
    "f32": (torch.float32,),
    "i64": (torch.int64, torch.uint64),
}


def _arg(fn, name, t, kind, numel=0):
    """Device pointer of an optional tensor argument, after checking that its
    elements have the C type's width and kind and that it holds at least
    `numel` of them (the library cannot see buffer sizes)."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise Csa2Error(-1, fn, f"{name}: expected a torch tensor, got {type(t).__name__}")
    if t.dtype not in _KINDS[kind]:
        raise Csa2Error(-1, fn, f"{name}: {kind} elements expected, got {t.dtype}")
    if t.numel() < numel:
        raise Csa2Error(-1, fn, f"{name}: at least {numel} elements expected, got {t.numel()}")
    return _ptr(t)


def _queries(fn, n, q_codes, q_scales, w):
    """Pointers of n indexer queries: codes [n][4][64], scales [n][4][4], weights [n][4]."""
    return (_arg(fn, "q_codes", q_codes, "u8", n * IDX_HEADS * IDX_DIM // 2),
            _arg(fn, "q_scales", q_scales, "u8", n * IDX_HEADS * IDX_DIM // 32),
            _arg(fn, "w", w, "f32", n * IDX_HEADS))


def _window(fn, n, win, win_scale, win_len):
    return (_arg(fn, "win", win, "u8", n * WINDOW * MAIN_DIM), _arg(fn, "win_scale", win_scale, "f32", n),
            _arg(fn, "win_len", win_len, "i32", n))


def _attn_out(fn, n, out, lse):
    return _arg(fn, "out", out, "f32", n * Q_HEADS * MAIN_DIM), _arg(fn, "lse", lse, "f32", n * Q_HEADS)


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


def _full_args(fn, q_codes, q_scales, w, seq_len, max_len, pool_blocks, k, pool_out, topk_out, scores_out):
    B = seq_len.shape[0]
    return (B, *_queries(fn, B, q_codes, q_scales, w), _arg(fn, "seq_len", seq_len, "i32", B),
            _arg(fn, "pool_out", pool_out, "i32", B * pool_blocks), _arg(fn, "topk_out", topk_out, "i32", B * k),
            _arg(fn, "scores_out", scores_out, "f32", B * max_len))


def _row_off(fn, seq_row_off, B):
    return _arg(fn, "seq_row_off", seq_row_off, "i64", B)


def _pages(fn, pt, B):
    return _arg(fn, "pages", pt.pages, "i32", B * pt.max_pages)


def csa2_index_full(idx_k, q_codes, q_scales, w, seq_row_off, seq_len, max_len, pool_blocks, k, pool_out, topk_out,
                    ws, scores_out=None, stream=None):
    wp, wn = _ws(ws)
    if isinstance(seq_row_off, PageTable):
        fn, pt = "csa2_index_full_paged", seq_row_off
        B, qc, qs, wv, sl, po, to, so = _full_args(fn, q_codes, q_scales, w, seq_len, max_len, pool_blocks, k,
                                                   pool_out, topk_out, scores_out)
        rc = lib().csa2_index_full_paged(idx_k, qc, qs, wv, _pages(fn, pt, B), pt.page_rows, pt.max_pages, sl, B,
                                         max_len, pool_blocks, k, po, to, so, wp, wn, _stream(stream))
        _check(rc, fn)
        return
    fn = "csa2_index_full"
    B, qc, qs, wv, sl, po, to, so = _full_args(fn, q_codes, q_scales, w, seq_len, max_len, pool_blocks, k, pool_out,
                                               topk_out, scores_out)
    rc = lib().csa2_index_full(idx_k, qc, qs, wv, _row_off(fn, seq_row_off, B), sl, B, max_len, pool_blocks, k, po,
                               to, so, wp, wn, _stream(stream))
    _check(rc, fn)


def csa2_index_full_pool(idx_k, q_codes, q_scales, w, seq_row_off, seq_len, max_len, pool_blocks, k, pool_out, ws,
                         scores_out=None, stream=None):
    fn = "csa2_index_full_pool"
    wp, wn = _ws(ws)
    B, qc, qs, wv, sl, po, _, so = _full_args(fn, q_codes, q_scales, w, seq_len, max_len, pool_blocks, k, pool_out,
                                              None, scores_out)
    rc = lib().csa2_index_full_pool(idx_k, qc, qs, wv, _row_off(fn, seq_row_off, B), sl, B, max_len, pool_blocks, k,
                                    po, so, wp, wn, _stream(stream))
    _check(rc, fn)


def csa2_index_full_topk(idx_k, q_codes, q_scales, w, seq_row_off, seq_len, max_len, pool_blocks, k, pool, topk_out,
                         ws, scores_out=None, stream=None):
    fn = "csa2_index_full_topk"
    wp, wn = _ws(ws)
    B, qc, qs, wv, sl, po, to, so = _full_args(fn, q_codes, q_scales, w, seq_len, max_len, pool_blocks, k, pool,
                                               topk_out, scores_out)
    rc = lib().csa2_index_full_topk(idx_k, qc, qs, wv, _row_off(fn, seq_row_off, B), sl, B, max_len, pool_blocks, k,
                                    po, to, so, wp, wn, _stream(stream))
    _check(rc, fn)


def csa2_index_reindex_workspace_bytes(B, pool_blocks, k):
    return lib().csa2_index_reindex_workspace_bytes(B, pool_blocks, k)


def csa2_index_reindex(idx_k, q_codes, q_scales, w, seq_row_off, seq_len, pool, k, topk_out, ws, stream=None):
    B, P = pool.shape
    wp, wn = _ws(ws)
    paged = isinstance(seq_row_off, PageTable)
    fn = "csa2_index_reindex_paged" if paged else "csa2_index_reindex"
    qc, qs, wv = _queries(fn, B, q_codes, q_scales, w)
    sl, pp = _arg(fn, "seq_len", seq_len, "i32", B), _arg(fn, "pool", pool, "i32", B * P)
    to = _arg(fn, "topk_out", topk_out, "i32", B * k)
    if paged:
        pt = seq_row_off
        rc = lib().csa2_index_reindex_paged(idx_k, qc, qs, wv, _pages(fn, pt, B), pt.page_rows, pt.max_pages, sl, pp,
                                            B, P, k, to, wp, wn, _stream(stream))
    else:
        rc = lib().csa2_index_reindex(idx_k, qc, qs, wv, _row_off(fn, seq_row_off, B), sl, pp, B, P, k, to, wp, wn,
                                      _stream(stream))
    _check(rc, fn)


def csa2_sparse_attn_decode_workspace_bytes(B, k):
    return lib().csa2_sparse_attn_decode_workspace_bytes(B, k)


def _decode_args(fn, q, seq_len, topk, win, win_scale, win_len, out, lse):
    B, k = topk.shape
    return (B, k, _arg(fn, "q", q, "bf16", B * Q_HEADS * MAIN_DIM), _arg(fn, "seq_len", seq_len, "i32", B),
            _arg(fn, "topk", topk, "i32", B * k), *_window(fn, B, win, win_scale, win_len), *_attn_out(fn, B, out, lse))


def csa2_sparse_attn_decode(q, main_kv, seq_row_off, seq_len, topk, win, win_scale, win_len, sm_scale, out, ws,
                            lse=None, stream=None):
    wp, wn = _ws(ws)
    paged = isinstance(seq_row_off, PageTable)
    fn = "csa2_sparse_attn_decode_paged" if paged else "csa2_sparse_attn_decode"
    B, k, qp, sl, tp, wi, wsc, wl, op, lp = _decode_args(fn, q, seq_len, topk, win, win_scale, win_len, out, lse)
    if paged:
        pt = seq_row_off
        rc = lib().csa2_sparse_attn_decode_paged(qp, main_kv, _pages(fn, pt, B), pt.page_rows, pt.max_pages, sl, tp,
                                                 k, wi, wsc, wl, float(sm_scale), op, lp, B, wp, wn, _stream(stream))
    else:
        rc = lib().csa2_sparse_attn_decode(qp, main_kv, _row_off(fn, seq_row_off, B), sl, tp, k, wi, wsc, wl,
                                           float(sm_scale), op, lp, B, wp, wn, _stream(stream))
    _check(rc, fn)


def csa2_compress_append_workspace_bytes(B):
    return lib().csa2_compress_append_workspace_bytes(B)


def _append_args(fn, raw, logits, w_idx, idx_raw, tok_off, seq_len_in, seq_len_out):
    """Pointers of the token inputs and lengths shared by the append calls."""
    B = seq_len_in.shape[0]
    n_tok = raw.shape[0] if raw is not None else 0
    return (B, n_tok, _arg(fn, "raw", raw, "bf16", n_tok * MAIN_DIM), _arg(fn, "logits", logits, "f32", n_tok),
            _arg(fn, "w_idx", w_idx, "f32", MAIN_DIM * IDX_DIM), _arg(fn, "idx_raw", idx_raw, "bf16", n_tok * IDX_DIM),
            _arg(fn, "tok_off", tok_off, "i64", B + 1), _arg(fn, "seq_len_in", seq_len_in, "i32", B),
            _arg(fn, "seq_len_out", seq_len_out, "i32", B))


def csa2_compress_append(main_kv, idx_k, raw, logits, tok_off, seq_row_off, seq_len_in, seq_len_out, ratio, max_new,
                         ws, w_idx=None, idx_raw=None, stream=None):
    fn = "csa2_compress_append"
    wp, wn = _ws(ws)
    B, n_tok, rp, lg, wi, ir, to, li, lo = _append_args(fn, raw, logits, w_idx, idx_raw, tok_off, seq_len_in,
                                                        seq_len_out)
    rc = lib().csa2_compress_append(main_kv, idx_k, rp, lg, wi, ir, to, _row_off(fn, seq_row_off, B), li, lo, B,
                                    ratio, n_tok, int(max_new), wp, wn, _stream(stream))
    _check(rc, fn)


def csa2_compress_stream_workspace_bytes(B):
    return lib().csa2_compress_stream_workspace_bytes(B)


def csa2_compress_stream(main_kv, idx_k, raw, logits, tok_off, seq_row_off, seq_len_in, seq_len_out, pend_n, pend_raw,
                         pend_logit, max_new, ws, w_idx=None, idx_raw=None, pend_idx=None, stream=None):
    """seq_len_out may be seq_len_in (in place) or None; raw may be None when no token is appended."""
    wp, wn = _ws(ws)
    paged = isinstance(seq_row_off, PageTable)
    fn = "csa2_compress_stream_paged" if paged else "csa2_compress_stream"
    B, n_tok, rp, lg, wi, ir, to, li, lo = _append_args(fn, raw, logits, w_idx, idx_raw, tok_off, seq_len_in,
                                                        seq_len_out)
    pend = (_arg(fn, "pend_n", pend_n, "i32", B), _arg(fn, "pend_raw", pend_raw, "bf16", B * MAIN_DIM),
            _arg(fn, "pend_logit", pend_logit, "f32", B), _arg(fn, "pend_idx", pend_idx, "bf16", B * IDX_DIM))
    if paged:
        pt = seq_row_off
        rc = lib().csa2_compress_stream_paged(main_kv, idx_k, rp, lg, wi, ir, to, _pages(fn, pt, B), pt.page_rows,
                                              pt.max_pages, li, lo, *pend, B, n_tok, int(max_new), wp, wn,
                                              _stream(stream))
    else:
        rc = lib().csa2_compress_stream(main_kv, idx_k, rp, lg, wi, ir, to, _row_off(fn, seq_row_off, B), li, lo,
                                        *pend, B, n_tok, int(max_new), wp, wn, _stream(stream))
    _check(rc, fn)


def csa2_index_multi_workspace_bytes(B, Q, max_vis, pool_blocks, k):
    return lib().csa2_index_multi_workspace_bytes(B, Q, max_vis, pool_blocks, k)


def csa2_index_multi(idx_k, q_codes, q_scales, w, seq_row_off, q_off, q_vis, max_vis, pool_blocks, k, pool_out,
                     topk_out, ws, q_row_off_out=None, stream=None):
    fn = "csa2_index_multi"
    B, Q = seq_row_off.shape[0], q_vis.shape[0]
    wp, wn = _ws(ws)
    rc = lib().csa2_index_multi(idx_k, *_queries(fn, Q, q_codes, q_scales, w), _row_off(fn, seq_row_off, B),
                                _arg(fn, "q_off", q_off, "i32", B + 1), _arg(fn, "q_vis", q_vis, "i32", Q), B, Q,
                                int(max_vis), pool_blocks, k, _arg(fn, "pool_out", pool_out, "i32", Q * pool_blocks),
                                _arg(fn, "topk_out", topk_out, "i32", Q * k),
                                _arg(fn, "q_row_off_out", q_row_off_out, "i64", Q), wp, wn, _stream(stream))
    _check(rc, fn)


def csa2_score_positions_workspace_bytes(B):
    return lib().csa2_score_positions_workspace_bytes(B)


def csa2_score_positions(idx_k, q_codes, q_scales, w, seq_row_off, seq_len, ids, block, keys_out, ws, stream=None):
    """keys_out [B, n] uint32 (int32 tensors carry the bits) <- rank keys of ids [B, n] (block 1 or 8)."""
    fn = "csa2_score_positions"
    B, n = ids.shape
    wp, wn = _ws(ws)
    rc = lib().csa2_score_positions(idx_k, *_queries(fn, B, q_codes, q_scales, w), _row_off(fn, seq_row_off, B),
                                    _arg(fn, "seq_len", seq_len, "i32", B), _arg(fn, "ids", ids, "i32", B * n), B, n,
                                    int(block), _arg(fn, "keys_out", keys_out, "i32", B * n), wp, wn, _stream(stream))
    _check(rc, fn)


def csa2_topk_merge_workspace_bytes(G, B, n):
    return lib().csa2_topk_merge_workspace_bytes(G, B, n)


def csa2_topk_merge(keys, ids, src_off, k, out, ws, lo=None, hi=None, out_local=None, stream=None):
    """keys / ids [G, B, n] from the shards -> out [B, k] (and out_local [B, k] for [lo, hi))."""
    fn = "csa2_topk_merge"
    G, B, n = ids.shape
    wp, wn = _ws(ws)
    rc = lib().csa2_topk_merge(_arg(fn, "keys", keys, "i32", G * B * n), _arg(fn, "ids", ids, "i32", G * B * n),
                               _arg(fn, "src_off", src_off, "i64", G * B), G, B, n, k, _arg(fn, "lo", lo, "i64", B),
                               _arg(fn, "hi", hi, "i64", B), _arg(fn, "out", out, "i32", B * k),
                               _arg(fn, "out_local", out_local, "i32", B * k), wp, wn, _stream(stream))
    _check(rc, fn)


def csa2_attn_combine(out_parts, lse_parts, out, lse=None, stream=None):
    """out_parts [G, B, 16, 512], lse_parts [G, B, 16] -> out [B, 16, 512], lse [B, 16]."""
    fn = "csa2_attn_combine"
    G, B = lse_parts.shape[0], lse_parts.shape[1]
    rc = lib().csa2_attn_combine(_arg(fn, "out_parts", out_parts, "f32", G * B * Q_HEADS * MAIN_DIM),
                                 _arg(fn, "lse_parts", lse_parts, "f32", G * B * Q_HEADS), G, B,
                                 *_attn_out(fn, B, out, lse), _stream(stream))
    _check(rc, fn)


def csa2_index_prefill_workspace_bytes(T, n_entries, pool_blocks, k):
    return lib().csa2_index_prefill_workspace_bytes(T, n_entries, pool_blocks, k)


def csa2_index_prefill(idx_k, q_codes, q_scales, w, q_pos, row0, n_entries, ratio, pool_blocks, k, pool_out,
                       topk_out, ws, stream=None):
    fn = "csa2_index_prefill"
    T = q_pos.shape[0]
    wp, wn = _ws(ws)
    rc = lib().csa2_index_prefill(idx_k, *_queries(fn, T, q_codes, q_scales, w), _arg(fn, "q_pos", q_pos, "i32", T), T,
                                  row0, n_entries, ratio, pool_blocks, k,
                                  _arg(fn, "pool_out", pool_out, "i32", T * pool_blocks),
                                  _arg(fn, "topk_out", topk_out, "i32", T * k), wp, wn, _stream(stream))
    _check(rc, fn)


def csa2_sparse_attn_prefill_workspace_bytes(T, k):
    return lib().csa2_sparse_attn_prefill_workspace_bytes(T, k)


def csa2_sparse_attn_prefill(q, q_pos, main_kv, row0, n_entries, ratio, topk, raw_win, win_scale, sm_scale, out, ws,
                             lse=None, stream=None):
    fn = "csa2_sparse_attn_prefill"
    T, k = topk.shape
    wp, wn = _ws(ws)
    rc = lib().csa2_sparse_attn_prefill(_arg(fn, "q", q, "bf16", T * Q_HEADS * MAIN_DIM),
                                        _arg(fn, "q_pos", q_pos, "i32", T), T, main_kv, row0, n_entries, ratio,
                                        _arg(fn, "topk", topk, "i32", T * k), k,
                                        _arg(fn, "raw_win", raw_win, "u8", raw_win.shape[0] * MAIN_DIM),
                                        raw_win.shape[0], float(win_scale), float(sm_scale), *_attn_out(fn, T, out, lse),
                                        wp, wn, _stream(stream))
    _check(rc, fn)


def noalloc_setup(stream=None):
    """The B = 0 call of csa2_sparse_attn_decode_noalloc: loads the library's
    scratch array and the attention kernel on the current device (the one
    time that call may allocate device memory) and launches nothing."""
    fn = "csa2_sparse_attn_decode_noalloc"
    rc = lib().csa2_sparse_attn_decode_noalloc(None, MXFP4Cache(None, None, 0), None, None, None, 1, None, None, None,
                                               0.0, None, None, None, 0, _stream(stream))
    _check(rc, fn)


def csa2_sparse_attn_decode_noalloc(q, main_kv, seq_row_off, seq_len, topk, win, win_scale, win_len, sm_scale, out,
                                    lse=None, flags_out=None, stream=None):
    """csa2_sparse_attn_decode without a workspace (fixed library scratch; B <= 64, k <= 512).

    For callers that may not allocate device memory while they run.  All calls
    on one device share the scratch, so calls that overlap on the GPU race."""
    fn = "csa2_sparse_attn_decode_noalloc"
    B, k, qp, sl, tp, wi, wsc, wl, op, lp = _decode_args(fn, q, seq_len, topk, win, win_scale, win_len, out, lse)
    if B == 0:
        return noalloc_setup(stream)
    rc = lib().csa2_sparse_attn_decode_noalloc(qp, main_kv, _row_off(fn, seq_row_off, B), sl, tp, k, wi, wsc, wl,
                                               float(sm_scale), op, lp, _arg(fn, "flags_out", flags_out, "i32", 1), B,
                                               _stream(stream))
    _check(rc, fn)
