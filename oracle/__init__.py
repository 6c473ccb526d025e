"""CPU oracle for the CSA2 sparse-attention path -- TEST INFRASTRUCTURE.

Thin ctypes wrapper over ``csa2_oracle.cpp`` (plain C++17, fp64 where the
definitions ask for it).  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference leg may import this package.  The CUDA
library never loads it and shares no code with it.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa2_oracle.cpp")
_LIB = os.path.join(_HERE, "_build", "libcsa2_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no fp contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        os.makedirs(os.path.dirname(_LIB), exist_ok=True)
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math",
                               "-shared", "-fPIC", "-pthread", _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        L = _lib
        P = C.c_void_p
        L.orc_e2m1_value.restype = C.c_double
        L.orc_e2m1_value.argtypes = [C.c_int]
        L.orc_e8m0_value.restype = C.c_double
        L.orc_e8m0_value.argtypes = [C.c_int]
        L.orc_e4m3_value.restype = C.c_double
        L.orc_e4m3_value.argtypes = [C.c_int]
        L.orc_exp.restype = C.c_double
        L.orc_exp.argtypes = [C.c_double]
        L.orc_rank_key.restype = C.c_uint32
        L.orc_rank_key.argtypes = [C.c_float]
        L.orc_mxfp4_encode.restype = None
        L.orc_mxfp4_encode.argtypes = [P, C.c_int64, C.c_int, P, P]
        L.orc_mxfp4_decode.restype = None
        L.orc_mxfp4_decode.argtypes = [P, P, C.c_int64, C.c_int, P]
        L.orc_index_scores.restype = None
        L.orc_index_scores.argtypes = [P, P, P, C.c_int64, P, P, P, P]
        L.orc_topk.restype = None
        L.orc_topk.argtypes = [P, P, C.c_int64, C.c_int, P]
        L.orc_index_full.restype = C.c_int
        L.orc_index_full.argtypes = [P, P, P, P, P, P, P, C.c_int, C.c_int, C.c_int, P, P, P,
                                     C.c_int64, C.c_int]
        L.orc_index_reindex.restype = C.c_int
        L.orc_index_reindex.argtypes = [P, P, P, P, P, P, P, P, C.c_int, C.c_int, C.c_int, P, C.c_int]
        L.orc_attn_decode.restype = C.c_int
        L.orc_attn_decode.argtypes = [P, P, P, P, P, P, C.c_int, P, P, P, C.c_double, P, P, C.c_int,
                                      C.c_int]
        L.orc_compress.restype = C.c_int
        L.orc_compress.argtypes = [P, P, P, P, C.c_int64, C.c_int, P, P, P, P, P, P, C.c_int]
        L.orc_index_prefill.restype = C.c_int
        L.orc_index_prefill.argtypes = [P, P, C.c_int64, C.c_int64, P, P, P, P, P, C.c_int64, C.c_int,
                                        C.c_int, C.c_int, P, P, C.c_int]
        L.orc_attn_prefill.restype = C.c_int
        L.orc_attn_prefill.argtypes = [P, P, P, C.c_int64, P, P, C.c_int64, C.c_int64, C.c_int, P,
                                       C.c_int, P, C.c_float, C.c_double, P, P, C.c_int]
    return _lib


# ----------------------------------------------------------------------------
# formats
# ----------------------------------------------------------------------------

def e2m1_value(code: int) -> float:
    return lib().orc_e2m1_value(int(code))


def e8m0_value(byte: int) -> float:
    return lib().orc_e8m0_value(int(byte))


def e4m3_value(byte: int) -> float:
    return lib().orc_e4m3_value(int(byte))


def own_exp(x: float) -> float:
    return lib().orc_exp(float(x))


def rank_key(s) -> int:
    return int(lib().orc_rank_key(float(np.float32(s))))


def mxfp4_encode(x: np.ndarray):
    """x fp32 [rows, n] -> (codes uint8 [rows, n/2], scales uint8 [rows, n/32])."""
    x = np.ascontiguousarray(x, np.float32)
    rows, n = x.shape
    codes = np.zeros((rows, n // 2), np.uint8)
    scales = np.zeros((rows, n // 32), np.uint8)
    lib().orc_mxfp4_encode(x.ctypes.data, rows, n, codes.ctypes.data, scales.ctypes.data)
    return codes, scales


def mxfp4_decode(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    rows = codes.shape[0]
    n = codes.shape[1] * 2
    out = np.zeros((rows, n), np.float64)
    lib().orc_mxfp4_decode(codes.ctypes.data, scales.ctypes.data, rows, n, out.ctypes.data)
    return out


# ----------------------------------------------------------------------------
# indexer
# ----------------------------------------------------------------------------

class _Hold:
    """Keeps converted arrays alive until the C call returns."""

    def __init__(self):
        self.keep = []

    def __call__(self, a, dt):
        if a is None:
            return None
        a = np.ascontiguousarray(a, dtype=dt)
        self.keep.append(a)
        return a.ctypes.data


def index_scores(kcodes, kscales, rows, qc, qs, w) -> np.ndarray:
    """Scores of cache rows `rows` for one indexer query (qc [4,64], qs [4,4], w [4])."""
    h = _Hold()
    rows = np.ascontiguousarray(rows, np.int64)
    out = np.zeros(rows.shape[0], np.float32)
    lib().orc_index_scores(h(kcodes, np.uint8), h(kscales, np.uint8), h(rows, np.int64), rows.shape[0],
                           h(qc, np.uint8), h(qs, np.uint8), h(w, np.float32), h(out, np.float32))
    return out


def topk(keys, ids, k) -> np.ndarray:
    h = _Hold()
    keys = np.ascontiguousarray(keys, np.uint32)
    out = np.zeros(k, np.int32)
    lib().orc_topk(h(keys, np.uint32), h(ids, np.int64), keys.shape[0], k, h(out, np.int32))
    return out


def index_full(kcodes, kscales, qc, qs, w, seq_row_off, seq_len, P, k, want_scores=False, nthreads=0):
    """Full-mode indexer.  Returns (pool [B,P], topk [B,k], scores [B,max_len] or None)."""
    h = _Hold()
    seq_len = np.ascontiguousarray(seq_len, np.int32)
    B = seq_len.shape[0]
    max_len = max(int(seq_len.max()) if B else 0, 1)
    pool = np.full((B, P), -1, np.int32)
    top = np.full((B, k), -1, np.int32)
    sc = np.zeros((B, max_len), np.float32) if want_scores else None
    rc = lib().orc_index_full(h(kcodes, np.uint8), h(kscales, np.uint8), h(qc, np.uint8), h(qs, np.uint8),
                              h(w, np.float32), h(seq_row_off, np.int64), h(seq_len, np.int32), B, P, k,
                              h(pool, np.int32), h(top, np.int32), h(sc, np.float32), max_len, nthreads)
    assert rc == 0
    return pool, top, sc


def multi_query_rows(seq_row_off, q_off, q_vis):
    """Per query of a batch with several queries per sequence: its sequence's
    first cache row and its visible entry count (queries of no sequence: row
    0, nothing visible)."""
    q_vis = np.asarray(q_vis, np.int64)
    rows = np.zeros(q_vis.shape[0], np.int64)
    vis = np.zeros(q_vis.shape[0], np.int32)
    for b in range(len(q_off) - 1):
        for i in range(int(q_off[b]), int(q_off[b + 1])):
            rows[i] = seq_row_off[b]
            vis[i] = max(0, int(q_vis[i]))
    return rows, vis


def index_multi(kcodes, kscales, qc, qs, w, seq_row_off, q_off, q_vis, P, k, nthreads=0):
    """Full-mode indexer for several queries per sequence (speculative
    verification, "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache
    Compression", section "DSpark"): every query is its own Full-mode query
    over the first q_vis[i] entries of its sequence.  Returns (pool [Q,P],
    topk [Q,k])."""
    rows, vis = multi_query_rows(seq_row_off, q_off, q_vis)
    pool, top, _ = index_full(kcodes, kscales, qc, qs, w, rows, vis, P, k, nthreads=nthreads)
    return pool, top


def index_reindex(kcodes, kscales, qc, qs, w, seq_row_off, seq_len, pool, k, nthreads=0):
    h = _Hold()
    pool = np.ascontiguousarray(pool, np.int32)
    B, P = pool.shape
    top = np.full((B, k), -1, np.int32)
    rc = lib().orc_index_reindex(h(kcodes, np.uint8), h(kscales, np.uint8), h(qc, np.uint8), h(qs, np.uint8),
                                 h(w, np.float32), h(seq_row_off, np.int64), h(seq_len, np.int32),
                                 h(pool, np.int32), B, P, k, h(top, np.int32), nthreads)
    assert rc == 0
    return top


def attn_decode(q_bf16, mcodes, mscales, seq_row_off, seq_len, topk_idx, win, win_scale, win_len, sm_scale,
                nthreads=0):
    """Returns (out fp64 [B,16,512], lse fp64 [B,16])."""
    h = _Hold()
    topk_idx = np.ascontiguousarray(topk_idx, np.int32)
    B, k = topk_idx.shape
    out = np.zeros((B, 16, 512), np.float64)
    lse = np.zeros((B, 16), np.float64)
    rc = lib().orc_attn_decode(h(q_bf16, np.uint16), h(mcodes, np.uint8), h(mscales, np.uint8),
                               h(seq_row_off, np.int64), h(seq_len, np.int32), h(topk_idx, np.int32), k,
                               h(win, np.uint8), h(win_scale, np.float32), h(win_len, np.int32),
                               float(sm_scale), h(out, np.float64), h(lse, np.float64), B, nthreads)
    if rc != 0:
        raise ValueError("oracle: a selected index lies outside the visible context")
    return out, lse


def compress(raw_bf16, logits, ratio, w_idx=None, idx_raw_bf16=None, nthreads=0, want_rows=False):
    """Compress + MXFP4-encode.

    Returns (main codes, main scales, idx codes, idx scales) and, with
    want_rows, also the fp32 rows before quantisation (c [n,512], r [n,128]).
    """
    h = _Hold()
    raw_bf16 = np.ascontiguousarray(raw_bf16, np.uint16)
    n = raw_bf16.shape[0] // ratio
    mc = np.zeros((n, 256), np.uint8)
    ms = np.zeros((n, 16), np.uint8)
    ic = np.zeros((n, 64), np.uint8)
    isc = np.zeros((n, 4), np.uint8)
    c_rows = np.zeros((n, 512), np.float32) if want_rows else None
    r_rows = np.zeros((n, 128), np.float32) if want_rows else None
    rc = lib().orc_compress(h(raw_bf16, np.uint16), h(logits, np.float32), h(w_idx, np.float32),
                            h(idx_raw_bf16, np.uint16), n, ratio, h(mc, np.uint8), h(ms, np.uint8),
                            h(ic, np.uint8), h(isc, np.uint8), h(c_rows, np.float32), h(r_rows, np.float32),
                            nthreads)
    assert rc == 0
    if want_rows:
        return mc, ms, ic, isc, c_rows, r_rows
    return mc, ms, ic, isc


def compress_stream(pend, raw_bf16, logits, tok_off, w_idx=None, idx_raw_bf16=None, nthreads=0):
    """Ratio-2 append with a pending half-pair per sequence.

    Entries are the disjoint pairs (2j, 2j+1) of each sequence's raw token
    stream ("DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache
    Compression", architecture figure caption and section
    "三个方向一起压小缓存": no overlap between entries), however the stream is
    cut into calls.  Sequence b's stream for this call is its pending token
    (pend[b], or None) followed by raw tokens tok_off[b] .. tok_off[b+1]-1;
    its complete pairs are compressed with ``compress`` and an odd trailing
    token becomes the new pending one.

    pend[b]: None or dict(raw=[512] uint16, logit=float, idx=[128] uint16 or None).
    Returns (entries, new_pend): entries[b] = (mc, ms, ic, isc) of the new
    entries (possibly empty), new_pend[b] as pend[b].
    """
    raw_bf16 = np.ascontiguousarray(raw_bf16, np.uint16).reshape(-1, 512)
    logits = np.ascontiguousarray(logits, np.float32).reshape(-1)
    use_idx = w_idx is None
    if use_idx:
        idx_raw_bf16 = np.ascontiguousarray(idx_raw_bf16, np.uint16).reshape(-1, 128)
    entries, new_pend = [], []
    for b in range(len(tok_off) - 1):
        t0, t1 = int(tok_off[b]), int(tok_off[b + 1])
        rows, zs, idx = [raw_bf16[t0:t1]], [logits[t0:t1]], [idx_raw_bf16[t0:t1]] if use_idx else None
        if pend[b] is not None:
            rows.insert(0, np.asarray(pend[b]["raw"], np.uint16).reshape(1, 512))
            zs.insert(0, np.array([pend[b]["logit"]], np.float32))
            if use_idx:
                idx.insert(0, np.asarray(pend[b]["idx"], np.uint16).reshape(1, 128))
        x, z = np.concatenate(rows), np.concatenate(zs)
        xi = np.concatenate(idx) if use_idx else None
        n = x.shape[0]
        m = n // 2 * 2
        entries.append(compress(x[:m], z[:m], 2, w_idx=w_idx, idx_raw_bf16=xi[:m] if use_idx else None,
                                nthreads=nthreads))
        new_pend.append(None if n == m else dict(raw=x[m].copy(), logit=float(z[m]),
                                                 idx=xi[m].copy() if use_idx else None))
    return entries, new_pend


def index_prefill(kcodes, kscales, row0, n_entries, qc, qs, w, q_pos, ratio, P, k, q_ids=None, nthreads=0):
    """Causal prefill indexer; q_ids selects a subset of queries (rows of the outputs)."""
    h = _Hold()
    q_pos = np.ascontiguousarray(q_pos, np.int32)
    nq = q_pos.shape[0] if q_ids is None else len(q_ids)
    pool = np.full((nq, P), -1, np.int32)
    top = np.full((nq, k), -1, np.int32)
    rc = lib().orc_index_prefill(h(kcodes, np.uint8), h(kscales, np.uint8), int(row0), int(n_entries),
                                 h(qc, np.uint8), h(qs, np.uint8), h(w, np.float32), h(q_pos, np.int32),
                                 h(q_ids, np.int32), nq, ratio, P, k, h(pool, np.int32), h(top, np.int32),
                                 nthreads)
    assert rc == 0
    return pool, top


def attn_prefill(q_bf16, q_pos, mcodes, mscales, row0, n_entries, ratio, topk_idx, raw_win, win_scale,
                 sm_scale, q_ids=None, nthreads=0):
    h = _Hold()
    topk_idx = np.ascontiguousarray(topk_idx, np.int32)
    nq, k = topk_idx.shape
    out = np.zeros((nq, 16, 512), np.float64)
    lse = np.zeros((nq, 16), np.float64)
    rc = lib().orc_attn_prefill(h(q_bf16, np.uint16), h(q_pos, np.int32), h(q_ids, np.int32), nq,
                                h(mcodes, np.uint8), h(mscales, np.uint8), int(row0), int(n_entries), ratio,
                                h(topk_idx, np.int32), k, h(raw_win, np.uint8), float(win_scale),
                                float(sm_scale), h(out, np.float64), h(lse, np.float64), nthreads)
    if rc != 0:
        raise ValueError("oracle: a selected index lies outside the visible context")
    return out, lse


# ----------------------------------------------------------------------------
# a whole decode step through a layer pattern (F / R / U)
# ----------------------------------------------------------------------------

def decode_step(pattern, caches, seq_row_off, seq_len, layers, P, k, sm_scale, full_rescan=False, nthreads=0,
                attention=True):
    """Oracle decode step.  caches: per Full layer dict(idx_codes, idx_scales,
    main_codes, main_scales); layers: per layer dict(q, q_codes, q_scales, w,
    win, win_scale, win_len).  Modes per the pages: the first Full layer scans
    and builds the pool; a later Full layer selects inside that pool with its
    own caches (or rescans when full_rescan); Reindex selects inside the pool
    with the nearest Full layer's indexer K; Reuse repeats the latest Top-k.
    Returns dict(pools, topk, out, lse) with one entry per layer (pools: per
    Full layer that scanned)."""
    full_idx = -1
    scanned = False
    pool = None
    last = None
    res = dict(pools={}, topk=[], out=[], lse=[])
    for layer, mode in enumerate(pattern):
        L = layers[layer]
        if mode == "F":
            full_idx += 1
        c = caches[full_idx]
        if mode == "F" and (not scanned or full_rescan):
            pool, top, _ = index_full(c["idx_codes"], c["idx_scales"], L["q_codes"], L["q_scales"], L["w"],
                                      seq_row_off, seq_len, P, k, nthreads=nthreads)
            res["pools"][layer] = pool
            scanned = True
            last = top
        elif mode in ("F", "R"):
            last = index_reindex(c["idx_codes"], c["idx_scales"], L["q_codes"], L["q_scales"], L["w"], seq_row_off,
                                 seq_len, pool, k, nthreads=nthreads)
        elif mode != "U":
            raise ValueError(mode)
        res["topk"].append(last)
        if attention:
            o, l = attn_decode(L["q"], c["main_codes"], c["main_scales"], seq_row_off, seq_len, last, L["win"],
                               L["win_scale"], L["win_len"], sm_scale, nthreads=nthreads)
            res["out"].append(o)
            res["lse"].append(l)
    return res
