"""The C-ABI library loads, exports every function include/csa2.h declares,
and rejects bad arguments on the host before any launch (no GPU needed)."""
import ctypes as Cc
import os
import re

import pytest

from long_context_decode_csa2_b200 import _build
from long_context_decode_csa2_b200 import csa2 as C

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "csa2.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(csa2_\w+)\s*\(", text)))


def test_library_builds_and_exports_every_declared_symbol():
    path = _build.build()
    lib = Cc.CDLL(path)
    names = _declared()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings():
    L = C.lib()
    assert L.csa2_status_string(0) == b"ok"
    assert L.csa2_status_string(-3) == b"workspace too small"


FAKE = 0x10000  # an aligned non-null address; never dereferenced (rejected first)


def _cache(rows=1024, codes=FAKE, scales=FAKE):
    return C.MXFP4Cache(codes, scales, rows)


def test_index_full_validation():
    L = C.lib()
    ws = L.csa2_index_full_workspace_bytes(2, 1000, 64, 64)
    args = dict(q=FAKE, qs=FAKE, w=FAKE, off=FAKE, ln=FAKE, pool=FAKE, top=FAKE)

    def call(cache=None, B=2, max_len=1000, P=64, k=64, ws_bytes=ws, wsp=FAKE, q=FAKE):
        return L.csa2_index_full(cache or _cache(), q, FAKE, FAKE, FAKE, FAKE, B, max_len, P, k, FAKE, FAKE, None,
                                 wsp, ws_bytes, None)

    assert call(P=0) == -1 and call(k=4096) == -1 and call(B=-1) == -1
    assert call(cache=_cache(rows=1001)) == -1                 # capacity not a multiple of 8
    assert call(cache=_cache(codes=FAKE + 4)) == -1            # misaligned
    assert call(q=0) == -1                                     # null pointer
    assert call(wsp=FAKE + 64) == -1                           # workspace not 256-aligned
    assert call(ws_bytes=ws - 1) == -3
    assert call(B=0) == 0                                      # nothing to do
    assert b"workspace" in L.csa2_last_error()


def test_other_calls_validation():
    L = C.lib()
    assert L.csa2_index_reindex(_cache(), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 0, 64, FAKE, FAKE, 1 << 20, None) == -1
    assert L.csa2_sparse_attn_decode(FAKE, _cache(), FAKE, FAKE, FAKE, 0, FAKE, FAKE, FAKE, 0.1, FAKE, None, 2, FAKE,
                                     1 << 30, None) == -1
    assert L.csa2_sparse_attn_decode(FAKE, _cache(), FAKE, FAKE, FAKE, 512, FAKE, FAKE, FAKE, 0.1, FAKE, None, 2, FAKE,
                                     16, None) == -3
    # ratio 3, and ratio 2 without logits, and both / neither indexer sources
    base = [_cache(), _cache(), FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, FAKE, 1]
    assert L.csa2_compress_append(*base, 3, 10, 5, FAKE, 256, None) == -1
    b2 = list(base)
    b2[3] = None
    assert L.csa2_compress_append(*b2, 2, 10, 5, FAKE, 256, None) == -1
    b3 = list(base)
    b3[4] = FAKE
    assert L.csa2_compress_append(*b3, 2, 10, 5, FAKE, 256, None) == -1
    b4 = list(base)
    b4[4], b4[5] = FAKE + 4, None                              # W_idx not 8-byte aligned
    assert L.csa2_compress_append(*b4, 1, 10, 5, FAKE, 256, None) == -1
    assert b"w_idx" in L.csa2_last_error()
    ws = L.csa2_compress_append_workspace_bytes(1)
    b5 = list(base)
    b5[4], b5[5] = FAKE, None
    assert L.csa2_compress_append(*b5, 1, 10, 5, FAKE, ws - 1, None) == -3
    assert L.csa2_compress_append(*b5, 1, 10, 5, FAKE + 64, ws, None) == -1   # workspace alignment
    assert L.csa2_index_prefill(_cache(), FAKE, FAKE, FAKE, FAKE, 4, 0, 100, 2, 64, 512, FAKE, FAKE, FAKE, 1 << 30,
                                None) == -2                    # pool smaller than k
    assert L.csa2_index_prefill(_cache(rows=64), FAKE, FAKE, FAKE, FAKE, 4, 0, 100, 2, 64, 64, FAKE, FAKE, FAKE,
                                1 << 30, None) == -1           # entries beyond the capacity
    assert L.csa2_sparse_attn_prefill(FAKE, FAKE, 4, _cache(), 0, 100, 3, FAKE, 512, FAKE, 300, 0.1, 0.1, FAKE, None,
                                      FAKE, 1 << 30, None) == -1


def test_workspace_sizes_grow_with_the_problem():
    L = C.lib()
    a = L.csa2_index_full_workspace_bytes(4, 1 << 16, 2048, 512)
    b = L.csa2_index_full_workspace_bytes(8, 1 << 16, 2048, 512)
    assert 256 < a < b and a % 256 == 0
    assert L.csa2_index_full_workspace_bytes(1, 8192, 256, 512) > L.csa2_index_full_workspace_bytes(1, 8192, 512, 512)
    # attention at B = 64: four CTAs per sequence, one partial each (O [16 x 512] + max + sum per
    # head, fp32); a segment's only CTA (many segments) writes no partial
    assert L.csa2_sparse_attn_decode_workspace_bytes(64, 512) >= 64 * 4 * (16 * 512 + 32) * 4
    assert L.csa2_sparse_attn_decode_workspace_bytes(4096, 512) < 4096 * (16 * 512 + 32) * 4
    assert L.csa2_sparse_attn_decode_workspace_bytes(128, 512) > L.csa2_sparse_attn_decode_workspace_bytes(16, 512)


def test_compress_stream_validation():
    """csa2_compress_stream: arguments checked on the host, nothing launched."""
    L = C.lib()
    ws = L.csa2_compress_stream_workspace_bytes(4)
    assert ws >= 256 + 4 * 4 and ws % 256 == 0
    assert L.csa2_compress_stream_workspace_bytes(1000) > ws

    def call(raw=FAKE, logits=FAKE, w_idx=FAKE, idx_raw=None, pend_n=FAKE, pend_raw=FAKE, pend_idx=None, B=4,
             n_tok=4, ws_bytes=1 << 20):
        return L.csa2_compress_stream(_cache(), _cache(), raw, logits, w_idx, idx_raw, FAKE, FAKE, FAKE, FAKE, pend_n,
                                      pend_raw, FAKE, pend_idx, B, n_tok, 1, FAKE, ws_bytes, None)

    assert call(B=0) == 0                                   # nothing to do
    assert call(logits=None) == -1                          # logits are required
    assert call(pend_n=None) == -1                          # pending state is required
    assert call(w_idx=None) == -1                           # no indexer source
    assert call(w_idx=None, idx_raw=FAKE) == -1             # idx_raw without a pending idx buffer
    assert call(idx_raw=FAKE, pend_idx=FAKE) == -1          # both sources
    assert call(pend_raw=FAKE + 8) == -1                    # misaligned pending row
    assert call(w_idx=FAKE + 4) == -1                       # W_idx read as float2: 8-byte alignment
    assert call(raw=None) == -1                             # tokens but no raw rows
    assert call(ws_bytes=256) == -3                         # no room for the counters


def test_widened_calls_validation():
    """The verification, paged, context-parallel and split calls check their
    arguments on the host and launch nothing when they fail."""
    L = C.lib()
    c = _cache()
    # csa2_index_multi: pool smaller than k, queries without sequences, max_vis past the cache
    args = [c, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE]
    assert L.csa2_index_multi(*args, 2, 6, 100, 64, 512, FAKE, FAKE, None, FAKE, 1 << 30, None) == -2
    assert L.csa2_index_multi(*args, 0, 6, 100, 512, 512, FAKE, FAKE, None, FAKE, 1 << 30, None) == -1
    assert L.csa2_index_multi(*args, 2, 6, 4096, 512, 512, FAKE, FAKE, None, FAKE, 1 << 30, None) == -1
    assert L.csa2_index_multi(*args, 2, 6, 100, 512, 512, FAKE, FAKE, None, FAKE, 16, None) == -3
    assert L.csa2_index_multi(*args, 2, 0, 100, 512, 512, FAKE, FAKE, None, FAKE, 16, None) == 0
    # paged calls: page size not a power of two / below 512, cache not a whole number of pages
    assert L.csa2_index_full_paged(_cache(rows=2048), FAKE, FAKE, FAKE, FAKE, 768, 4, FAKE, 2, 1000, 64, 64, FAKE,
                                   FAKE, None, FAKE, 1 << 30, None) == -1
    assert L.csa2_index_full_paged(_cache(rows=2048), FAKE, FAKE, FAKE, FAKE, 256, 4, FAKE, 2, 1000, 64, 64, FAKE,
                                   FAKE, None, FAKE, 1 << 30, None) == -1
    assert L.csa2_index_full_paged(_cache(rows=1000), FAKE, FAKE, FAKE, FAKE, 512, 4, FAKE, 2, 1000, 64, 64, FAKE,
                                   FAKE, None, FAKE, 1 << 30, None) == -1
    assert L.csa2_sparse_attn_decode_paged(FAKE, _cache(rows=1024), None, 512, 4, FAKE, FAKE, 512, FAKE, FAKE, FAKE,
                                           0.1, FAKE, None, 2, FAKE, 1 << 30, None) == -1
    assert L.csa2_index_reindex_paged(_cache(rows=1024), FAKE, FAKE, FAKE, FAKE, 512, 0, FAKE, FAKE, 2, 64, 64, FAKE,
                                      FAKE, 1 << 30, None) == -1
    # context parallelism: block must be 1 or 8; merge k out of range; too small a workspace; combine needs G >= 1
    assert L.csa2_score_positions(c, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 10, 4, FAKE, FAKE, 256, None) == -1
    assert L.csa2_topk_merge(FAKE, FAKE, None, 2, 3, 100, 0, None, None, FAKE, None, FAKE, 1 << 20, None) == -1
    assert L.csa2_topk_merge(FAKE, FAKE, None, 2, 3, 100, 64, None, None, FAKE, None, FAKE, 256, None) == -3
    assert L.csa2_topk_merge(FAKE, FAKE, None, 2, 3, 100, 64, None, None, FAKE, FAKE, FAKE, 1 << 20, None) == -1
    assert L.csa2_attn_combine(FAKE, FAKE, 0, 2, FAKE, None, None) == -1
    assert L.csa2_topk_merge_workspace_bytes(3, 4, 100) > L.csa2_topk_merge_workspace_bytes(2, 4, 100)
    # split Full layer: the same checks as csa2_index_full
    assert L.csa2_index_full_pool(c, FAKE, FAKE, FAKE, None, FAKE, 2, 1000, 0, 64, FAKE, None, FAKE, 1 << 30,
                                  None) == -1
    assert L.csa2_index_full_topk(c, FAKE, FAKE, FAKE, None, FAKE, 2, 1000, 64, 64, FAKE, FAKE, None, FAKE, 1 << 30,
                                  None) == -1


def test_every_entry_point_cites_its_source():
    """Each operation declared in include/csa2.h sits under a comment block
    that names the passage defining it (or says the pages have none)."""
    src = open(HEADER).read()
    decls = [(m.start(), m.group(1)) for m in re.finditer(r"^csa2_status (csa2_\w+)\(", src, re.M)]
    assert len(decls) >= 15
    helpers = {"csa2_device_status"}  # reads the status word back; no operation of the method
    for pos, name in decls:
        if name in helpers:
            continue
        block = src[src.rfind("/*", 0, pos):pos]
        assert "Source:" in block or "no counterpart" in block, name
