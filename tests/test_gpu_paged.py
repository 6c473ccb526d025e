"""Paged caches (block tables): the *_paged calls read and write the same
rows through a page table and give the same bits as the contiguous layout
(Top-k and appended cache bytes bit-exact, attention outputs identical), and
the oracle agrees."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
import synth.workloads as W
from long_context_decode_csa2_b200 import csa2 as C
from long_context_decode_csa2_b200.decode import DecodeStep, FullCache
from tests._gpu import check_attention, dev, host

pytestmark = pytest.mark.gpu

PLANES = (("idx_codes", 64), ("idx_scales", 4), ("main_codes", 256), ("main_scales", 16))


def _page_table(caps, page_rows, n_spare, seed):
    """A random assignment of physical pages to every sequence's logical
    pages (spare pages stay unused)."""
    need = [(c + page_rows - 1) // page_rows for c in caps]
    n_pages = sum(need) + n_spare
    perm = np.random.default_rng(seed).permutation(n_pages).astype(np.int32)
    max_pages = max(need)
    table = np.full((len(caps), max_pages), 0, np.int32)
    o = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[o:o + n]
        o += n
    return table, n_pages


def _to_pages(cache_h, off, caps, table, page_rows, n_pages, seed):
    """Copies each sequence's contiguous rows into its pages; unused rows get
    random bytes (a wrong page read would show)."""
    rng = np.random.default_rng(seed)
    out = {}
    for key, width in PLANES:
        phys = rng.integers(0, 256, (n_pages * page_rows, width), dtype=np.uint8)
        if key.endswith("scales"):
            phys[:] = rng.integers(120, 135, phys.shape, dtype=np.uint8)
        for b, cap in enumerate(caps):
            for lp in range((cap + page_rows - 1) // page_rows):
                n = min(page_rows, cap - lp * page_rows)
                src = cache_h[key][off[b] + lp * page_rows: off[b] + lp * page_rows + n]
                dst = int(table[b, lp]) * page_rows
                phys[dst:dst + n] = src
        out[key] = phys
    return out


def _device_caches(c):
    return FullCache(C.cache(dev(c["idx_codes"]), dev(c["idx_scales"])),
                     C.cache(dev(c["main_codes"]), dev(c["main_scales"])))


def _layers_dev(layers):
    keys = ("q", "q_codes", "q_scales", "w", "win", "win_scale", "win_len")
    return [{k: dev(L[k]) for k in keys} for L in layers]


@pytest.mark.parametrize("page_rows", [512, 2048])
def test_paged_decode_step_equals_contiguous(page_rows):
    wl = W.DecodeWorkload("paged_small", np.array([9001, 4096, 20000, 700]), "FRUFR", needles=16, lognormal=True)
    layers = [W.layer_inputs_host(wl, l) for l in range(len(wl.pattern))]
    caches_h = [W.full_cache_host(wl, f, layers[f]["q_codes"], layers[f]["q_scales"]) for f in wl.full_layers()]
    off = caches_h[0]["seq_row_off"]
    caps = [int(x) for x in (wl.lengths + 7) // 8 * 8]
    table, n_pages = _page_table(caps, page_rows, 3, seed=page_rows)
    paged_h = [_to_pages(c, off, caps, table, page_rows, n_pages, seed=11 + i) for i, c in enumerate(caches_h)]
    lens = dev(wl.lengths.astype(np.int32))
    dl = _layers_dev(layers)

    plain = DecodeStep(wl.pattern, wl.B, wl.max_len, wl.P, wl.k)
    plain.run([_device_caches(c) for c in caches_h], dev(off), lens, dl)
    paged = DecodeStep(wl.pattern, wl.B, wl.max_len, wl.P, wl.k)
    paged.run([_device_caches(c) for c in paged_h], C.PageTable(dev(table), page_rows), lens, dl)
    torch.cuda.synchronize()
    assert plain.device_flags() == 0 and paged.device_flags() == 0
    for layer in range(len(wl.pattern)):
        assert np.array_equal(host(paged.topk[layer]), host(plain.topk[layer])), f"layer {layer} Top-k"
    assert np.array_equal(host(paged.out), host(plain.out)) and np.array_equal(host(paged.lse), host(plain.lse))
    assert np.array_equal(host(paged.pool), host(plain.pool))
    ref = oracle.decode_step(wl.pattern, caches_h, off, wl.lengths.astype(np.int32), layers, wl.P, wl.k,
                             1 / math.sqrt(512))
    for layer in range(len(wl.pattern)):
        assert np.array_equal(host(paged.topk[layer]), ref["topk"][layer])
        check_attention(host(paged.out[layer]), ref["out"][layer], what=f"layer {layer}")


def test_paged_stream_append_writes_the_pages():
    """Ratio-2 appends through a page table land in the sequences' pages,
    crossing page boundaries, bit-exact with the oracle."""
    B, page_rows = 3, 512
    start = np.array([500, 0, 1020], np.int32)      # entries already held; appends cross page ends
    caps = [2048, 1024, 2048]
    table, n_pages = _page_table(caps, page_rows, 2, seed=5)
    rows = n_pages * page_rows
    mc = torch.zeros((rows, 256), dtype=torch.uint8, device="cuda")
    ms = torch.zeros((rows, 16), dtype=torch.uint8, device="cuda")
    ic = torch.zeros((rows, 64), dtype=torch.uint8, device="cuda")
    isc = torch.zeros((rows, 4), dtype=torch.uint8, device="cuda")
    seq_len = dev(start)
    pend_n = torch.zeros(B, dtype=torch.int32, device="cuda")
    pend_raw = torch.zeros((B, 512), dtype=torch.bfloat16, device="cuda")
    pend_logit = torch.zeros(B, dtype=torch.float32, device="cuda")
    w_idx = synth.normal_f32(60, synth.T_WIDX, 0, 0, 512 * 128, log2_div=13).reshape(512, 128)
    ws = C.workspace(C.csa2_compress_stream_workspace_bytes(B))
    pt = C.PageTable(dev(table), page_rows)
    pend = [None] * B
    lens = start.astype(np.int64).copy()
    expect = {}  # (b, logical entry) -> (mc, ms, ic, isc)
    for call, ntok in enumerate([np.array([27, 3, 9]), np.array([0, 40, 2]), np.array([1, 1, 33])]):
        tok_off = np.concatenate([[0], np.cumsum(ntok)]).astype(np.int64)
        n = int(tok_off[-1])
        raw = synth.normal_bf16(61 + call, synth.T_RAW, 0, 0, n * 512).reshape(n, 512)
        z = synth.normal_f32(61 + call, synth.T_LOGITS, 0, 0, n)
        max_new = int(((ntok + host(pend_n)) // 2).max())
        C.csa2_compress_stream(C.cache(mc, ms), C.cache(ic, isc), dev(raw), dev(z), dev(tok_off), pt, seq_len, seq_len,
                               pend_n, pend_raw, pend_logit, max_new, ws, w_idx=dev(w_idx))
        ent, pend = oracle.compress_stream(pend, raw, z, tok_off, w_idx=w_idx)
        for b in range(B):
            for j in range(ent[b][0].shape[0]):
                expect[(b, int(lens[b]) + j)] = tuple(e[j] for e in ent[b])
            lens[b] += ent[b][0].shape[0]
    torch.cuda.synchronize()
    assert C.device_status(ws) == 0
    assert host(seq_len).tolist() == lens.tolist()
    planes = [host(t) for t in (mc, ms, ic, isc)]
    for (b, e), want in expect.items():
        r = int(table[b, e // page_rows]) * page_rows + e % page_rows
        for g, w_ in zip(planes, want):
            assert np.array_equal(g[r], w_), (b, e)


def test_paged_bad_page_id_is_flagged():
    """A page id outside the cache sets the row-layout flag; the call reads
    page 0 instead and finishes."""
    wl = W.DecodeWorkload("paged_bad", np.array([4096, 2048]), "F", P=256)
    L0 = W.layer_inputs_host(wl, 0)
    c = W.full_cache_host(wl, 0, L0["q_codes"], L0["q_scales"])
    table = np.array([[0, 1, 2, 3, 4, 5, 6, 7], [8, 9, 99, 11, 0, 0, 0, 0]], np.int32)  # page 99 does not exist
    step = DecodeStep(wl.pattern, wl.B, wl.max_len, wl.P, wl.k)
    step.run([_device_caches(c)], C.PageTable(dev(table), 512), dev(wl.lengths.astype(np.int32)), _layers_dev([L0]))
    torch.cuda.synchronize()
    assert step.device_flags() & 2  # CSA2_DEV_ROW_LAYOUT


def test_paged_ratio2_decode_steps_equal_contiguous():
    """Ratio-2 decode through a page table: appends land in the pages and
    every step's results equal the contiguous layout's."""
    lens0 = np.array([4000, 1030, 2048], np.int64)
    room, steps, page_rows = 24, 5, 512
    wl = W.DecodeWorkload("paged_r2", lens0, "FRRU", needles=8, ratio=2, room=room)
    layers = [W.layer_inputs_host(wl, l) for l in range(len(wl.pattern))]
    c = W.full_cache_host(wl, 0, layers[0]["q_codes"], layers[0]["q_scales"])
    off = c["seq_row_off"]
    caps = [int(x) for x in (lens0 + room + 7) // 8 * 8]
    table, n_pages = _page_table(caps, page_rows, 2, seed=9)
    paged_c = _to_pages(c, off, caps, table, page_rows, n_pages, seed=10)
    dl = _layers_dev(layers)
    plain = DecodeStep(wl.pattern, wl.B, wl.max_len + room, wl.P, wl.k, ratio=2, projection=False)
    paged = DecodeStep(wl.pattern, wl.B, wl.max_len + room, wl.P, wl.k, ratio=2, projection=False)
    cp, cg = _device_caches(c), _device_caches(paged_c)
    len_p, len_g = dev(lens0.astype(np.int32)), dev(lens0.astype(np.int32))
    pt = C.PageTable(dev(table), page_rows)
    import synth
    for t in range(steps):
        tok = dict(raw=dev(synth.normal_bf16(90, synth.T_RAW, t, 0, wl.B * 512).reshape(wl.B, 512)),
                   logit=dev(synth.normal_f32(90, synth.T_LOGITS, t, 0, wl.B)),
                   idx_raw=dev(synth.normal_bf16(90, synth.T_IDXRAW, t, 0, wl.B * 128).reshape(wl.B, 128)))
        plain.run([cp], dev(off), len_p, dl, new_tokens=[tok])
        paged.run([cg], pt, len_g, dl, new_tokens=[tok])
        torch.cuda.synchronize()
        for layer in range(len(wl.pattern)):
            assert np.array_equal(host(paged.topk[layer]), host(plain.topk[layer])), (t, layer)
        assert np.array_equal(host(paged.out), host(plain.out)), t
    assert plain.device_flags() == 0 and paged.device_flags() == 0
    assert host(len_g).tolist() == host(len_p).tolist() == (lens0 + steps // 2).tolist()
