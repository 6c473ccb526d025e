"""Prefill workload (ratio-2 compression, then a causal chunk): compressed
cache bytes, per-query pools and Top-k bit-exact; attention within tolerance."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth.workloads as W
from long_context_decode_csa2_b200 import csa2 as C
from tests._gpu import check_attention, dev, host

pytestmark = pytest.mark.gpu


def _gpu_prefill(inp, n_raw, T, ratio, P, k, use_proj):
    n_ent = n_raw // ratio
    rows = (n_ent + 7) // 8 * 8
    mc = torch.zeros((rows, 256), dtype=torch.uint8, device="cuda")
    ms = torch.zeros((rows, 16), dtype=torch.uint8, device="cuda")
    ic = torch.zeros((rows, 64), dtype=torch.uint8, device="cuda")
    isc = torch.zeros((rows, 4), dtype=torch.uint8, device="cuda")
    main, idx = C.cache(mc, ms), C.cache(ic, isc)
    d = {k_: dev(v) for k_, v in inp.items() if isinstance(v, np.ndarray)}
    ws = C.workspace(C.csa2_compress_append_workspace_bytes(1))
    out_len = torch.zeros(1, dtype=torch.int32, device="cuda")
    C.csa2_compress_append(main, idx, d["raw"], d["logits"], dev(np.array([0, n_raw], np.int64)),
                           dev(np.array([0], np.int64)), dev(np.array([0], np.int32)), out_len, ratio, n_ent, ws,
                           w_idx=d["w_idx"] if use_proj else None, idx_raw=None if use_proj else d["idx_raw"])
    pool = torch.full((T, P), -7, dtype=torch.int32, device="cuda")
    top = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    ws2 = C.workspace(C.csa2_index_prefill_workspace_bytes(T, n_ent, P, k))
    C.csa2_index_prefill(idx, d["q_codes"], d["q_scales"], d["w"], d["q_pos"], 0, n_ent, ratio, P, k, pool, top, ws2)
    out = torch.zeros((T, 16, 512), dtype=torch.float32, device="cuda")
    lse = torch.zeros((T, 16), dtype=torch.float32, device="cuda")
    ws3 = C.workspace(C.csa2_sparse_attn_prefill_workspace_bytes(T, k))
    C.csa2_sparse_attn_prefill(d["q"], d["q_pos"], main, 0, n_ent, ratio, top, d["raw_win"], float(inp["win_scale"]),
                               1 / math.sqrt(512), out, ws3, lse=lse)
    torch.cuda.synchronize()
    assert C.device_status(ws) == 0 and C.device_status(ws2) == 0 and C.device_status(ws3) == 0
    return dict(mc=host(mc), ms=host(ms), ic=host(ic), isc=host(isc), pool=host(pool), top=host(top), out=host(out),
                lse=host(lse), n_ent=n_ent)


@pytest.mark.parametrize("P,k,use_proj,T", [(2048, 512, True, 48), (64, 64, False, 45), (2048, 2048, True, 20)])
def test_prefill_reduced(P, k, use_proj, T):
    """T = 45 leaves a partial group of queries on the tensor-core scan; the
    first 16 queries see only a few entries each (causal masking)."""
    pw = W.prefill_workload()
    n_raw = 16384
    inp = W.prefill_inputs_host(pw, n_raw=n_raw, T=T)
    inp["q_pos"] = np.concatenate([np.arange(0, 16, dtype=np.int32) * 37, inp["q_pos"][16:]])
    g = _gpu_prefill(inp, n_raw, T, 2, P, k, use_proj)
    mc, ms, ic, isc = oracle.compress(inp["raw"], inp["logits"], 2, w_idx=inp["w_idx"] if use_proj else None,
                                      idx_raw_bf16=None if use_proj else inp["idx_raw"])
    n = g["n_ent"]
    for a, b in ((g["mc"], mc), (g["ms"], ms), (g["ic"], ic), (g["isc"], isc)):
        assert np.array_equal(a[:n], b)
    pool, top = oracle.index_prefill(ic, isc, 0, n, inp["q_codes"], inp["q_scales"], inp["w"], inp["q_pos"], 2, P, k)
    assert np.array_equal(g["pool"], pool) and np.array_equal(g["top"], top)
    ro, rl = oracle.attn_prefill(inp["q"], inp["q_pos"], mc, ms, 0, n, 2, top, inp["raw_win"], inp["win_scale"],
                                 1 / math.sqrt(512))
    check_attention(g["out"], ro, g["lse"], rl)


def test_prefill_full_size_512_queries():
    """The full prefill workload (262144 raw tokens, 4096 queries): every
    compressed and quantised byte, and a seeded subset of 512 query rows (the
    first 8, the last 8 and 496 drawn at random) for pools, Top-k and
    attention."""
    pw = W.prefill_workload()
    inp = W.prefill_inputs_host(pw)
    g = _gpu_prefill(inp, pw.n_raw, pw.T, pw.ratio, pw.P, pw.k, pw.use_projection)
    mc, ms, ic, isc = oracle.compress(inp["raw"], inp["logits"], 2, w_idx=inp["w_idx"])
    n = g["n_ent"]
    for a, b in ((g["mc"], mc), (g["ms"], ms), (g["ic"], ic), (g["isc"], isc)):
        assert np.array_equal(a[:n], b)
    rng = np.random.default_rng(4096)
    middle = rng.choice(np.arange(8, pw.T - 8), 496, replace=False)
    ids = np.sort(np.concatenate([np.arange(8), middle, np.arange(pw.T - 8, pw.T)])).astype(np.int32)
    assert len(np.unique(ids)) == 512
    pool, top = oracle.index_prefill(ic, isc, 0, n, inp["q_codes"], inp["q_scales"], inp["w"], inp["q_pos"], 2, pw.P,
                                     pw.k, q_ids=ids)
    assert np.array_equal(g["pool"][ids], pool) and np.array_equal(g["top"][ids], top)
    ro, rl = oracle.attn_prefill(inp["q"], inp["q_pos"], mc, ms, 0, n, 2, top, inp["raw_win"], inp["win_scale"],
                                 1 / math.sqrt(512), q_ids=ids)
    check_attention(g["out"][ids], ro, g["lse"][ids], rl)


@pytest.mark.parametrize("distinct", [1, 3])
def test_prefill_index_heavy_ties(distinct):
    """Indexer rows drawn from `distinct` different rows, so block keys and
    candidate keys tie massively (with one row, every present key of a query
    is the same): the selections' shared-prefix and equal-key rules decide
    almost everything.  Pools and Top-k bit-exact."""
    pw = W.prefill_workload()
    T, n_raw, ratio, P, k = 24, 8192, 2, 64, 64
    inp = W.prefill_inputs_host(pw, n_raw=n_raw, T=T)
    n = n_raw // ratio
    rows = (n + 7) // 8 * 8
    rng = np.random.default_rng(100 + distinct)
    pick = rng.integers(0, distinct, rows)
    ic = rng.integers(0, 256, (distinct, 64), dtype=np.uint8)[pick]
    isc = rng.integers(124, 129, (distinct, 4)).astype(np.uint8)[pick]
    pool = torch.full((T, P), -7, dtype=torch.int32, device="cuda")
    top = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    ws = C.workspace(C.csa2_index_prefill_workspace_bytes(T, n, P, k))
    C.csa2_index_prefill(C.cache(dev(ic), dev(isc)), dev(inp["q_codes"]), dev(inp["q_scales"]), dev(inp["w"]),
                         dev(inp["q_pos"]), 0, n, ratio, P, k, pool, top, ws)
    torch.cuda.synchronize()
    assert C.device_status(ws) == 0
    want_pool, want_top = oracle.index_prefill(ic, isc, 0, n, inp["q_codes"], inp["q_scales"], inp["w"],
                                               inp["q_pos"], ratio, P, k)
    assert np.array_equal(host(pool), want_pool) and np.array_equal(host(top), want_top)
