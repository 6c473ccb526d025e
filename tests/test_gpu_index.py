"""GPU parity of the indexer calls against the oracle: bit-exact pools and
Top-k (and scores), on seeded inputs spanning several tiles, ragged tails and
edge cases.  Calls go through the C ABI (ctypes binding)."""
import numpy as np
import pytest
import torch

import oracle
import synth
import synth.workloads as W
from long_context_decode_csa2_b200 import csa2 as C
from tests._gpu import dev, host

pytestmark = pytest.mark.gpu


def _random_cache(rng, lengths, smin=124, smax=128, ties=False):
    pad = (np.asarray(lengths) + 7) // 8 * 8
    off = np.concatenate([[0], np.cumsum(pad)[:-1]]).astype(np.int64)
    rows = int(pad.sum()) + 8
    kc = rng.integers(0, 256, (rows, 64), dtype=np.uint8)
    ks = rng.integers(smin, smax + 1, (rows, 4), dtype=np.uint8)
    if ties:
        kc[::3] = kc[0]
        ks[::3] = ks[0]
    return kc, ks, off, rows


def _queries(rng, B, smin=124, smax=128):
    qc = rng.integers(0, 256, (B, 4, 64), dtype=np.uint8)
    qs = rng.integers(smin, smax + 1, (B, 4, 4), dtype=np.uint8)
    w = (0.5 + rng.random((B, 4))).astype(np.float32)
    return qc, qs, w


def _run_full(kc, ks, off, lengths, qc, qs, w, P, k, want_scores=False):
    B = len(lengths)
    max_len = max(int(np.max(lengths)) if B else 0, 1)
    cache = C.cache(dev(kc), dev(ks))
    keep = [cache]
    pool = torch.full((B, P), -7, dtype=torch.int32, device="cuda")
    top = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
    sc = torch.zeros((B, max_len), dtype=torch.float32, device="cuda") if want_scores else None
    ws = C.workspace(C.csa2_index_full_workspace_bytes(B, max_len, P, k))
    args = [dev(qc), dev(qs), dev(w), dev(off), dev(np.asarray(lengths, np.int32))]
    keep += args
    C.csa2_index_full(cache, *args, max_len, P, k, pool, top, ws, scores_out=sc)
    torch.cuda.synchronize()
    assert C.device_status(ws) == 0
    return host(pool), host(top), (host(sc) if want_scores else None)


@pytest.mark.parametrize("lengths,P,k", [
    ([8192], 256, 512),                     # P < k: Top-k over stored scores
    ([5000, 777, 3, 0, 4096, 12345], 64, 64),
    ([20000, 1, 9, 600], 2048, 512),        # nb <= P for short sequences
    ([100000, 65536], 2048, 512),
    # more than 16384 blocks: the pool is collected by several CTAs per sequence first
    ([300001, 150000, 70, 140000], 2048, 512),
    ([40000, 20001, 16384], 2048, 2048),    # the largest pool and Top-k the calls accept
    ([9000, 8, 1], 1, 1),                   # the smallest
])
def test_index_full_matches_oracle(lengths, P, k):
    rng = np.random.default_rng(sum(lengths) + P)
    kc, ks, off, _ = _random_cache(rng, lengths, ties=True)
    qc, qs, w = _queries(rng, len(lengths))
    gp, gt, gs = _run_full(kc, ks, off, lengths, qc, qs, w, P, k, want_scores=True)
    op, ot, osc = oracle.index_full(kc, ks, qc, qs, w, off, np.asarray(lengths), P, k, want_scores=True)
    assert np.array_equal(gt, ot)
    assert np.array_equal(gp, op)
    for b, L in enumerate(lengths):
        assert np.array_equal(gs[b, :L].view(np.uint32), osc[b, :L].view(np.uint32))


def test_index_full_tiny_config_with_needles():
    wl = W.decode_workloads()["tiny_decode_b1_l8192"]
    L0 = W.layer_inputs_host(wl, 0)
    c = W.full_cache_host(wl, 0, L0["q_codes"], L0["q_scales"])
    gp, gt, _ = _run_full(c["idx_codes"], c["idx_scales"], c["seq_row_off"], wl.lengths, L0["q_codes"],
                          L0["q_scales"], L0["w"], wl.P, wl.k)
    op, ot, _ = oracle.index_full(c["idx_codes"], c["idx_scales"], L0["q_codes"], L0["q_scales"], L0["w"],
                                  c["seq_row_off"], wl.lengths, wl.P, wl.k)
    assert np.array_equal(gt, ot) and np.array_equal(gp, op)
    pos = synth.needle_positions(wl.seed, 0, 0, 8192, wl.needles)
    assert set(pos.tolist()) <= set(gt[0].tolist())


def test_index_extreme_scales_and_all_ties():
    rng = np.random.default_rng(5)
    lengths = [3000, 2048]
    kc, ks, off, _ = _random_cache(rng, lengths, smin=90, smax=160)
    qc, qs, w = _queries(rng, 2, smin=100, smax=150)
    gp, gt, gs = _run_full(kc, ks, off, lengths, qc, qs, w, 128, 100, want_scores=True)
    op, ot, osc = oracle.index_full(kc, ks, qc, qs, w, off, np.asarray(lengths), 128, 100, want_scores=True)
    assert np.array_equal(gt, ot) and np.array_equal(gp, op)
    assert np.array_equal(gs[0, :3000].view(np.uint32), osc[0, :3000].view(np.uint32))
    # every key identical -> lowest positions win
    kc[:] = kc[0]
    ks[:] = ks[0]
    gp, gt, _ = _run_full(kc, ks, off, lengths, qc, qs, w, 16, 64)
    assert gt[0].tolist() == list(range(64)) and gp[0].tolist() == list(range(16))


@pytest.mark.parametrize("lengths,P,k", [([9000, 70000, 5], 2048, 512), ([4096, 333], 64, 100),
                                         ([70000, 20000], 2048, 2048), ([5000], 1, 1)])
def test_index_reindex_matches_oracle(lengths, P, k):
    rng = np.random.default_rng(len(lengths) * 7 + k)
    kc, ks, off, _ = _random_cache(rng, lengths)
    qc, qs, w = _queries(rng, len(lengths))
    pool, _, _ = oracle.index_full(kc, ks, qc, qs, w, off, np.asarray(lengths), P, k)
    qc2, qs2, w2 = _queries(rng, len(lengths))
    want = oracle.index_reindex(kc, ks, qc2, qs2, w2, off, np.asarray(lengths), pool, k)
    B = len(lengths)
    cache = C.cache(dev(kc), dev(ks))
    top = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
    ws = C.workspace(C.csa2_index_reindex_workspace_bytes(B, P, k))
    keep = [dev(qc2), dev(qs2), dev(w2), dev(off), dev(np.asarray(lengths, np.int32)), dev(pool)]
    C.csa2_index_reindex(cache, *keep[:5], keep[5], k, top, ws)
    torch.cuda.synchronize()
    assert C.device_status(ws) == 0
    assert np.array_equal(host(top), want)


def test_reindex_flags_out_of_range_pool_block():
    rng = np.random.default_rng(9)
    kc, ks, off, _ = _random_cache(rng, [1000])
    qc, qs, w = _queries(rng, 1)
    pool = np.full((1, 8), -1, np.int32)
    pool[0, :3] = [1, 5, 200]           # block 200 starts at position 1600 >= 1000
    cache = C.cache(dev(kc), dev(ks))
    top = torch.zeros((1, 16), dtype=torch.int32, device="cuda")
    ws = C.workspace(C.csa2_index_reindex_workspace_bytes(1, 8, 16))
    keep = [dev(qc), dev(qs), dev(w), dev(off), dev(np.array([1000], np.int32)), dev(pool)]
    C.csa2_index_reindex(cache, *keep[:5], keep[5], 16, top, ws)
    assert C.device_status(ws) == 1       # CSA2_DEV_INDEX_RANGE
    got = host(top)[0]
    assert set(got[got >= 0].tolist()) == set(range(8, 16)) | set(range(40, 48))


@pytest.mark.parametrize("qmin,qmax", [(100, 150), (2, 200), (2, 253), (180, 253)])
def test_index_multi_extreme_scales(qmin, qmax):
    """The multi-query scan with wide key and query exponent spreads (its
    fp64 epilogue path) and query scale bytes over the whole E8M0 range stays
    bit-exact.  Near the top of the range head dots overflow to +-inf and
    head sums of +inf and -inf give NaN; every NaN ranks below every number
    on both sides."""
    rng = np.random.default_rng(qmin + qmax)
    lengths = [3000, 2048, 777]
    kc, ks, off, _ = _random_cache(rng, lengths, smin=90, smax=160)
    m = np.array([3, 9, 2])
    q_off = np.concatenate([[0], np.cumsum(m)]).astype(np.int32)
    Q = int(q_off[-1])
    qc, qs, w = _queries(rng, Q, smin=qmin, smax=qmax)
    q_vis = np.concatenate([lengths[b] - np.arange(m[b])[::-1] * 5 for b in range(3)]).astype(np.int32)
    P, k = 128, 100
    pool = torch.full((Q, P), -7, dtype=torch.int32, device="cuda")
    top = torch.full((Q, k), -7, dtype=torch.int32, device="cuda")
    ws = C.workspace(C.csa2_index_multi_workspace_bytes(3, Q, max(lengths), P, k))
    C.csa2_index_multi(C.cache(dev(kc), dev(ks)), dev(qc), dev(qs), dev(w), dev(off), dev(q_off), dev(q_vis),
                       max(lengths), P, k, pool, top, ws)
    torch.cuda.synchronize()
    assert C.device_status(ws) == 0
    wp, wt = oracle.index_multi(kc, ks, qc, qs, w, off, q_off, q_vis, P, k)
    assert np.array_equal(host(pool), wp) and np.array_equal(host(top), wt)


def test_index_infinite_and_nan_scores():
    """Scores that overflow fp32 to +-inf, and head sums of +inf and -inf
    (NaN), on both Full-layer paths (stored scores when P < k, the pool
    re-score when P >= k), Reindex and the multi-query scan: pools and Top-k
    bit-exact with the oracle (every NaN ranks below every number, NaNs by
    position); stored scores equal bit for bit, NaN where the oracle's is."""
    from tests.test_oracle_index import _overflow_case

    kc0, ks0, qc0, qs0, w0, kinds = _overflow_case(1000)
    rng = np.random.default_rng(92)
    kc1, ks1, _, _ = _random_cache(rng, [3001])
    kc = np.concatenate([kc0, kc1])      # sequence 0: rows 0..999, sequence 1: rows 1000..4000
    ks = np.concatenate([ks0, ks1])
    off = np.array([0, 1000], np.int64)
    lengths = [1000, 3001]
    qc, qs, w = np.stack([qc0, qc0]), np.stack([qs0, qs0]), np.stack([w0, w0])
    # P < k: Top-k over the stored scores
    gp, gt, gs = _run_full(kc, ks, off, lengths, qc, qs, w, 64, 512, want_scores=True)
    op, ot, osc = oracle.index_full(kc, ks, qc, qs, w, off, np.asarray(lengths), 64, 512, want_scores=True)
    assert np.array_equal(gp, op) and np.array_equal(gt, ot)
    for b, L in enumerate(lengths):
        nan = np.isnan(osc[b, :L])
        assert np.array_equal(np.isnan(gs[b, :L]), nan)
        assert np.array_equal(gs[b, :L][~nan].view(np.uint32), osc[b, :L][~nan].view(np.uint32))
    assert np.isnan(osc[0, 120:860]).all() and (osc[0, 100:120] == np.inf).all()
    # P >= k: the pool re-score path, with NaN positions inside the Top-k
    gp, gt, _ = _run_full(kc, ks, off, lengths, qc, qs, w, 512, 400)
    op, ot, _ = oracle.index_full(kc, ks, qc, qs, w, off, np.asarray(lengths), 512, 400)
    assert np.array_equal(gp, op) and np.array_equal(gt, ot)
    assert set(range(120, 260)) <= set(gt[0].tolist())   # the first 140 NaN positions
    # Reindex inside that pool
    want = oracle.index_reindex(kc, ks, qc, qs, w, off, np.asarray(lengths), op, 400)
    top = torch.full((2, 400), -7, dtype=torch.int32, device="cuda")
    ws = C.workspace(C.csa2_index_reindex_workspace_bytes(2, 512, 400))
    keep = [dev(qc), dev(qs), dev(w), dev(off), dev(np.asarray(lengths, np.int32)), dev(op)]
    C.csa2_index_reindex(C.cache(dev(kc), dev(ks)), *keep[:5], keep[5], 400, top, ws)
    torch.cuda.synchronize()
    assert C.device_status(ws) == 0
    assert np.array_equal(host(top), want)
    # the multi-query scan: two queries on sequence 0, one on sequence 1
    q_off = np.array([0, 2, 3], np.int32)
    q_vis = np.array([1000, 950, 3001], np.int32)
    qm, qsm, wm = qc[[0, 0, 1]], qs[[0, 0, 1]], w[[0, 0, 1]]
    pool = torch.full((3, 512), -7, dtype=torch.int32, device="cuda")
    top = torch.full((3, 400), -7, dtype=torch.int32, device="cuda")
    ws = C.workspace(C.csa2_index_multi_workspace_bytes(2, 3, 3001, 512, 400))
    C.csa2_index_multi(C.cache(dev(kc), dev(ks)), dev(qm), dev(qsm), dev(wm), dev(off), dev(q_off), dev(q_vis), 3001,
                       512, 400, pool, top, ws)
    torch.cuda.synchronize()
    assert C.device_status(ws) == 0
    wp, wt = oracle.index_multi(kc, ks, qm, qsm, wm, off, q_off, q_vis, 512, 400)
    assert np.array_equal(host(pool), wp) and np.array_equal(host(top), wt)


@pytest.mark.parametrize("P,k", [(2048, 512), (256, 512)])
def test_select_overfull_threshold_bucket(P, k):
    """Every indexer-K row identical: all keys tie, so the threshold bucket
    holds every key (far more than the 12288 the in-block lists take) and the
    selections fall back to global radix passes, which a diagnostic counter
    in the status block (word 4) records.  The pool must be blocks 0..P-1 and
    the Top-k positions 0..k-1, as the oracle says."""
    rng = np.random.default_rng(17)
    lengths = [300001, 140000]
    kc, ks, off, _ = _random_cache(rng, lengths)
    kc[:] = kc[0]
    ks[:] = ks[0]
    qc, qs, w = _queries(rng, 2)
    B, max_len = 2, max(lengths)
    cache = C.cache(dev(kc), dev(ks))
    args = [dev(qc), dev(qs), dev(w), dev(off), dev(np.asarray(lengths, np.int32))]
    pool = torch.full((B, P), -7, dtype=torch.int32, device="cuda")
    top = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
    ws = C.workspace(C.csa2_index_full_workspace_bytes(B, max_len, P, k))
    C.csa2_index_full(cache, *args, max_len, P, k, pool, top, ws)
    torch.cuda.synchronize()
    overfull = int(ws[:32].view(torch.int32)[4].item())
    assert C.device_status(ws) == 0
    # the pool select of both sequences (and with P < k the Top-k over the
    # stored scores as well) took the global radix path
    assert overfull == (2 if P >= k else 4), overfull
    op, ot, _ = oracle.index_full(kc, ks, qc, qs, w, off, np.asarray(lengths), P, k)
    assert np.array_equal(host(pool), op) and np.array_equal(host(top), ot)
    assert host(pool)[0].tolist() == list(range(P)) and host(top)[1].tolist() == list(range(k))
