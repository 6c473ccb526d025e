"""The bounded-wait failure path of the tensor-core scans.

Every pipeline wait inside the scans gives up after a time limit, flags
CSA2_DEV_TIMEOUT, drains the kernel's own copies and tensor-core operations,
frees its tensor memory and returns.  To exercise that path without any GPU
fault, a test control in the workspace's status block (word 3) makes each
CTA's producer withhold the copies of its first work item: stage 0 never
fills, so the waits on it must run out, after the short limit of word 2.  The
call must come back with the flag set; after the workspace is zero-filled
again (the contract after any flag), the next call on the same stream must be
bit-exact with the oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth.workloads as W
from long_context_decode_csa2_b200 import csa2 as C
from tests._gpu import dev, host

pytestmark = pytest.mark.gpu

CSA2_DEV_TIMEOUT = 16
CTL_WAIT_US, CTL_WITHHOLD = 2, 3     # int32 words of the workspace's status block


def _arm(ws, wait_us=2000):
    """Sets the test controls: a 2 ms wait limit and the withheld first item."""
    ctl = ws[:16].view(torch.int32)
    ctl[CTL_WAIT_US] = wait_us
    ctl[CTL_WITHHOLD] = 1


def _cache(rng, lengths):
    pad = (np.asarray(lengths) + 7) // 8 * 8
    off = np.concatenate([[0], np.cumsum(pad)[:-1]]).astype(np.int64)
    rows = int(pad.sum()) + 8
    kc = rng.integers(0, 256, (rows, 64), dtype=np.uint8)
    ks = rng.integers(124, 129, (rows, 4), dtype=np.uint8)
    return kc, ks, off


def _queries(rng, n):
    return (rng.integers(0, 256, (n, 4, 64), dtype=np.uint8), rng.integers(124, 129, (n, 4, 4), dtype=np.uint8),
            (0.5 + rng.random((n, 4))).astype(np.float32))


def test_scan_timeout_flags_returns_and_recovers():
    rng = np.random.default_rng(301)
    lengths = [70000, 5000, 777]
    kc, ks, off = _cache(rng, lengths)
    qc, qs, w = _queries(rng, 3)
    B, P, k, max_len = 3, 2048, 512, max(lengths)
    cache = C.cache(dev(kc), dev(ks))
    args = [dev(qc), dev(qs), dev(w), dev(off), dev(np.asarray(lengths, np.int32))]
    pool = torch.full((B, P), -7, dtype=torch.int32, device="cuda")
    top = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
    ws = C.workspace(C.csa2_index_full_workspace_bytes(B, max_len, P, k))
    _arm(ws)
    C.csa2_index_full(cache, *args, max_len, P, k, pool, top, ws)
    torch.cuda.synchronize()                       # the call came back
    flags = C.device_status(ws)
    assert flags & CSA2_DEV_TIMEOUT, f"flags {flags}"
    ws.zero_()
    C.csa2_index_full(cache, *args, max_len, P, k, pool, top, ws)
    torch.cuda.synchronize()
    assert C.device_status(ws) == 0
    op, ot, _ = oracle.index_full(kc, ks, qc, qs, w, off, np.asarray(lengths), P, k)
    assert np.array_equal(host(pool), op) and np.array_equal(host(top), ot)


def test_prefill_scan_timeout_flags_returns_and_recovers():
    pw = W.prefill_workload()
    n_raw, T, P, k = 40000, 37, 2048, 512
    inp = W.prefill_inputs_host(pw, n_raw=n_raw, T=T)
    n_ent = n_raw // 2
    rng = np.random.default_rng(302)
    kc, ks, _ = _cache(rng, [n_ent])
    cache = C.cache(dev(kc), dev(ks))
    d = [dev(inp["q_codes"]), dev(inp["q_scales"]), dev(inp["w"]), dev(inp["q_pos"])]
    pool = torch.full((T, P), -7, dtype=torch.int32, device="cuda")
    top = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    ws = C.workspace(C.csa2_index_prefill_workspace_bytes(T, n_ent, P, k))
    _arm(ws)
    C.csa2_index_prefill(cache, *d, 0, n_ent, 2, P, k, pool, top, ws)
    torch.cuda.synchronize()
    flags = C.device_status(ws)
    assert flags & CSA2_DEV_TIMEOUT, f"flags {flags}"
    ws.zero_()
    C.csa2_index_prefill(cache, *d, 0, n_ent, 2, P, k, pool, top, ws)
    torch.cuda.synchronize()
    assert C.device_status(ws) == 0
    wp, wt = oracle.index_prefill(kc, ks, 0, n_ent, inp["q_codes"], inp["q_scales"], inp["w"], inp["q_pos"], 2, P, k)
    assert np.array_equal(host(pool), wp) and np.array_equal(host(top), wt)


def test_multi_query_scan_timeout_flags_returns_and_recovers():
    rng = np.random.default_rng(303)
    lengths = [9000, 20000]
    kc, ks, off = _cache(rng, lengths)
    m = np.array([5, 2])
    q_off = np.concatenate([[0], np.cumsum(m)]).astype(np.int32)
    Q = int(q_off[-1])
    qc, qs, w = _queries(rng, Q)
    q_vis = np.concatenate([lengths[b] - np.arange(m[b])[::-1] for b in range(2)]).astype(np.int32)
    P, k = 2048, 512
    cache = C.cache(dev(kc), dev(ks))
    d = [dev(qc), dev(qs), dev(w), dev(off), dev(q_off), dev(q_vis)]
    pool = torch.full((Q, P), -7, dtype=torch.int32, device="cuda")
    top = torch.full((Q, k), -7, dtype=torch.int32, device="cuda")
    ws = C.workspace(C.csa2_index_multi_workspace_bytes(2, Q, max(lengths), P, k))
    _arm(ws)
    C.csa2_index_multi(cache, *d, max(lengths), P, k, pool, top, ws)
    torch.cuda.synchronize()
    flags = C.device_status(ws)
    assert flags & CSA2_DEV_TIMEOUT, f"flags {flags}"
    ws.zero_()
    C.csa2_index_multi(cache, *d, max(lengths), P, k, pool, top, ws)
    torch.cuda.synchronize()
    assert C.device_status(ws) == 0
    wp, wt = oracle.index_multi(kc, ks, qc, qs, w, off, q_off, q_vis, P, k)
    assert np.array_equal(host(pool), wp) and np.array_equal(host(top), wt)
