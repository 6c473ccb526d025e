"""End-to-end decode steps (layer patterns F / FRRU / (FRURU)x) on the GPU
against the oracle's own step: pools and Top-k bit-exact, attention within
tolerance.  Includes the full-size configurations (sampled for the 1M one)."""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth.workloads as W
from long_context_decode_csa2_b200 import csa2 as C
from long_context_decode_csa2_b200.decode import DecodeStep, FullCache
from tests._gpu import check_attention, dev, host

pytestmark = pytest.mark.gpu


def _device_layers(layers):
    keys = ("q", "q_codes", "q_scales", "w", "win", "win_scale", "win_len")
    return [{k: dev(L[k]) for k in keys} for L in layers]


def _run_and_compare(wl, full_rescan=False, host_caches=True, concurrent=True):
    layers = [W.layer_inputs_host(wl, l) for l in range(len(wl.pattern))]
    fulls = wl.full_layers()
    caches_h = [W.full_cache_host(wl, f, layers[f]["q_codes"], layers[f]["q_scales"]) for f in fulls]
    caches_d = [FullCache(C.cache(dev(c["idx_codes"]), dev(c["idx_scales"])),
                          C.cache(dev(c["main_codes"]), dev(c["main_scales"]))) for c in caches_h]
    off = caches_h[0]["seq_row_off"]
    lens = wl.lengths.astype(np.int32)
    step = DecodeStep(wl.pattern, wl.B, wl.max_len, wl.P, wl.k, full_rescan=full_rescan, concurrent=concurrent)
    dl = _device_layers(layers)
    off_d, len_d = dev(off), dev(lens)
    for _ in range(2):  # the second step reuses the workspaces (counters and histograms back at zero)
        step.run(caches_d, off_d, len_d, dl)
    torch.cuda.synchronize()
    assert step.device_flags() == 0
    ref = oracle.decode_step(wl.pattern, caches_h, off, lens, layers, wl.P, wl.k, 1 / math.sqrt(512),
                             full_rescan=full_rescan)
    for layer in range(len(wl.pattern)):
        assert np.array_equal(host(step.topk[layer]), ref["topk"][layer]), f"layer {layer} Top-k"
        check_attention(host(step.out[layer]), ref["out"][layer], host(step.lse[layer]), ref["lse"][layer],
                        what=f"layer {layer}")
    first_full = wl.full_layers()[0]
    assert np.array_equal(host(step.pool), ref["pools"][max(ref["pools"])])
    return step, ref


def test_decode_tiny_config():
    _run_and_compare(W.decode_workloads()["tiny_decode_b1_l8192"])


@pytest.mark.parametrize("concurrent", [True, False])
def test_decode_stack_reduced(concurrent):
    wl = W.DecodeWorkload("stack_small", np.array([131072, 50001, 9000, 333, 8]), "FRRU", needles=64)
    _run_and_compare(wl, concurrent=concurrent)


@pytest.mark.parametrize("rescan", [False, True])
def test_decode_ragged_reduced(rescan):
    wl = W.DecodeWorkload("ragged_small", np.array([4096, 65536, 7777, 20000, 4100, 33333]), "FRURU" * 2,
                          needles=32, lognormal=True)
    _run_and_compare(wl, full_rescan=rescan)


def test_decode_stack_full_size():
    _run_and_compare(W.decode_workloads()["stack_decode_b32_l128k"])


def _host_cores():
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def _compare_streamed(wl, step, caches_dev, layers, full_rescan=False, group_bytes=4 << 30):
    """Every sequence of a step that ran on device-resident caches, against
    the oracle's decode step.  The sequences' cache rows are copied to the
    host a group at a time (at most `group_bytes` of cache rows, at most one
    sequence per host core), so host memory stays bounded; the oracle runs
    each group on all host cores.  Top-k of every layer and the pool of every
    scanning layer bit-exact; attention within tolerance per sequence and
    layer."""
    off = caches_dev[0]["seq_row_off"]
    lens = wl.lengths.astype(np.int64)
    per_pos = 340 * len(caches_dev)  # 68 B indexer K + 272 B main KV per Full layer
    sm = 1 / math.sqrt(512)
    topk = [host(t) for t in step.topk]
    pools = {layer: host(t) for layer, t in step.pools.items()}
    out, lse = host(step.out), host(step.lse)
    b = 0
    while b < wl.B:
        group, size = [], 0
        while b < wl.B and len(group) < _host_cores() and (not group or size + lens[b] * per_pos <= group_bytes):
            group.append(b)
            size += int(lens[b]) * per_pos
            b += 1
        pad = (lens[group] + 7) // 8 * 8
        off_h = np.concatenate([[0], np.cumsum(pad)[:-1]]).astype(np.int64)
        rows = int(pad.sum())
        caches_h = []
        for c in caches_dev:
            h = dict(idx_codes=np.zeros((rows, 64), np.uint8), idx_scales=np.zeros((rows, 4), np.uint8),
                     main_codes=np.zeros((rows, 256), np.uint8), main_scales=np.zeros((rows, 16), np.uint8))
            for j, bb in enumerate(group):
                o, L, oh = int(off[bb]), int(lens[bb]), int(off_h[j])
                for key in h:
                    h[key][oh:oh + L] = host(c[key][o:o + L])
            caches_h.append(h)
        lg = [{k: (v[group] if isinstance(v, np.ndarray) and v.ndim >= 1 and v.shape[0] == wl.B else v)
               for k, v in L_.items()} for L_ in layers]
        ref = oracle.decode_step(wl.pattern, caches_h, off_h, lens[group].astype(np.int32), lg, wl.P, wl.k, sm,
                                 full_rescan=full_rescan)
        for layer in range(len(wl.pattern)):
            assert np.array_equal(topk[layer][group], ref["topk"][layer]), (group, layer)
            for j, bb in enumerate(group):
                check_attention(out[layer][bb], ref["out"][layer][j], lse[layer][bb], ref["lse"][layer][j],
                                what=f"seq {bb} layer {layer}")
        assert sorted(ref["pools"]) == sorted(pools)
        for layer, pool in ref["pools"].items():
            assert np.array_equal(pools[layer][group], pool), (group, layer)


def _full_size_step(wl, full_rescan=False):
    layers = [W.layer_inputs_host(wl, l) for l in range(len(wl.pattern))]
    caches = [W.full_cache_device(wl, f, layers[f]["q_codes"], layers[f]["q_scales"]) for f in wl.full_layers()]
    fc = [FullCache(C.cache(c["idx_codes"], c["idx_scales"]), C.cache(c["main_codes"], c["main_scales"]))
          for c in caches]
    step = DecodeStep(wl.pattern, wl.B, wl.max_len, wl.P, wl.k, full_rescan=full_rescan)
    step.run(fc, dev(caches[0]["seq_row_off"]), dev(wl.lengths.astype(np.int32)), _device_layers(layers))
    torch.cuda.synchronize()
    assert step.device_flags() == 0
    return step, caches, layers


def test_decode_long_full_size_all_sequences():
    """B = 64, L = 2^20, F R R U, the bench's launch configuration: every one
    of the 64 sequences checked against the oracle (cache rows streamed to
    the host from the device generator, which equals the NumPy generator
    byte for byte)."""
    wl = W.decode_workloads()["long_decode_b64_l1m"]
    step, caches, layers = _full_size_step(wl)
    _compare_streamed(wl, step, caches, layers)


@pytest.mark.parametrize("rescan", [False, True])
def test_decode_ragged_20_layers_full_size(rescan):
    """B = 48, lengths log-uniform on [4096, 2^20], 20 layers (F R U R U) x 4
    with four Full layers' own caches, at full size, under the pages' plan
    (only the first Full layer scans; later Full layers select inside its
    pool with their own caches) and with every Full layer rescanning: every
    sequence, every layer, against the oracle."""
    wl = W.decode_workloads()["ragged_decode_b48_20l"]
    step, caches, layers = _full_size_step(wl, full_rescan=rescan)
    _compare_streamed(wl, step, caches, layers, full_rescan=rescan)


def test_decode_with_input_events_and_layer_callbacks():
    """Inputs arriving on a copy stream (per-layer events) and outputs copied
    out per layer give the same results as the plain step."""
    wl = W.DecodeWorkload("stack_tiny", np.array([20000, 777, 4096]), "FRRU", needles=8)
    layers = [W.layer_inputs_host(wl, l) for l in range(len(wl.pattern))]
    caches_h = [W.full_cache_host(wl, f, layers[f]["q_codes"], layers[f]["q_scales"]) for f in wl.full_layers()]
    caches_d = [FullCache(C.cache(dev(c["idx_codes"]), dev(c["idx_scales"])),
                          C.cache(dev(c["main_codes"]), dev(c["main_scales"]))) for c in caches_h]
    off_d, len_d = dev(caches_h[0]["seq_row_off"]), dev(wl.lengths.astype(np.int32))
    plain = DecodeStep(wl.pattern, wl.B, wl.max_len, wl.P, wl.k)
    plain.run(caches_d, off_d, len_d, _device_layers(layers))
    torch.cuda.synchronize()
    step = DecodeStep(wl.pattern, wl.B, wl.max_len, wl.P, wl.k)
    keys = ("q", "q_codes", "q_scales", "w", "win", "win_scale", "win_len")
    dl = [{k: torch.empty_like(dev(L[k])) for k in keys} for L in layers]
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    ev = [torch.cuda.Event() for _ in layers]
    with torch.cuda.stream(h2d):
        for l, L in enumerate(layers):
            for k in keys:
                dl[l][k].copy_(torch.from_numpy(np.ascontiguousarray(
                    L[k].view(np.int16) if L[k].dtype == np.uint16 else L[k])).pin_memory().view(dl[l][k].dtype),
                    non_blocking=True)
            ev[l].record(h2d)
    outs = torch.empty((len(layers),) + tuple(step.out.shape[1:]), dtype=torch.float32).pin_memory()
    done = []

    def copy_out(layer, e):
        done.append(layer)
        d2h.wait_event(e)
        with torch.cuda.stream(d2h):
            outs[layer].copy_(step.out[layer], non_blocking=True)

    step.run(caches_d, off_d, len_d, dl, ready=ev, on_layer_done=copy_out)
    torch.cuda.synchronize()
    assert done == list(range(len(layers)))
    assert step.device_flags() == 0 and plain.device_flags() == 0
    for layer in range(len(layers)):
        assert np.array_equal(host(step.topk[layer]), host(plain.topk[layer]))
        assert np.array_equal(outs[layer].numpy(), host(plain.out[layer]))


def test_decode_step_replayed_from_a_cuda_graph():
    """A captured step replays to the same bits as the eager step."""
    wl = W.DecodeWorkload("graph_small", np.array([70000, 4096, 777]), "FRRU", needles=8)
    layers = [W.layer_inputs_host(wl, l) for l in range(len(wl.pattern))]
    caches_h = [W.full_cache_host(wl, f, layers[f]["q_codes"], layers[f]["q_scales"]) for f in wl.full_layers()]
    caches_d = [FullCache(C.cache(dev(c["idx_codes"]), dev(c["idx_scales"])),
                          C.cache(dev(c["main_codes"]), dev(c["main_scales"]))) for c in caches_h]
    off_d, len_d = dev(caches_h[0]["seq_row_off"]), dev(wl.lengths.astype(np.int32))
    dl = _device_layers(layers)
    step = DecodeStep(wl.pattern, wl.B, wl.max_len, wl.P, wl.k)
    step.run(caches_d, off_d, len_d, dl)
    torch.cuda.synchronize()
    eager = [host(t).copy() for t in step.topk], host(step.out).copy()
    graph = step.capture(caches_d, off_d, len_d, dl)
    step.out.zero_()
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    assert step.device_flags() == 0
    for layer in range(len(wl.pattern)):
        assert np.array_equal(host(step.topk[layer]), eager[0][layer])
    assert np.array_equal(host(step.out), eager[1])


def _new_tokens(seed, B, n_full, step, proj):
    """Per Full layer: one raw bf16 token per sequence, its logit, and the
    layer's W_idx (or a raw indexer row)."""
    import synth

    out = []
    for f in range(n_full):
        t = dict(raw=synth.normal_bf16(seed, synth.T_RAW, step, f, B * 512).reshape(B, 512),
                 logit=synth.normal_f32(seed, synth.T_LOGITS, step, f, B) * 2)
        if proj:
            t["w_idx"] = synth.normal_f32(seed, synth.T_WIDX, 0, f, 512 * 128, log2_div=13).reshape(512, 128)
        else:
            t["idx_raw"] = synth.normal_bf16(seed, synth.T_IDXRAW, step, f, B * 128).reshape(B, 128)
        out.append(t)
    return out


@pytest.mark.parametrize("proj", [True, False])
def test_ratio2_decode_steps(proj):
    """Ratio-2 decode: every step appends one raw token per sequence to each
    Full layer's caches (an entry every second step, the odd token pending
    on the device) and then runs the layer pattern over the grown caches.
    Cache bytes, lengths and the last step's Top-k are bit-exact with the
    oracle (streaming appends, then its decode step); attention within
    tolerance."""
    lens0 = np.array([9001, 4096, 20000, 333], np.int64)
    room, steps, pattern = 16, 5, "FRUFR"
    wl = W.DecodeWorkload("r2_small", lens0, pattern, needles=16, ratio=2, room=room)
    layers = [W.layer_inputs_host(wl, l) for l in range(len(pattern))]
    fulls = wl.full_layers()
    caches_h = [W.full_cache_host(wl, f, layers[f]["q_codes"], layers[f]["q_scales"]) for f in fulls]
    caches_d = [FullCache(C.cache(dev(c["idx_codes"]), dev(c["idx_scales"])),
                          C.cache(dev(c["main_codes"]), dev(c["main_scales"]))) for c in caches_h]
    off = caches_h[0]["seq_row_off"]
    off_d, len_d = dev(off), dev(lens0.astype(np.int32))
    step = DecodeStep(pattern, wl.B, wl.max_len + room, wl.P, wl.k, ratio=2, projection=proj)
    dl = _device_layers(layers)
    pend = [[None] * wl.B for _ in fulls]
    lens = lens0.copy()
    for t in range(steps):
        toks = _new_tokens(77, wl.B, len(fulls), t, proj)
        step.run(caches_d, off_d, len_d, dl, new_tokens=[{k: dev(v) for k, v in tk.items()} for tk in toks])
        # the oracle's appends into its own copies of the caches
        tok_off = np.arange(wl.B + 1, dtype=np.int64)
        new_lens = lens.copy()
        for f, (c, tk) in enumerate(zip(caches_h, toks)):
            ent, pend[f] = oracle.compress_stream(pend[f], tk["raw"], tk["logit"], tok_off, w_idx=tk.get("w_idx"),
                                                  idx_raw_bf16=tk.get("idx_raw"))
            for b in range(wl.B):
                ne = ent[b][0].shape[0]
                r0 = int(off[b] + lens[b])
                for key, arr in zip(("main_codes", "main_scales", "idx_codes", "idx_scales"), ent[b]):
                    c[key][r0:r0 + ne] = arr
                new_lens[b] = lens[b] + ne
        lens = new_lens
    torch.cuda.synchronize()
    assert step.device_flags() == 0
    assert host(len_d).tolist() == lens.tolist()
    assert lens.tolist() == (lens0 + steps // 2).tolist()
    for c_h, c_d in zip(caches_h, caches_d):
        for key, t in (("main_codes", c_d.main._keep[0]), ("main_scales", c_d.main._keep[1]),
                       ("idx_codes", c_d.idx._keep[0]), ("idx_scales", c_d.idx._keep[1])):
            assert np.array_equal(host(t), c_h[key]), key
    ref = oracle.decode_step(pattern, caches_h, off, lens.astype(np.int32), layers, wl.P, wl.k, 1 / math.sqrt(512))
    for layer in range(len(pattern)):
        assert np.array_equal(host(step.topk[layer]), ref["topk"][layer]), f"layer {layer} Top-k"
        check_attention(host(step.out[layer]), ref["out"][layer], host(step.lse[layer]), ref["lse"][layer],
                        what=f"layer {layer}")


def _verify_case(lens, m_per_seq, pattern, needles=16, lognormal=False, seqs_checked=None):
    """A verification step: sequence b carries m_per_seq[b] candidate queries
    whose entries are already in its cache; candidate i sees all but the
    last m_b - 1 - i entries."""
    wl = W.DecodeWorkload("verify_small", np.asarray(lens), pattern, needles=needles, lognormal=lognormal)
    m = np.asarray(m_per_seq)
    q_off = np.concatenate([[0], np.cumsum(m)]).astype(np.int32)
    q_vis = np.concatenate([wl.lengths[b] - (m[b] - 1 - np.arange(m[b])) for b in range(wl.B)]).astype(np.int32)
    Q = int(q_off[-1])
    wq = W.DecodeWorkload("verify_small_q", q_vis.astype(np.int64), pattern, seed=wl.seed + 7)
    layers = [W.layer_inputs_host(wq, l) for l in range(len(pattern))]
    return wl, q_off, q_vis, Q, layers


def test_verify_step_ragged_queries():
    """Speculative verification: 6, 0, 3 and 9 candidate queries on four
    sequences (9 spans two query groups of the scan); Top-k bit-exact and
    attention within tolerance against the oracle's step over the queries
    as their own segments."""
    wl, q_off, q_vis, Q, layers = _verify_case([9001, 4096, 20000, 333], [6, 0, 3, 9], "FRUFR")
    fulls = wl.full_layers()
    first = np.minimum(q_off[:-1], Q - 1)  # needles aimed at each sequence's first query
    caches_h = [W.full_cache_host(wl, f, layers[f]["q_codes"][first], layers[f]["q_scales"][first]) for f in fulls]
    caches_d = [FullCache(C.cache(dev(c["idx_codes"]), dev(c["idx_scales"])),
                          C.cache(dev(c["main_codes"]), dev(c["main_scales"]))) for c in caches_h]
    off = caches_h[0]["seq_row_off"]
    step = DecodeStep(wl.pattern, wl.B, wl.max_len, wl.P, wl.k, queries=Q)
    step.run(caches_d, dev(off), None, _device_layers(layers), q_off=dev(q_off), q_vis=dev(q_vis))
    torch.cuda.synchronize()
    assert step.device_flags() == 0
    rows, vis = oracle.multi_query_rows(off, q_off, q_vis)
    assert np.array_equal(host(step.q_row_off), rows)
    ref = oracle.decode_step(wl.pattern, caches_h, rows, vis, layers, wl.P, wl.k, 1 / math.sqrt(512))
    for layer in range(len(wl.pattern)):
        assert np.array_equal(host(step.topk[layer]), ref["topk"][layer]), f"layer {layer} Top-k"
        check_attention(host(step.out[layer]), ref["out"][layer], host(step.lse[layer]), ref["lse"][layer],
                        what=f"layer {layer}")
    assert np.array_equal(host(step.pool), ref["pools"][max(ref["pools"])])


def test_verify_index_multi_matches_oracle_and_single_queries():
    """csa2_index_multi alone: equal to the oracle, and to csa2_index_full
    run once per query (the same sequence repeated as a segment)."""
    wl, q_off, q_vis, Q, layers = _verify_case([70000, 8, 131072], [5, 2, 8], "F", needles=8)
    first = np.minimum(q_off[:-1], Q - 1)
    c = W.full_cache_host(wl, 0, layers[0]["q_codes"][first], layers[0]["q_scales"][first])
    idx = C.cache(dev(c["idx_codes"]), dev(c["idx_scales"]))
    L = layers[0]
    pool = torch.full((Q, wl.P), -1, dtype=torch.int32, device="cuda")
    top = torch.full((Q, wl.k), -1, dtype=torch.int32, device="cuda")
    ws = C.workspace(C.csa2_index_multi_workspace_bytes(wl.B, Q, wl.max_len, wl.P, wl.k))
    C.csa2_index_multi(idx, dev(L["q_codes"]), dev(L["q_scales"]), dev(L["w"]), dev(c["seq_row_off"]), dev(q_off),
                       dev(q_vis), wl.max_len, wl.P, wl.k, pool, top, ws)
    torch.cuda.synchronize()
    assert C.device_status(ws) == 0
    want_p, want_t = oracle.index_multi(c["idx_codes"], c["idx_scales"], L["q_codes"], L["q_scales"], L["w"],
                                        c["seq_row_off"], q_off, q_vis, wl.P, wl.k)
    assert np.array_equal(host(pool), want_p) and np.array_equal(host(top), want_t)
    rows, vis = oracle.multi_query_rows(c["seq_row_off"], q_off, q_vis)
    pool1 = torch.full((Q, wl.P), -1, dtype=torch.int32, device="cuda")
    top1 = torch.full((Q, wl.k), -1, dtype=torch.int32, device="cuda")
    ws1 = C.workspace(C.csa2_index_full_workspace_bytes(Q, wl.max_len, wl.P, wl.k))
    C.csa2_index_full(idx, dev(L["q_codes"]), dev(L["q_scales"]), dev(L["w"]), dev(rows), dev(vis), wl.max_len, wl.P,
                      wl.k, pool1, top1, ws1)
    torch.cuda.synchronize()
    assert np.array_equal(host(pool1), host(pool)) and np.array_equal(host(top1), host(top))


def test_verify_step_full_size_sampled():
    """B = 64, L = 2^20, six candidate queries per sequence, F R R U: the
    whole batch runs on the GPU; the queries of two sequences are recomputed
    by the oracle."""
    base = W.decode_workloads()["long_decode_b64_l1m"]
    m = 6
    wl, q_off, q_vis, Q, layers = _verify_case(base.lengths, [m] * base.B, base.pattern, needles=base.needles,
                                               lognormal=True)
    c = W.full_cache_device(wl, 0, layers[0]["q_codes"][::m], layers[0]["q_scales"][::m])
    cache = FullCache(C.cache(c["idx_codes"], c["idx_scales"]), C.cache(c["main_codes"], c["main_scales"]))
    off = c["seq_row_off"]
    step = DecodeStep(wl.pattern, wl.B, wl.max_len, wl.P, wl.k, queries=Q)
    step.run([cache], dev(off), None, _device_layers(layers), q_off=dev(q_off), q_vis=dev(q_vis))
    torch.cuda.synchronize()
    assert step.device_flags() == 0
    for b in (0, 41):
        o = int(off[b])
        Lb = int(wl.lengths[b])
        ch = dict(idx_codes=host(c["idx_codes"][o:o + Lb]), idx_scales=host(c["idx_scales"][o:o + Lb]),
                  main_codes=host(c["main_codes"][o:o + Lb]), main_scales=host(c["main_scales"][o:o + Lb]))
        qs = slice(int(q_off[b]), int(q_off[b + 1]))
        lb = [{k: v[qs] for k, v in L_.items()} for L_ in layers]
        ref = oracle.decode_step(wl.pattern, [ch], np.zeros(m, np.int64), q_vis[qs], lb, wl.P, wl.k,
                                 1 / math.sqrt(512))
        for layer in range(len(wl.pattern)):
            assert np.array_equal(host(step.topk[layer][qs]), ref["topk"][layer]), (b, layer)
            check_attention(host(step.out[layer][qs]), ref["out"][layer], what=f"seq {b} layer {layer}")


def test_decode_with_the_full_layer_split_in_two_calls():
    """csa2_index_full_pool + csa2_index_full_topk (split_full) give the same
    bits as the single call, with the Reindex layers started from the pool."""
    wl = W.DecodeWorkload("split_small", np.array([70000, 4096, 777]), "FRRU", needles=8)
    layers = [W.layer_inputs_host(wl, l) for l in range(len(wl.pattern))]
    caches_h = [W.full_cache_host(wl, f, layers[f]["q_codes"], layers[f]["q_scales"]) for f in wl.full_layers()]
    caches_d = [FullCache(C.cache(dev(c["idx_codes"]), dev(c["idx_scales"])),
                          C.cache(dev(c["main_codes"]), dev(c["main_scales"]))) for c in caches_h]
    off_d, len_d = dev(caches_h[0]["seq_row_off"]), dev(wl.lengths.astype(np.int32))
    dl = _device_layers(layers)
    plain = DecodeStep(wl.pattern, wl.B, wl.max_len, wl.P, wl.k)
    split = DecodeStep(wl.pattern, wl.B, wl.max_len, wl.P, wl.k, split_full=True)
    plain.run(caches_d, off_d, len_d, dl)
    split.run(caches_d, off_d, len_d, dl)
    torch.cuda.synchronize()
    assert plain.device_flags() == 0 and split.device_flags() == 0
    assert np.array_equal(host(split.pool), host(plain.pool))
    for layer in range(len(wl.pattern)):
        assert np.array_equal(host(split.topk[layer]), host(plain.topk[layer]))
    assert np.array_equal(host(split.out), host(plain.out))


@pytest.mark.parametrize("groups,rescan", [(2, False), (3, True)])
def test_decode_grouped_layer_order_matches_layer_order(groups, rescan):
    """groups > 1 (layer order per group of sequences, groups on their own
    streams, graph-captured too) gives the bits of the plain layer-order
    step: every call sees its sequences alike in both.  With a rescan the
    second Full layer scans again, after every group's earlier layers."""
    wl = W.DecodeWorkload("grouped_small", np.array([70000, 4096, 777, 20000, 9]), "FRRUFR", needles=8)
    layers = [W.layer_inputs_host(wl, l) for l in range(len(wl.pattern))]
    caches_h = [W.full_cache_host(wl, f, layers[f]["q_codes"], layers[f]["q_scales"]) for f in wl.full_layers()]
    caches_d = [FullCache(C.cache(dev(c["idx_codes"]), dev(c["idx_scales"])),
                          C.cache(dev(c["main_codes"]), dev(c["main_scales"]))) for c in caches_h]
    off_d, len_d = dev(caches_h[0]["seq_row_off"]), dev(wl.lengths.astype(np.int32))
    dl = _device_layers(layers)
    plain = DecodeStep(wl.pattern, wl.B, wl.max_len, wl.P, wl.k, concurrent=False, full_rescan=rescan)
    grouped = DecodeStep(wl.pattern, wl.B, wl.max_len, wl.P, wl.k, concurrent=False, groups=groups,
                         full_rescan=rescan)
    plain.run(caches_d, off_d, len_d, dl)
    done = []
    grouped.run(caches_d, off_d, len_d, dl, on_layer_done=lambda layer, ev: done.append(layer))
    torch.cuda.synchronize()
    assert done == list(range(len(wl.pattern)))
    assert plain.device_flags() == 0 and grouped.device_flags() == 0

    def same(a, b):
        for p in a.pools:
            assert np.array_equal(host(a.pools[p]), host(b.pools[p])), f"pool of layer {p}"
        for layer in range(len(wl.pattern)):
            assert np.array_equal(host(a.topk[layer]), host(b.topk[layer])), f"layer {layer} Top-k"
        assert np.array_equal(host(a.out), host(b.out))
        assert np.array_equal(host(a.lse), host(b.lse))

    same(grouped, plain)
    grouped.out.zero_()
    g = grouped.capture(caches_d, off_d, len_d, dl)
    g.replay()
    torch.cuda.synchronize()
    same(grouped, plain)
    del g

