"""Pins of the oracle's decode step through a layer pattern (no GPU).

"DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression", section
"三个方向一起压小缓存", and the "DeepSeek-V4.1" reading notes: the first Full
layer scans every visible position and builds the pool of best blocks; a
Reindex layer ranks only the pool's positions with its own indexer query
against the nearest Full layer's indexer K; a Reuse layer takes the previous
Top-k unchanged; every layer attends with the main KV of its nearest Full
layer.  Each selection below is checked by brute force (scores of the
candidate positions, a full sort by (score desc, position asc)).
"""
import math

import numpy as np
import pytest

import synth.workloads as W

PATTERN = "FRUFRU"           # two Full layers, each followed by a Reindex and a Reuse layer
NEAREST_F = [0, 0, 0, 3, 3, 3]


def _setup():
    wl = W.DecodeWorkload("decode_step_pins", np.array([700, 1500]), PATTERN, P=16, k=32, needles=2)
    layers = [W.layer_inputs_host(wl, l) for l in range(len(PATTERN))]
    caches = {f: W.full_cache_host(wl, f, layers[f]["q_codes"], layers[f]["q_scales"]) for f in wl.full_layers()}
    return wl, layers, caches


def _rank(orc, cache, lay, b, positions):
    off = int(cache["seq_row_off"][b])
    s = orc.index_scores(cache["idx_codes"], cache["idx_scales"], off + np.asarray(positions, np.int64),
                         lay["q_codes"][b], lay["q_scales"][b], lay["w"][b])
    return [orc.rank_key(v) for v in s]


def _best(keys, ids, n):
    order = sorted(range(len(ids)), key=lambda i: (-keys[i], ids[i]))[:n]
    out = sorted(ids[i] for i in order)
    return out + [-1] * (n - len(out))


def _brute_full(orc, cache, lay, b, L, P, k):
    key = _rank(orc, cache, lay, b, range(L))
    nb = (L + 7) // 8
    bkey = [max(key[8 * j:min(L, 8 * j + 8)]) for j in range(nb)]
    return _best(bkey, list(range(nb)), P), _best(key, list(range(L)), k)


def _brute_in_pool(orc, cache, lay, b, L, pool, k):
    pos = [8 * int(j) + i for j in pool if j >= 0 for i in range(8) if 8 * int(j) + i < L]
    return _best(_rank(orc, cache, lay, b, pos), pos, k)


@pytest.mark.parametrize("full_rescan", [False, True])
def test_decode_step_layer_modes_by_brute_force(orc, full_rescan):
    wl, layers, caches = _setup()
    lens = wl.lengths.astype(np.int32)
    off = caches[0]["seq_row_off"]
    sm = 1 / math.sqrt(512)
    res = orc.decode_step(PATTERN, [caches[0], caches[3]], off, lens, layers, wl.P, wl.k, sm,
                          full_rescan=full_rescan, nthreads=1)
    assert sorted(res["pools"]) == ([0, 3] if full_rescan else [0])
    for b in range(wl.B):
        L = int(lens[b])
        pool0, top0 = _brute_full(orc, caches[0], layers[0], b, L, wl.P, wl.k)
        assert res["pools"][0][b].tolist() == pool0
        assert res["topk"][0][b].tolist() == top0
        assert res["topk"][1][b].tolist() == _brute_in_pool(orc, caches[0], layers[1], b, L, pool0, wl.k)
        pool = pool0
        if full_rescan:                                   # the second Full layer scans its own cache again
            pool3, top3 = _brute_full(orc, caches[3], layers[3], b, L, wl.P, wl.k)
            assert res["pools"][3][b].tolist() == pool3
            assert res["topk"][3][b].tolist() == top3
            pool = pool3
        else:                                             # it ranks the first pool with its own cache
            assert res["topk"][3][b].tolist() == _brute_in_pool(orc, caches[3], layers[3], b, L, pool0, wl.k)
        assert res["topk"][4][b].tolist() == _brute_in_pool(orc, caches[3], layers[4], b, L, pool, wl.k)
    # Reuse layers repeat the Top-k before them
    assert np.array_equal(res["topk"][2], res["topk"][1])
    assert np.array_equal(res["topk"][5], res["topk"][4])
    # each layer attends its own Top-k in its nearest Full layer's main KV, with its own window
    for l in range(len(PATTERN)):
        c, lay = caches[NEAREST_F[l]], layers[l]
        o, lse = orc.attn_decode(lay["q"], c["main_codes"], c["main_scales"], off, lens, res["topk"][l], lay["win"],
                                 lay["win_scale"], lay["win_len"], sm, nthreads=1)
        assert np.array_equal(res["out"][l], o) and np.array_equal(res["lse"][l], lse), l
