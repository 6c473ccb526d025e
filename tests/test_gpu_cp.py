"""Context-parallel decode on one GPU (every shard driven by this process):
the shards' local selections, ranked by csa2_score_positions and merged by
csa2_topk_merge, give the single-device pool and Top-k bit for bit; the
shards' attention partials combined by csa2_attn_combine match the oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth.workloads as W
from long_context_decode_csa2_b200 import csa2 as C
from long_context_decode_csa2_b200.cp import Shard, ShardedStep, shard_bounds, split_caches, to_full_cache
from long_context_decode_csa2_b200.decode import DecodeStep, FullCache
from tests._gpu import check_attention, dev, host

pytestmark = pytest.mark.gpu


def _layers_dev(layers, rows=None):
    keys = ("q", "q_codes", "q_scales", "w", "win", "win_scale", "win_len")
    return [{k: dev(L[k]) for k in keys} for L in layers]


def test_score_positions_match_the_oracle():
    wl = W.DecodeWorkload("cp_score", np.array([5000, 777]), "F", needles=8, lognormal=True)
    L0 = W.layer_inputs_host(wl, 0)
    c = W.full_cache_host(wl, 0, L0["q_codes"], L0["q_scales"])
    off = c["seq_row_off"]
    rng = np.random.default_rng(3)
    ids = np.stack([np.sort(rng.choice(int(L), 200, replace=False)) for L in wl.lengths]).astype(np.int32)
    ids[1, -3:] = -1
    blocks = np.stack([np.sort(rng.choice(int((L + 7) // 8), 64, replace=False)) for L in wl.lengths]).astype(np.int32)
    keys = torch.zeros(ids.shape, dtype=torch.int32, device="cuda")
    bkeys = torch.zeros(blocks.shape, dtype=torch.int32, device="cuda")
    ws = C.workspace(C.csa2_score_positions_workspace_bytes(wl.B))
    args = (C.cache(dev(c["idx_codes"]), dev(c["idx_scales"])), dev(L0["q_codes"]), dev(L0["q_scales"]), dev(L0["w"]),
            dev(off), dev(wl.lengths.astype(np.int32)))
    C.csa2_score_positions(*args, dev(ids), 1, keys, ws)
    C.csa2_score_positions(*args, dev(blocks), 8, bkeys, ws)
    torch.cuda.synchronize()
    assert C.device_status(ws) == 0
    gk, gb = host(keys).view(np.uint32), host(bkeys).view(np.uint32)
    for b in range(wl.B):
        L = int(wl.lengths[b])
        s = oracle.index_scores(c["idx_codes"], c["idx_scales"], off[b] + np.arange(L), L0["q_codes"][b],
                                L0["q_scales"][b], L0["w"][b])
        rk = np.array([oracle.rank_key(v) for v in s], np.uint32)
        want = np.array([rk[i] if i >= 0 else 0 for i in ids[b]], np.uint32)
        assert np.array_equal(gk[b], want)
        wantb = np.array([rk[8 * j:min(L, 8 * j + 8)].max() for j in blocks[b]], np.uint32)
        assert np.array_equal(gb[b], wantb)


def test_topk_merge_matches_a_full_sort():
    """Three shards' ascending candidate lists with ties and padding: the
    merge equals sorting the union by (key desc, id asc)."""
    rng = np.random.default_rng(4)
    G, B, n, k = 3, 2, 300, 128
    lo = np.array([[0, 0], [5000, 4000], [9000, 8000]], np.int64)
    ids = np.full((G, B, n), -1, np.int32)
    keys = np.zeros((G, B, n), np.uint32)
    for g in range(G):
        for b in range(B):
            m = n - 17 * g
            ids[g, b, :m] = np.sort(rng.choice(4000, m, replace=False))
            keys[g, b, :m] = rng.integers(1, 40, m).astype(np.uint32) | 0x80000000  # many ties
    out = torch.full((B, k), -1, dtype=torch.int32, device="cuda")
    mine = torch.full((B, k), -1, dtype=torch.int32, device="cuda")
    ws = C.workspace(C.csa2_topk_merge_workspace_bytes(G, B, n))
    C.csa2_topk_merge(dev(keys.view(np.int32)), dev(ids), dev(lo), k, out, ws, lo=dev(lo[1]),
                      hi=dev(lo[2]), out_local=mine)
    torch.cuda.synchronize()
    for b in range(B):
        cand = [(int(keys[g, b, i]), int(ids[g, b, i] + lo[g, b])) for g in range(G) for i in range(n)
                if ids[g, b, i] >= 0]
        best = sorted(cand, key=lambda t: (-t[0], t[1]))[:k]
        want = sorted(i for _, i in best)
        assert host(out[b]).tolist() == want + [-1] * (k - len(want))
        loc = [i - lo[1, b] if lo[1, b] <= i < lo[2, b] else -1 for i in host(out[b])]
        assert host(mine[b]).tolist() == [(-1 if i < 0 else int(x)) for i, x in zip(host(out[b]), loc)]


@pytest.mark.parametrize("G", [2, 3])
def test_sharded_step_equals_single_device(G):
    wl = W.DecodeWorkload("cp_small", np.array([60000, 33001, 20480]), "FRURU", needles=32, lognormal=True)
    layers = [W.layer_inputs_host(wl, l) for l in range(len(wl.pattern))]
    caches_h = [W.full_cache_host(wl, f, layers[f]["q_codes"], layers[f]["q_scales"]) for f in wl.full_layers()]
    off = caches_h[0]["seq_row_off"]
    lens = wl.lengths.astype(np.int32)
    single = DecodeStep(wl.pattern, wl.B, wl.max_len, wl.P, wl.k)
    single.run([FullCache(C.cache(dev(c["idx_codes"]), dev(c["idx_scales"])),
                          C.cache(dev(c["main_codes"]), dev(c["main_scales"]))) for c in caches_h],
               dev(off), dev(lens), _layers_dev(layers))

    bounds = shard_bounds(wl.lengths, G)
    parts = [split_caches(c, off, bounds) for c in caches_h]  # [cache][shard] -> (arrays, row offsets)
    shards = []
    for g in range(G):
        lg = []
        for L in layers:
            Lg = dict(L)
            if g != G - 1:  # the window belongs to the shard with the newest entries
                Lg["win_len"] = np.zeros_like(L["win_len"])
            lg.append(Lg)
        shards.append(Shard(caches=[to_full_cache(parts[f][g][0], "cuda") for f in range(len(caches_h))],
                            seq_row_off=dev(parts[0][g][1]), seq_len=dev((bounds[g + 1] - bounds[g]).astype(np.int32)),
                            lo=dev(bounds[g]), hi=dev(bounds[g + 1]), layers=_layers_dev(lg)))
    src_pos = dev(bounds[:-1])
    max_shard = int((bounds[1:] - bounds[:-1]).max())
    cp = ShardedStep(wl.pattern, wl.B, max_shard, G, G, wl.P, wl.k)
    cp.run(shards, src_pos, dev(bounds[:-1] // 8))
    torch.cuda.synchronize()
    assert cp.device_flags() == 0 and single.device_flags() == 0
    assert np.array_equal(host(cp.pool), host(single.pool))
    ref = oracle.decode_step(wl.pattern, caches_h, off, lens, layers, wl.P, wl.k, 1 / math.sqrt(512))
    for layer in range(len(wl.pattern)):
        assert np.array_equal(host(cp.topk[layer]), host(single.topk[layer])), f"layer {layer} Top-k"
        check_attention(host(cp.out[layer]), ref["out"][layer], host(cp.lse[layer]), ref["lse"][layer],
                        what=f"layer {layer}")
