"""GPU parity of sparse attention (decode and prefill windows) against the
fp64 oracle, within max-abs 2e-3 and relative-L2 1e-3, plus edge cases."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from long_context_decode_csa2_b200 import csa2 as C
from tests._gpu import check_attention, dev, host

pytestmark = pytest.mark.gpu


def _case(seed, lengths, k, win_len, lognormal=False):
    rng = np.random.default_rng(seed)
    B = len(lengths)
    pad = (np.asarray(lengths) + 7) // 8 * 8
    off = np.concatenate([[0], np.cumsum(pad)[:-1]]).astype(np.int64)
    rows = int(pad.sum())
    mc = np.zeros((rows, 256), np.uint8)
    ms = np.zeros((rows, 16), np.uint8)
    for b in range(B):
        nk = synth.stream_key(seed, synth.T_ROWNORM, b, 0) if lognormal else None
        c, s = synth.mxfp4_rows(seed, synth.T_MAIN_CODES, synth.T_MAIN_SCALES, b, 0, 0, int(pad[b]), 512, nk)
        mc[off[b]:off[b] + pad[b]], ms[off[b]:off[b] + pad[b]] = c, s
    top = np.full((B, k), -1, np.int32)
    for b in range(B):
        m = min(k, lengths[b])
        if m:
            sel = np.sort(rng.choice(lengths[b], m, replace=False))
            top[b, :m] = sel
            top[b, rng.integers(0, k, 3)] = -1
    q = np.stack([synth.normal_bf16(seed, synth.T_Q, b, 0, 16 * 512).reshape(16, 512) for b in range(B)])
    win = np.stack([synth.e4m3_rows(seed, synth.T_WIN, b, 0, 0, 128) for b in range(B)])
    ws = np.array([synth.window_scale(seed, b, 0) for b in range(B)], np.float32)
    wl = np.asarray(win_len, np.int32)
    return dict(q=q, mc=mc, ms=ms, off=off, lens=np.asarray(lengths, np.int32), top=top, win=win, ws=ws, wl=wl)


def _gpu_decode(d, sm):
    B, k = d["top"].shape
    out = torch.zeros((B, 16, 512), dtype=torch.float32, device="cuda")
    lse = torch.zeros((B, 16), dtype=torch.float32, device="cuda")
    ws = C.workspace(C.csa2_sparse_attn_decode_workspace_bytes(B, k))
    cache = C.cache(dev(d["mc"]), dev(d["ms"]))
    args = [dev(d["q"]), cache, dev(d["off"]), dev(d["lens"]), dev(d["top"]), dev(d["win"]), dev(d["ws"]),
            dev(d["wl"])]
    C.csa2_sparse_attn_decode(*args, sm, out, ws, lse=lse)
    torch.cuda.synchronize()
    return host(out), host(lse), C.device_status(ws)


@pytest.mark.parametrize("lengths,k,win_len,lognormal", [
    ([8192], 512, [128], False),
    ([5000, 700, 131072], 512, [128, 37, 128], True),
    ([300, 64], 100, [0, 128], False),
    ([2000], 700, [5], False),
    ([30000, 5000, 2047], 2048, [128, 128, 1], True),   # the largest Top-k the call accepts
    ([40], 4, [0], False),                               # one to three selected rows, no window
    ([40], 1, [1], False),                               # a single window row (the one selected is -1)
])
def test_attention_decode_matches_oracle(lengths, k, win_len, lognormal):
    d = _case(len(lengths) * 31 + k, lengths, k, win_len, lognormal)
    sm = 1 / math.sqrt(512)
    out, lse, flags = _gpu_decode(d, sm)
    assert flags == 0
    ro, rl = oracle.attn_decode(d["q"], d["mc"], d["ms"], d["off"], d["lens"], d["top"], d["win"], d["ws"], d["wl"],
                                sm)
    check_attention(out, ro, lse, rl, what=str(lengths))


def test_attention_empty_and_out_of_range():
    d = _case(3, [100, 50], 16, [0, 4])
    d["top"][0] = -1
    d["top"][1, 0] = 77          # >= seq_len 50: skipped and flagged
    out, lse, flags = _gpu_decode(d, 0.05)
    assert flags == 1
    assert not out[0].any() and np.all(np.isneginf(lse[0]))
    d2 = dict(d)
    d2["top"] = d["top"].copy()
    d2["top"][1, 0] = -1
    ro, rl = oracle.attn_decode(d2["q"], d2["mc"], d2["ms"], d2["off"], d2["lens"], d2["top"], d2["win"], d2["ws"],
                                d2["wl"], 0.05)
    check_attention(out[1], ro[1], lse[1], rl[1])


def test_attention_prefill_window_matches_oracle():
    rng = np.random.default_rng(12)
    n_raw, ratio, k, T = 3000, 2, 512, 9
    n_ent = n_raw // ratio
    mc, ms = synth.mxfp4_rows(4, synth.T_MAIN_CODES, synth.T_MAIN_SCALES, 0, 0, 0, (n_ent + 7) // 8 * 8, 512)
    raw_win = synth.e4m3_rows(4, synth.T_RAWWIN, 0, 0, 0, n_raw)
    q_pos = np.array([0, 1, 2, 126, 127, 128, 255, 1500, 2999], np.int32)
    q = synth.normal_bf16(4, synth.T_Q, 0, 0, T * 8192).reshape(T, 16, 512)
    top = np.full((T, k), -1, np.int32)
    for i, p in enumerate(q_pos):
        vis = (p + 1) // ratio
        m = min(vis, k)
        if m:
            top[i, :m] = np.sort(rng.choice(vis, m, replace=False))
    sm, sig = 1 / math.sqrt(512), float(synth.window_scale(4, 0, 0))
    out = torch.zeros((T, 16, 512), dtype=torch.float32, device="cuda")
    lse = torch.zeros((T, 16), dtype=torch.float32, device="cuda")
    ws = C.workspace(C.csa2_sparse_attn_prefill_workspace_bytes(T, k))
    cache = C.cache(dev(mc), dev(ms))
    keep = [dev(q), dev(q_pos), dev(top), dev(raw_win)]
    C.csa2_sparse_attn_prefill(keep[0], keep[1], cache, 0, n_ent, ratio, keep[2], keep[3], sig, sm, out, ws, lse=lse)
    torch.cuda.synchronize()
    assert C.device_status(ws) == 0
    ro, rl = oracle.attn_prefill(q, q_pos, mc, ms, 0, n_ent, ratio, top, raw_win, sig, sm)
    check_attention(host(out), ro, host(lse), rl)
