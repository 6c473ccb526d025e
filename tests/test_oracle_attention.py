"""Pins of the oracle's sparse attention (decode and causal prefill): closed
forms and a brute-force dense softmax written independently here (no GPU)."""
import numpy as np
import pytest
import torch
from scipy.special import logsumexp, softmax

import synth


def _main_decode_indep(codes, scales):
    """Dequantise MXFP4 rows with vectorised NumPy (independent of the oracle)."""
    lo = codes & 15
    hi = codes >> 4
    c = np.stack([lo, hi], -1).reshape(codes.shape[0], -1).astype(np.int64)
    mag = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])[c & 7]
    val = np.where(c & 8, -mag, mag)
    return val * np.exp2(np.repeat(scales.astype(np.float64) - 127, 32, axis=1))


def _e4m3_indep(b):
    return torch.from_numpy(np.ascontiguousarray(b)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _bf16(x):
    return synth.f32_to_bf16_bits(np.asarray(x, np.float32))


def _setup(seed, B=2, L=700, k=64, win_len=(128, 37)):
    rng = np.random.default_rng(seed)
    rows = B * L
    mc = rng.integers(0, 256, (rows, 256), dtype=np.uint8)
    ms = rng.integers(124, 128, (rows, 16), dtype=np.uint8)
    off = np.arange(B, dtype=np.int64) * L
    lens = np.array([L, L - 11][:B], np.int32)
    top = np.full((B, k), -1, np.int32)
    for b in range(B):
        sel = np.sort(rng.choice(lens[b], k - 5, replace=False))
        top[b, :k - 5] = sel
    win = synth.e4m3_rows(seed, synth.T_WIN, 0, 0, 0, B * 128).reshape(B, 128, 512)
    ws = np.array([synth.window_scale(seed, b, 0) for b in range(B)], np.float32)
    wl = np.array(win_len[:B], np.int32)
    q = _bf16(rng.standard_normal((B, 16, 512)))
    return dict(q=q, mc=mc, ms=ms, off=off, lens=lens, top=top, win=win, ws=ws, wl=wl)


def test_attention_bruteforce_dense_softmax(orc):
    d = _setup(20)
    sm = 1 / np.sqrt(512)
    out, lse = orc.attn_decode(d["q"], d["mc"], d["ms"], d["off"], d["lens"], d["top"], d["win"], d["ws"], d["wl"], sm)
    main = _main_decode_indep(d["mc"], d["ms"])
    for b in range(2):
        sel = d["top"][b][d["top"][b] >= 0]
        keys = np.concatenate([main[d["off"][b] + sel],
                               _e4m3_indep(d["win"][b, :d["wl"][b]]) * float(d["ws"][b])])
        q = synth.bf16_bits_to_f32(d["q"][b]).astype(np.float64)
        logits = sm * q @ keys.T
        ref = softmax(logits, axis=1) @ keys
        assert np.allclose(out[b], ref, rtol=1e-11, atol=1e-13)
        assert np.allclose(lse[b], logsumexp(logits, axis=1), rtol=1e-12)


def test_attention_identical_keys_return_the_key(orc):
    d = _setup(21, win_len=(0, 0))
    d["mc"][:] = d["mc"][3]
    d["ms"][:] = d["ms"][3]
    out, _ = orc.attn_decode(d["q"], d["mc"], d["ms"], d["off"], d["lens"], d["top"], d["win"], d["ws"], d["wl"], 0.3)
    key = _main_decode_indep(d["mc"][3:4], d["ms"][3:4])[0]
    assert np.allclose(out, key[None, None, :], rtol=0, atol=1e-14)


def test_attention_zero_query_gives_mean_of_keys(orc):
    d = _setup(22)
    d["q"][:] = 0
    out, lse = orc.attn_decode(d["q"], d["mc"], d["ms"], d["off"], d["lens"], d["top"], d["win"], d["ws"], d["wl"], 0.1)
    main = _main_decode_indep(d["mc"], d["ms"])
    for b in range(2):
        sel = d["top"][b][d["top"][b] >= 0]
        keys = np.concatenate([main[d["off"][b] + sel], _e4m3_indep(d["win"][b, :d["wl"][b]]) * float(d["ws"][b])])
        assert np.allclose(out[b], keys.mean(0)[None], atol=1e-13)
        assert np.allclose(lse[b], np.log(len(keys)))


def test_attention_needle_dominates(orc):
    d = _setup(23, B=1, win_len=(128,))
    main = _main_decode_indep(d["mc"], d["ms"])
    needle_t = int(d["top"][0, 7])
    key = main[needle_t]
    q = np.tile(key / np.linalg.norm(key) * 40.0, (16, 1))          # logit ~ 40*|key|*sm
    d["q"] = _bf16(q)[None]
    out, _ = orc.attn_decode(d["q"], d["mc"], d["ms"], d["off"], d["lens"], d["top"], d["win"], d["ws"], d["wl"], 1.0)
    assert np.allclose(out[0], key[None], atol=1e-6)


def test_attention_empty_selection(orc):
    d = _setup(24, B=1, win_len=(0,))
    d["top"][:] = -1
    out, lse = orc.attn_decode(d["q"], d["mc"], d["ms"], d["off"], d["lens"], d["top"], d["win"], d["ws"], d["wl"], 0.1)
    assert not out.any() and np.all(np.isneginf(lse))


def test_attention_rejects_out_of_range_index(orc):
    d = _setup(25, B=1)
    d["top"][0, 0] = d["lens"][0]
    with pytest.raises(ValueError):
        orc.attn_decode(d["q"], d["mc"], d["ms"], d["off"], d["lens"], d["top"], d["win"], d["ws"], d["wl"], 0.1)


def test_prefill_attention_equals_decode_with_explicit_window(orc):
    """Causal prefill = decode with the window rows max(0,p-127)..p copied out."""
    rng = np.random.default_rng(26)
    n_raw, ratio, k = 600, 2, 32
    n_ent = n_raw // ratio
    mc = rng.integers(0, 256, (n_ent, 256), dtype=np.uint8)
    ms = rng.integers(124, 128, (n_ent, 16), dtype=np.uint8)
    raw_win = synth.e4m3_rows(1, synth.T_RAWWIN, 0, 0, 0, n_raw)
    q_pos = np.array([0, 1, 2, 60, 127, 128, 599], np.int32)
    T = len(q_pos)
    q = _bf16(rng.standard_normal((T, 16, 512)))
    top = np.full((T, k), -1, np.int32)
    for i, p in enumerate(q_pos):
        vis = (p + 1) // ratio
        m = min(vis, k)
        if m:
            top[i, :m] = np.sort(rng.choice(vis, m, replace=False))
    out, lse = orc.attn_prefill(q, q_pos, mc, ms, 0, n_ent, ratio, top, raw_win, 0.0123, 0.05)
    for i, p in enumerate(q_pos):
        lo = max(0, p - 127)
        win = np.zeros((1, 128, 512), np.uint8)
        win[0, :p - lo + 1] = raw_win[lo:p + 1]
        o2, l2 = orc.attn_decode(q[i:i + 1], mc, ms, np.array([0]), np.array([n_ent]), top[i:i + 1], win,
                                 np.array([0.0123], np.float32), np.array([p - lo + 1]), 0.05)
        assert np.array_equal(out[i], o2[0]) and np.array_equal(lse[i], l2[0])
    bad = top.copy()
    bad[1, 0] = 1                  # entry 1 is not yet complete at raw position 1
    with pytest.raises(ValueError):
        orc.attn_prefill(q, q_pos, mc, ms, 0, n_ent, ratio, bad, raw_win, 0.0123, 0.05)
