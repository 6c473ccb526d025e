"""csa2_sparse_attn_decode_noalloc: the attention call for callers that may
not allocate device memory while running (a plugin inside a runtime that owns
every allocation, a serving loop held to a fixed footprint).  Its scratch is a
fixed array inside the library.  After the one set-up call per device (B = 0),
two calls in a row must allocate nothing (the device's free memory does not
move) and give exactly the regular workspace call's bits, which themselves
match the oracle within the attention tolerance.  This file runs last so that
a failure here stops nothing else."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from long_context_decode_csa2_b200 import csa2 as C
from tests._gpu import check_attention, dev, host

pytestmark = pytest.mark.gpu


def _inputs(seed, lengths, k):
    rng = np.random.default_rng(seed)
    B = len(lengths)
    pad = (np.asarray(lengths) + 7) // 8 * 8
    off = np.concatenate([[0], np.cumsum(pad)[:-1]]).astype(np.int64)
    mc, ms = synth.mxfp4_rows(seed, synth.T_MAIN_CODES, synth.T_MAIN_SCALES, 0, 0, 0, int(pad.sum()), 512)
    top = np.full((B, k), -1, np.int32)
    for b in range(B):
        m = min(k, lengths[b])
        top[b, :m] = np.sort(rng.choice(lengths[b], m, replace=False))
    q = synth.normal_bf16(seed, synth.T_Q, 0, 0, B * 16 * 512).reshape(B, 16, 512)
    win = synth.e4m3_rows(seed, synth.T_WIN, 0, 0, 0, B * 128).reshape(B, 128, 512)
    ws = np.array([synth.window_scale(seed, b, 0) for b in range(B)], np.float32)
    wl = np.minimum(128, np.asarray(lengths)).astype(np.int32)
    h = dict(q=q, mc=mc, ms=ms, off=off, lens=np.asarray(lengths, np.int32), top=top, win=win, ws=ws, wl=wl)
    d = dict(q=dev(q), off=dev(off), lens=dev(h["lens"]), top=dev(top), win=dev(win), ws=dev(ws), wl=dev(wl))
    d["cache"] = C.cache(dev(mc), dev(ms))
    return d, h


def test_noalloc_matches_workspace_call_twice_without_allocating():
    sm = 1 / math.sqrt(512)
    C.noalloc_setup()  # the one call per device that may allocate (module load)
    torch.cuda.synchronize()
    for seed, lengths in ((41, [70000, 512, 9000]), (42, [1000] * 64)):
        d, h = _inputs(seed, lengths, 512)
        B = len(lengths)
        ref = torch.zeros((B, 16, 512), dtype=torch.float32, device="cuda")
        ref_lse = torch.zeros((B, 16), dtype=torch.float32, device="cuda")
        ws = C.workspace(C.csa2_sparse_attn_decode_workspace_bytes(B, 512))
        C.csa2_sparse_attn_decode(d["q"], d["cache"], d["off"], d["lens"], d["top"], d["win"], d["ws"], d["wl"], sm,
                                  ref, ws, lse=ref_lse)
        outs = [torch.full((B, 16, 512), float("nan"), dtype=torch.float32, device="cuda") for _ in range(2)]
        lses = [torch.full((B, 16), float("nan"), dtype=torch.float32, device="cuda") for _ in range(2)]
        flags = [torch.full((1,), 7, dtype=torch.int32, device="cuda") for _ in range(2)]
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        for i in range(2):
            C.csa2_sparse_attn_decode_noalloc(d["q"], d["cache"], d["off"], d["lens"], d["top"], d["win"], d["ws"],
                                              d["wl"], sm, outs[i], lse=lses[i], flags_out=flags[i])
        torch.cuda.synchronize()
        free1 = torch.cuda.mem_get_info()[0]
        assert free1 == free0, f"device free memory moved by {free0 - free1} bytes across the two calls"
        for i in range(2):
            assert int(flags[i].item()) == 0
            # same kernel, same split, same combine order: the same bits
            assert torch.equal(outs[i], ref), f"call {i}: out differs from the workspace call"
            assert torch.equal(lses[i], ref_lse), f"call {i}: lse differs from the workspace call"
        if seed == 41:  # and the workspace call (hence both) against the oracle
            o, l = oracle.attn_decode(h["q"], h["mc"], h["ms"], h["off"], h["lens"], h["top"], h["win"], h["ws"],
                                      h["wl"], sm)
            check_attention(host(outs[1]), o, host(lses[1]), l, what="noalloc vs oracle")


def test_noalloc_rejects_problems_beyond_its_scratch():
    d, _ = _inputs(43, [100] * 65, 64)
    out = torch.zeros((65, 16, 512), dtype=torch.float32, device="cuda")
    with pytest.raises(C.Csa2Error) as e:
        C.csa2_sparse_attn_decode_noalloc(d["q"], d["cache"], d["off"], d["lens"], d["top"], d["win"], d["ws"],
                                          d["wl"], 0.1, out)
    assert e.value.status == -2
    d, _ = _inputs(44, [2000], 600)
    with pytest.raises(C.Csa2Error) as e:
        C.csa2_sparse_attn_decode_noalloc(d["q"], d["cache"], d["off"], d["lens"], d["top"], d["win"], d["ws"],
                                          d["wl"], 0.1, out[:1])
    assert e.value.status == -2
