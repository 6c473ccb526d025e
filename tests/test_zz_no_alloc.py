"""csa2_sparse_attn_decode_noalloc: the attention call for callers that may
not allocate device memory while running (its scratch is a fixed array inside
the library).  Its results must match the regular workspace call on two calls
in a row.  This file runs last so that a failure here stops nothing else."""
import math

import numpy as np
import pytest
import torch

import synth
from long_context_decode_csa2_b200 import csa2 as C
from tests._gpu import ATTN_MAX_ABS, ATTN_REL_L2, dev, host

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
    d = dict(q=dev(q), off=dev(off), lens=dev(np.asarray(lengths, np.int32)), top=dev(top), win=dev(win),
             ws=dev(ws), wl=dev(wl))
    d["cache"] = C.cache(dev(mc), dev(ms))
    return d


def _close(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    assert np.abs(a - b).max() <= ATTN_MAX_ABS
    assert np.linalg.norm(a - b) <= ATTN_REL_L2 * np.linalg.norm(b)


def test_noalloc_matches_workspace_call_twice():
    sm = 1 / math.sqrt(512)
    for seed, lengths in ((41, [70000, 512, 9000]), (42, [1000] * 64)):
        d = _inputs(seed, lengths, 512)
        B = len(lengths)
        ref = torch.zeros((B, 16, 512), dtype=torch.float32, device="cuda")
        ref_lse = torch.zeros((B, 16), dtype=torch.float32, device="cuda")
        ws = C.workspace(C.csa2_sparse_attn_decode_workspace_bytes(B, 512))
        C.csa2_sparse_attn_decode(d["q"], d["cache"], d["off"], d["lens"], d["top"], d["win"], d["ws"], d["wl"], sm,
                                  ref, ws, lse=ref_lse)
        for _ in range(2):
            out = torch.full((B, 16, 512), float("nan"), dtype=torch.float32, device="cuda")
            lse = torch.full((B, 16), float("nan"), dtype=torch.float32, device="cuda")
            flags = torch.full((1,), 7, dtype=torch.int32, device="cuda")
            C.csa2_sparse_attn_decode_noalloc(d["q"], d["cache"], d["off"], d["lens"], d["top"], d["win"], d["ws"],
                                              d["wl"], sm, out, lse=lse, flags_out=flags)
            torch.cuda.synchronize()
            assert int(flags.item()) == 0
            _close(host(out), host(ref))
            _close(host(lse), host(ref_lse))


def test_noalloc_rejects_problems_beyond_its_scratch():
    d = _inputs(43, [100] * 65, 64)
    out = torch.zeros((65, 16, 512), dtype=torch.float32, device="cuda")
    with pytest.raises(C.Csa2Error) as e:
        C.csa2_sparse_attn_decode_noalloc(d["q"], d["cache"], d["off"], d["lens"], d["top"], d["win"], d["ws"],
                                          d["wl"], 0.1, out)
    assert e.value.status == -2
    d = _inputs(44, [2000], 600)
    with pytest.raises(C.Csa2Error) as e:
        C.csa2_sparse_attn_decode_noalloc(d["q"], d["cache"], d["off"], d["lens"], d["top"], d["win"], d["ws"],
                                          d["wl"], 0.1, out[:1])
    assert e.value.status == -2
