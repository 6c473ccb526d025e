"""GPU parity of compression + MXFP4 append: cache bytes bit-exact with the
oracle (ratio 1 and 2, projection and raw indexer rows, ragged appends)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from long_context_decode_csa2_b200 import csa2 as C
from tests._gpu import dev, host

pytestmark = pytest.mark.gpu


def _append(raw, logits, tok_off, seq_row_off, seq_len_in, rows, ratio, w_idx=None, idx_raw=None):
    B = len(seq_len_in)
    mc = torch.zeros((rows, 256), dtype=torch.uint8, device="cuda")
    ms = torch.zeros((rows, 16), dtype=torch.uint8, device="cuda")
    ic = torch.zeros((rows, 64), dtype=torch.uint8, device="cuda")
    isc = torch.zeros((rows, 4), dtype=torch.uint8, device="cuda")
    out_len = torch.zeros(B, dtype=torch.int32, device="cuda")
    ws = C.workspace(C.csa2_compress_append_workspace_bytes(B))
    ntok = np.diff(tok_off)
    max_new = int((ntok // ratio).max()) if B else 0
    keep = [dev(raw), dev(logits) if logits is not None else None, dev(tok_off), dev(seq_row_off), dev(seq_len_in),
            dev(w_idx) if w_idx is not None else None, dev(idx_raw) if idx_raw is not None else None]
    C.csa2_compress_append(C.cache(mc, ms), C.cache(ic, isc), keep[0], keep[1], keep[2], keep[3], keep[4], out_len,
                           ratio, max_new, ws, w_idx=keep[5], idx_raw=keep[6])
    torch.cuda.synchronize()
    return host(mc), host(ms), host(ic), host(isc), host(out_len), C.device_status(ws)


@pytest.mark.parametrize("ratio,proj", [(2, True), (2, False), (1, True), (1, False)])
def test_compress_single_sequence_bit_exact(ratio, proj):
    n = 4100
    raw = synth.normal_bf16(7, synth.T_RAW, 0, 0, n * 512).reshape(n, 512)
    logits = synth.normal_f32(7, synth.T_LOGITS, 0, 0, n) * 3
    w_idx = synth.normal_f32(7, synth.T_WIDX, 0, 0, 512 * 128, log2_div=13).reshape(512, 128) if proj else None
    idx_raw = None if proj else synth.normal_bf16(7, synth.T_IDXRAW, 0, 0, n * 128).reshape(n, 128)
    rows = (n // ratio + 7) // 8 * 8
    got = _append(raw, logits if ratio == 2 else None, np.array([0, n]), np.array([0]), np.array([0], np.int32),
                  rows, ratio, w_idx, idx_raw)
    want = oracle.compress(raw, logits if ratio == 2 else None, ratio, w_idx=w_idx, idx_raw_bf16=idx_raw)
    ne = n // ratio
    assert got[5] == 0 and got[4][0] == ne
    for g, w_ in zip(got[:4], want):
        assert np.array_equal(g[:ne], w_)
    assert not got[0][ne:].any()


def test_compress_ragged_batch_appends_at_offsets():
    rng = np.random.default_rng(3)
    ntok = np.array([7, 0, 1, 64, 2, 33])          # odd tails are not emitted
    tok_off = np.concatenate([[0], np.cumsum(ntok)]).astype(np.int64)
    n = int(tok_off[-1])
    raw = synth.normal_bf16(8, synth.T_RAW, 0, 0, n * 512).reshape(n, 512)
    logits = synth.normal_f32(8, synth.T_LOGITS, 0, 0, n)
    idx_raw = synth.normal_bf16(8, synth.T_IDXRAW, 0, 0, n * 128).reshape(n, 128)
    seq_len_in = np.array([5, 0, 16, 3, 100, 9], np.int32)
    seq_row_off = np.array([0, 64, 128, 192, 256, 512], np.int64)
    rows = 640
    mc, ms, ic, isc, out_len, flags = _append(raw, logits, tok_off, seq_row_off, seq_len_in, rows, 2,
                                              idx_raw=idx_raw)
    assert flags == 0
    assert out_len.tolist() == (seq_len_in + ntok // 2).tolist()
    for b in range(6):
        t0, t1 = tok_off[b], tok_off[b + 1]
        ne = (t1 - t0) // 2
        if ne == 0:
            continue
        want = oracle.compress(raw[t0:t0 + 2 * ne], logits[t0:t0 + 2 * ne], 2, idx_raw_bf16=idx_raw[t0:t0 + 2 * ne])
        r0 = seq_row_off[b] + seq_len_in[b]
        for g, w_ in zip((mc, ms, ic, isc), want):
            assert np.array_equal(g[r0:r0 + ne], w_)


def test_compress_rejects_bad_arguments():
    with pytest.raises(C.Csa2Error):
        _append(np.zeros((4, 512), np.uint16), None, np.array([0, 4]), np.array([0]), np.array([0], np.int32), 8, 2,
                idx_raw=np.zeros((4, 128), np.uint16))   # ratio 2 without logits
