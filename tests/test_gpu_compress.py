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


def _append(raw, logits, tok_off, seq_row_off, seq_len_in, rows, ratio, w_idx=None, idx_raw=None, max_new=None):
    B = len(seq_len_in)
    mc = torch.zeros((rows, 256), dtype=torch.uint8, device="cuda")
    ms = torch.zeros((rows, 16), dtype=torch.uint8, device="cuda")
    ic = torch.zeros((rows, 64), dtype=torch.uint8, device="cuda")
    isc = torch.zeros((rows, 4), dtype=torch.uint8, device="cuda")
    out_len = torch.zeros(B, dtype=torch.int32, device="cuda")
    ws = C.workspace(C.csa2_compress_append_workspace_bytes(B))
    ntok = np.diff(tok_off)
    if max_new is None:
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


@pytest.mark.parametrize("max_new", [2, 40])
def test_compress_beyond_max_new_is_flagged(max_new):
    """More entries than the host bound: the first max_new are written (bit-exact;
    at most two per CTA take the one-chain projection, more the shared one), the
    rest are not, and CSA2_DEV_LENGTH is raised."""
    n = 100
    raw = synth.normal_bf16(9, synth.T_RAW, 0, 0, n * 512).reshape(n, 512)
    w_idx = synth.normal_f32(9, synth.T_WIDX, 0, 0, 512 * 128, log2_div=13).reshape(512, 128)
    got = _append(raw, None, np.array([0, n]), np.array([0]), np.array([0], np.int32), 104, 1, w_idx,
                  max_new=max_new)
    want = oracle.compress(raw, None, 1, w_idx=w_idx)
    assert got[5] == 8                             # CSA2_DEV_LENGTH
    assert got[4][0] == n                          # the length the call was asked for
    for g, w_ in zip(got[:4], want):
        assert np.array_equal(g[:max_new], w_[:max_new])
        assert not g[max_new:].any()


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


# --- streaming appends (ratio-2 decode: a pending half-pair per sequence) ---

class _StreamState:
    """Device caches, lengths and pending buffers of B sequences, mirrored by
    the oracle's state on the host."""

    def __init__(self, B, cap, proj, seed):
        self.B, self.cap, self.proj = B, cap, proj
        rows = B * cap
        self.mc = torch.zeros((rows, 256), dtype=torch.uint8, device="cuda")
        self.ms = torch.zeros((rows, 16), dtype=torch.uint8, device="cuda")
        self.ic = torch.zeros((rows, 64), dtype=torch.uint8, device="cuda")
        self.isc = torch.zeros((rows, 4), dtype=torch.uint8, device="cuda")
        self.seq_row_off = dev(np.arange(B, dtype=np.int64) * cap)
        self.seq_len = torch.zeros(B, dtype=torch.int32, device="cuda")
        self.pend_n = torch.zeros(B, dtype=torch.int32, device="cuda")
        self.pend_raw = torch.zeros((B, 512), dtype=torch.bfloat16, device="cuda")
        self.pend_logit = torch.zeros(B, dtype=torch.float32, device="cuda")
        self.pend_idx = None if proj else torch.zeros((B, 128), dtype=torch.bfloat16, device="cuda")
        self.w_idx = (synth.normal_f32(seed, synth.T_WIDX, 0, 0, 512 * 128, log2_div=13).reshape(512, 128)
                      if proj else None)
        self.w_idx_d = dev(self.w_idx) if proj else None
        self.ws = C.workspace(C.csa2_compress_stream_workspace_bytes(B))
        # oracle side
        self.o_pend = [None] * B
        self.o_len = np.zeros(B, np.int64)
        self.o_cache = [np.zeros((rows, 256), np.uint8), np.zeros((rows, 16), np.uint8),
                        np.zeros((rows, 64), np.uint8), np.zeros((rows, 4), np.uint8)]

    def append(self, raw, logits, idx_raw, ntok, out_mode="inplace"):
        tok_off = np.concatenate([[0], np.cumsum(ntok)]).astype(np.int64)
        pend_now = host(self.pend_n)
        max_new = int(((ntok + pend_now) // 2).max())
        keep = [dev(raw), dev(logits), dev(tok_off), dev(idx_raw) if idx_raw is not None else None]
        out = {"inplace": self.seq_len, "none": None}[out_mode]
        C.csa2_compress_stream(C.cache(self.mc, self.ms), C.cache(self.ic, self.isc), keep[0], keep[1], keep[2],
                               self.seq_row_off, self.seq_len, out, self.pend_n, self.pend_raw, self.pend_logit,
                               max_new, self.ws, w_idx=self.w_idx_d, idx_raw=keep[3], pend_idx=self.pend_idx)
        ent, self.o_pend = oracle.compress_stream(self.o_pend, raw, logits, tok_off, w_idx=self.w_idx,
                                                  idx_raw_bf16=idx_raw)
        for b in range(self.B):
            ne = ent[b][0].shape[0]
            r0 = b * self.cap + self.o_len[b]
            for dst, src in zip(self.o_cache, ent[b]):
                dst[r0:r0 + ne] = src
            if out_mode == "inplace":
                self.o_len[b] += ne
        torch.cuda.synchronize()

    def check(self):
        assert C.device_status(self.ws) == 0
        for g, w_ in zip((self.mc, self.ms, self.ic, self.isc), self.o_cache):
            assert np.array_equal(host(g), w_)
        assert host(self.seq_len).tolist() == self.o_len.tolist()
        pn = host(self.pend_n)
        pr, pl = host(self.pend_raw), host(self.pend_logit)
        pi = host(self.pend_idx) if self.pend_idx is not None else None
        for b in range(self.B):
            p = self.o_pend[b]
            assert pn[b] == (0 if p is None else 1)
            if p is not None:
                assert np.array_equal(pr[b], p["raw"]) and np.float32(p["logit"]) == pl[b]
                if pi is not None:
                    assert np.array_equal(pi[b], p["idx"])


def _tokens(seed, n):
    raw = synth.normal_bf16(seed, synth.T_RAW, 0, 0, n * 512).reshape(n, 512)
    logits = synth.normal_f32(seed, synth.T_LOGITS, 0, 0, n) * 2
    idx_raw = synth.normal_bf16(seed, synth.T_IDXRAW, 0, 0, n * 128).reshape(n, 128)
    return raw, logits, idx_raw


@pytest.mark.parametrize("proj", [True, False])
def test_compress_stream_ragged_calls_bit_exact(proj):
    """Ragged token counts per call (0 .. 70, so up to three CTAs per
    sequence), pending tokens carried between calls, lengths in place."""
    B, cap = 6, 256
    st = _StreamState(B, cap, proj, seed=40)
    rng = np.random.default_rng(41)
    for call in range(5):
        ntok = rng.integers(0, 8, B)
        ntok[call % B] = 70 if call < 3 else 33
        n = int(ntok.sum())
        raw, logits, idx_raw = _tokens(100 + call, n)
        st.append(raw, logits, None if proj else idx_raw, ntok)
        st.check()


@pytest.mark.parametrize("proj", [True, False])
def test_compress_stream_one_token_per_step(proj):
    """The decode pattern: one token per sequence per call; an entry every
    second call.  Equal to the one-shot append of all tokens."""
    B, cap, steps = 64, 16, 9
    st = _StreamState(B, cap, proj, seed=42)
    ntok = np.ones(B, np.int64)
    all_raw, all_z, all_i = [], [], []
    for t in range(steps):
        raw, logits, idx_raw = _tokens(200 + t, B)
        all_raw.append(raw), all_z.append(logits), all_i.append(idx_raw)
        st.append(raw, logits, None if proj else idx_raw, ntok)
    st.check()
    for b in range(0, B, 7):
        x = np.stack([r[b] for r in all_raw])
        z = np.array([zz[b] for zz in all_z], np.float32)
        xi = np.stack([r[b] for r in all_i])
        m = steps // 2 * 2
        want = oracle.compress(x[:m], z[:m], 2, w_idx=st.w_idx, idx_raw_bf16=None if proj else xi[:m])
        for g, w_ in zip((st.mc, st.ms, st.ic, st.isc), want):
            assert np.array_equal(host(g)[b * cap:b * cap + m // 2], w_)


def test_compress_stream_lengths_not_written():
    """seq_len_out = NULL leaves the lengths alone (several caches appended
    from one length array); the pending state still advances."""
    B, cap = 3, 64
    st = _StreamState(B, cap, False, seed=43)
    ntok = np.array([3, 0, 4])
    raw, logits, idx_raw = _tokens(300, int(ntok.sum()))
    st.append(raw, logits, idx_raw, ntok, out_mode="none")
    st.check()
