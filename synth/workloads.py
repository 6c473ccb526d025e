"""Workload shapes of the CSA2 decode / prefill configurations and their
seeded inputs (host NumPy for small cases, device generation for large ones).

Only input generation lives here: no quantisation, scoring, selection or
attention.  The five workloads:

* ``tiny_decode_b1_l8192``   - batch 1, L = 8192, one Full layer, pool 256 blocks
* ``stack_decode_b32_l128k`` - batch 32, L = 131072, layers F R R U
* ``long_decode_b64_l1m``    - batch 64, L = 2^20, layers F R R U, log-normal key norms
* ``prefill_r2_262144``      - ratio-2 compression of 262144 raw tokens, then a
                               4096-query causal prefill chunk
* ``ragged_decode_b48_20l``  - batch 48, lengths log-uniform on [4096, 2^20],
                               20 layers (F R U R U) x 4
* ``verify_decode_b64_l1m_m6`` - as ``long_decode_b64_l1m`` with six candidate
                               queries per sequence (speculative verification):
                               query i sees all entries but the last 5 - i
* ``paged_decode_b64_l1m``   - as ``long_decode_b64_l1m`` with the caches read
                               through a page table (4096-row pages, the
                               whole pool's pages shuffled across sequences)
* ``ratio2_decode_b64_l1m``  - as ``long_decode_b64_l1m`` over ratio-2 entries
                               (2^20 entries = 2^21 raw tokens); each step also
                               appends one raw token per sequence, so the
                               caches carry spare rows
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

import synth


@dataclass
class DecodeWorkload:
    name: str
    lengths: np.ndarray
    pattern: str
    P: int = 2048
    k: int = 512
    needles: int = 0
    lognormal: bool = False
    seed: int = 2026
    ratio: int = 1      # 2: entries are compressed pairs, appended during decode
    room: int = 0       # spare cache rows per sequence beyond its length
    queries_per_seq: int = 0  # > 0: a verification step with this many candidate queries per sequence
    page_rows: int = 0  # > 0: the caches are read through a page table of pages this size

    def page_table(self):
        """[B, max_pages] int32: the contiguous layout's pages (sequence b
        owns pages off[b] / page_rows ..) dealt out in a seeded random order,
        so sequence b's logical page i is some other physical page."""
        off, rows = self.row_offsets()
        pr = self.page_rows
        assert rows % pr == 0 and (off % pr == 0).all(), "sequences must start on page boundaries"
        n_pages = rows // pr
        need = (self.lengths + self.room + pr - 1) // pr
        perm = np.random.default_rng(self.seed + 17).permutation(n_pages).astype(np.int32)
        table = np.zeros((self.B, int(need.max())), np.int32)
        o = 0
        for b, n in enumerate(need):
            table[b, :n] = perm[o:o + n]
            o += n
        return table

    @property
    def B(self):
        return len(self.lengths)

    @property
    def max_len(self):
        return int(self.lengths.max())

    def row_offsets(self):
        """Sequence b starts at a multiple of 8; total capacity is a multiple of 8."""
        pad = (self.lengths + self.room + 7) // 8 * 8
        off = np.concatenate([[0], np.cumsum(pad)[:-1]]).astype(np.int64)
        return off, int(pad.sum())

    def verify_queries(self):
        """q_off [B+1], q_vis [Q]: candidate i of sequence b sees all of its
        entries but the last m - 1 - i (the later candidates' own)."""
        m = self.queries_per_seq
        q_off = (np.arange(self.B + 1) * m).astype(np.int32)
        q_vis = (np.repeat(self.lengths, m) - (m - 1 - np.tile(np.arange(m), self.B))).astype(np.int32)
        return q_off, q_vis

    def full_layers(self):
        return [i for i, m in enumerate(self.pattern) if m == "F"]

    def scan_bytes(self):
        return int(self.lengths.sum()) * 68


@dataclass
class PrefillWorkload:
    name: str
    n_raw: int
    T: int
    ratio: int = 2
    P: int = 2048
    k: int = 512
    seed: int = 2026
    use_projection: bool = True

    @property
    def n_entries(self):
        return self.n_raw // self.ratio

    def q_pos(self):
        return np.arange(self.n_raw - self.T, self.n_raw, dtype=np.int32)


def decode_workloads():
    return {
        "tiny_decode_b1_l8192": DecodeWorkload("tiny_decode_b1_l8192", np.array([8192]), "F", P=256, needles=8),
        "stack_decode_b32_l128k": DecodeWorkload("stack_decode_b32_l128k", np.full(32, 131072), "FRRU", needles=64),
        "long_decode_b64_l1m": DecodeWorkload("long_decode_b64_l1m", np.full(64, 1 << 20), "FRRU", needles=256,
                                              lognormal=True),
        "ragged_decode_b48_20l": DecodeWorkload("ragged_decode_b48_20l", synth.log_uniform_lengths(2026, 48),
                                                "FRURU" * 4, needles=32),
        "verify_decode_b64_l1m_m6": DecodeWorkload("verify_decode_b64_l1m_m6", np.full(64, 1 << 20), "FRRU",
                                                   needles=256, lognormal=True, queries_per_seq=6),
        "paged_decode_b64_l1m": DecodeWorkload("paged_decode_b64_l1m", np.full(64, 1 << 20), "FRRU", needles=256,
                                               lognormal=True, page_rows=4096),
        "ratio2_decode_b64_l1m": DecodeWorkload("ratio2_decode_b64_l1m", np.full(64, 1 << 20), "FRRU", needles=256,
                                                lognormal=True, ratio=2, room=1024),
    }


def prefill_workload():
    return PrefillWorkload("prefill_r2_262144", n_raw=262144, T=4096)


# ----------------------------------------------------------------------------
# per-layer query-side inputs (small; always generated on the host)
# ----------------------------------------------------------------------------

def layer_inputs_host(wl: DecodeWorkload, layer: int) -> dict:
    B, seed = wl.B, wl.seed
    q = np.stack([synth.normal_bf16(seed, synth.T_Q, b, layer, 16 * 512).reshape(16, 512) for b in range(B)])
    qc, qs = zip(*[synth.mxfp4_rows(seed, synth.T_QIDX_CODES, synth.T_QIDX_SCALES, b, layer, 0, 4, 128)
                   for b in range(B)])
    w = np.stack([synth.head_weights(seed, b, layer) for b in range(B)])
    win = np.stack([synth.e4m3_rows(seed, synth.T_WIN, b, layer, 0, 128) for b in range(B)])
    ws = np.array([synth.window_scale(seed, b, layer) for b in range(B)], np.float32)
    wlen = np.minimum(128, wl.lengths).astype(np.int32)
    return dict(q=q, q_codes=np.stack(qc), q_scales=np.stack(qs), w=w, win=win, win_scale=ws, win_len=wlen)


def needles_for(wl: DecodeWorkload, layer: int, b: int, q_codes_b: np.ndarray, q_scales_b: np.ndarray):
    """Needle positions and indexer-K rows of sequence b for Full layer `layer`."""
    pos = synth.needle_positions(wl.seed, b, layer, int(wl.lengths[b]), wl.needles)
    nc, ns = synth.needle_rows(q_codes_b[0], q_scales_b[0], len(pos))
    return pos, nc, ns


def full_cache_host(wl: DecodeWorkload, layer: int, q_codes, q_scales) -> dict:
    """Indexer-K and main-KV caches of Full layer `layer` (host; small cases)."""
    off, rows = wl.row_offsets()
    ic = np.zeros((rows, 64), np.uint8)
    isc = np.zeros((rows, 4), np.uint8)
    mc = np.zeros((rows, 256), np.uint8)
    msc = np.zeros((rows, 16), np.uint8)
    for b in range(wl.B):
        n = int((wl.lengths[b] + wl.room + 7) // 8 * 8)
        nk = synth.stream_key(wl.seed, synth.T_ROWNORM, b, 0) if wl.lognormal else None
        c, s = synth.mxfp4_rows(wl.seed, synth.T_IDXK_CODES, synth.T_IDXK_SCALES, b, layer, 0, n, 128, nk)
        ic[off[b]:off[b] + n], isc[off[b]:off[b] + n] = c, s
        c, s = synth.mxfp4_rows(wl.seed, synth.T_MAIN_CODES, synth.T_MAIN_SCALES, b, layer, 0, n, 512, nk)
        mc[off[b]:off[b] + n], msc[off[b]:off[b] + n] = c, s
        if wl.needles:
            pos, nc, ns = needles_for(wl, layer, b, q_codes[b], q_scales[b])
            ic[off[b] + pos], isc[off[b] + pos] = nc, ns
    return dict(idx_codes=ic, idx_scales=isc, main_codes=mc, main_scales=msc, seq_row_off=off, rows=rows)


def full_cache_device(wl: DecodeWorkload, layer: int, q_codes, q_scales, device="cuda") -> dict:
    """Same bytes as full_cache_host, generated on the device."""
    import torch

    import synth.gpu as sg

    off, rows = wl.row_offsets()
    ic = torch.empty((rows, 64), dtype=torch.uint8, device=device)
    isc = torch.empty((rows, 4), dtype=torch.uint8, device=device)
    mc = torch.empty((rows, 256), dtype=torch.uint8, device=device)
    msc = torch.empty((rows, 16), dtype=torch.uint8, device=device)
    for b in range(wl.B):
        n = int((wl.lengths[b] + wl.room + 7) // 8 * 8)
        o = int(off[b])
        sg.mxfp4_rows_into(ic[o:o + n], isc[o:o + n], wl.seed, synth.T_IDXK_CODES, synth.T_IDXK_SCALES, b, layer, 0,
                           n, 128, wl.lognormal)
        sg.mxfp4_rows_into(mc[o:o + n], msc[o:o + n], wl.seed, synth.T_MAIN_CODES, synth.T_MAIN_SCALES, b, layer, 0,
                           n, 512, wl.lognormal)
        if wl.needles:
            pos, nc, ns = needles_for(wl, layer, b, q_codes[b], q_scales[b])
            idx = torch.from_numpy(o + pos).to(device)
            ic[idx] = torch.from_numpy(nc).to(device)
            isc[idx] = torch.from_numpy(ns).to(device)
    return dict(idx_codes=ic, idx_scales=isc, main_codes=mc, main_scales=msc, seq_row_off=off, rows=rows)


# ----------------------------------------------------------------------------
# prefill (ratio-2 compression + causal chunk)
# ----------------------------------------------------------------------------

def prefill_inputs_host(pw: PrefillWorkload, n_raw=None, T=None) -> dict:
    """Host inputs of the prefill workload; n_raw / T override the sizes."""
    n_raw = n_raw or pw.n_raw
    T = T or pw.T
    seed = pw.seed
    raw = synth.normal_bf16(seed, synth.T_RAW, 0, 0, n_raw * 512).reshape(n_raw, 512)
    logits = synth.normal_f32(seed, synth.T_LOGITS, 0, 0, n_raw)
    w_idx = synth.normal_f32(seed, synth.T_WIDX, 0, 0, 512 * 128, log2_div=13).reshape(512, 128)
    idx_raw = synth.normal_bf16(seed, synth.T_IDXRAW, 0, 0, n_raw * 128).reshape(n_raw, 128)
    q = synth.normal_bf16(seed, synth.T_Q, 0, 0, T * 16 * 512).reshape(T, 16, 512)
    qc, qs = synth.mxfp4_rows(seed, synth.T_QIDX_CODES, synth.T_QIDX_SCALES, 0, 0, 0, T * 4, 128)
    w = synth.head_weights(seed, 0, 0, T * 4).reshape(T, 4)
    raw_win = synth.e4m3_rows(seed, synth.T_RAWWIN, 0, 0, 0, n_raw)
    q_pos = np.arange(n_raw - T, n_raw, dtype=np.int32)
    return dict(raw=raw, logits=logits, w_idx=w_idx, idx_raw=idx_raw, q=q, q_codes=qc.reshape(T, 4, 64),
                q_scales=qs.reshape(T, 4, 4), w=w, raw_win=raw_win, win_scale=synth.window_scale(seed, 0, 0),
                q_pos=q_pos)
