"""Seeded synthetic inputs for the CSA2 decode / prefill path.

This module is the ONLY code shared by the CUDA library's tests/bench and the
CPU oracle.  It holds none of the method's arithmetic: it never quantises,
scores, selects or attends.  Everything is produced from a counter-based
SplitMix64 stream with integer operations only (plus exact power-of-two
scalings and the round-to-nearest-even bf16 narrowing), so the NumPy code here
and the CUDA generator kernel in ``synth_kernels.cu`` produce bit-identical
bytes.

Inputs are drawn directly in the storage domain:

* MXFP4 rows (indexer K, main KV, indexer q): each E2M1 code has a random sign
  and a magnitude index drawn from a fixed categorical table that mimics
  ``N(0,1)`` values after OCP MXFP4 block scaling (most blocks scaled by
  2^-1); each E8M0 block scale is 125/126/127.  A per-row integer exponent
  shift (-2..+2) mimics log-normal key norms (sigma = 0.5 in natural log).
* needles: an indexer-K row replaced by the layer's head-0 indexer-q codes with
  every block scale raised by 2, which makes it score far above the bulk.
* FP8 E4M3 window rows: sign, 3-bit mantissa and an exponent drawn from a
  table that mimics ``|N(0, 100^2)|``; NaN codes are never produced.
* bf16 / fp32 reals (queries, raw tokens, compression logits, projection
  weights): Irwin-Hall sums of twelve uniform bytes, an exact dyadic
  approximation of ``N(0,1)``.
"""
from __future__ import annotations

import math
import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_FNV = np.uint64(0x100000001B3)

# tensor ids of the seeded streams
T_IDXK_CODES, T_IDXK_SCALES, T_MAIN_CODES, T_MAIN_SCALES = 1, 2, 3, 4
T_ROWNORM, T_NEEDLE, T_QIDX_CODES, T_QIDX_SCALES = 5, 6, 7, 8
T_W, T_Q, T_WIN, T_WIN_SCALE = 9, 10, 11, 12
T_RAW, T_LOGITS, T_WIDX, T_IDXRAW, T_LEN, T_RAWWIN = 13, 14, 15, 16, 17, 18

# cumulative thresholds (out of 128) for the E2M1 magnitude index 0..7
E2M1_CUM = np.array([13, 38, 60, 79, 101, 118, 127, 128], dtype=np.uint32)
# E8M0 byte from one uniform byte: <64 -> 125, <243 -> 126, else 127
SCALE_CUT = (64, 243)
# per-row exponent shift from one uniform byte: -2,-1,0,+1,+2
ROWNORM_CUM = np.array([5, 63, 193, 251, 256], dtype=np.uint32)
# E4M3 exponent category (field = 9 + cat) out of 256
E4M3_CUM = np.array([16, 40, 64, 123, 205, 253, 256], dtype=np.uint32)


def mix64(z):
    """SplitMix64 finaliser (Steele, Lea, Flood 2014), elementwise on uint64."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, tensor: int, seq: int = 0, layer: int = 0) -> np.uint64:
    """Key of one counter stream; every (seed, tensor, sequence, layer) differs."""
    with np.errstate(over="ignore"):
        z = np.uint64(seed) * _FNV
        z ^= np.uint64(tensor) << np.uint64(48)
        z ^= np.uint64(layer) << np.uint64(32)
        z ^= np.uint64(seq)
    return mix64(z)


def hashes(key, start: int, count: int) -> np.ndarray:
    """Counter-mode draws: element i = mix64(key + (start+i+1) * golden)."""
    i = np.arange(start, start + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return mix64(np.uint64(key) + (i + np.uint64(1)) * GOLDEN)


def _bytes_of(h: np.ndarray) -> np.ndarray:
    """Little-endian bytes of uint64 draws, shape (..., 8)."""
    return h.astype("<u8").view(np.uint8).reshape(h.shape + (8,))


# ----------------------------------------------------------------------------
# MXFP4 rows in the storage domain
# ----------------------------------------------------------------------------

def mxfp4_rows(seed, t_codes, t_scales, seq, layer, r0, nrows, n, rownorm_key=None):
    """Rows r0..r0+nrows-1 of one (sequence, layer) MXFP4 tensor of width n.

    Returns (codes uint8 [nrows, n/2], scales uint8 [nrows, n/32]).
    Code for element e of row r uses byte (e % 8) of draw r*(n/8) + e//8.
    """
    assert n % 32 == 0
    kc = stream_key(seed, t_codes, seq, layer)
    h = hashes(kc, r0 * (n // 8), nrows * (n // 8)).reshape(nrows, n // 8)
    b = _bytes_of(h).reshape(nrows, n).astype(np.uint32)       # one byte per element
    mag = np.searchsorted(E2M1_CUM, b & 127, side="right").astype(np.uint8)
    code = mag | ((b >> 7).astype(np.uint8) << 3)
    codes = (code[:, 0::2] | (code[:, 1::2] << 4)).astype(np.uint8)

    ks = stream_key(seed, t_scales, seq, layer)
    nh = (n // 32 + 7) // 8
    hs = hashes(ks, r0 * nh, nrows * nh).reshape(nrows, nh)
    sb = _bytes_of(hs).reshape(nrows, nh * 8)[:, : n // 32].astype(np.int32)
    scales = np.where(sb < SCALE_CUT[0], 125, np.where(sb < SCALE_CUT[1], 126, 127))
    if rownorm_key is not None:
        scales = scales + rownorm_shift(rownorm_key, r0, nrows)[:, None]
    return codes, scales.astype(np.uint8)


def rownorm_shift(key, r0, nrows) -> np.ndarray:
    """Per-row exponent shift in -2..+2 (log-normal key norms)."""
    u = (hashes(key, r0, nrows) & np.uint64(255)).astype(np.uint32)
    return np.searchsorted(ROWNORM_CUM, u, side="right").astype(np.int32) - 2


def needle_positions(seed, seq, layer, L, n_needles) -> np.ndarray:
    """n_needles distinct positions, one per equal stratum of [0, L-128)."""
    span = L - 128 if L > 256 else L
    n = min(n_needles, span)
    if n <= 0:
        return np.zeros(0, dtype=np.int64)
    key = stream_key(seed, T_NEEDLE, seq, layer)
    h = hashes(key, 0, n)
    lo = (np.arange(n, dtype=np.int64) * span) // n
    hi = (np.arange(1, n + 1, dtype=np.int64) * span) // n
    return lo + (h % (hi - lo).astype(np.uint64)).astype(np.int64)


def needle_rows(qidx_codes_h0, qidx_scales_h0, count):
    """Needle indexer-K rows: head-0 query codes, every block scale + 2."""
    c = np.broadcast_to(qidx_codes_h0, (count,) + qidx_codes_h0.shape).copy()
    s = np.minimum(qidx_scales_h0.astype(np.int32) + 2, 254).astype(np.uint8)
    return c, np.broadcast_to(s, (count,) + s.shape).copy()


# ----------------------------------------------------------------------------
# FP8 E4M3 window rows
# ----------------------------------------------------------------------------

def e4m3_rows(seed, tensor, seq, layer, r0, nrows, n=512) -> np.ndarray:
    """uint8 [nrows, n] E4M3 codes; 4 values per draw (16 bits each)."""
    key = stream_key(seed, tensor, seq, layer)
    h = hashes(key, r0 * (n // 4), nrows * (n // 4)).reshape(nrows, n // 4)
    b = _bytes_of(h).reshape(nrows, n // 4, 4, 2).astype(np.uint32)
    lo, hi = b[..., 0], b[..., 1]
    cat = np.searchsorted(E4M3_CUM, hi, side="right").astype(np.uint32)
    field = 9 + cat
    mant = lo & 7
    mant = np.where((field == 15) & (mant == 7), 6, mant)
    code = ((lo >> 7) << 7) | (field << 3) | mant
    return code.reshape(nrows, n).astype(np.uint8)


def window_scale(seed, seq, layer) -> np.float32:
    """Per-(sequence, layer) FP8 scale in [400, 528) * 2^-15."""
    h = hashes(stream_key(seed, T_WIN_SCALE, seq, layer), 0, 1)[0]
    return np.float32((400 + int(h & np.uint64(127))) / 32768.0)


# ----------------------------------------------------------------------------
# real-valued inputs
# ----------------------------------------------------------------------------

def irwin_hall_int(key, start, count) -> np.ndarray:
    """Sum of twelve uniform bytes minus 1530, as int32 (two draws per value)."""
    h = hashes(key, 2 * start, 2 * count).reshape(count, 2)
    b = _bytes_of(h).reshape(count, 16)[:, :12].astype(np.int32)
    return b.sum(axis=1) - 1530


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16, returned as uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_bf16(seed, tensor, seq, layer, count) -> np.ndarray:
    """~N(0,1) values as bf16 bit patterns (uint16)."""
    v = irwin_hall_int(stream_key(seed, tensor, seq, layer), 0, count).astype(np.float32) / np.float32(256)
    return f32_to_bf16_bits(v)


def normal_f32(seed, tensor, seq, layer, count, log2_div=8) -> np.ndarray:
    """~N(0, 2^(16-2*log2_div)) fp32 values (exact dyadic)."""
    v = irwin_hall_int(stream_key(seed, tensor, seq, layer), 0, count).astype(np.float32)
    return v / np.float32(2.0 ** log2_div)


def head_weights(seed, seq, layer, n=4) -> np.ndarray:
    """Indexer head weights U(0.5, 1.5) on a 2^-23 grid (exact fp32)."""
    h = hashes(stream_key(seed, T_W, seq, layer), 0, n)
    return (np.float32(0.5) + (h >> np.uint64(41)).astype(np.float32) * np.float32(2.0 ** -23)).astype(np.float32)


def log_uniform_lengths(seed, B, lo=4096, hi=1 << 20) -> np.ndarray:
    """Ragged lengths, log-uniform on [lo, hi], rounded down to a multiple of 8 is NOT applied."""
    h = hashes(stream_key(seed, T_LEN, 0, 0), 0, B)
    u = (h >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
    L = np.floor(np.exp(math.log(lo) + u * (math.log(hi) - math.log(lo)))).astype(np.int64)
    return np.clip(L, lo, hi)
