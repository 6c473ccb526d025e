"""Pins of the oracle's number formats: E2M1, E8M0, MXFP4 encode/decode, E4M3,
and its own exp (test-only; no GPU)."""
import math
import os

import numpy as np
import pytest
import torch

from tests._exact import brute_block as _brute_block, e2m1_from_bits, e4m3_from_bits, pow2

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load_golden_table(name):
    vals = []
    for line in open(os.path.join(GOLDEN, name)):
        line = line.split("#", 1)[0].strip()
        if line:
            code, val = line.split()
            vals.append((int(code, 0), float(val)))
    return vals


def test_e2m1_table_matches_ocp_golden(orc):
    table = _load_golden_table("e2m1_values.txt")
    assert len(table) == 16
    for code, val in table:
        assert orc.e2m1_value(code) == val
        assert float(e2m1_from_bits(code)) == val


def test_e8m0_scales(orc):
    for byte in range(255):
        assert orc.e8m0_value(byte) == math.ldexp(1.0, byte - 127)


def test_e4m3_matches_torch_and_bitfields(orc):
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for b in range(256):
        v = orc.e4m3_value(b)
        exact = e4m3_from_bits(b)
        if exact is None:
            assert math.isnan(v) and math.isnan(ref[b])
        else:
            assert v == float(exact) == ref[b], hex(b)
    assert orc.e4m3_value(0x7E) == 448.0 and orc.e4m3_value(0x01) == 2.0 ** -9


def _unpack(codes_row):
    out = []
    for b in codes_row:
        out += [int(b) & 15, int(b) >> 4]
    return out


def test_mxfp4_encode_matches_bruteforce_random(orc):
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal((64, 32)),
        rng.standard_normal((32, 32)) * np.exp(rng.uniform(-20, 20, (32, 1))),
        np.round(rng.standard_normal((32, 32)) * 4) / 4,          # many exact ties
    ]).astype(np.float32)
    codes, scales = orc.mxfp4_encode(x)
    for r in range(x.shape[0]):
        bc, bs = _brute_block(x[r])
        assert int(scales[r, 0]) == bs, r
        assert _unpack(codes[r]) == bc, r


def test_mxfp4_ties_to_even_and_sign(orc):
    # anchor 6.0 fixes X = 0 (scale byte 127), so values are taken as is
    vals = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, -0.2, 0.0, -0.0, 6.0]
    expect = [0, 2, 2, 4, 4, 6, 6, 7, 8, 0, 8, 7]
    x = np.zeros((1, 32), np.float32)
    x[0, :len(vals)] = vals
    x[0, 31] = 6.0
    codes, scales = orc.mxfp4_encode(x)
    assert scales[0, 0] == 127
    assert _unpack(codes[0])[:len(vals)] == expect


def test_mxfp4_all_zero_block(orc):
    codes, scales = orc.mxfp4_encode(np.zeros((1, 32), np.float32))
    assert scales[0, 0] == 0 and not codes.any()


def test_mxfp4_roundtrip_all_codes_and_scales(orc):
    # every (code, scale): a block holding decode(code, scale) and an anchor 6*2^X
    xs, want = [], []
    for s in range(1, 255):
        for c in range(16):
            v = float(e2m1_from_bits(c) * pow2(s - 127))
            anchor = float(6 * pow2(s - 127))
            with np.errstate(over="ignore"):                # scales past fp32's range are skipped
                a32, v32 = np.float32(anchor), np.float32(v)
            if not (np.isfinite(a32) and a32 == anchor and v32 == v):
                continue
            blk = np.full(32, 0.0, np.float32)
            blk[0], blk[1] = v, anchor
            xs.append(blk)
            want.append((c, s))
    x = np.stack(xs)
    codes, scales = orc.mxfp4_encode(x)
    dec = orc.mxfp4_decode(codes, scales)
    for r, (c, s) in enumerate(want):
        assert scales[r, 0] == s
        got = int(codes[r, 0]) & 15
        # +0/-0 both decode to zero; all other codes are recovered exactly
        assert got == c or (c & 7) == 0 and (got & 7) == 0
        assert dec[r, 0] == x[r, 0] and dec[r, 1] == x[r, 1]


def test_mxfp4_error_bound(orc):
    """|decode(encode(x)) - x| <= half an E2M1 step at the block scale (or clip)."""
    rng = np.random.default_rng(2)
    x = rng.standard_normal((256, 128)).astype(np.float32)
    codes, scales = orc.mxfp4_encode(x)
    dec = orc.mxfp4_decode(codes, scales)
    for r in range(x.shape[0]):
        for b in range(4):
            X = int(scales[r, b]) - 127
            blk = x[r, 32 * b:32 * b + 32].astype(np.float64) * 2.0 ** (-X)
            got = dec[r, 32 * b:32 * b + 32] * 2.0 ** (-X)
            half_step = np.where(np.abs(blk) < 2, 0.25, np.where(np.abs(blk) < 4, 0.5, 1.0))
            clipped = np.abs(blk) > 6
            assert np.all((np.abs(got - blk) <= half_step) | clipped)
            assert np.all(np.abs(got[clipped]) == 6.0)


def test_own_exp_close_to_libm(orc):
    """Within 1 ulp of the C library's exp over the pair-weight range (x <= 0)
    and the whole finite range."""
    rng = np.random.default_rng(3)
    xs = np.concatenate([rng.uniform(-60, 0, 20000), -np.logspace(-12, 2.5, 2000), rng.uniform(-745, 709, 20000),
                         [0.0, -1e-300, -700.0]])
    for x in xs:
        got, ref = orc.own_exp(x), math.exp(x)
        assert abs(got - ref) <= math.ulp(ref), (x, got, ref)
    assert orc.own_exp(0.0) == 1.0
    assert orc.own_exp(-800.0) == 0.0
