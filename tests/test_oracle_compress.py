"""Pins of the oracle's pair compression, projection, MXFP4 append, and the
causal prefill indexer's visibility rule (no GPU)."""
from fractions import Fraction

import numpy as np

import synth
from tests._exact import brute_block, rn32


def _unpack(row):
    out = []
    for b in row:
        out += [int(b) & 15, int(b) >> 4]
    return out


def _raw(n, seed=30, width=512):
    bits = synth.normal_bf16(seed, synth.T_RAW, 0, 0, n * width).reshape(n, width)
    return bits, synth.bf16_bits_to_f32(bits).astype(np.float64)


def test_equal_logits_give_plain_average(orc):
    bits, x = _raw(64)
    z = np.zeros(64, np.float32)
    _, _, _, _, c, _ = orc.compress(bits, z, 2, idx_raw_bf16=bits[:, :128], want_rows=True)
    for j in range(32):
        for i in range(0, 512, 37):
            want = rn32(Fraction(x[2 * j, i]) / 2 + Fraction(x[2 * j + 1, i]) / 2)
            assert c[j, i] == want


def test_dominant_logit_returns_first_row(orc):
    bits, x = _raw(16)
    z = np.zeros(16, np.float32)
    z[0::2] = 50.0
    _, _, _, _, c, _ = orc.compress(bits, z, 2, idx_raw_bf16=bits[:, :128], want_rows=True)
    x0 = x[0::2].astype(np.float32)
    big = np.abs(x0) > 1e-6
    assert np.array_equal(c[big], x0[big])


def test_pair_weights_match_softmax(orc):
    bits, x = _raw(512)
    z = synth.normal_f32(3, synth.T_LOGITS, 0, 0, 512) * 4
    _, _, _, _, c, _ = orc.compress(bits, z, 2, idx_raw_bf16=bits[:, :128], want_rows=True)
    zz = z.astype(np.float64).reshape(-1, 2)
    e = np.exp(zz - zz.max(1, keepdims=True))
    w = e / e.sum(1, keepdims=True)
    ref = w[:, :1] * x[0::2] + w[:, 1:] * x[1::2]
    assert np.allclose(c, ref, rtol=2 ** -22, atol=1e-30)


def test_ratio1_is_identity_then_ocp_encode(orc):
    bits, x = _raw(8)
    mc, ms, ic, isc, c, r = orc.compress(bits, None, 1, idx_raw_bf16=bits[:, :128], want_rows=True)
    assert np.array_equal(c, x.astype(np.float32))
    assert np.array_equal(r, x[:, :128].astype(np.float32))
    for j in range(8):
        for b in range(16):
            codes, scale = brute_block(c[j, 32 * b:32 * b + 32])
            assert ms[j, b] == scale and _unpack(mc[j, 16 * b:16 * b + 16]) == codes


def test_projection_matches_float64_matmul(orc):
    bits, x = _raw(64)
    z = synth.normal_f32(4, synth.T_LOGITS, 0, 0, 64)
    W = synth.normal_f32(5, synth.T_WIDX, 0, 0, 512 * 128, log2_div=13).reshape(512, 128)
    mc, ms, ic, isc, c, r = orc.compress(bits, z, 2, w_idx=W, want_rows=True)
    ref = c.astype(np.float64) @ W.astype(np.float64)
    assert np.allclose(r, ref, rtol=3e-7, atol=1e-9)
    for j in range(32):
        for b in range(4):
            codes, scale = brute_block(r[j, 32 * b:32 * b + 32])
            assert isc[j, b] == scale and _unpack(ic[j, 16 * b:16 * b + 16]) == codes


def test_idx_raw_merged_like_main(orc):
    bits, x = _raw(32)
    z = synth.normal_f32(6, synth.T_LOGITS, 0, 0, 32)
    idx_bits = synth.normal_bf16(9, synth.T_IDXRAW, 0, 0, 32 * 128).reshape(32, 128)
    _, _, _, _, c, r = orc.compress(bits, z, 2, idx_raw_bf16=idx_bits, want_rows=True)
    # merging the idx rows alone (as the first 128 columns of a main row) gives r
    wide = np.zeros((32, 512), np.uint16)
    wide[:, :128] = idx_bits
    _, _, _, _, c2, _ = orc.compress(wide, z, 2, idx_raw_bf16=idx_bits, want_rows=True)
    assert np.array_equal(r, c2[:, :128])


def test_prefill_visibility_rule(orc):
    rng = np.random.default_rng(31)
    n_ent, ratio, P, k = 500, 2, 16, 24
    kc = rng.integers(0, 256, (n_ent, 64), dtype=np.uint8)
    ks = rng.integers(125, 128, (n_ent, 4), dtype=np.uint8)
    T = 5
    qc = rng.integers(0, 256, (T, 4, 64), dtype=np.uint8)
    qs = rng.integers(125, 128, (T, 4, 4), dtype=np.uint8)
    w = (0.5 + rng.random((T, 4))).astype(np.float32)
    q_pos = np.array([0, 1, 17, 998, 2000], np.int32)
    pool, top = orc.index_prefill(kc, ks, 0, n_ent, qc, qs, w, q_pos, ratio, P, k)
    for i, p in enumerate(q_pos):
        vis = min(n_ent, (p + 1) // 2)
        s = orc.index_scores(kc, ks, np.arange(vis), qc[i], qs[i], w[i])
        key = [orc.rank_key(v) for v in s]
        want = sorted(sorted(range(vis), key=lambda t: (-key[t], t))[:k])
        assert top[i].tolist() == want + [-1] * (k - len(want))
        nb = (vis + 7) // 8
        bkey = [max(key[8 * b:min(vis, 8 * b + 8)]) for b in range(nb)]
        wp = sorted(sorted(range(nb), key=lambda b: (-bkey[b], b))[:P])
        assert pool[i].tolist() == wp + [-1] * (P - len(wp))


# --- streaming (ratio-2 decode) appends -------------------------------------

def _stream_inputs(n, seed=31):
    bits = synth.normal_bf16(seed, synth.T_RAW, 0, 0, n * 512).reshape(n, 512)
    ibits = synth.normal_bf16(seed, synth.T_IDXRAW, 0, 0, n * 128).reshape(n, 128)
    z = synth.normal_f32(seed, synth.T_LOGITS, 0, 0, n) * 2
    return bits, ibits, z


def test_stream_chunks_equal_one_shot_append(orc):
    """Entries are the disjoint pairs (2j, 2j+1) of the token stream, so any
    cut of the stream into calls gives the one-shot append's bytes."""
    n = 45
    bits, ibits, z = _stream_inputs(n)
    one = orc.compress(bits[:n - 1], z[:n - 1], 2, idx_raw_bf16=ibits[:n - 1])
    rng = np.random.default_rng(5)
    cuts = [0]
    while cuts[-1] < n:
        cuts.append(min(n, cuts[-1] + int(rng.integers(0, 6))))
    pend, got = [None], [[], [], [], []]
    for a, b in zip(cuts[:-1], cuts[1:]):
        ent, pend = orc.compress_stream(pend, bits[a:b], z[a:b], [0, b - a], idx_raw_bf16=ibits[a:b])
        for part, arr in zip(got, ent[0]):
            part.append(arr)
    for want, part in zip(one, got):
        assert np.array_equal(np.concatenate(part), want)
    # n is odd: the last token is pending, bit for bit
    assert pend[0] is not None
    assert np.array_equal(pend[0]["raw"], bits[n - 1]) and np.array_equal(pend[0]["idx"], ibits[n - 1])
    assert np.float32(pend[0]["logit"]) == z[n - 1]


def test_stream_one_token_per_call_pairs_consecutive_tokens(orc):
    """With equal logits, entry j is the average of tokens 2j and 2j+1 (the
    pending token is the first of the pair, the new token the second)."""
    n = 12
    bits, ibits, _ = _stream_inputs(n, seed=32)
    x = synth.bf16_bits_to_f32(bits).astype(np.float64)
    z = np.zeros(n, np.float32)
    pend, entries = [None], []
    for t in range(n):
        ent, pend = orc.compress_stream(pend, bits[t:t + 1], z[t:t + 1], [0, 1], idx_raw_bf16=ibits[t:t + 1])
        assert ent[0][0].shape[0] == (t % 2)          # an entry every second token
        assert (pend[0] is None) == (t % 2 == 1)
        if t % 2:
            entries.append(ent[0])
    for j, (mc, ms, _, _) in enumerate(entries):
        avg = np.array([[rn32(Fraction(x[2 * j, i]) / 2 + Fraction(x[2 * j + 1, i]) / 2) for i in range(512)]],
                       np.float32)
        wc, ws = orc.mxfp4_encode(avg)
        assert np.array_equal(mc, wc) and np.array_equal(ms, ws)


def test_stream_projection_and_ragged_batch(orc):
    """Several sequences in one call, some with a pending token, some empty,
    with the W_idx projection: per sequence equal to the one-shot append of
    the pending token followed by the new tokens."""
    bits, _, z = _stream_inputs(40, seed=33)
    w_idx = synth.normal_f32(33, synth.T_WIDX, 0, 0, 512 * 128, log2_div=13).reshape(512, 128)
    tok_off = np.array([0, 0, 1, 6, 6, 15], np.int64)
    pend = [None, dict(raw=bits[30], logit=float(z[30]), idx=None), None,
            dict(raw=bits[31], logit=float(z[31]), idx=None), dict(raw=bits[32], logit=float(z[32]), idx=None)]
    ent, new = orc.compress_stream(pend, bits[:15], z[:15], tok_off, w_idx=w_idx)
    for b in range(5):
        t0, t1 = tok_off[b], tok_off[b + 1]
        rows = list(range(t0, t1))
        xs = ([bits[30 + [None, 0, None, 1, 2][b]]] if pend[b] is not None else []) + [bits[t] for t in rows]
        zs = ([z[30 + [None, 0, None, 1, 2][b]]] if pend[b] is not None else []) + [z[t] for t in rows]
        m = len(xs) // 2 * 2
        if m:
            want = orc.compress(np.stack(xs[:m]), np.array(zs[:m], np.float32), 2, w_idx=w_idx)
            for w_, g_ in zip(want, ent[b]):
                assert np.array_equal(w_, g_)
        else:
            assert ent[b][0].shape[0] == 0
        assert (new[b] is None) == (len(xs) % 2 == 0)
        if new[b] is not None:
            assert np.array_equal(new[b]["raw"], xs[-1])
