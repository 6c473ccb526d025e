"""Pins of the oracle's indexer: exact score, ranking keys, Top-k, block-max
pool, Full/Reindex/Reuse selection and the needle closed form (no GPU)."""
import numpy as np
import pytest

import synth
from tests._exact import exact_score


def _rand_rows(rng, n, width, smin=120, smax=134):
    codes = rng.integers(0, 256, (n, width // 2), dtype=np.uint8)
    scales = rng.integers(smin, smax + 1, (n, width // 32), dtype=np.uint8)
    return codes, scales


def _rand_query(rng, smin=120, smax=134):
    qc = rng.integers(0, 256, (4, 64), dtype=np.uint8)
    qs = rng.integers(smin, smax + 1, (4, 4), dtype=np.uint8)
    w = (0.5 + rng.random(4)).astype(np.float32)
    return qc, qs, w


def test_score_equals_exact_rational(orc):
    rng = np.random.default_rng(10)
    for trial in range(6):
        smin, smax = [(120, 134), (100, 140), (125, 127)][trial % 3]
        kc, ks = _rand_rows(rng, 24, 128, smin, smax)
        qc, qs, w = _rand_query(rng, smin, smax)
        got = orc.index_scores(kc, ks, np.arange(24), qc, qs, w)
        for t in range(24):
            want = exact_score(kc[t], ks[t], qc, qs, w)
            assert got[t].tobytes() == want.tobytes(), (trial, t, got[t], want)


def test_score_one_hot_weight_is_rounded_dot(orc):
    """w = (1,0,0,0) leaves exactly d_0 = fp32(q_0 . k)."""
    rng = np.random.default_rng(11)
    kc, ks = _rand_rows(rng, 16, 128)
    qc, qs, _ = _rand_query(rng)
    w = np.array([1, 0, 0, 0], np.float32)
    got = orc.index_scores(kc, ks, np.arange(16), qc, qs, w)
    dk = orc.mxfp4_decode(kc, ks)
    dq = orc.mxfp4_decode(qc, qs)
    ref = (dk @ dq[0]).astype(np.float32)       # exact in fp64 for these scales
    assert np.array_equal(got, ref)


def test_rank_key_order(orc):
    rng = np.random.default_rng(12)
    vals = np.concatenate([rng.standard_normal(300).astype(np.float32),
                           np.array([0.0, -0.0, 1e-45, -1e-45, np.inf, -np.inf, 3.4e38, -3.4e38], np.float32)])
    keys = np.array([orc.rank_key(v) for v in vals], np.uint64)
    assert orc.rank_key(-0.0) == orc.rank_key(0.0)
    for i in range(len(vals)):
        for j in range(0, len(vals), 7):
            if vals[i] < vals[j]:
                assert keys[i] < keys[j]
            elif vals[i] == vals[j]:
                assert keys[i] == keys[j]


def test_topk_matches_full_sort(orc):
    rng = np.random.default_rng(13)
    for n, k, levels in [(1000, 64, 5), (5000, 512, 50), (300, 512, 3), (0, 8, 1), (700, 700, 2)]:
        keys = rng.integers(0, levels, n).astype(np.uint32) * 1000 + 7
        ids = rng.permutation(n).astype(np.int64)
        got = orc.topk(keys, ids, k)
        order = sorted(range(n), key=lambda i: (-int(keys[i]), int(ids[i])))[:k]
        want = sorted(int(ids[i]) for i in order)
        want += [-1] * (k - len(want))
        assert got.tolist() == want


def test_topk_all_equal_picks_lowest_positions(orc):
    keys = np.full(4096, 12345, np.uint32)
    got = orc.topk(keys, np.arange(4096), 512)
    assert got.tolist() == list(range(512))


def _brute_full(orc, kc, ks, qc, qs, w, L, P, k):
    s = orc.index_scores(kc, ks, np.arange(L), qc, qs, w)
    key = [orc.rank_key(v) for v in s]
    nb = (L + 7) // 8
    bkey = [max(key[8 * b:min(L, 8 * b + 8)]) for b in range(nb)]
    pool = sorted(sorted(range(nb), key=lambda b: (-bkey[b], b))[:P])
    top = sorted(sorted(range(L), key=lambda t: (-key[t], t))[:k])
    return pool + [-1] * (P - len(pool)), top + [-1] * (k - len(top)), s


@pytest.mark.parametrize("L,P,k", [(203, 8, 16), (64, 16, 16), (5, 4, 8), (0, 4, 4), (1000, 16, 100)])
def test_index_full_bruteforce(orc, L, P, k):
    rng = np.random.default_rng(L + P)
    cap = max(L, 1) + 16
    kc, ks = _rand_rows(rng, cap, 128, 125, 127)
    kc[8:40] = kc[0]                                   # runs of equal scores (ties)
    ks[8:40] = ks[0]
    qc, qs, w = _rand_query(rng, 125, 127)
    off = np.array([8], np.int64)
    pool, top, sc = orc.index_full(kc, ks, qc[None], qs[None], w[None], off, np.array([L]), P, k, want_scores=True)
    bp, bt, bs = _brute_full(orc, kc[8:], ks[8:], qc, qs, w, L, P, k)
    assert pool[0].tolist() == bp
    assert top[0].tolist() == bt
    assert np.array_equal(sc[0, :L], bs)


def test_pool_contains_full_topk_when_P_ge_k(orc):
    """Containment: every Full Top-k position's block is in the pool when P >= k."""
    rng = np.random.default_rng(14)
    B, L, P, k = 3, 4096, 64, 64
    kc, ks = _rand_rows(rng, B * L, 128, 124, 128)
    # heavy ties: repeat a few rows everywhere
    kc[::5] = kc[0]
    ks[::5] = ks[0]
    qc, qs, w = _rand_query(rng, 124, 128)
    off = np.arange(B, dtype=np.int64) * L
    lens = np.array([L, L - 3, 777], np.int32)
    pool, top, _ = orc.index_full(kc, ks, np.repeat(qc[None], B, 0), np.repeat(qs[None], B, 0),
                                  np.repeat(w[None], B, 0), off, lens, P, k)
    for b in range(B):
        blocks = set(pool[b][pool[b] >= 0].tolist())
        assert all((t // 8) in blocks for t in top[b] if t >= 0)


def test_reindex_with_full_pool_equals_full_topk(orc):
    rng = np.random.default_rng(15)
    L, P, k = 2000, 256, 128
    kc, ks = _rand_rows(rng, L, 128)
    qc, qs, w = _rand_query(rng)
    off, lens = np.array([0], np.int64), np.array([L], np.int32)
    pool, top, _ = orc.index_full(kc, ks, qc[None], qs[None], w[None], off, lens, P, k)
    assert (pool[0] >= 0).sum() == 250                # all ceil(2000/8) blocks
    re = orc.index_reindex(kc, ks, qc[None], qs[None], w[None], off, lens, pool, k)
    assert np.array_equal(re, top)
    # a Reindex layer with another query over a partial pool = brute force
    qc2, qs2, w2 = _rand_query(rng)
    part = np.full((1, P), -1, np.int32)
    part[0, :40] = np.sort(rng.choice(250, 40, replace=False))
    re2 = orc.index_reindex(kc, ks, qc2[None], qs2[None], w2[None], off, lens, part, k)
    pos = [8 * b + j for b in part[0, :40] for j in range(8)]
    s = orc.index_scores(kc, ks, np.array(pos), qc2, qs2, w2)
    key = [orc.rank_key(v) for v in s]
    best = sorted(sorted(range(len(pos)), key=lambda i: (-key[i], pos[i]))[:k])
    assert re2[0].tolist() == sorted(pos[i] for i in best)


def test_needles_always_selected(orc):
    """Closed form: needle keys (head-0 query codes, scales +2) are in the Top-512."""
    seed, L = 7, 8192
    qc = synth.mxfp4_rows(seed, synth.T_QIDX_CODES, synth.T_QIDX_SCALES, 0, 0, 0, 4, 128)
    w = synth.head_weights(seed, 0, 0)
    kc, ks = synth.mxfp4_rows(seed, synth.T_IDXK_CODES, synth.T_IDXK_SCALES, 0, 0, 0, L, 128)
    pos = synth.needle_positions(seed, 0, 0, L, 8)
    nc, ns = synth.needle_rows(qc[0][0], qc[1][0], len(pos))
    kc[pos], ks[pos] = nc, ns
    pool, top, _ = orc.index_full(kc, ks, qc[0][None], qc[1][None], w[None], np.array([0]), np.array([L]), 256, 512)
    assert set(pos.tolist()) <= set(top[0].tolist())
    assert set((pos // 8).tolist()) <= set(pool[0].tolist())


def test_index_multi_each_query_sees_its_own_prefix(orc):
    """Several queries per sequence (speculative verification): query i of
    sequence b ranks exactly the first q_vis[i] entries of b, checked by
    brute force (scores of those entries, full sort); queries of no sequence
    select nothing."""
    rng = np.random.default_rng(15)
    L, P, k = 300, 16, 8
    kc, ks = _rand_rows(rng, 3 * 304, 128, 125, 127)
    seq_row_off = np.array([0, 304, 608], np.int64)
    q_off = np.array([0, 3, 3, 7], np.int32)            # 3 queries, none, 4 queries; query 7 belongs to none
    q_vis = np.array([L, L - 1, 5, 299, 300, 64, 1, 200], np.int32)
    Q = len(q_vis)
    qs_ = [_rand_query(rng, 125, 127) for _ in range(Q)]
    qc = np.stack([q[0] for q in qs_])
    qsc = np.stack([q[1] for q in qs_])
    w = np.stack([q[2] for q in qs_])
    pool, top = orc.index_multi(kc, ks, qc, qsc, w, seq_row_off, q_off, q_vis, P, k)
    owner = [0, 0, 0, 2, 2, 2, 2, None]
    for i in range(Q):
        if owner[i] is None:
            assert (top[i] == -1).all() and (pool[i] == -1).all()
            continue
        r0, v = int(seq_row_off[owner[i]]), int(q_vis[i])
        bp, bt, _ = _brute_full(orc, kc[r0:], ks[r0:], qc[i], qsc[i], w[i], v, P, k)
        assert pool[i].tolist() == bp and top[i].tolist() == bt, i


def test_index_multi_one_query_per_sequence_is_index_full(orc):
    rng = np.random.default_rng(16)
    B, L = 4, 512
    kc, ks = _rand_rows(rng, B * L, 128, 124, 128)
    qc = rng.integers(0, 256, (B, 4, 64), dtype=np.uint8)
    qsc = rng.integers(124, 129, (B, 4, 4), dtype=np.uint8)
    w = (0.5 + rng.random((B, 4))).astype(np.float32)
    off = np.arange(B, dtype=np.int64) * L
    lens = np.array([512, 17, 400, 256], np.int32)
    pool_f, top_f, _ = orc.index_full(kc, ks, qc, qsc, w, off, lens, 64, 32)
    pool_m, top_m = orc.index_multi(kc, ks, qc, qsc, w, off, np.arange(B + 1, dtype=np.int32), lens, 64, 32)
    assert np.array_equal(pool_f, pool_m) and np.array_equal(top_f, top_m)


def _overflow_case(L=1000):
    """Rows whose exact head dots overflow fp32: query head 0 is +6 on blocks
    0-1 and head 1 is -6 on blocks 2-3 (zeros elsewhere), at scale byte 200
    (2^73); planted key rows of +6 at scale byte 250 (2^123) give block dots
    of +-(32*12*12)*2^(73+123-2), far above fp32's range; heads 2, 3 (random
    codes) sit at scale bytes 10 and 12, finite against every row.  Rows 100..119 (+6 on blocks 0-1): d0 = +inf, d1 = 0,
    score +inf.  Rows 120..859 (+6 everywhere): d0 = +inf, d1 = -inf, score
    NaN.  Rows 860..899 (+6 on blocks 2-3): d0 = 0, d1 = -inf, score -inf.
    Other rows are random at normal scales (finite scores)."""
    rng = np.random.default_rng(91)
    kc, ks = _rand_rows(rng, L, 128, 124, 128)
    qc = rng.integers(0, 256, (4, 64), dtype=np.uint8)
    qs = rng.integers(124, 129, (4, 4), dtype=np.uint8)
    qc[0, :32], qc[0, 32:] = 0x77, 0x00      # head 0: +6 on blocks 0, 1
    qc[1, :32], qc[1, 32:] = 0x00, 0xFF      # head 1: -6 on blocks 2, 3
    qs[0], qs[1] = 200, 200
    qs[2], qs[3] = 10, 12                    # heads 2, 3 stay finite against the planted rows
    w = np.array([1.0, 0.75, 1.25, 0.5], np.float32)
    kinds = np.zeros(L, np.int8)
    for lo, hi, code, kind in ((100, 120, (0x77, 0x00), 1), (120, 860, (0x77, 0x77), 2), (860, 900, (0x00, 0x77), 3)):
        kc[lo:hi, :32], kc[lo:hi, 32:] = code
        ks[lo:hi] = 250
        kinds[lo:hi] = kind
    return kc, ks, qc, qs, w, kinds


def test_rank_key_nan_ranks_below_every_number(orc):
    """Every NaN (any sign or payload) ranks below every number, -inf
    included, and NaNs tie among themselves; key 0 stays "absent"."""
    nans = np.array([0x7FC00000, 0xFFC00000, 0x7F800001, 0xFFFFFFFF, 0x7FFFFFFF], np.uint32).view(np.float32)
    assert all(orc.rank_key(v) == 1 for v in nans)
    assert orc.rank_key(-np.inf) == 0x007FFFFF
    assert orc.rank_key(np.inf) == 0xFF800000
    # scores [NaN, -inf, 1, NaN, -3], best 4 by (score desc, position asc):
    # 1 (pos 2), -3 (pos 4), -inf (pos 1), the first NaN (pos 0)
    s = np.array([np.nan, -np.inf, 1.0, np.nan, -3.0], np.float32)
    key = [orc.rank_key(v) for v in s]
    assert orc.topk(key, np.arange(5), 4).tolist() == [0, 1, 2, 4]


def test_overflowing_scores_are_inf_and_nan(orc):
    kc, ks, qc, qs, w, kinds = _overflow_case()
    s = orc.index_scores(kc, ks, np.arange(len(kinds)), qc, qs, w)
    assert np.all(s[kinds == 1] == np.inf)
    assert np.all(np.isnan(s[kinds == 2]))
    assert np.all(s[kinds == 3] == -np.inf)
    assert np.all(np.isfinite(s[kinds == 0]))
    # the Top-512: the 20 +inf rows, the 200 finite rows, the 40 -inf rows and
    # then the first 252 NaN rows by position (brute force over the sort rule)
    _, top, _ = orc.index_full(kc, ks, qc, qs, w, np.array([0]), np.array([len(kinds)], np.int32), 64, 512)
    want = sorted(list(range(100, 120)) + list(range(100)) + list(range(900, 1000)) + list(range(860, 900))
                  + list(range(120, 120 + 252)))
    assert top[0].tolist() == want


def test_score_with_wide_exponent_spread_is_the_ordered_fp64_sum(orc):
    """Beyond a block-exponent spread of 38 the four block terms of a head no
    longer add exactly in fp64 (13-bit integers 2^39 apart and more).  The
    definition is then the fp64 sum in block order 0..3, rounded once to fp32;
    this pins the oracle to that order on rows where it differs from the exact
    sum."""
    from fractions import Fraction

    from tests._exact import frac32, rn32, row_values

    rng = np.random.default_rng(93)
    differs = 0
    for trial in range(40):
        kc, ks = _rand_rows(rng, 1, 128)
        qc, qs, w = _rand_query(rng, 125, 129)
        # block 0 huge, blocks 1..3 tiny: spreads of 60..90 exponents
        ks[0] = [127 + 40, 127 - rng.integers(20, 50), 127 - rng.integers(20, 50), 127 - 20]
        got = orc.index_scores(kc, ks, np.arange(1), qc, qs, w)[0]
        k = row_values(kc[0], ks[0])
        d = []
        for h in range(4):
            q = row_values(qc[h], qs[h])
            acc = 0.0
            exact = Fraction(0)
            for b in range(4):
                term = sum(q[i] * k[i] for i in range(32 * b, 32 * b + 32))   # exact block dot
                acc = acc + float(term)           # fp64 add in block order (each term exact in fp64)
                exact += term
            d.append(np.float32(acc))
            differs += int(Fraction(acc) != exact)
        s = rn32(frac32(w[0]) * frac32(d[0]))
        for h in range(1, 4):
            s = rn32(frac32(w[h]) * frac32(d[h]) + frac32(s))
        assert got.tobytes() == np.float32(0.0 if s == 0 else s).tobytes(), trial
    assert differs > 0     # the ordered sum really differs from the exact one somewhere
