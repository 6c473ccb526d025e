"""The oracle's pins catch plausible mistakes.

Each mutant below is a copy of the oracle with one planted mistake of the
kinds a restatement of the definitions can make: a wrong table entry or
exponent bias, a dropped term or factor, a transposed operand, a swapped
nibble order or tie-break, an off-by-one window, the wrong cache or query in
the layer-mode composition.  For every mutant a scratch tree is made with a
copy of the oracle (C++ source and Python wrapper, one of them mutated), of
the seeded input generators and of the oracle pin tests; the pins run there
in a child process, which builds that copy of the oracle itself, and at
least one of them must fail.  An unmutated copy run the same way must pass
them all (which shows that each child loads the copy it was given).

Only memory-safe mutants are planted: none moves a read or write outside the
buffers that the unmutated oracle touches.
"""
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PIN_FILES = ["test_oracle_formats.py", "test_oracle_index.py", "test_oracle_attention.py",
             "test_oracle_compress.py", "test_oracle_decode_step.py"]
CPP, PY = "oracle/csa2_oracle.cpp", "oracle/__init__.py"

# (name, text in the C++ oracle, replacement); each text occurs once.
MUTANTS = [
    # formats (OCP MX v1.0: E2M1, E8M0; FP8 E4M3)
    ("e2m1 table entry", "{0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0}", "{0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 5.0}"),
    ("doubled e2m1 table entry", "{0, 1, 2, 3, 4, 6, 8, 12}", "{0, 1, 2, 3, 4, 6, 8, 10}"),
    ("doubled e2m1 drops the sign", "return (code & 8) ? -t[code & 7] : t[code & 7];", "return t[code & 7];"),
    ("e8m0 bias", "std::ldexp(1.0, byte - 127)", "std::ldexp(1.0, byte - 128)"),
    ("e4m3 subnormal exponent", "std::ldexp(m / 8.0, -6)", "std::ldexp(m / 8.0, -7)"),
    ("e4m3 bias", "std::ldexp(1.0 + m / 8.0, e - 7)", "std::ldexp(1.0 + m / 8.0, e - 8)"),
    ("e4m3 has no NaN", '  if (e == 15 && m == 7) return std::nan("");\n', ""),
    ("nibble order", "return (e & 1) ? (b >> 4) : (b & 15);", "return (e & 1) ? (b & 15) : (b >> 4);"),
    ("ties round down", "return (i % 2 == 0) ? i : i + 1;", "return i;"),
    ("ties round up", "return (i % 2 == 0) ? i : i + 1;", "return i + 1;"),
    ("no saturation below 6", "if (a >= 6.0) return 7;", "if (a > 6.0) return 7;\n  if (a == 6.0) return 6;"),
    ("block scale emax", "(e - 1) - 2))", "(e - 1) - 1))"),
    ("negative zero loses its sign", "(std::signbit(x[i + j]) ? 8 : 0)", "(x[i + j] < 0.0f ? 8 : 0)"),
    # own exp
    ("exp drops the low ln2 part", "double r = (x - k * kLn2Hi) - k * kLn2Lo;", "double r = x - k * kLn2Hi;"),
    ("exp series one term short", "for (int i = 13; i >= 0; --i)", "for (int i = 12; i >= 0; --i)"),
    # indexer score
    ("score misses the doubling factor", "(int(ks[b]) - 127) - 2;", "(int(ks[b]) - 127) - 1;"),
    ("score uses one key scale", "(int(ks[b]) - 127)", "(int(ks[0]) - 127)"),
    ("score transposes the query scales", "int(qs[4 * h + b])", "int(qs[4 * b + h])"),
    ("score reuses head 0", "std::fma(w[h], d[h], s)", "std::fma(w[h], d[0], s)"),
    ("score drops head 0", "float s = w[0] * d[0];", "float s = 0.0f;"),
    ("score head chain in one step", "for (int h = 1; h < 4; ++h) s = std::fma(w[h], d[h], s);",
     "for (int h = 1; h < 4; ++h) s = s + w[h] * d[h];"),
    ("score block sum rounded per block", "acc = acc + term;", "acc = double(float(acc + term));"),
    # selection
    ("rank key keeps negative bits", "(u & 0x80000000u) ? ~u : (u | 0x80000000u)", "(u & 0x80000000u) ? u : (u | 0x80000000u)"),
    ("tie-break by higher id", "return ids[a] < ids[b];", "return ids[a] > ids[b];"),
    ("top-k padded with 0", "int32_t(sel[i]) : -1;", "int32_t(sel[i]) : 0;"),
    ("top-k left unsorted", "std::sort(sel.begin(), sel.end());", ""),
    ("block key is the last position", "bkey[b] = std::max(bkey[b], rank_key(s[t]));", "bkey[b] = rank_key(s[t]);"),
    ("block drops its last position", "std::min(L, (b + 1) * kBlk)", "std::min(L, b * kBlk + kBlk - 1)"),
    ("pool one block short", "topk_select(bkey, bid, P, pool_out)", "topk_select(bkey, bid, P - 1, pool_out)"),
    ("reindex drops each block's last position", "for (int j = 0; j < kBlk; ++j) {",
     "for (int j = 0; j < kBlk - 1; ++j) {"),
    ("rank key keeps the sign of zero", "  if (s == 0.0f) s = 0.0f;\n  uint32_t u;", "  uint32_t u;"),
    ("NaN ranked by its bits", "  if (std::isnan(s)) return 1u;\n", ""),
    ("NaN ranked first", "  if (std::isnan(s)) return 1u;", "  if (std::isnan(s)) return 0xFFFFFFFFu;"),
    ("reindex block is not scaled by 8", "int64_t t = int64_t(blk) * kBlk + j;", "int64_t t = int64_t(blk) + j;"),
    # attention
    ("attention drops sm_scale", "lg[j] = sm_scale * acc;", "lg[j] = acc;"),
    ("lse drops the max", "lse[h] = m + std::log(l);", "lse[h] = std::log(l);"),
    ("attention not normalised", "for (int d = 0; d < kD; ++d) o[d] /= l;", ""),
    ("window scale dropped", "int64_t(kD), double(win_scale[b]))", "int64_t(kD), 1.0)"),
    ("window skips its first row", "for (int r = 0; r < win_len[b]; ++r)", "for (int r = 1; r < win_len[b]; ++r)"),
    ("window ignores its length", "for (int r = 0; r < win_len[b]; ++r)", "for (int r = 0; r < 128; ++r)"),
    ("prefill window one row wider", "std::max<int64_t>(0, p - 127)", "std::max<int64_t>(0, p - 128)"),
    # compression
    ("pair weights swapped", "w0 = a / s;", "w0 = b / s;"),
    ("pair merges the first token twice", "src[(2 * j + 1) * stride + i]", "src[(2 * j) * stride + i]"),
    ("pair merge rounded twice", "c[i] = float(std::fma(w0, x0, w1 * x1));", "c[i] = float(w0 * x0) + float(w1 * x1);"),
    ("projection transposed", "double(w_idx[i * kDi + o])", "double(w_idx[o * kD + i])"),
    ("prefill index visibility off by one", "(int64_t(q_pos[i]) + 1) / ratio", "int64_t(q_pos[i]) / ratio"),
    ("prefill attention visibility off by one", "(p + 1) / ratio", "p / ratio"),
]

# (name, text in the Python wrapper, replacement): the compositions written there.
PY_MUTANTS = [
    # several queries per sequence
    ("query rows from the first sequence", "rows[i] = seq_row_off[b]", "rows[i] = seq_row_off[0]"),
    ("query sees one entry less", "vis[i] = max(0, int(q_vis[i]))", "vis[i] = max(0, int(q_vis[i]) - 1)"),
    ("last sequence's queries dropped", "for b in range(len(q_off) - 1):\n        for i in",
     "for b in range(len(q_off) - 2):\n        for i in"),
    # streamed ratio-2 append
    ("pending token placed after the new ones",
     'rows.insert(0, np.asarray(pend[b]["raw"], np.uint16).reshape(1, 512))',
     'rows.append(np.asarray(pend[b]["raw"], np.uint16).reshape(1, 512))'),
    ("odd trailing token dropped", "None if n == m else dict(", "None if True else dict("),
    ("pending logit of the wrong token", "logit=float(z[m])", "logit=float(z[m - 1])"),
    # layer modes of a decode step
    ("every layer uses the first Full layer's cache", "c = caches[full_idx]", "c = caches[0]"),
    ("rescan switch ignored", 'if mode == "F" and (not scanned or full_rescan):', 'if mode == "F" and not scanned:'),
    ("Reuse layers rank again", 'elif mode in ("F", "R"):', 'elif mode in ("F", "R", "U"):'),
    ("attention reads the first Full layer's main KV",
     'o, l = attn_decode(L["q"], c["main_codes"], c["main_scales"],',
     'o, l = attn_decode(L["q"], caches[0]["main_codes"], caches[0]["main_scales"],'),
]


def _scratch_tree(dst: str, path: str, old: str, new: str) -> str:
    """A copy of the oracle, the input generators and the pin tests, with
    `old` replaced by `new` in `path` (nothing replaced when path is None)."""
    os.makedirs(os.path.join(dst, "oracle"))
    for f in (CPP, PY):
        shutil.copy(os.path.join(ROOT, f), os.path.join(dst, f))
    shutil.copytree(os.path.join(ROOT, "synth"), os.path.join(dst, "synth"),
                    ignore=shutil.ignore_patterns("_build", "__pycache__", "*.so", "*.cu", "gpu.py"))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(dst, "tests", "golden"))
    for f in ["conftest.py", "_exact.py"] + PIN_FILES:
        shutil.copy(os.path.join(ROOT, "tests", f), os.path.join(dst, "tests", f))
    if path is not None:
        with open(os.path.join(dst, path)) as f:
            src = f.read()
        assert src.count(old) == 1, f"{old!r}: the planted text must occur exactly once in {path}"
        with open(os.path.join(dst, path), "w") as f:
            f.write(src.replace(old, new))
    return dst


def _run_pins(tree: str) -> subprocess.CompletedProcess:
    env = {k: v for k, v in os.environ.items() if k != "PYTHONPATH"}
    return subprocess.run([sys.executable, "-m", "pytest", *[f"tests/{f}" for f in PIN_FILES], "-x", "-q",
                           "-m", "not gpu", "-p", "no:cacheprovider", "-W", "ignore"],
                          cwd=tree, env=env, capture_output=True, text=True, timeout=900)


def test_every_planted_mistake_fails_a_pin(tmp_path):
    muts = [(name, CPP, old, new) for name, old, new in MUTANTS] + [(name, PY, old, new) for name, old, new in PY_MUTANTS]
    names = [m[0] for m in muts]
    assert len(set(names)) == len(names)
    jobs = [("control", None, None, None)] + muts

    def run(i_job):
        i, (_, path, old, new) = i_job
        return _run_pins(_scratch_tree(str(tmp_path / f"t{i}"), path, old, new))

    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        res = list(ex.map(run, enumerate(jobs)))
    ctl = res[0]
    assert ctl.returncode == 0, "the unmutated copy must pass its pins:\n" + ctl.stdout[-3000:] + ctl.stderr[-2000:]
    survivors, broken = [], []
    for (name, _, _, _), r in zip(jobs[1:], res[1:]):
        if r.returncode == 0:
            survivors.append(name)
        elif r.returncode != 1 or " failed" not in r.stdout:  # 1 = a test failed (not a crash or usage error)
            broken.append((name, r.returncode, r.stdout[-800:] + r.stderr[-800:]))
    assert not broken, broken
    assert not survivors, f"mistakes no pin detects: {survivors}"
