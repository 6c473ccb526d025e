"""Host side of the Python binding and of the step orchestration (no GPU).

1. The binding checks every tensor argument's element type and size against
   the C declaration before anything reaches the library (the library sees
   only pointers), and refuses host tensors.
2. DecodeStep and ShardedStep are driven with host tensors against a
   recording stand-in of the library (the binding's pointer and stream
   lookups are patched to accept host memory).  This runs the real
   orchestration code and the binding's checks on every call it makes, and
   pins which calls a layer pattern issues, with which caches, pools and
   Top-k buffers ("DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache
   Compression", section "三个方向一起压小缓存": the first Full layer scans
   and builds the pool, Reindex layers rank inside it with the nearest Full
   layer's caches, Reuse layers repeat the last Top-k).
"""
import ctypes

import numpy as np
import pytest
import torch

import synth.workloads as W
from long_context_decode_csa2_b200 import csa2 as C
from long_context_decode_csa2_b200.cp import Shard, ShardedStep, stack_gather
from long_context_decode_csa2_b200.decode import DecodeStep, FullCache


def t(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    return torch.from_numpy(a)


def _decode_args(B=2, k=16):
    return dict(q=torch.zeros((B, 16, 512), dtype=torch.bfloat16), main_kv=C.MXFP4Cache(0, 0, 0),
                seq_row_off=torch.zeros(B, dtype=torch.int64), seq_len=torch.ones(B, dtype=torch.int32),
                topk=torch.zeros((B, k), dtype=torch.int32), win=torch.zeros((B, 128, 512), dtype=torch.uint8),
                win_scale=torch.ones(B), win_len=torch.ones(B, dtype=torch.int32), sm_scale=0.05,
                out=torch.zeros((B, 16, 512)), ws=torch.zeros(256, dtype=torch.uint8),
                lse=torch.zeros((B, 16)))


# ---------------------------------------------------------------------------
# orchestration against a recording stand-in of the library
# ---------------------------------------------------------------------------

class FakeLib:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        if not name.startswith("csa2_"):
            raise AttributeError(name)

        def f(*args):
            if name.endswith("_workspace_bytes"):
                return 256
            self.calls.append((name, args))
            return 0

        return f


class FakeStream:
    cuda_stream = 0

    def wait_event(self, ev):
        raise AssertionError("a sequential step waits on no event")


@pytest.fixture
def fake(monkeypatch):
    lib = FakeLib()
    monkeypatch.setattr(C, "_lib", lib)
    monkeypatch.setattr(C, "_ptr", lambda x: None if x is None else x.data_ptr())
    monkeypatch.setattr(C, "_stream", lambda s: ctypes.c_void_p(0))
    return lib


@pytest.mark.parametrize("name,bad", [
    ("q", torch.zeros((2, 16, 512), dtype=torch.float32)),        # fp32 where bf16 bits are read
    ("q", torch.zeros((2, 16, 512), dtype=torch.float16)),        # same width, another format
    ("seq_row_off", torch.zeros(2, dtype=torch.int32)),           # int32 where int64 is read
    ("seq_len", torch.zeros(2, dtype=torch.int64)),
    ("win_scale", torch.ones(2, dtype=torch.float64)),
    ("out", torch.zeros((1, 16, 512))),                           # one sequence short
    ("lse", torch.zeros((2, 15))),
    ("win", torch.zeros((2, 127, 512), dtype=torch.uint8)),
    ("q", np.zeros((2, 16, 512), np.uint16)),                     # not a tensor
])
def test_binding_rejects_wrong_element_types_and_short_buffers(fake, name, bad):
    args = _decode_args()
    args[name] = bad
    with pytest.raises(C.Csa2Error) as e:
        C.csa2_sparse_attn_decode(**args)
    assert e.value.status == -1 and name in str(e.value)
    assert not fake.calls
    C.csa2_sparse_attn_decode(**_decode_args())                   # the same call with every argument right
    assert [n for n, _ in fake.calls] == ["csa2_sparse_attn_decode"]


def test_binding_refuses_host_tensors():
    with pytest.raises(ValueError, match="CUDA"):
        C.csa2_sparse_attn_decode(**_decode_args())


def _inputs(wl, queries=None):
    layers = [W.layer_inputs_host(wl if queries is None else queries, l) for l in range(len(wl.pattern))]
    keys = ("q", "q_codes", "q_scales", "w", "win", "win_scale", "win_len")
    dev = [{k: t(L[k]) for k in keys} for L in layers]
    caches = []
    for f in wl.full_layers():
        n = int(wl.row_offsets()[1])
        z = lambda w: torch.zeros((n, w), dtype=torch.uint8)  # noqa: E731
        caches.append(FullCache(C.cache(z(64), z(4)), C.cache(z(256), z(16))))
    off = t(wl.row_offsets()[0])
    return dev, caches, off, t(wl.lengths.astype(np.int32))


def _nearest_full(pattern):
    f, out = -1, []
    for m in pattern:
        f += m == "F"
        out.append(f)
    return out


@pytest.mark.parametrize("rescan", [False, True])
def test_decode_step_issues_the_layer_modes(fake, rescan):
    pattern = "FRUFRU"
    wl = W.DecodeWorkload("orchestration", np.array([700, 1500, 64]), pattern, P=16, k=32)
    layers, caches, off, lens = _inputs(wl)
    step = DecodeStep(pattern, wl.B, wl.max_len, wl.P, wl.k, full_rescan=rescan, device="cpu", concurrent=False)
    step.run(caches, off, lens, layers, stream=FakeStream())
    near = _nearest_full(pattern)
    scans = [0, 3] if rescan else [0]
    want = []
    for l, m in enumerate(pattern):
        if l in scans:
            want.append("csa2_index_full")
        elif m != "U":
            want.append("csa2_index_reindex")
        want.append("csa2_sparse_attn_decode")
    assert [n for n, _ in fake.calls] == want
    it = iter(fake.calls)
    for l, m in enumerate(pattern):
        c = caches[near[l]]
        if m != "U":
            name, a = next(it)
            assert a[0] is c.idx                                     # the nearest Full layer's indexer K
            assert a[1] == layers[l]["q_codes"].data_ptr()           # this layer's own query
            pool_layer = max(s for s in scans if s <= l)
            pool_arg = a[10] if name == "csa2_index_full" else a[6]
            assert pool_arg == step.pools[pool_layer].data_ptr()
        name, a = next(it)
        assert a[1] is c.main and a[0] == layers[l]["q"].data_ptr()
        src = l - 1 if m == "U" else l                              # Reuse attends the Top-k before it
        assert a[4] == step.topk[src].data_ptr() and step.topk[l] is step.topk[src]
        assert a[10] == step.out[l].data_ptr() and a[11] == step.lse[l].data_ptr()


def test_ratio2_step_appends_each_full_layer_first(fake):
    pattern = "FRFU"
    wl = W.DecodeWorkload("orchestration_r2", np.array([100, 333]), pattern, P=16, k=32, ratio=2)
    layers, caches, off, lens = _inputs(wl)
    step = DecodeStep(pattern, wl.B, wl.max_len, wl.P, wl.k, device="cpu", concurrent=False, ratio=2)
    tok = [dict(raw=torch.zeros((wl.B, 512), dtype=torch.bfloat16), logit=torch.zeros(wl.B),
                w_idx=torch.zeros((512, 128))) for _ in range(2)]
    step.run(caches, off, lens, layers, stream=FakeStream(), new_tokens=tok)
    names = [n for n, _ in fake.calls]
    assert names[:2] == ["csa2_compress_stream"] * 2 and "csa2_compress_stream" not in names[2:]
    (_, a0), (_, a1) = fake.calls[:2]
    assert a0[0] is caches[0].main and a0[1] is caches[0].idx and a1[0] is caches[1].main
    assert a0[9] is None and a1[9] == lens.data_ptr()   # lengths advance once, after the last Full layer's append


def test_verification_step_takes_queries_as_segments(fake):
    pattern = "FRU"
    wl = W.DecodeWorkload("orchestration_verify", np.array([900, 4000]), pattern, P=16, k=32, queries_per_seq=3)
    q_off, q_vis = wl.verify_queries()
    wq = W.DecodeWorkload("orchestration_verify_q", q_vis.astype(np.int64), pattern, P=16, k=32)
    layers, caches, off, lens = _inputs(wl, queries=wq)
    Q = len(q_vis)
    step = DecodeStep(pattern, wl.B, wl.max_len, wl.P, wl.k, device="cpu", concurrent=False, queries=Q)
    step.run(caches, off, lens, layers, stream=FakeStream(), q_off=t(q_off), q_vis=t(q_vis))
    names = [n for n, _ in fake.calls]
    assert names == ["csa2_index_multi", "csa2_sparse_attn_decode", "csa2_index_reindex", "csa2_sparse_attn_decode",
                     "csa2_sparse_attn_decode"]
    _, multi = fake.calls[0]
    assert multi[14] == step.q_row_off.data_ptr()
    for name, a in fake.calls[1:]:                                 # segments = queries: rows and lengths per query
        row_off, seg_len = (a[2], a[3]) if name == "csa2_sparse_attn_decode" else (a[4], a[5])
        assert row_off == step.q_row_off.data_ptr() and seg_len != lens.data_ptr()


def test_sharded_step_merges_each_selection(fake):
    pattern = "FRU"
    B, G, P, k = 2, 2, 64, 32
    wl = W.DecodeWorkload("orchestration_cp", np.array([600, 1000]), pattern, P=P, k=k)
    layers, _, _, _ = _inputs(wl)
    shards = []
    for g in range(G):
        z = lambda w: torch.zeros((512, w), dtype=torch.uint8)  # noqa: E731
        caches = [FullCache(C.cache(z(64), z(4)), C.cache(z(256), z(16)))]
        lo = torch.tensor([0, 0], dtype=torch.int64) + g * 256
        shards.append(Shard(caches=caches, seq_row_off=torch.tensor([0, 256], dtype=torch.int64),
                            seq_len=torch.full((B,), 256, dtype=torch.int32), lo=lo, hi=lo + 256, layers=layers))
    src_pos = torch.tensor([[0, 0], [256, 256]], dtype=torch.int64)
    step = ShardedStep(pattern, B, 256, G, G, P, k, device="cpu", gather=stack_gather)
    step.run(shards, src_pos, src_pos // 8)
    names = [n for n, _ in fake.calls]
    per_shard_scan = ["csa2_index_full", "csa2_score_positions", "csa2_score_positions"]
    attn = ["csa2_sparse_attn_decode"] * G + ["csa2_attn_combine"]
    assert names == (per_shard_scan * G + ["csa2_topk_merge"] * (2 * G) + attn
                     + ["csa2_index_reindex", "csa2_score_positions"] * G + ["csa2_topk_merge"] * G + attn + attn)
    combines = [a for n, a in fake.calls if n == "csa2_attn_combine"]
    assert [a[4] for a in combines] == [step.out[l].data_ptr() for l in range(3)]


def test_paged_step_reads_through_the_page_table(fake):
    pattern = "FRU"
    wl = W.DecodeWorkload("orchestration_paged", np.array([1024, 1536]), pattern, P=16, k=32, room=0,
                          page_rows=512)
    layers, caches, _, lens = _inputs(wl)
    pt = C.PageTable(t(wl.page_table()), wl.page_rows)
    step = DecodeStep(pattern, wl.B, wl.max_len, wl.P, wl.k, device="cpu", concurrent=False)
    step.run(caches, pt, lens, layers, stream=FakeStream())
    names = [n for n, _ in fake.calls]
    assert names == ["csa2_index_full_paged", "csa2_sparse_attn_decode_paged", "csa2_index_reindex_paged",
                     "csa2_sparse_attn_decode_paged", "csa2_sparse_attn_decode_paged"]
    for name, a in fake.calls:
        pages_arg = a[2] if name == "csa2_sparse_attn_decode_paged" else a[4]
        assert pages_arg == pt.pages.data_ptr()
        assert 512 in a and pt.max_pages in a


def test_every_wrapper_checks_its_tensors():
    """Outside the checked helper, raw pointers are taken only for the cache
    planes (checked in cache()), workspaces and the status read-back."""
    import ast
    import inspect

    tree = ast.parse(inspect.getsource(C))
    allowed = {"_arg", "cache", "_ws", "device_status", "_ptr"}
    for fn in [n for n in tree.body if isinstance(n, ast.FunctionDef)]:
        uses = [c for c in ast.walk(fn) if isinstance(c, ast.Call) and getattr(c.func, "id", None) == "_ptr"]
        assert not uses or fn.name in allowed, fn.name
