"""Host-side logic of the bench and the workloads (no GPU): algorithmic byte
counts, the verification queries' visibility, page tables, layer plans."""
import numpy as np
import pytest

import bench
import synth.workloads as W
from long_context_decode_csa2_b200.decode import DecodeStep, layer_plan


def test_algorithmic_bytes_of_the_default_step():
    wl = W.decode_workloads()["long_decode_b64_l1m"]
    ab = bench.algorithmic_bytes(wl)
    L = 1 << 20
    assert ab["scan"] == 64 * L * 68
    assert ab["pool"] == 2 * 64 * 16384 * 68                 # the two Reindex layers
    assert ab["attn"] == 4 * 64 * (512 * 272 + 128 * 512)
    assert ab["total"] == ab["scan"] + ab["pool"] + ab["attn"]
    assert abs(ab["total"] / 1e9 - 4.758) < 1e-3              # 74.35 MB per sequence


def test_algorithmic_bytes_of_the_variants():
    ragged = W.decode_workloads()["ragged_decode_b48_20l"]
    one, every = bench.algorithmic_bytes(ragged), bench.algorithmic_bytes(ragged, full_rescan=True)
    # FRURU x 4: 8 Reindex layers select in the pool; under the pages' plan the
    # three later Full layers do too, with every Full layer rescanning they scan
    assert every["scan"] == 4 * one["scan"] and every["pool"] * 11 == one["pool"] * 8
    verify = W.decode_workloads()["verify_decode_b64_l1m_m6"]
    v = bench.algorithmic_bytes(verify)
    assert v["scan"] == 64 * (1 << 20) * 68                    # indexer K read once per sequence
    assert v["attn"] == 4 * 384 * (512 * 272 + 128 * 512)      # attention per candidate
    r2 = bench.algorithmic_bytes(W.decode_workloads()["ratio2_decode_b64_l1m"])
    assert r2["append"] == 64 * (1024 + 4) + 512 * 128 * 4 + 64 * 340 // 2


def test_verification_queries_see_their_own_prefix():
    wl = W.decode_workloads()["verify_decode_b64_l1m_m6"]
    q_off, q_vis = wl.verify_queries()
    assert q_off.tolist() == list(range(0, 6 * 64 + 1, 6))
    L = 1 << 20
    assert q_vis[:6].tolist() == [L - 5, L - 4, L - 3, L - 2, L - 1, L]
    assert len(q_vis) == 384


def test_page_table_is_a_permutation_of_the_pool():
    wl = W.decode_workloads()["paged_decode_b64_l1m"]
    t = wl.page_table()
    off, rows = wl.row_offsets()
    assert t.shape == (64, (1 << 20) // 4096)
    assert sorted(t.ravel().tolist()) == list(range(rows // 4096))   # every page used once
    small = W.DecodeWorkload("pt", np.array([1948, 412]), "F", page_rows=512, room=100)  # capacities 2048, 512
    ts = small.page_table()
    need = (np.array([1948, 412]) + 100 + 511) // 512
    assert ts.shape == (2, need.max())
    used = np.concatenate([ts[b, :n] for b, n in enumerate(need)])
    assert sorted(used.tolist()) == list(range(need.sum()))
    with pytest.raises(AssertionError):  # sequences that do not start on a page boundary
        W.DecodeWorkload("pt2", np.array([5000, 12]), "F", page_rows=512).page_table()


def test_capacity_rows_leave_room_for_appends():
    wl = W.decode_workloads()["ratio2_decode_b64_l1m"]
    off, rows = wl.row_offsets()
    assert (np.diff(off) == (1 << 20) + 1024).all() and rows == 64 * ((1 << 20) + 1024)


@pytest.mark.parametrize("pattern,rescan,acts", [
    ("FRRU", False, ["scan", "reindex", "reindex", "reuse"]),
    ("FRUFR", False, ["scan", "reindex", "reuse", "reindex", "reindex"]),
    ("FRUFR", True, ["scan", "reindex", "reuse", "scan", "reindex"]),
])
def test_layer_plans(pattern, rescan, acts):
    plan = layer_plan(pattern, rescan)
    assert [a for *_, a in plan] == acts
    if pattern == "FRUFR":  # layers 3 and 4 use the second Full layer's caches
        assert [f for _, _, f, _ in plan] == [0, 0, 0, 1, 1]


def test_layer_plan_rejects_bad_patterns():
    for bad in ("RF", "UF", "FX"):
        with pytest.raises(ValueError):
            layer_plan(bad)


def test_decode_grouped_rejects_other_schedules():
    """Grouped layer order is for plain decode steps (checked before any device memory is taken)."""
    with pytest.raises(ValueError):
        DecodeStep("FR", 4, 8192, groups=2)                      # concurrent steps overlap layers instead
    with pytest.raises(ValueError):
        DecodeStep("FR", 4, 8192, concurrent=False, groups=5)    # more groups than sequences
    with pytest.raises(ValueError):
        DecodeStep("FR", 4, 8192, concurrent=False, groups=2, queries=8)


def test_deferred_copy_gates():
    """The layers that must wait for the previous step's last-layer copy: the
    last layer, and the layer whose Top-k tensor a final Reuse layer shares."""
    from long_context_decode_csa2_b200.decode import layer_plan

    assert bench.deferred_copy_gates(layer_plan("FRRU")) == {3, 2}
    assert bench.deferred_copy_gates(layer_plan("FRUU")) == {3, 1}
    assert bench.deferred_copy_gates(layer_plan("FRURU" * 4)) == {19, 18}
    assert bench.deferred_copy_gates(layer_plan("FRRR")) == {3}
    assert bench.deferred_copy_gates(layer_plan("F")) == {0}
    assert bench.deferred_copy_gates(layer_plan("FU")) == {1, 0}
    assert bench.deferred_copy_gates(layer_plan("FRFU", full_rescan=True)) == {3, 2}
