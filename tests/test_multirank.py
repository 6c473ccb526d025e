"""The multi-rank (torchrun) bookkeeping of bench.py, run as two gloo ranks on
the CPU: each rank decodes its own batch (weak scaling, no data-path
exchange), timings are reduced as the maximum over ranks, and the job
throughput counts every rank's queries.  The decode itself is the oracle here
(no GPU in these tests); the GPU path is the same per-rank code."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle
import synth.workloads as W

WORLD = 2


def small_workload():
    return W.DecodeWorkload("multirank_small", np.array([1500, 2048]), "FRRU", P=64, k=64, needles=4)


def rank_decode(wl):
    layers = [W.layer_inputs_host(wl, l) for l in range(len(wl.pattern))]
    caches = [W.full_cache_host(wl, f, layers[f]["q_codes"], layers[f]["q_scales"]) for f in wl.full_layers()]
    off = caches[0]["seq_row_off"]
    res = oracle.decode_step(wl.pattern, caches, off, wl.lengths.astype(np.int32), layers, wl.P, wl.k,
                             1 / math.sqrt(512), nthreads=1)
    return caches[0]["idx_codes"], res


def _worker(rank, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(WORLD))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=120))
    try:
        wl = bench.rank_workload(small_workload(), rank)
        codes, res = rank_decode(wl)
        fake_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        ms = bench.max_over_ranks(fake_ms, torch.device("cpu"), WORLD)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), seed=wl.seed, ms=ms,
                 codes_sum=np.int64(codes.astype(np.int64).sum()),
                 topk=np.stack([t for t in res["topk"]]), out=np.stack(res["out"]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_run_independent_batches(tmp_path):
    mp.start_processes(_worker, args=(_free_port(), str(tmp_path)), nprocs=WORLD, start_method="spawn", join=True)
    r = [np.load(tmp_path / f"rank{i}.npz") for i in range(WORLD)]
    # timings: every rank reports the slowest rank's time
    assert float(r[0]["ms"]) == float(r[1]["ms"]) == 15.0
    # weak scaling: distinct seeds, so the ranks hold different caches
    assert int(r[0]["seed"]) != int(r[1]["seed"])
    assert int(r[0]["codes_sum"]) != int(r[1]["codes_sum"])
    # no exchange: each rank's result equals a single-process decode of its batch
    for rank in range(WORLD):
        _, ref = rank_decode(bench.rank_workload(small_workload(), rank))
        np.testing.assert_array_equal(r[rank]["topk"], np.stack(ref["topk"]))
        np.testing.assert_array_equal(r[rank]["out"], np.stack(ref["out"]))


def test_job_throughput_counts_every_rank():
    assert bench.job_throughput(1, 64, 1.0) == pytest.approx(64000.0)
    assert bench.job_throughput(8, 64, 2.0) == pytest.approx(256000.0)
    assert bench.max_over_ranks(3.5, torch.device("cpu"), 1) == 3.5


def test_reference_arm_runs_on_rank0_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        workload = "tiny_decode_b1_l8192"
        steps = 1
        warmup = 0

    assert bench.run_reference(Args()) is None
    assert capsys.readouterr().out == ""


# --- context-parallel exchange: one sequence split over two gloo ranks ---

def _cp_worker(rank, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(WORLD))
    import datetime

    from long_context_decode_csa2_b200.cp import dist_gather, shard_bounds

    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=120))
    try:
        wl = W.DecodeWorkload("cp_gloo", np.array([6001]), "F", P=64, k=64, needles=4)
        L0 = W.layer_inputs_host(wl, 0)
        c = W.full_cache_host(wl, 0, L0["q_codes"], L0["q_scales"])
        bounds = shard_bounds(wl.lengths, WORLD)
        lo, hi = int(bounds[rank, 0]), int(bounds[rank + 1, 0])
        # this rank's own winners over its range (the oracle stands in for the GPU calls here)
        _, top, sc = oracle.index_full(c["idx_codes"][lo:hi], c["idx_scales"][lo:hi], L0["q_codes"], L0["q_scales"],
                                       L0["w"], np.array([0]), np.array([hi - lo], np.int32), wl.P, wl.k,
                                       want_scores=True)
        keys = np.array([oracle.rank_key(sc[0, t]) if t >= 0 else 0 for t in top[0]], np.uint32)
        ids = np.where(top[0] >= 0, top[0] + lo, -1).astype(np.int64)
        g_keys = dist_gather()([torch.from_numpy(keys.view(np.int32).astype(np.int64))])
        g_ids = dist_gather()([torch.from_numpy(ids)])
        np.savez(os.path.join(out_dir, f"cp{rank}.npz"), keys=g_keys.numpy(), ids=g_ids.numpy(), bounds=bounds)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_context_parallel_exchange_two_gloo_ranks(tmp_path):
    """Each rank's Top-k over its shard, all-gathered in rank order, holds
    the whole sequence's Top-k: merging the union by (key desc, position
    asc) equals the single-process selection."""
    mp.start_processes(_cp_worker, args=(_free_port(), str(tmp_path)), nprocs=WORLD, start_method="spawn", join=True)
    r = [np.load(tmp_path / f"cp{i}.npz") for i in range(WORLD)]
    assert np.array_equal(r[0]["keys"], r[1]["keys"]) and np.array_equal(r[0]["ids"], r[1]["ids"])
    b = r[0]["bounds"]
    assert b[0, 0] == 0 and b[-1, 0] == 6001 and b[1, 0] % 8 == 0
    keys = (r[0]["keys"].astype(np.int64) & 0xFFFFFFFF).ravel()
    ids = r[0]["ids"].ravel()
    assert (np.diff(ids[ids >= 0]) > 0).all()  # shard order = position order
    ok = ids >= 0
    merged = oracle.topk(keys[ok].astype(np.uint32), ids[ok], 64)
    wl = W.DecodeWorkload("cp_gloo", np.array([6001]), "F", P=64, k=64, needles=4)
    L0 = W.layer_inputs_host(wl, 0)
    c = W.full_cache_host(wl, 0, L0["q_codes"], L0["q_scales"])
    _, whole, _ = oracle.index_full(c["idx_codes"], c["idx_scales"], L0["q_codes"], L0["q_scales"], L0["w"],
                                    np.array([0]), np.array([6001], np.int32), 64, 64)
    assert merged.tolist() == whole[0].tolist()


def test_shard_bounds_cover_each_sequence_in_whole_blocks():
    from long_context_decode_csa2_b200.cp import shard_bounds

    L = np.array([0, 7, 8, 1000, 1 << 20, 33001])
    for G in (1, 2, 3, 8):
        b = shard_bounds(L, G)
        assert b.shape == (G + 1, len(L))
        assert (b[0] == 0).all() and (b[-1] == L).all() and (np.diff(b, axis=0) >= 0).all()
        assert (b[1:-1] % 8 == 0).all()
        assert (np.diff(b, axis=0).max(axis=0) <= L // G + 8).all()
