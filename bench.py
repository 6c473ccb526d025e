"""Benchmark of the CSA2 decode step (default: batch 64, L = 2^20, layers F R R U).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-cpu-baseline]

One step = the whole hot path for one decode token per sequence: the Full
layer's full-context FP4 scan + block-max pool + Top-512, two Reindex layers,
one Reuse layer, and four sparse attentions (MXFP4 selection + FP8 window).
Inputs are synthetic and already resident in HBM; the scan alone streams
4.56 GB per step, more than L2, so no extra L2 flush is needed.  Under
torchrun each rank runs its own batch of 64 different sequences (weak scaling,
no data-path collective); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode queries/sec at L=1M batch 64; achieved HBM GB/s as % of B200 peak"
NOMINAL_HBM_GBS = 8000.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="long_decode_b64_l1m")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--groups", type=lambda v: [int(x) for x in v.split(",") if x], default=[2, 4],
                    help="group counts of the grouped layer-order step also timed (comma list; empty: none)")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--batch", type=int, default=0, help="override the batch size (small profiling captures)")
    ap.add_argument("--no-graph", action="store_true",
                    help="time eager steps instead of replays of one captured CUDA graph")
    ap.add_argument("--schedule", choices=["layer", "concurrent"], default="layer",
                    help="the timed step: every call in layer order on one stream (the order a model runs; "
                         "default), or the tail of every layer overlapped on side streams (needs every layer's "
                         "inputs up front); the other one is timed as well and reported beside it")
    ap.add_argument("--sequential", action="store_true", help="the same as --schedule layer")
    ap.add_argument("--context", type=int, default=0,
                    help="override every sequence's length (small profiling captures of the attention)")
    ap.add_argument("--full-rescan", action="store_true",
                    help="every Full layer scans its whole context and rebuilds the pool (default: only the first)")
    ap.add_argument("--peaks", action="store_true",
                    help="measure the roofline denominators a copy and a GEMM do not give: read-only HBM stream "
                         "(128-bit loads, bulk copies), tcgen05 FP4 rate at N = 16 and 128, FP64 FMA rate")
    ap.add_argument("--cp", type=int, default=0,
                    help="context-parallel step over this many shards of every sequence: one per rank under "
                         "torchrun, all in this process on one GPU")
    return ap.parse_args()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def deferred_copy_gates(plan) -> set:
    """Layers of a decode step that overwrite what the previous step's last
    layer copies out (its attention output and Top-k): the last layer itself
    and, when it reuses a Top-k, the latest earlier layer that selected one
    (a Reuse layer's Top-k is that layer's tensor).  plan: [(layer, mode,
    full_index, action)] as decode.layer_plan returns."""
    last = plan[-1][0]
    writer = last
    if plan[-1][3] == "reuse":
        writer = max(layer for layer, _, _, act in plan if act != "reuse" and layer < last)
    return {last, writer}


def algorithmic_bytes(wl, full_rescan=False):
    """Per step, from the method's own reads (no scratch traffic): each
    scanning Full layer L*68 B; each layer that selects inside the pool (a
    Reindex layer, or a later Full layer under the pages' plan)
    min(16384, 8*ceil(L/8))*68 B; each attention 512*272 + 128*512 B.  The
    scanning Full layer's own Top-512, taken by re-scoring the positions of
    its best 512 blocks (8*512*68 B per sequence), is an implementation step
    and not counted."""
    L = wl.lengths.astype(np.int64)
    n_scan = sum(1 for _, m in enumerate(wl.pattern) if m == "F")
    # pool-scored layers: Reindex, and the Full layers after the first unless they rescan
    n_pool = sum(1 for m in wl.pattern if m == "R") + (0 if full_rescan else max(0, n_scan - 1))
    # only the first Full layer scans (default plan); with full_rescan every one does
    scan = int((L * 68).sum()) * (n_scan if full_rescan else 1)
    # a verification step scores and attends per query, but reads each
    # sequence's indexer K once
    Lq = wl.verify_queries()[1].astype(np.int64) if wl.queries_per_seq else L
    pooled = np.minimum(wl.P * 8, (Lq + 7) // 8 * 8)
    pool = int((pooled * 68).sum()) * n_pool
    attn = len(Lq) * (wl.k * 272 + 128 * 512) * len(wl.pattern)
    # ratio 2: per Full layer one raw token + logit per sequence, W_idx, and
    # one 340-byte entry per sequence every second step
    append = n_scan * (wl.B * (512 * 2 + 4) + 512 * 128 * 4 + wl.B * 340 // 2) if wl.ratio == 2 else 0
    return dict(scan=scan, pool=pool, attn=attn, append=append, total=scan + pool + attn + append, n_full=n_scan)


class ClockSampler:
    """nvidia-smi clocks during the timed region (median SM MHz, reasons)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = tempfile.mktemp(suffix=".csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------
# oracle timing (CPU baseline and the reference arm)
# ----------------------------------------------------------------------------

def oracle_sample_inputs(wl, layers, caches_dev, seqs):
    """Host copies of the sampled sequences' cache rows and per-layer inputs."""
    import torch

    off = wl.row_offsets()[0]
    m = wl.queries_per_seq
    table = wl.page_table() if wl.page_rows else None
    out = []
    for b in seqs:
        o, L = int(off[b]), int(wl.lengths[b])
        if table is None:
            rows = slice(o, o + L)
        else:  # the sequence's rows through its page table
            t = np.arange(L, dtype=np.int64)
            rows = torch.from_numpy(table[b][t // wl.page_rows].astype(np.int64) * wl.page_rows
                                    + t % wl.page_rows).to(caches_dev[0]["idx_codes"].device)
        ch = [dict(idx_codes=c["idx_codes"][rows].cpu().numpy(), idx_scales=c["idx_scales"][rows].cpu().numpy(),
                   main_codes=c["main_codes"][rows].cpu().numpy(),
                   main_scales=c["main_scales"][rows].cpu().numpy()) for c in caches_dev]
        rows = slice(b * m, (b + 1) * m) if m else slice(b, b + 1)
        lb = [{k: v[rows] for k, v in Ld.items()} for Ld in layers]
        vis = wl.verify_queries()[1][rows] if m else np.array([L], np.int32)
        out.append((ch, vis, lb))
    torch.cuda.synchronize()
    return out


def time_oracle(wl, samples, nthreads, jobs=None):
    """Runs the oracle's decode step (one query: every layer of the pattern
    for one sequence) once per job, `nthreads` jobs at a time on the host
    cores; job j uses sample j % len(samples).  Returns (seconds, queries)."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle

    toks = None
    if wl.ratio == 2:
        import synth

        toks = [dict(raw=synth.normal_bf16(wl.seed, synth.T_RAW, 0, f, 512).reshape(1, 512),
                     logit=synth.normal_f32(wl.seed, synth.T_LOGITS, 0, f, 1),
                     w_idx=synth.normal_f32(wl.seed, synth.T_WIDX, 0, f, 512 * 128, log2_div=13).reshape(512, 128))
                for f in wl.full_layers()]

    def one(j):
        ch, vis, lb = samples[j % len(samples)]
        if toks:  # ratio 2: the step's append (a pending token completes an entry)
            for t in toks:
                pend = [dict(raw=t["raw"][0], logit=float(t["logit"][0]), idx=None)]
                oracle.compress_stream(pend, t["raw"], t["logit"], np.array([0, 1]), w_idx=t["w_idx"], nthreads=1)
        oracle.decode_step(wl.pattern, ch, np.zeros(len(vis), np.int64), np.asarray(vis, np.int32), lb, wl.P, wl.k,
                           1 / math.sqrt(512), nthreads=1)

    n = len(samples) if jobs is None else jobs
    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=nthreads) as ex:
        list(ex.map(one, range(n)))
    return time.perf_counter() - t0, n * max(1, wl.queries_per_seq)


def host_cores():
    """Host cores this process may run on (the oracle baselines use them all)."""
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def single_thread_oracle(wl, samples):
    """The oracle on one host thread (one query of the first sample), and the
    host's core count, for the cpu_baseline object."""
    secs, nq = time_oracle(wl, samples[:1], 1, jobs=1)
    return {"single_thread": {"value": nq / secs, "unit": "queries/s", "sample": f"{nq} query, one thread, "
                              f"{secs:.2f} s"}, "host_cores": host_cores()}


# ----------------------------------------------------------------------------

def decode_config(wl, l2_bytes, concurrent, graph=True, full_rescan=False):
    """The `config` object of a decode line (both arms)."""
    extra = ({"ratio": 2, "append": "one raw token per sequence per Full layer per step (csa2_compress_stream, "
                                    "W_idx projection)"} if wl.ratio == 2 else {})
    if wl.page_rows:
        extra["paged"] = "%d-row pages, page table shuffled over the whole cache pool" % wl.page_rows
    if wl.pattern.count("F") > 1:
        extra["full_layers"] = "every Full layer scans" if full_rescan else "the first Full layer scans, the others select in its pool"
    if wl.queries_per_seq:
        extra["queries_per_seq"] = wl.queries_per_seq
        extra["verify"] = ("candidate i sees all entries but the last %d - i; value counts candidate queries"
                           % (wl.queries_per_seq - 1))
    return {"workload": wl.name, "batch_per_gpu": wl.B, "context": wl.max_len, "layers": wl.pattern, **extra,
            "pool_blocks": wl.P, "topk": wl.k, "window": 128,
            "l2": "no flush: inputs larger than L2 (%.2f GB read per step)" % (l2_bytes / 1e9),
            "schedule": ("concurrent tail (side streams: every layer's inputs given up front)" if concurrent
                         else "layer order (one stream)") + (", one CUDA graph per step" if graph else "")}


def rank_workload(wl, rank):
    """Weak scaling: rank r runs its own batch of the same shape, drawn with
    seed + 1000 r, so no two ranks share a sequence and no data crosses ranks."""
    import synth.workloads as W

    if rank == 0:
        return wl
    return dataclasses.replace(wl, seed=wl.seed + 1000 * rank)


def max_over_ranks(x, device, world):
    """The slowest rank's value (timings are reported as the max over ranks)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, batch_per_rank, ms_per_step):
    """Whole-job queries/s: every rank decodes its batch once per step."""
    return world * batch_per_rank / (ms_per_step * 1e-3)


def build_workload(wl, rank, device):
    import torch

    import synth.workloads as W
    from long_context_decode_csa2_b200 import csa2 as C
    from long_context_decode_csa2_b200.decode import FullCache

    wl = rank_workload(wl, rank)
    m = wl.queries_per_seq
    if m:  # one set of layer inputs per candidate query; needles aimed at each sequence's first one
        wq = dataclasses.replace(wl, lengths=wl.verify_queries()[1].astype(np.int64), queries_per_seq=0,
                                 seed=wl.seed + 7)
        layers = [W.layer_inputs_host(wq, l) for l in range(len(wl.pattern))]
    else:
        layers = [W.layer_inputs_host(wl, l) for l in range(len(wl.pattern))]
    first = slice(None, None, m) if m else slice(None)
    caches_dev = [W.full_cache_device(wl, f, layers[f]["q_codes"][first], layers[f]["q_scales"][first], device)
                  for f in wl.full_layers()]
    caches = [FullCache(C.cache(c["idx_codes"], c["idx_scales"]), C.cache(c["main_codes"], c["main_scales"]))
              for c in caches_dev]

    def to_dev(a):
        a = np.ascontiguousarray(a)
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
        return torch.from_numpy(a).to(device)

    keys = ("q", "q_codes", "q_scales", "w", "win", "win_scale", "win_len")
    layers_dev = [{k: to_dev(L[k]) for k in keys} for L in layers]
    off = caches_dev[0]["seq_row_off"]
    if wl.page_rows:  # the same cache pool read through a shuffled page table
        from long_context_decode_csa2_b200 import csa2 as C2

        off_d = C2.PageTable(to_dev(wl.page_table()), wl.page_rows)
    else:
        off_d = to_dev(off)
    return wl, layers, caches_dev, caches, layers_dev, off_d, to_dev(wl.lengths.astype(np.int32))


def new_token_inputs(wl, device):
    """Ratio 2: per Full layer the step's new raw token of every sequence
    (bf16), its logit and the layer's W_idx (host arrays and device copies)."""
    import synth

    host, devs = [], []
    for i, f in enumerate(wl.full_layers()):
        h = dict(raw=synth.normal_bf16(wl.seed, synth.T_RAW, 0, f, wl.B * 512).reshape(wl.B, 512),
                 logit=synth.normal_f32(wl.seed, synth.T_LOGITS, 0, f, wl.B) * 2,
                 w_idx=synth.normal_f32(wl.seed, synth.T_WIDX, 0, f, 512 * 128, log2_div=13).reshape(512, 128))
        host.append(h)
        d = {}
        import torch

        for k, v in h.items():
            v = np.ascontiguousarray(v)
            d[k] = (torch.from_numpy(v.view(np.int16)).to(device).view(torch.bfloat16) if v.dtype == np.uint16
                    else torch.from_numpy(v).to(device))
        devs.append(d)
    return host, devs


def run_ours(args):
    import torch
    import torch.distributed as dist

    import synth.workloads as W
    from long_context_decode_csa2_b200 import csa2 as C
    from long_context_decode_csa2_b200.decode import DecodeStep

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600), device_id=device)

    wl = W.decode_workloads()[args.workload]
    if args.batch:
        wl = dataclasses.replace(wl, name=wl.name + f"_b{args.batch}", lengths=wl.lengths[:args.batch])
    if args.context:
        wl = dataclasses.replace(wl, name=wl.name + f"_l{args.context}", lengths=np.full(wl.B, args.context),
                                 needles=min(wl.needles, max(1, args.context // 1024)))
    wl, layers, caches_dev, caches, layers_dev, off_d, len_d = build_workload(wl, rank, device)
    C.lib()
    m = wl.queries_per_seq
    n_q = wl.B * m if m else wl.B  # queries per step on this rank
    concurrent = args.schedule == "concurrent" and not args.sequential
    step = DecodeStep(wl.pattern, wl.B, wl.max_len + wl.room, wl.P, wl.k, concurrent=concurrent,
                      ratio=wl.ratio, queries=n_q if m else None, full_rescan=args.full_rescan)
    vq = {}
    if m:
        q_off_h, q_vis_h = wl.verify_queries()
        vq = dict(q_off=torch.from_numpy(q_off_h).to(device), q_vis=torch.from_numpy(q_vis_h).to(device))
    stream = torch.cuda.current_stream()
    toks_host, toks_dev = new_token_inputs(wl, device) if wl.ratio == 2 else (None, None)
    len0 = len_d.clone()
    if wl.ratio == 2 and max(args.steps, args.e2e_steps + 1, args.warmup + 3) > 2 * wl.room:
        raise SystemExit(f"at most {2 * wl.room} steps per timed phase fit the caches' spare rows")

    def reset_lengths():
        """Ratio 2: every phase starts from the initial lengths (the steps
        append into the spare rows again)."""
        if wl.ratio == 2:
            len_d.copy_(len0)
            for pair in step.pairs:
                pair.pend_n.zero_()

    # events around every C-ABI call of the timed region, on the stream the
    # call runs on; csa2_index_full (full-context scan, block max, pool,
    # Top-512) is the dominant call and runs alone.  The other calls overlap
    # one another on side streams, so their times include that sharing.
    n_layers = len(wl.pattern)
    ev_calls = {}
    recording = [False]

    def hook(name, phase, on_stream):
        if not recording[0]:
            return
        lst = ev_calls.setdefault(name, [])
        if phase == "begin":
            lst.append([torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)])
            lst[-1][0].record(on_stream)
        else:
            lst[-1][1].record(on_stream)

    step.hook = hook

    def run_step(record=False):
        recording[0] = record
        step.run(caches, off_d, len_d, layers_dev, new_tokens=toks_dev, **vq)
        recording[0] = False

    for _ in range(args.warmup):
        run_step()
    torch.cuda.synchronize()
    if step.device_flags():
        raise RuntimeError("device status flags set during warm-up")

    # the timed steps replay one captured CUDA graph of the whole step (the
    # default); the per-call times come from a separate eager pass
    graph = None
    if not args.no_graph:
        graph = step.capture(caches, off_d, len_d, layers_dev, new_tokens=toks_dev, **vq)
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
    reset_lengths()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        time.sleep(0.5)  # let the sampler start before the timed region
        t0.record(stream)
        for _ in range(args.steps):
            if graph is not None:
                graph.replay()
            else:
                run_step(record=True)
        t1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = t0.elapsed_time(t1) / args.steps
    reset_lengths()
    # the same step in the other schedule (layer order: the order a model whose
    # layer inputs depend on the previous layer imposes; concurrent: the tails
    # of all layers overlapped, possible only with every layer's inputs given
    # up front), and layer order per group of sequences, each replayed from a
    # graph
    def schedule_ms(conc, groups=1):
        step_seq = DecodeStep(wl.pattern, wl.B, wl.max_len + wl.room, wl.P, wl.k, concurrent=conc, ratio=wl.ratio,
                              queries=n_q if m else None, full_rescan=args.full_rescan, groups=groups)
        step_seq.run(caches, off_d, len_d, layers_dev, new_tokens=toks_dev, **vq)
        g_seq = step_seq.capture(caches, off_d, len_d, layers_dev, new_tokens=toks_dev, **vq)
        for _ in range(3):
            g_seq.replay()
        reset_lengths()
        torch.cuda.synchronize()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for _ in range(args.steps):
            g_seq.replay()
        s1.record(stream)
        torch.cuda.synchronize()
        t = max_over_ranks(s0.elapsed_time(s1) / args.steps, device, world)
        if step_seq.device_flags():
            raise RuntimeError("device status flags set in the layer-order step")
        del g_seq, step_seq
        reset_lengths()
        return t

    other_ms = None
    group_ms = {}
    if graph is not None:
        other_ms = schedule_ms(not concurrent)
        # layer order per group of sequences (groups overlap each other)
        if not m and isinstance(off_d, torch.Tensor):
            for G in args.groups:
                if 1 < G <= wl.B:
                    group_ms[G] = schedule_ms(False, G)
    if graph is not None:
        for _ in range(min(args.steps, 50)):
            run_step(record=True)
        torch.cuda.synchronize()
    per_call = {name: sum(a.elapsed_time(b) for a, b in lst) / len(lst) for name, lst in ev_calls.items()}
    scan_call = "csa2_index_multi" if m else "csa2_index_full"
    full_ms = [a.elapsed_time(b) for a, b in ev_calls[scan_call]]
    ms = max_over_ranks(ms, device, world)

    # end to end: host (pinned) query inputs -> device, step, outputs -> host
    keys_in = ("q", "q_codes", "q_scales", "w")
    host_in = [{k: torch.from_numpy(np.ascontiguousarray(
        L[k].view(np.int16) if L[k].dtype == np.uint16 else L[k])).pin_memory() for k in keys_in} for L in layers]
    h2d = sum(t.numel() * t.element_size() for L in host_in for t in L.values())
    # ratio 2: the new raw tokens and logits come from the host every step
    tok_in = ([{k: torch.from_numpy(np.ascontiguousarray(h[k].view(np.int16) if h[k].dtype == np.uint16 else h[k]))
                .pin_memory() for k in ("raw", "logit")} for h in toks_host] if toks_host else [])
    h2d += sum(t.numel() * t.element_size() for T in tok_in for t in T.values())
    full_of_layer = {l: i for i, l in enumerate(wl.full_layers())}
    out_host = torch.empty(step.out.shape, dtype=torch.float32).pin_memory()
    top_host = torch.empty((n_layers, n_q, wl.k), dtype=torch.int32).pin_memory()
    d2h = out_host.numel() * 4 + top_host.numel() * 4
    # inputs go in on one copy stream, results come out on another
    h2d_stream, d2h_stream = torch.cuda.Stream(device=device), torch.cuda.Stream(device=device)

    def copy_now(layer):
        with torch.cuda.stream(d2h_stream):
            out_host[layer].copy_(step.out[layer], non_blocking=True)
            top_host[layer].copy_(step.topk[layer], non_blocking=True)

    last_layer = n_layers - 1

    def copy_out(layer, ev):
        if layer == last_layer:  # leaves while the next step starts (see e2e_step)
            return
        d2h_stream.wait_event(ev)
        copy_now(layer)

    # The last layer's results are copied out at the start of the next step,
    # beside its scan; of that step only the layers that overwrite those
    # tensors wait for the copy.
    gated = deferred_copy_gates(step.plan)

    # Inputs are double-buffered: every step copies the NEXT step's inputs
    # from pinned host memory into the other buffer set while it computes, so
    # the copy overlaps the step (a serving loop prefetches its next batch the
    # same way); each layer's results leave as soon as its attention is done.
    bufs = [layers_dev, [{k: t.clone() for k, t in L.items()} for L in layers_dev]]
    tbufs = [toks_dev, [{k: t.clone() for k, t in T.items()} for T in toks_dev] if toks_dev else None]

    def copy_in(p):
        for l in range(n_layers):
            for k in keys_in:
                dst = bufs[p][l][k]
                (dst.view(torch.int16) if dst.dtype == torch.bfloat16 else dst).copy_(host_in[l][k], non_blocking=True)
            if tok_in and l in full_of_layer:
                for k, src in tok_in[full_of_layer[l]].items():
                    dst = tbufs[p][full_of_layer[l]][k]
                    (dst.view(torch.int16) if dst.dtype == torch.bfloat16 else dst).copy_(src, non_blocking=True)

    def e2e_step(p):
        cur = torch.cuda.current_stream()
        start = torch.cuda.Event()
        start.record(cur)
        h2d_stream.wait_stream(cur)  # the step that last read buffer 1 - p has finished
        with torch.cuda.stream(h2d_stream):
            copy_in(1 - p)
        # the previous step's last layer results (that step has completed)
        d2h_stream.wait_stream(cur)
        copy_now(last_layer)
        out_gone = torch.cuda.Event()
        out_gone.record(d2h_stream)
        ready = [out_gone if layer in gated else start for layer in range(n_layers)]
        step.run(caches, off_d, len_d, bufs[p], ready=ready, on_layer_done=copy_out, new_tokens=tbufs[p], **vq)
        cur.wait_stream(d2h_stream)  # this step's copies of its other layers are on the host
        cur.wait_stream(h2d_stream)

    e2e_graphs = None
    if graph is not None:  # the whole end-to-end step (copies included) as one graph per buffer set
        e2e_graphs = []
        for p in (0, 1):
            e2e_step(p)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            cap = torch.cuda.Stream(device=device)
            cap.wait_stream(stream)
            with torch.cuda.graph(g, stream=cap, capture_error_mode="thread_local"):
                e2e_step(p)
            stream.wait_stream(cap)
            e2e_graphs.append(g)
        torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    reset_lengths()
    copy_in(0)  # the first step's inputs (each timed step copies the next step's)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(args.e2e_steps):
        if e2e_graphs is not None:
            e2e_graphs[i % 2].replay()
        else:
            e2e_step(i % 2)
    d2h_stream.wait_stream(stream)  # the last step's last layer
    copy_now(last_layer)
    stream.wait_stream(d2h_stream)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / args.e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, device, world)
    flags = step.device_flags()

    ab = algorithmic_bytes(wl, args.full_rescan)
    peak, peak_kind = measured_peaks()
    full_avg = sum(full_ms) / len(full_ms)
    # the dominant call's algorithmic bytes: its scan (one Full layer's)
    full_bytes = ab["scan"] // (ab["n_full"] if args.full_rescan else 1)
    achieved = full_bytes / (full_avg * 1e-3) / 1e9
    traffic = None
    prof = os.path.join(ROOT, "profiles", "index_full_traffic.json")
    if os.path.exists(prof):
        try:
            traffic = json.load(open(prof)).get(wl.name)
        except Exception:
            traffic = None

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        nthreads = host_cores()
        seqs = list(range(0, wl.B, max(1, wl.B // nthreads)))[:nthreads]
        samples = oracle_sample_inputs(wl, layers, caches_dev, seqs)
        jobs = 3 * len(samples)
        secs, nq = time_oracle(wl, samples, nthreads, jobs=jobs)
        cpu = {"value": nq / secs, "unit": "queries/s", "cores": min(nthreads, len(samples)), "kind": "oracle",
               "sample": f"{nq} queries (each sequence {seqs} of the batch decoded 3 times; L={wl.max_len}, "
                         f"one full {wl.pattern} step per query, one host thread per query); {secs:.1f} s wall, "
                         f"{secs * min(nthreads, len(samples)):.0f} core-seconds",
               **single_thread_oracle(wl, samples)}

    if rank == 0:
        launches_per_step = 0
        for _, m in enumerate(step.plan):
            act = m[3]
            # index_full: prep, scan, pool select, pool score, Top-k select;
            # reindex: pool score, select; attention: one kernel
            launches_per_step += {"scan": 5, "reindex": 2, "reuse": 0}[act] + 1
        launches_per_step += len(step.pairs)  # ratio 2: one append per Full layer
        res = {
            "metric": METRIC,
            "value": job_throughput(world, n_q, ms),
            "unit": "queries/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "int32+f64 indexer, f16 tensor-core attention (f32 accumulate)",
            "data": "synthetic",
            "config": decode_config(wl, ab["total"], concurrent, graph is not None, args.full_rescan),
            "tokens_per_s": job_throughput(world, n_q, ms),
            "hbm_algorithmic_gbs": ab["total"] / (ms * 1e-3) / 1e9,
            "hbm_frac_of_8tbs": ab["total"] / (ms * 1e-3) / 1e9 / NOMINAL_HBM_GBS,
            "roofline": {"kernel": scan_call + " (scan + block max + pool + Top-512)", "bound": "hbm",
                         "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                         "peak_kind": peak_kind, "traffic": traffic, "algorithmic_bytes": full_bytes,
                         "avg_ms": full_avg},
            "cpu_baseline": cpu,
            "e2e": {"value": job_throughput(world, n_q, e2e_ms), "unit": "queries/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": launches_per_step * args.steps,
            "per_call_ms": per_call,
            ("layer_order_graph" if concurrent else "concurrent_layers_graph"):
                (None if other_ms is None else
                 {"ms_per_step": other_ms, "queries_per_s": job_throughput(world, n_q, other_ms)}),
            "layer_order_groups_graph": {str(G): {"ms_per_step": t, "queries_per_s": job_throughput(world, n_q, t)}
                                         for G, t in group_ms.items()},
            "clocks": clk.summary(),
            "device_flags": flags,
        }
        print(json.dumps(res))
    if world > 1:
        dist.destroy_process_group()


def prefill_cpu_baseline(pw, seed, nthreads, nq=64, n_comp=8192):
    """The oracle's prefill step estimated from a bounded sample: the
    indexer and attention of `nq` queries spread over the chunk (each sees
    about 131072 entries) and the compression of `n_comp` raw tokens (W_idx
    projection), scaled to T queries and n_raw tokens.  The oracle's cache
    rows are drawn by the input generator, not taken from the GPU."""
    import oracle
    import synth

    n_raw, T, ratio, P, k = pw.n_raw, pw.T, pw.ratio, pw.P, pw.k
    n_ent = n_raw // ratio
    ic, isc = synth.mxfp4_rows(seed, synth.T_IDXK_CODES, synth.T_IDXK_SCALES, 0, 0, 0, n_ent, 128)
    mc, msc = synth.mxfp4_rows(seed, synth.T_MAIN_CODES, synth.T_MAIN_SCALES, 0, 0, 0, n_ent, 512)
    raw_win = synth.e4m3_rows(seed, synth.T_RAWWIN, 0, 0, 0, n_raw)
    q_pos = np.linspace(n_raw - T, n_raw - 1, nq).astype(np.int32)
    qc, qs = synth.mxfp4_rows(seed, synth.T_QIDX_CODES, synth.T_QIDX_SCALES, 0, 0, 0, nq * 4, 128)
    qc, qs = qc.reshape(nq, 4, 64), qs.reshape(nq, 4, 4)
    w = synth.head_weights(seed, 0, 0, nq * 4).reshape(nq, 4)
    q = synth.normal_bf16(seed, synth.T_Q, 0, 0, nq * 16 * 512).reshape(nq, 16, 512)
    raw = synth.normal_bf16(seed, synth.T_RAW, 0, 0, n_comp * 512).reshape(n_comp, 512)
    z = synth.normal_f32(seed, synth.T_LOGITS, 0, 0, n_comp)
    w_idx = synth.normal_f32(seed, synth.T_WIDX, 0, 0, 512 * 128, log2_div=13).reshape(512, 128)
    t0 = time.perf_counter()
    _, top = oracle.index_prefill(ic, isc, 0, n_ent, qc, qs, w, q_pos, ratio, P, k, nthreads=nthreads)
    oracle.attn_prefill(q, q_pos, mc, msc, 0, n_ent, ratio, top, raw_win, float(synth.window_scale(seed, 0, 0)),
                        1 / math.sqrt(512), nthreads=nthreads)
    t1 = time.perf_counter()
    oracle.compress(raw, z, ratio, w_idx=w_idx, nthreads=nthreads)
    t2 = time.perf_counter()
    est = (t1 - t0) * T / nq + (t2 - t1) * n_raw / n_comp
    return {"value": T / est, "unit": "queries/s", "cores": nthreads, "kind": "oracle",
            "sample": f"indexer + attention of {nq} of the {T} queries ({t1 - t0:.1f} s) and compression of "
                      f"{n_comp} of the {n_raw} raw tokens ({t2 - t1:.1f} s), scaled to one whole prefill step "
                      f"({est:.0f} s)"}


def run_prefill(args):
    """Prefill workload: ratio-2 compression of n_raw tokens into a fresh
    cache (with the W_idx projection), the causal indexer for T queries, and
    their sparse attention; one step = those three calls.  Reports prefill
    queries/s and per-call times (compressed tokens/s for the first call)."""
    import torch

    import synth
    import synth.gpu as sg
    import synth.workloads as W
    from long_context_decode_csa2_b200 import csa2 as C

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600), device_id=device)
    pw = W.prefill_workload()
    seed = pw.seed + 1000 * rank
    n_raw, T, ratio, P, k = pw.n_raw, pw.T, pw.ratio, pw.P, pw.k
    n_ent = n_raw // ratio
    rows = (n_ent + 7) // 8 * 8
    raw = torch.empty((n_raw, 512), dtype=torch.bfloat16, device=device)
    sg.normal_bf16_into(raw, seed, synth.T_RAW, 0, 0)
    q = torch.empty((T, 16, 512), dtype=torch.bfloat16, device=device)
    sg.normal_bf16_into(q, seed, synth.T_Q, 0, 0)
    raw_win = torch.empty((n_raw, 512), dtype=torch.uint8, device=device)
    sg.e4m3_rows_into(raw_win, seed, synth.T_RAWWIN, 0, 0, 0, n_raw)
    logits = torch.from_numpy(synth.normal_f32(seed, synth.T_LOGITS, 0, 0, n_raw)).to(device)
    w_idx = torch.from_numpy(synth.normal_f32(seed, synth.T_WIDX, 0, 0, 512 * 128, log2_div=13)).to(device)
    qc, qs = synth.mxfp4_rows(seed, synth.T_QIDX_CODES, synth.T_QIDX_SCALES, 0, 0, 0, T * 4, 128)
    q_codes = torch.from_numpy(np.ascontiguousarray(qc.reshape(T, 4, 64))).to(device)
    q_scales = torch.from_numpy(np.ascontiguousarray(qs.reshape(T, 4, 4))).to(device)
    w = torch.from_numpy(synth.head_weights(seed, 0, 0, T * 4).reshape(T, 4)).to(device)
    win_scale = float(synth.window_scale(seed, 0, 0))
    q_pos = torch.arange(n_raw - T, n_raw, dtype=torch.int32, device=device)
    main = C.cache(torch.zeros((rows, 256), dtype=torch.uint8, device=device),
                   torch.zeros((rows, 16), dtype=torch.uint8, device=device))
    idx = C.cache(torch.zeros((rows, 64), dtype=torch.uint8, device=device),
                  torch.zeros((rows, 4), dtype=torch.uint8, device=device))
    tok_off = torch.tensor([0, n_raw], dtype=torch.int64, device=device)
    row_off = torch.zeros(1, dtype=torch.int64, device=device)
    len_in = torch.zeros(1, dtype=torch.int32, device=device)
    len_out = torch.zeros(1, dtype=torch.int32, device=device)
    pool = torch.empty((T, P), dtype=torch.int32, device=device)
    top = torch.empty((T, k), dtype=torch.int32, device=device)
    out = torch.empty((T, 16, 512), dtype=torch.float32, device=device)
    lse = torch.empty((T, 16), dtype=torch.float32, device=device)
    ws1 = C.workspace(C.csa2_compress_append_workspace_bytes(1), device)
    ws2 = C.workspace(C.csa2_index_prefill_workspace_bytes(T, n_ent, P, k), device)
    ws3 = C.workspace(C.csa2_sparse_attn_prefill_workspace_bytes(T, k), device)
    stream = torch.cuda.current_stream()
    names = ("csa2_compress_append", "csa2_index_prefill", "csa2_sparse_attn_prefill")
    times = {n: [] for n in names}

    dev_in = {"raw": raw, "logits": logits, "q": q, "q_codes": q_codes, "q_scales": q_scales, "w": w,
              "raw_win": raw_win}
    dev_out = {"top": top, "out": out}

    def step(record, x=None, y=None):
        x = x or dev_in
        y = y or dev_out
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)] if record else None
        if record:
            ev[0].record(stream)
        C.csa2_compress_append(main, idx, x["raw"], x["logits"], tok_off, row_off, len_in, len_out, ratio, n_ent, ws1,
                               w_idx=w_idx)
        if record:
            ev[1].record(stream)
        C.csa2_index_prefill(idx, x["q_codes"], x["q_scales"], x["w"], q_pos, 0, n_ent, ratio, P, k, pool, y["top"],
                             ws2)
        if record:
            ev[2].record(stream)
        C.csa2_sparse_attn_prefill(x["q"], q_pos, main, 0, n_ent, ratio, y["top"], x["raw_win"], win_scale,
                                   1 / math.sqrt(512), y["out"], ws3, lse=lse)
        if record:
            ev[3].record(stream)
            for i, n in enumerate(names):
                times[n].append((ev[i], ev[i + 1]))

    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize()
    flags = C.device_status(ws1) | C.device_status(ws2) | C.device_status(ws3)
    if flags:
        raise RuntimeError(f"device status flags {flags} during warm-up")
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        time.sleep(0.5)
        t0.record(stream)
        for _ in range(args.steps):
            step(True)
        t1.record(stream)
        torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, device, world)
    per_call = {n: sum(a.elapsed_time(b) for a, b in v) / len(v) for n, v in times.items()}

    # end to end: every input of the step from pinned host memory (raw tokens,
    # logits, queries and their indexer inputs, the raw FP8 window rows), the
    # outputs (attention output, Top-k) back to the host.  Prefill chunks are
    # independent requests, so, as a serving loop would, each step's inputs
    # are copied in on one copy stream while the previous step computes
    # (double-buffered), and each step's results leave on another while the
    # next one computes; the timed region ends when the last results are on
    # the host.
    host_in = {name: t.cpu().pin_memory() for name, t in dev_in.items()}
    ins = [dev_in, {name: t.clone() for name, t in dev_in.items()}]
    outs = [dev_out, {name: t.clone() for name, t in dev_out.items()}]
    out_h = torch.empty(out.shape, dtype=torch.float32).pin_memory()
    top_h = torch.empty(top.shape, dtype=torch.int32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = out_h.numel() * 4 + top_h.numel() * 4
    e_steps = max(1, min(args.e2e_steps, 10))
    h2d_stream, d2h_stream = torch.cuda.Stream(device=device), torch.cuda.Stream(device=device)

    def copy_in(x):
        with torch.cuda.stream(h2d_stream):
            for name, src in host_in.items():
                x[name].copy_(src, non_blocking=True)

    out_done = [None, None]  # per output set: its last results are on the host
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    copy_in(ins[0])  # the first step's inputs (each step copies the next step's)
    for i in range(e_steps):
        p = i % 2
        stream.wait_stream(h2d_stream)  # this step's inputs are on the device
        if i + 1 < e_steps:
            h2d_stream.wait_stream(stream)  # the step that last read the other input set has finished
            copy_in(ins[1 - p])
        if out_done[p] is not None:
            stream.wait_event(out_done[p])  # the results last written to this output set have left
        step(False, ins[p], outs[p])
        d2h_stream.wait_stream(stream)
        with torch.cuda.stream(d2h_stream):
            out_h.copy_(outs[p]["out"], non_blocking=True)
            top_h.copy_(outs[p]["top"], non_blocking=True)
            out_done[p] = torch.cuda.Event()
            out_done[p].record(d2h_stream)
    stream.wait_stream(d2h_stream)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e_steps, device, world)

    # roofline of the indexer (the dominant call): the causal FP4 score GEMM's
    # useful FLOPs against the FP4 tensor peak at the kernel's MMA shape
    # (kind::mxf4, N = 128), measured here by the peak probe; its time is the
    # exact epilogue's, not the MMAs'
    n_vis = np.minimum(np.arange(n_raw - T, n_raw, dtype=np.int64) + 1, n_raw) // ratio
    flops = float(n_vis.sum()) * 4 * 128 * 2
    fp4_peak, fp4_kind = fp4_peak_tflops()
    achieved = flops / (per_call["csa2_index_prefill"] * 1e-3) / 1e12
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = prefill_cpu_baseline(pw, seed, host_cores())
    if rank == 0:
        print(json.dumps({
            "metric": "prefill queries/sec (ratio-2 compression of 262144 tokens, 4096-query causal chunk)",
            "value": job_throughput(world, T, ms), "unit": "queries/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int32+f64 indexer, f16 tensor-core attention (f32 accumulate)",
            "data": "synthetic",
            "config": {"workload": pw.name, "raw_tokens": n_raw, "entries": n_ent, "queries": T, "pool_blocks": P,
                       "topk": k, "window": 128},
            "compress_tokens_per_s": n_raw / (per_call["csa2_compress_append"] * 1e-3),
            "roofline": {"kernel": "csa2_index_prefill (causal FP4 score GEMM + block max + pool + Top-512)",
                         "bound": "tensor", "achieved": achieved, "peak": fp4_peak, "unit": "TFLOP/s",
                         "frac": achieved / fp4_peak, "peak_kind": fp4_kind,
                         "traffic": None, "note": "bound in fact by the exact CUDA-core epilogue"},
            "cpu_baseline": cpu,
            "e2e": {"value": job_throughput(world, T, e2e_ms), "unit": "queries/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            # compress 1; indexer: visibility, scan, pool select, pool scoring, Top-k select; attention:
            # visibility, attention
            "gpu_launches": 8 * args.steps,
            "per_call_ms": per_call, "clocks": clk.summary(), "device_flags": flags}))
    if world > 1:
        dist.destroy_process_group()


def run_reference(args):
    """The oracle as the reference arm: K timed steps, each one oracle decode
    step over a bounded sample of the workload's sequences on the host cores."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import torch

    import synth.workloads as W

    nthreads = host_cores()
    if args.workload.startswith("prefill"):
        # the oracle's prefill step, estimated from a bounded sample per timed step
        pw = W.prefill_workload()
        runs = [prefill_cpu_baseline(pw, pw.seed, nthreads) for _ in range(max(1, min(args.steps, 3)))]
        value = statistics.median(r["value"] for r in runs)
        ms = 1e3 * pw.T / value
        print(json.dumps({"impl": "reference", "metric": "prefill queries/sec (ratio-2 compression of 262144 tokens, "
                          "4096-query causal chunk)", "value": value, "unit": "queries/s", "n_gpus": world,
                          "steps": len(runs), "warmup": 0, "ms_per_step": ms, "higher_is_better": True,
                          "scaling": "weak", "vs_baseline": None, "dtype": "int32+f64 (CPU oracle)",
                          "data": "synthetic",
                          "config": {"workload": pw.name, "raw_tokens": pw.n_raw, "entries": pw.n_entries,
                                     "queries": pw.T, "pool_blocks": pw.P, "topk": pw.k, "window": 128},
                          "cpu_baseline": dict(runs[0], value=value),
                          "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0,
                                  "d2h_bytes_per_step": 0}}))
        return
    wl = W.decode_workloads()[args.workload]
    on_gpu = torch.cuda.is_available()
    if on_gpu:
        # inputs from the device generator (same bytes as the NumPy generator)
        wl2, layers, caches_dev, _, _, _, _ = build_workload(wl, 0, torch.device("cuda", 0))
        seqs = list(range(min(nthreads, wl.B)))
        samples = oracle_sample_inputs(wl2, layers, caches_dev, seqs)
        del caches_dev
    else:
        # no GPU to generate the full-size caches: shorter contexts (named in the config)
        small = dataclasses.replace(wl, name=wl.name + "_l65536_host", lengths=np.full(nthreads, min(wl.max_len, 65536)))
        wl = small
        m = small.queries_per_seq
        if m:
            wq = dataclasses.replace(small, lengths=small.verify_queries()[1].astype(np.int64), queries_per_seq=0,
                                     seed=small.seed + 7)
            layers = [W.layer_inputs_host(wq, l) for l in range(len(small.pattern))]
        else:
            layers = [W.layer_inputs_host(small, l) for l in range(len(small.pattern))]
        first = slice(None, None, m) if m else slice(None)
        caches = [W.full_cache_host(small, f, layers[f]["q_codes"][first], layers[f]["q_scales"][first])
                  for f in small.full_layers()]
        samples = []
        off = small.row_offsets()[0]
        for b in range(nthreads):
            o, L = int(off[b]), int(small.lengths[b])
            ch = [{k: c[k][o:o + L] for k in ("idx_codes", "idx_scales", "main_codes", "main_scales")} for c in caches]
            rows = slice(b * m, (b + 1) * m) if m else slice(b, b + 1)
            vis = small.verify_queries()[1][rows] if m else np.array([L], np.int32)
            samples.append((ch, vis, [{k: v[rows] for k, v in Ld.items()} for Ld in layers]))
    # one timed step = one query (a full decode step of one sequence); the K
    # steps run nthreads at a time, so K steps take about K/nthreads queries'
    # time (about a minute for K = 400 on 8 cores)
    time_oracle(wl, samples, nthreads, jobs=max(1, args.warmup))
    secs, nseq = time_oracle(wl, samples, nthreads, jobs=args.steps)
    value = nseq / secs
    res = {"impl": "reference", "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int32+f64 (CPU oracle)",
           "data": "synthetic", "config": decode_config(wl, algorithmic_bytes(wl)["total"],
                                                        args.schedule == "concurrent" and not args.sequential,
                                                        not args.no_graph),
           "cpu_baseline": {"value": value, "unit": "queries/s", "cores": nthreads, "kind": "oracle",
                            "sample": f"{nseq} queries ({max(1, wl.queries_per_seq)} per step) over "
                                      f"{len(samples)} sequences of the workload, {nthreads} host threads at a "
                                      f"time; {secs:.1f} s", **single_thread_oracle(wl, samples)},
           "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    if not on_gpu:  # the GPU arm's cache and launch notes do not describe a host-only run
        res["config"]["l2"] = "host-only run (no GPU): contexts shortened to %d" % wl.max_len
        res["config"].pop("schedule")
    print(json.dumps(res))


def run_cp(args):
    """Context-parallel decode step (cp.py): the workload's sequences split
    into G shards.  Under torchrun G = the world size, one shard per rank,
    exchanging through NCCL all-gathers (strong scaling: the sequences are
    fixed, each rank holds 1/G of them); in one process all G shards run on
    this GPU one after the other."""
    import torch
    import torch.distributed as dist

    import synth.workloads as W
    from long_context_decode_csa2_b200 import csa2 as C
    from long_context_decode_csa2_b200.cp import Shard, ShardedStep, dist_gather, shard_bounds, stack_gather
    from long_context_decode_csa2_b200.decode import FullCache

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600), device_id=device)
    G = world if world > 1 else args.cp
    mine = [rank] if world > 1 else list(range(G))
    wl = W.decode_workloads()[args.workload]
    if wl.queries_per_seq or wl.ratio != 1 or wl.page_rows:
        raise SystemExit("--cp runs the plain decode workloads")
    if args.batch:
        wl = dataclasses.replace(wl, name=wl.name + f"_b{args.batch}", lengths=wl.lengths[:args.batch])
    layers = [W.layer_inputs_host(wl, l) for l in range(len(wl.pattern))]
    caches_dev = [W.full_cache_device(wl, f, layers[f]["q_codes"], layers[f]["q_scales"], device)
                  for f in wl.full_layers()]
    off = caches_dev[0]["seq_row_off"]
    bounds = shard_bounds(wl.lengths, G)
    keys = ("q", "q_codes", "q_scales", "w", "win", "win_scale", "win_len")

    def to_dev(a):
        a = np.ascontiguousarray(a)
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
        return torch.from_numpy(a).to(device)

    shards = []
    for g in mine:
        lens = (bounds[g + 1] - bounds[g]).astype(np.int64)
        pad = (lens + 7) // 8 * 8
        soff = np.concatenate([[0], np.cumsum(pad)[:-1]]).astype(np.int64)
        rows = int(max(8, pad.sum()))
        shard_caches = []
        for c in caches_dev:  # this shard's rows of every sequence, gathered on the device
            idx = torch.cat([torch.arange(int(off[b] + bounds[g, b]), int(off[b] + bounds[g + 1, b]), device=device)
                             for b in range(wl.B)] or [torch.zeros(0, dtype=torch.int64, device=device)])
            planes = {}
            for key in ("idx_codes", "idx_scales", "main_codes", "main_scales"):
                t = torch.zeros((rows, c[key].shape[1]), dtype=torch.uint8, device=device)
                dst = torch.cat([torch.arange(int(soff[b]), int(soff[b] + lens[b]), device=device)
                                 for b in range(wl.B)])
                t[dst] = c[key][idx]
                planes[key] = t
            shard_caches.append(FullCache(C.cache(planes["idx_codes"], planes["idx_scales"]),
                                          C.cache(planes["main_codes"], planes["main_scales"])))
        lg = []
        for L in layers:
            Lg = {k: to_dev(L[k]) for k in keys}
            if g != G - 1:  # the window lives on the shard with the newest entries
                Lg["win_len"] = torch.zeros_like(Lg["win_len"])
            lg.append(Lg)
        shards.append(Shard(caches=shard_caches, seq_row_off=to_dev(soff), seq_len=to_dev(lens.astype(np.int32)),
                            lo=to_dev(bounds[g]), hi=to_dev(bounds[g + 1]), layers=lg))
    del caches_dev
    torch.cuda.empty_cache()
    src_pos = to_dev(bounds[:-1])
    src_blk = to_dev(bounds[:-1] // 8)
    max_shard = int((bounds[1:] - bounds[:-1]).max())
    step = ShardedStep(wl.pattern, wl.B, max_shard, len(mine), G, wl.P, wl.k,
                       gather=dist_gather() if world > 1 else stack_gather)
    for _ in range(args.warmup):
        step.run(shards, src_pos, src_blk)
    torch.cuda.synchronize()
    if step.device_flags():
        raise RuntimeError("device status flags set during warm-up")
    # one process: the step replays from a CUDA graph (its many small calls
    # would otherwise wait on the host); across ranks the steps stay eager
    graph = None
    if world == 1 and not args.no_graph:
        graph = step.capture(shards, src_pos, src_blk)
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        time.sleep(0.5)
        t0.record(stream)
        for _ in range(args.steps):
            if graph is not None:
                graph.replay()
            else:
                step.run(shards, src_pos, src_blk)
        t1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, device, world)

    # end to end: every shard's query inputs of every layer from pinned host
    # memory, then the step, then the merged outputs and Top-k back, all in
    # stream order on this stream (no overlap between steps)
    q_keys = ("q", "q_codes", "q_scales", "w")
    host_q = [[{k: t.cpu().pin_memory() for k, t in Lg.items() if k in q_keys} for Lg in sh.layers]
              for sh in shards]
    out_h = torch.empty(step.out.shape, dtype=torch.float32).pin_memory()
    top_h = [torch.empty(t.shape, dtype=torch.int32).pin_memory() for t in step.topk]
    h2d = sum(t.numel() * t.element_size() for hs in host_q for L in hs for t in L.values())
    d2h = out_h.numel() * 4 + sum(t.numel() * 4 for t in top_h)
    e_steps = max(1, min(args.e2e_steps, 10))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e_steps):
        for sh, hs in zip(shards, host_q):
            for Lg, L in zip(sh.layers, hs):
                for k, src in L.items():
                    Lg[k].copy_(src, non_blocking=True)  # same dtype: a plain byte copy
        if graph is not None:
            graph.replay()
        else:
            step.run(shards, src_pos, src_blk)
        out_h.copy_(step.out, non_blocking=True)
        for th, t in zip(top_h, step.topk):
            th.copy_(t, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e_steps, device, world)
    if rank == 0:
        ab = algorithmic_bytes(wl)
        print(json.dumps({
            "metric": METRIC, "value": wl.B / (ms * 1e-3), "unit": "queries/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None,
            "dtype": "int32+f64 indexer, f16 tensor-core attention (f32 accumulate)", "data": "synthetic",
            "config": dict(decode_config(wl, ab["total"], False, graph is not None), cp_shards=G,
                           cp_mode="one shard per rank (NCCL all-gather)" if world > 1 else
                           "all shards on this GPU, one after the other"),
            "hbm_algorithmic_gbs": ab["total"] / (ms * 1e-3) / 1e9,
            # the roofline and the oracle baseline are reported by the single-device step
            "roofline": None, "cpu_baseline": None,
            "e2e": {"value": wl.B / (e2e_ms * 1e-3), "unit": "queries/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "clocks": clk.summary(), "device_flags": step.device_flags()}))
    if world > 1:
        dist.destroy_process_group()


PEAKS_SRC = os.path.join(ROOT, "bench_peaks.cu")
PEAKS_LIB = os.path.join(ROOT, "_build", "libcsa2_peaks.so")


def build_peaks(force=False):
    """Compiles the peak probes (bench_peaks.cu) for sm_100a."""
    if force or not os.path.exists(PEAKS_LIB) or os.path.getmtime(PEAKS_LIB) < os.path.getmtime(PEAKS_SRC):
        os.makedirs(os.path.dirname(PEAKS_LIB), exist_ok=True)
        tmp = PEAKS_LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
                               "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"), "-I", ROOT,
                               PEAKS_SRC, "-o", tmp])
        os.replace(tmp, PEAKS_LIB)
    return PEAKS_LIB


def fp4_peak_tflops():
    """The FP4 tensor-core rate at the prefill indexer's MMA shape (kind::mxf4,
    M = N = 128, K = 64), measured now with the peak probe; if the probe
    cannot run, the measured bf16 rate x 4 (the nominal fp4 / bf16 ratio)."""
    import ctypes

    import torch

    try:
        lib = ctypes.CDLL(build_peaks())
        sms = lib.peaks_num_sms()
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        stream = torch.cuda.current_stream()
        iters, ms = 60000, []
        for rep in range(5):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            assert lib.peaks_mma_mxf4(128, iters, ctypes.c_void_p(err.data_ptr()),
                                      ctypes.c_void_p(stream.cuda_stream)) == 0
            e1.record(stream)
            torch.cuda.synchronize()
            if rep >= 2:
                ms.append(e0.elapsed_time(e1))
        if int(err.item()) == 0:
            return sms * iters * 2.0 * 128 * 128 * 64 / (statistics.median(ms) * 1e-3) / 1e12, \
                "measured now: tcgen05 kind::mxf4, N = 128 (bench_peaks.cu)"
    except Exception:
        pass
    pk = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pk):
        return 4 * float(json.load(open(pk))["bf16_tflops"]), "measured bf16 x 4 (nominal fp4 / bf16)"
    return 4 * 1590.0, "fallback bf16 x 4"


def run_peaks(args):
    """Roofline denominators measured on this GPU (one JSON line): the
    read-only HBM stream with 128-bit loads and with bulk copies into shared
    memory (4 GiB read once per repetition, more than L2), tcgen05.mma
    kind::mxf4 (unit scales) at M = 128, K = 64 and N = 16 / 128, and FP64
    FMA.  Median of 10 timed repetitions after 3 warm-ups, CUDA events."""
    import ctypes

    import torch

    lib = ctypes.CDLL(build_peaks())
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    sp = ctypes.c_void_p(stream.cuda_stream)
    sms = lib.peaks_num_sms()
    nbytes = 4 << 30
    buf = torch.ones(nbytes, dtype=torch.uint8, device=dev)
    sink = torch.zeros(sms * 8, dtype=torch.int64, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    P = ctypes.c_void_p

    def timed(launch, reps=10, warm=3):
        for _ in range(warm):
            assert launch() == 0
        ms = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            assert launch() == 0
            e1.record(stream)
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1))
        return statistics.median(ms)

    out = {}
    with ClockSampler(0) as clk:
        ms = timed(lambda: lib.peaks_read_ldg(P(buf.data_ptr()), ctypes.c_longlong(nbytes // 16),
                                              P(sink.data_ptr()), sp))
        out["hbm_read_ldg128_gbs"] = nbytes / (ms * 1e-3) / 1e9
        ms = timed(lambda: lib.peaks_read_bulk(P(buf.data_ptr()), ctypes.c_longlong(nbytes), P(err.data_ptr()), sp))
        out["hbm_read_bulk_gbs"] = nbytes / (ms * 1e-3) / 1e9
        for n, iters in ((16, 400000), (128, 60000)):
            ms = timed(lambda: lib.peaks_mma_mxf4(n, iters, P(err.data_ptr()), sp))
            out[f"fp4_mxf4_n{n}_tflops"] = sms * iters * 2.0 * 128 * n * 64 / (ms * 1e-3) / 1e12
        iters = 20000
        ms = timed(lambda: lib.peaks_fma64(iters, P(sink.data_ptr()), sp))
        out["fp64_fma_tflops"] = sms * 8 * 256 * 8 * iters * 2.0 / (ms * 1e-3) / 1e12
    torch.cuda.synchronize()
    out["probe_errors"] = int(err.item())
    out["sms"] = sms
    print(json.dumps({"peaks": out, "clocks": clk.summary(),
                      "method": "bench_peaks.cu kernels, CUDA events, median of 10 after 3 warm-ups; HBM probes read "
                                "4 GiB once per repetition"}))


def main():
    args = parse()
    if args.peaks:
        run_peaks(args)
        return
    if args.impl == "reference":
        run_reference(args)
    elif args.workload.startswith("prefill"):
        run_prefill(args)
    elif args.cp:
        run_cp(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
