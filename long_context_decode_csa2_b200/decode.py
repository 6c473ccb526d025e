"""One CSA2 decode step through a layer pattern, driven over the C ABI.

Layer modes ("DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache
Compression", section "三个方向一起压小缓存", and the "DeepSeek-V4.1" reading
notes):

* ``F`` (Full) computes its own main KV and indexer K.  The first Full layer
  of the step scans the whole visible context, builds the shared candidate
  pool and picks its own Top-k.  A later Full layer uses its OWN caches but,
  by default, selects inside the first Full layer's pool (only the first Full
  layer scans the full range); with ``full_rescan=True`` every Full layer scans
  and rebuilds the pool.
* ``R`` (Reindex) reuses the nearest Full layer's caches and selects again
  inside the pool with its own indexer query.
* ``U`` (Reuse) takes the most recent Top-k unchanged (no indexer call).

Every layer attends its selection plus its own FP8 window.  This module only
sequences C-ABI calls; all arithmetic runs in ``libcsa2.so``.

With ``ratio=2`` (compressed entries during generation) each step first
appends the new raw token of every Full layer's caches with
``csa2_compress_stream``: the odd token of a pair waits on the device, every
second step completes an entry, and the sequence lengths advance in place
before the indexer sees them.

With ``queries=Q`` (speculative verification, the page's section "DSpark":
several candidate positions per request checked in one forward) a step
carries up to Q queries in total, a ragged number per sequence (``q_off``),
each with its own visible entry count (``q_vis``).  The scanning Full layer
reads every sequence's indexer K once for all of its queries
(``csa2_index_multi``); the later calls take the queries as Q segments.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

from . import csa2 as C


@dataclass
class FullCache:
    idx: C.MXFP4Cache
    main: C.MXFP4Cache


def layer_plan(pattern: str, full_rescan: bool = False):
    """[(layer, mode, full_index, action)] with action in scan / reindex / reuse."""
    plan, f, seen_full = [], -1, False
    for layer, m in enumerate(pattern):
        if m == "F":
            f += 1
            act = "scan" if (not seen_full or full_rescan) else "reindex"
            seen_full = True
        elif m == "R":
            if f < 0:
                raise ValueError("a Reindex layer needs an earlier Full layer")
            act = "reindex"
        elif m == "U":
            if f < 0 or not plan:
                raise ValueError("a Reuse layer needs an earlier indexer output")
            act = "reuse"
        else:
            raise ValueError(f"unknown layer mode {m!r}")
        plan.append((layer, m, f, act))
    return plan


class PairStream:
    """Pending half-pairs of one Full layer's caches for ratio-2 appends
    during decode (one raw token per sequence per step)."""

    def __init__(self, B: int, device, projection: bool = True):
        dev = torch.device(device)
        self.pend_n = torch.zeros(B, dtype=torch.int32, device=dev)
        self.pend_raw = torch.zeros((B, C.MAIN_DIM), dtype=torch.bfloat16, device=dev)
        self.pend_logit = torch.zeros(B, dtype=torch.float32, device=dev)
        self.pend_idx = None if projection else torch.zeros((B, C.IDX_DIM), dtype=torch.bfloat16, device=dev)
        self.tok_off = torch.arange(B + 1, dtype=torch.int64, device=dev)
        self.ws = C.workspace(C.csa2_compress_stream_workspace_bytes(B), dev)

    def append(self, cache: FullCache, tok: dict, seq_row_off, seq_len, update_len: bool, stream=None):
        """tok: raw [B,512] bf16, logit [B] fp32, and w_idx [512,128] fp32 or
        idx_raw [B,128] bf16.  update_len: write the new lengths into seq_len."""
        C.csa2_compress_stream(cache.main, cache.idx, tok["raw"], tok["logit"], self.tok_off, seq_row_off, seq_len,
                               seq_len if update_len else None, self.pend_n, self.pend_raw, self.pend_logit, 1,
                               self.ws, w_idx=tok.get("w_idx"), idx_raw=tok.get("idx_raw"), pend_idx=self.pend_idx,
                               stream=stream)


class DecodeStep:
    """Owns the workspaces and outputs of one decode step; ``run`` enqueues it.

    With ``concurrent=True`` (default) the calls that do not depend on each
    other run on side streams: every Reindex layer waits only for the pool,
    every attention only for its layer's Top-k, so the latency-bound tail of
    the step (pool scoring, Top-k selection, attention) overlaps across
    layers.  Each such call then gets its own workspace.  The caller's stream
    waits for all of them before ``run`` returns, and the scans stay on the
    caller's stream in layer order.  That overlap needs every layer's inputs
    up front, which a model running layer after layer does not have.

    With ``concurrent=False`` every call runs in layer order.  ``groups=G``
    then splits the batch into G groups of consecutive sequences after each
    scanning layer: a group's calls stay in layer order on a stream of their
    own, and the groups overlap.  Sequences are independent, so this is an
    order a model can run (its layer l+1 queries of a group come from that
    group's layer l outputs)."""

    def __init__(self, pattern: str, B: int, max_len: int, P: int = 2048, k: int = 512, full_rescan: bool = False,
                 device="cuda", sm_scale: float | None = None, concurrent: bool = True, side_streams: int = 3,
                 ratio: int = 1, projection: bool = True, queries: int | None = None, split_full: bool = False,
                 groups: int = 1):
        if ratio not in (1, 2):
            raise ValueError("ratio must be 1 or 2")
        if groups < 1 or groups > B or (groups > 1 and (concurrent or queries is not None)):
            raise ValueError("groups > 1 is for layer-order steps over sequences, at most one group per sequence")
        if queries is not None and ratio != 1:
            raise ValueError("verification steps take their entries as given (ratio 1 appends are the caller's)")
        self.pattern, self.B, self.max_len, self.P, self.k = pattern, B, max_len, P, k
        self.ratio = ratio
        self.queries = queries
        # concurrent steps only: issue the scanning Full layer as pool + Top-k,
        # so that the Reindex layers start from the pool (they then compete
        # with the Full layer's own pool scoring; measured no faster at B = 64)
        self.split_full = split_full and concurrent
        nq = B if queries is None else queries  # segments of the calls after the scan
        self.plan = layer_plan(pattern, full_rescan)
        self.sm_scale = sm_scale if sm_scale is not None else 1.0 / math.sqrt(C.MAIN_DIM)
        self.concurrent = concurrent
        dev = torch.device(device)
        nL = len(pattern)
        if queries is None:
            self.ws_full = C.workspace(C.csa2_index_full_workspace_bytes(B, max_len, P, k), dev)
            self.q_row_off = None
        else:
            self.ws_full = C.workspace(C.csa2_index_multi_workspace_bytes(B, queries, max_len, P, k), dev)
            self.q_row_off = torch.zeros(queries, dtype=torch.int64, device=dev)
        re_bytes = C.csa2_index_reindex_workspace_bytes(nq, P, k)
        attn_bytes = C.csa2_sparse_attn_decode_workspace_bytes(nq, k)
        if concurrent:
            self.ws_re = [C.workspace(re_bytes, dev) if act == "reindex" else None for _, _, _, act in self.plan]
            self.ws_attn = [C.workspace(attn_bytes, dev) for _ in range(nL)]
            self.streams = [torch.cuda.Stream(device=dev) for _ in range(max(1, side_streams))]
            self.ev_idx = [torch.cuda.Event() for _ in range(nL)]
            self.ev_pool = [torch.cuda.Event() for _ in range(nL)]
            self.ev_done = [torch.cuda.Event() for _ in range(nL)]
        elif groups > 1:
            # group g: sequences bounds[g] .. bounds[g+1]-1, its own stream and workspaces
            self.bounds = [g * B // groups for g in range(groups + 1)]
            sizes = [self.bounds[g + 1] - self.bounds[g] for g in range(groups)]
            self.ws_re = [[C.workspace(C.csa2_index_reindex_workspace_bytes(n, P, k), dev) for n in sizes]
                          if act == "reindex" else None for _, _, _, act in self.plan]
            self.ws_attn = [[C.workspace(C.csa2_sparse_attn_decode_workspace_bytes(n, k), dev) for n in sizes]
                            for _ in range(nL)]
            self.gstreams = [torch.cuda.Stream(device=dev) for _ in range(groups)]
            self.join = torch.cuda.Stream(device=dev)  # layer-done events, off the groups' paths
            self.ev_scan = [torch.cuda.Event() for _ in range(nL)]
            self.ev_group = [[torch.cuda.Event() for _ in range(groups)] for _ in range(nL)]
            self.ev_layer = [torch.cuda.Event() for _ in range(nL)]
        else:
            ws_re, ws_attn = C.workspace(re_bytes, dev), C.workspace(attn_bytes, dev)
            self.ws_re = [ws_re] * nL
            self.ws_attn = [ws_attn] * nL
        self.groups = groups
        # one pool per scanning layer (a rescan must not overwrite a pool that
        # an earlier Reindex layer may still be reading)
        self.pools = {layer: torch.full((nq, P), -1, dtype=torch.int32, device=dev)
                      for layer, _, _, act in self.plan if act == "scan"}
        self.topk = [torch.full((nq, k), -1, dtype=torch.int32, device=dev) for _ in range(nL)]
        self.out = torch.zeros((nL, nq, C.Q_HEADS, C.MAIN_DIM), dtype=torch.float32, device=dev)
        self.lse = torch.zeros((nL, nq, C.Q_HEADS), dtype=torch.float32, device=dev)
        # ratio 2: one pending-token state per Full layer's caches
        n_full = sum(1 for m in pattern if m == "F")
        self.pairs = [PairStream(B, dev, projection) for _ in range(n_full)] if ratio == 2 else []
        # optional callable(call_name, "begin" | "end", stream), e.g. to record events
        self.hook = None

    @property
    def pool(self):
        """The pool of the last scanning Full layer."""
        return self.pools[max(self.pools)]

    def _hook(self, name, phase, stream):
        if self.hook is not None:
            self.hook(name, phase, stream)

    def run(self, caches, seq_row_off, seq_len, layers, stream=None, ready=None, on_layer_done=None,
            new_tokens=None, q_off=None, q_vis=None):
        """caches: [FullCache] per Full layer; layers: per layer dict of device
        tensors q, q_codes, q_scales, w, win, win_scale, win_len.

        ready: optional per-layer CUDA events; a layer's calls wait for its
        event (e.g. its inputs arriving on a copy stream).  on_layer_done:
        optional callable(layer, event), called once the layer's attention is
        enqueued, with an event that completes after it (e.g. to copy the
        layer's output out while later layers run).

        new_tokens (ratio 2 only): per Full layer a dict for
        ``PairStream.append``; the appends run first, on the caller's stream,
        and advance ``seq_len`` in place.

        q_off [B+1], q_vis [Q] (verification steps only, device int32): the
        queries of sequence b are q_off[b] .. q_off[b+1]-1, query i sees the
        first q_vis[i] entries; layer inputs are then per query and seq_len
        is not used."""
        if (self.queries is None) != (q_off is None and q_vis is None):
            raise ValueError("q_off / q_vis go with (and only with) a verification step")
        main = stream if stream is not None else torch.cuda.current_stream()
        if self.ratio == 2:
            if new_tokens is None or len(new_tokens) != len(self.pairs):
                raise ValueError("a ratio-2 step needs one new token dict per Full layer")
            full_layers = [layer for layer, m, _, _ in self.plan if m == "F"]
            for f, (pair, tok) in enumerate(zip(self.pairs, new_tokens)):
                if ready is not None:
                    main.wait_event(ready[full_layers[f]])
                self._hook("csa2_compress_stream", "begin", main)
                pair.append(caches[f], tok, seq_row_off, seq_len, update_len=f == len(self.pairs) - 1, stream=main)
                self._hook("csa2_compress_stream", "end", main)
        elif new_tokens is not None:
            raise ValueError("new_tokens is for ratio-2 steps")
        if self.groups > 1:
            return self._run_groups(caches, seq_row_off, seq_len, layers, main, ready, on_layer_done)
        pool, pool_ev = None, None
        last, last_ev = None, None
        # segments of the calls after the scan: sequences, or the queries of a
        # verification step (rows written by csa2_index_multi)
        seg_row_off, seg_len = (seq_row_off, seq_len) if self.queries is None else (self.q_row_off, q_vis)
        side = 0
        for layer, mode, f, act in self.plan:
            L = layers[layer]
            cache = caches[f]
            ev_ready = ready[layer] if ready is not None else None
            if act == "scan":
                if ev_ready is not None:
                    main.wait_event(ev_ready)
                pool = self.pools[layer]
                split = self.split_full and self.queries is None and isinstance(seq_row_off, torch.Tensor)
                if split:
                    # the pool is ready before the Full layer's own Top-k: the
                    # Reindex layers start from it while the Top-k is selected
                    self._hook("csa2_index_full", "begin", main)
                    C.csa2_index_full_pool(cache.idx, L["q_codes"], L["q_scales"], L["w"], seq_row_off, seq_len,
                                           self.max_len, self.P, self.k, pool, self.ws_full, stream=main)
                    self.ev_pool[layer].record(main)
                    C.csa2_index_full_topk(cache.idx, L["q_codes"], L["q_scales"], L["w"], seq_row_off, seq_len,
                                           self.max_len, self.P, self.k, pool, self.topk[layer], self.ws_full,
                                           stream=main)
                    self._hook("csa2_index_full", "end", main)
                elif self.queries is None:
                    self._hook("csa2_index_full", "begin", main)
                    C.csa2_index_full(cache.idx, L["q_codes"], L["q_scales"], L["w"], seq_row_off, seq_len,
                                      self.max_len, self.P, self.k, pool, self.topk[layer], self.ws_full, stream=main)
                    self._hook("csa2_index_full", "end", main)
                else:
                    self._hook("csa2_index_multi", "begin", main)
                    C.csa2_index_multi(cache.idx, L["q_codes"], L["q_scales"], L["w"], seq_row_off, q_off, q_vis,
                                       self.max_len, self.P, self.k, pool, self.topk[layer], self.ws_full,
                                       q_row_off_out=self.q_row_off, stream=main)
                    self._hook("csa2_index_multi", "end", main)
                last = self.topk[layer]
                if self.concurrent:
                    self.ev_idx[layer].record(main)
                    last_ev = self.ev_idx[layer]
                    pool_ev = self.ev_pool[layer] if split else self.ev_idx[layer]
            if self.concurrent:
                s = self.streams[side % len(self.streams)]
                side += 1
            else:
                s = main
            if ev_ready is not None and act != "scan":
                s.wait_event(ev_ready)
            if act == "reindex":
                if self.concurrent:
                    s.wait_event(pool_ev)
                self._hook("csa2_index_reindex", "begin", s)
                C.csa2_index_reindex(cache.idx, L["q_codes"], L["q_scales"], L["w"], seg_row_off, seg_len, pool,
                                     self.k, self.topk[layer], self.ws_re[layer], stream=s)
                self._hook("csa2_index_reindex", "end", s)
                last = self.topk[layer]
                if self.concurrent:
                    self.ev_idx[layer].record(s)
                    last_ev = self.ev_idx[layer]
            elif act == "reuse":
                self.topk[layer] = last  # Reuse: the same tensor, no copy
                if self.concurrent:
                    s.wait_event(last_ev)
            elif self.concurrent:  # scan: the attention runs beside the next layers
                s.wait_event(last_ev)
            self._hook("csa2_sparse_attn_decode", "begin", s)
            C.csa2_sparse_attn_decode(L["q"], cache.main, seg_row_off, seg_len, last, L["win"], L["win_scale"],
                                      L["win_len"], self.sm_scale, self.out[layer], self.ws_attn[layer],
                                      lse=self.lse[layer], stream=s)
            self._hook("csa2_sparse_attn_decode", "end", s)
            if self.concurrent:
                self.ev_done[layer].record(s)
            if on_layer_done is not None:
                if self.concurrent:
                    on_layer_done(layer, self.ev_done[layer])
                else:
                    ev = torch.cuda.Event()
                    ev.record(s)
                    on_layer_done(layer, ev)
        if self.concurrent:
            for ev in self.ev_done:
                main.wait_event(ev)
        return self.out

    def _run_groups(self, caches, seq_row_off, seq_len, layers, main, ready, on_layer_done):
        """Layer order per group of sequences (``groups`` > 1): scans on the
        caller's stream over the whole batch, everything else per group on
        the group's stream."""
        if not isinstance(seq_row_off, torch.Tensor):
            raise ValueError("groups > 1 takes the contiguous layout (seq_row_off tensor)")
        G, bd = self.groups, self.bounds
        pool, last = None, None
        started = False
        for layer, mode, f, act in self.plan:
            L = layers[layer]
            cache = caches[f]
            ev_ready = ready[layer] if ready is not None else None
            if act == "scan":
                if started:  # the batch's next scan follows every group's earlier layers
                    for g in range(G):
                        main.wait_event(self.ev_group[layer - 1][g])
                if ev_ready is not None:
                    main.wait_event(ev_ready)
                pool = self.pools[layer]
                self._hook("csa2_index_full", "begin", main)
                C.csa2_index_full(cache.idx, L["q_codes"], L["q_scales"], L["w"], seq_row_off, seq_len,
                                  self.max_len, self.P, self.k, pool, self.topk[layer], self.ws_full, stream=main)
                self._hook("csa2_index_full", "end", main)
                last = self.topk[layer]
                self.ev_scan[layer].record(main)
            started = True
            if act == "reuse":
                self.topk[layer] = last
            for g in range(G):
                b0, b1 = bd[g], bd[g + 1]
                s = self.gstreams[g]
                if act == "scan":
                    s.wait_event(self.ev_scan[layer])
                if ev_ready is not None and act != "scan":
                    s.wait_event(ev_ready)
                if act == "reindex":
                    self._hook("csa2_index_reindex", "begin", s)
                    C.csa2_index_reindex(cache.idx, L["q_codes"][b0:b1], L["q_scales"][b0:b1], L["w"][b0:b1],
                                         seq_row_off[b0:b1], seq_len[b0:b1], pool[b0:b1], self.k,
                                         self.topk[layer][b0:b1], self.ws_re[layer][g], stream=s)
                    self._hook("csa2_index_reindex", "end", s)
                self._hook("csa2_sparse_attn_decode", "begin", s)
                C.csa2_sparse_attn_decode(L["q"][b0:b1], cache.main, seq_row_off[b0:b1], seq_len[b0:b1],
                                          self.topk[layer][b0:b1], L["win"][b0:b1], L["win_scale"][b0:b1],
                                          L["win_len"][b0:b1], self.sm_scale, self.out[layer][b0:b1],
                                          self.ws_attn[layer][g], lse=self.lse[layer][b0:b1], stream=s)
                self._hook("csa2_sparse_attn_decode", "end", s)
                self.ev_group[layer][g].record(s)
            if act == "reindex":
                last = self.topk[layer]
            if on_layer_done is not None:
                # an event after every group's attention of this layer, on a
                # stream of its own (no group waits for another)
                for g in range(G):
                    self.join.wait_event(self.ev_group[layer][g])
                self.ev_layer[layer].record(self.join)
                on_layer_done(layer, self.ev_layer[layer])
        for g in range(G):
            main.wait_event(self.ev_group[self.plan[-1][0]][g])
        return self.out

    def capture(self, caches, seq_row_off, seq_len, layers, new_tokens=None, q_off=None, q_vis=None):
        """Records one step into a CUDA graph; ``graph.replay()`` then runs the
        whole step (every call, both schedules, with the same buffers) as one
        launch.  Call ``run`` once before capturing (warm-up), and do not
        change the tensors' addresses afterwards."""
        graph = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(device=self.out.device)
        cap.wait_stream(torch.cuda.current_stream())
        hook, self.hook = self.hook, None
        try:
            with torch.cuda.graph(graph, stream=cap, capture_error_mode="thread_local"):
                self.run(caches, seq_row_off, seq_len, layers, new_tokens=new_tokens, q_off=q_off, q_vis=q_vis)
        finally:
            self.hook = hook
        torch.cuda.current_stream().wait_stream(cap)
        return graph

    def device_flags(self) -> int:
        flags = C.device_status(self.ws_full)
        extra = [p.ws for p in self.pairs]
        flat = []
        for w in self.ws_re + self.ws_attn:
            flat.extend(w if isinstance(w, list) else [w])
        for ws in {id(w): w for w in flat + extra if w is not None}.values():
            flags |= C.device_status(ws)
        return flags
