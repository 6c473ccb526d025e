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


class DecodeStep:
    """Owns the workspaces and outputs of one decode step; ``run`` enqueues it."""

    def __init__(self, pattern: str, B: int, max_len: int, P: int = 2048, k: int = 512, full_rescan: bool = False,
                 device="cuda", sm_scale: float | None = None):
        self.pattern, self.B, self.max_len, self.P, self.k = pattern, B, max_len, P, k
        self.plan = layer_plan(pattern, full_rescan)
        self.sm_scale = sm_scale if sm_scale is not None else 1.0 / math.sqrt(C.MAIN_DIM)
        dev = torch.device(device)
        self.ws_full = C.workspace(C.csa2_index_full_workspace_bytes(B, max_len, P, k), dev)
        self.ws_re = C.workspace(C.csa2_index_reindex_workspace_bytes(B, P, k), dev)
        self.ws_attn = C.workspace(C.csa2_sparse_attn_decode_workspace_bytes(B, k), dev)
        self.pool = torch.full((B, P), -1, dtype=torch.int32, device=dev)
        nL = len(pattern)
        self.topk = [torch.full((B, k), -1, dtype=torch.int32, device=dev) for _ in range(nL)]
        self.out = torch.zeros((nL, B, C.Q_HEADS, C.MAIN_DIM), dtype=torch.float32, device=dev)
        self.lse = torch.zeros((nL, B, C.Q_HEADS), dtype=torch.float32, device=dev)
        self.scores = None
        # optional callable(call_name, "begin" | "end"), e.g. to record events
        self.hook = None

    def _hook(self, name, phase):
        if self.hook is not None:
            self.hook(name, phase)

    def run(self, caches, seq_row_off, seq_len, layers, stream=None):
        """caches: [FullCache] per Full layer; layers: per layer dict of device
        tensors q, q_codes, q_scales, w, win, win_scale, win_len."""
        last = None
        for layer, mode, f, act in self.plan:
            L = layers[layer]
            cache = caches[f]
            if act == "scan":
                self._hook("csa2_index_full", "begin")
                C.csa2_index_full(cache.idx, L["q_codes"], L["q_scales"], L["w"], seq_row_off, seq_len, self.max_len,
                                  self.P, self.k, self.pool, self.topk[layer], self.ws_full, stream=stream)
                self._hook("csa2_index_full", "end")
                last = self.topk[layer]
            elif act == "reindex":
                self._hook("csa2_index_reindex", "begin")
                C.csa2_index_reindex(cache.idx, L["q_codes"], L["q_scales"], L["w"], seq_row_off, seq_len, self.pool,
                                     self.k, self.topk[layer], self.ws_re, stream=stream)
                self._hook("csa2_index_reindex", "end")
                last = self.topk[layer]
            else:
                self.topk[layer] = last  # Reuse: the same tensor, no copy
            self._hook("csa2_sparse_attn_decode", "begin")
            C.csa2_sparse_attn_decode(L["q"], cache.main, seq_row_off, seq_len, last, L["win"], L["win_scale"],
                                      L["win_len"], self.sm_scale, self.out[layer], self.ws_attn,
                                      lse=self.lse[layer], stream=stream)
            self._hook("csa2_sparse_attn_decode", "end")
        return self.out

    def device_flags(self) -> int:
        return C.device_status(self.ws_full) | C.device_status(self.ws_re) | C.device_status(self.ws_attn)
