"""Context-parallel decode: every long sequence split over G shards.

Shard g holds entries [lo_g, hi_g) of each sequence in its own caches (one
GPU each in a deployment).  A decode step through the layer pattern then
needs one exchange per indexer call and one per attention:

* Full layer (scan): each shard runs ``csa2_index_full`` on its range, ranks
  its pool blocks and its Top-k with ``csa2_score_positions``; the shards
  all-gather the (key, id) lists and ``csa2_topk_merge`` picks the global
  pool and Top-k (the global winners lie in the union of the shards' own
  winners, ranked by the same keys) and gives every shard its own part;
* Reindex layer: each shard scores its part of the pool
  (``csa2_index_reindex``) and the same rank / gather / merge follows;
* Reuse layer: the last Top-k;
* attention: each shard attends its part of the Top-k (the window lives on
  the shard with the newest entries), then the partial outputs are gathered
  and mixed by their log-sum-exps (``csa2_attn_combine``).

This is the exchange the "DeepSeek-V4.1-Flash: Pushing the Limits of KV
Cache Compression" selection rules allow (section "三个方向一起压小缓存":
block pool and Top-512 are best-first selections); the pages themselves run
on one device.  ``ShardedStep.run`` takes the list of shards this process
drives: one shard per rank with ``gather`` = an all-gather over the process
group, or every shard in one process (``stack_gather``), which computes the
same step on one GPU.  All arithmetic runs in ``libcsa2.so``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

from . import csa2 as C
from .decode import FullCache, layer_plan


def shard_bounds(lengths, G: int, align: int = 8):
    """[G+1, B] int64 boundaries: shard g holds entries bounds[g, b] ..
    bounds[g+1, b] of sequence b; inner boundaries are multiples of `align`
    (whole 8-position blocks per shard) and as even as that allows."""
    L = np.asarray(lengths, np.int64)
    g = np.arange(G + 1, dtype=np.int64)[:, None]
    b = (L[None, :] * g // G) // align * align
    b[G] = L
    return b


def stack_gather(tensors):
    """The exchange when one process drives every shard: [G, ...] stacked."""
    return torch.stack(tensors)


def dist_gather(group=None):
    """The exchange across ranks (one shard per rank): an all-gather of each
    rank's tensor into [G, ...] over `group` (NCCL on GPUs)."""
    import torch.distributed as dist

    def gather(tensors):
        (t,) = tensors
        parts = [torch.empty_like(t) for _ in range(dist.get_world_size(group))]
        dist.all_gather(parts, t.contiguous(), group=group)
        return torch.stack(parts)

    return gather


@dataclass
class Shard:
    """One shard's inputs: its caches (one FullCache per Full layer, rows of
    its own entries), row offsets and lengths of its part of every sequence,
    its global range [lo, hi) per sequence, and the per-layer query inputs
    (``win_len`` zero except on the shard holding the newest entries)."""

    caches: list
    seq_row_off: torch.Tensor   # [B] int64
    seq_len: torch.Tensor       # [B] int32 (hi - lo)
    lo: torch.Tensor            # [B] int64
    hi: torch.Tensor            # [B] int64
    layers: list


class ShardedStep:
    """Workspaces and outputs of a context-parallel step for the shards one
    process drives.  ``src_pos`` / ``src_blk`` [G, B] int64 are every shard's
    lo (in positions / in blocks), the offsets that make shard-local ids
    global."""

    def __init__(self, pattern: str, B: int, max_shard_len: int, n_local: int, G: int, P: int = 2048, k: int = 512,
                 device="cuda", sm_scale: float | None = None, gather=stack_gather):
        if P < k:
            raise ValueError("the sharded step needs the pool fast path (P >= k)")
        self.pattern, self.B, self.P, self.k, self.G = pattern, B, P, k, G
        self.max_shard_len = max_shard_len
        self.plan = layer_plan(pattern)
        self.sm_scale = sm_scale if sm_scale is not None else 1.0 / math.sqrt(C.MAIN_DIM)
        self.gather = gather
        dev = torch.device(device)
        nL = len(pattern)
        z32 = dict(dtype=torch.int32, device=dev)

        def ws(nbytes):
            return C.workspace(nbytes, dev)

        self.local = []
        for _ in range(n_local):
            self.local.append(dict(
                ws_full=ws(C.csa2_index_full_workspace_bytes(B, max_shard_len, P, k)),
                ws_re=ws(C.csa2_index_reindex_workspace_bytes(B, P, k)),
                ws_attn=ws(C.csa2_sparse_attn_decode_workspace_bytes(B, k)),
                ws_score=ws(C.csa2_score_positions_workspace_bytes(B)),
                ws_mpool=ws(C.csa2_topk_merge_workspace_bytes(G, B, P)),
                ws_mtop=ws(C.csa2_topk_merge_workspace_bytes(G, B, k)),
                pool_l=torch.full((B, P), -1, **z32), top_l=torch.full((B, k), -1, **z32),
                pool_keys=torch.zeros((B, P), **z32), top_keys=torch.zeros((B, k), **z32),
                pool_mine=torch.full((B, P), -1, **z32),
                top_mine=[torch.full((B, k), -1, **z32) for _ in range(nL)],
                out_l=torch.zeros((B, C.Q_HEADS, C.MAIN_DIM), dtype=torch.float32, device=dev),
                lse_l=torch.zeros((B, C.Q_HEADS), dtype=torch.float32, device=dev)))
        self.pool = torch.full((B, P), -1, **z32)
        self.topk = [torch.full((B, k), -1, **z32) for _ in range(nL)]
        self.out = torch.zeros((nL, B, C.Q_HEADS, C.MAIN_DIM), dtype=torch.float32, device=dev)
        self.lse = torch.zeros((nL, B, C.Q_HEADS), dtype=torch.float32, device=dev)

    def _merge(self, shards, ids_key, keys_key, src_off, k, out, mine_key, lo_div, ws_key, layer=None):
        keys = self.gather([st[keys_key] for st in self.local[:len(shards)]])
        ids = self.gather([st[ids_key] for st in self.local[:len(shards)]])
        for sh, st in zip(shards, self.local):
            mine = st[mine_key] if layer is None else st[mine_key][layer]
            lo = sh.lo if lo_div == 1 else sh.lo // lo_div
            hi = sh.hi if lo_div == 1 else (sh.hi + lo_div - 1) // lo_div
            C.csa2_topk_merge(keys, ids, src_off, k, out, st[ws_key], lo=lo, hi=hi, out_local=mine)

    def run(self, shards, src_pos: torch.Tensor, src_blk: torch.Tensor):
        """shards: the Shard objects this process drives (all G with
        stack_gather, this rank's one with dist_gather)."""
        if len(shards) > len(self.local):
            raise ValueError("more shards than the step was built for")
        last = None
        for layer, mode, f, act in self.plan:
            if act == "scan":
                for sh, st in zip(shards, self.local):
                    L = sh.layers[layer]
                    cache = sh.caches[f]
                    C.csa2_index_full(cache.idx, L["q_codes"], L["q_scales"], L["w"], sh.seq_row_off, sh.seq_len,
                                      self.max_shard_len, self.P, self.k, st["pool_l"], st["top_l"], st["ws_full"])
                    C.csa2_score_positions(cache.idx, L["q_codes"], L["q_scales"], L["w"], sh.seq_row_off,
                                           sh.seq_len, st["pool_l"], C.BLOCK, st["pool_keys"], st["ws_score"])
                    C.csa2_score_positions(cache.idx, L["q_codes"], L["q_scales"], L["w"], sh.seq_row_off,
                                           sh.seq_len, st["top_l"], 1, st["top_keys"], st["ws_score"])
                self._merge(shards, "pool_l", "pool_keys", src_blk, self.P, self.pool, "pool_mine", C.BLOCK,
                            "ws_mpool")
                self._merge(shards, "top_l", "top_keys", src_pos, self.k, self.topk[layer], "top_mine", 1, "ws_mtop",
                            layer)
                last = layer
            elif act == "reindex":
                for sh, st in zip(shards, self.local):
                    L = sh.layers[layer]
                    cache = sh.caches[f]
                    C.csa2_index_reindex(cache.idx, L["q_codes"], L["q_scales"], L["w"], sh.seq_row_off, sh.seq_len,
                                         st["pool_mine"], self.k, st["top_l"], st["ws_re"])
                    C.csa2_score_positions(cache.idx, L["q_codes"], L["q_scales"], L["w"], sh.seq_row_off,
                                           sh.seq_len, st["top_l"], 1, st["top_keys"], st["ws_score"])
                self._merge(shards, "top_l", "top_keys", src_pos, self.k, self.topk[layer], "top_mine", 1, "ws_mtop",
                            layer)
                last = layer
            else:  # reuse
                self.topk[layer].copy_(self.topk[last])
                for st in self.local[:len(shards)]:
                    st["top_mine"][layer].copy_(st["top_mine"][last])
            for sh, st in zip(shards, self.local):
                L = sh.layers[layer]
                C.csa2_sparse_attn_decode(L["q"], sh.caches[f].main, sh.seq_row_off, sh.seq_len,
                                          st["top_mine"][layer], L["win"], L["win_scale"], L["win_len"],
                                          self.sm_scale, st["out_l"], st["ws_attn"], lse=st["lse_l"])
            outs = self.gather([st["out_l"] for st in self.local[:len(shards)]])
            lses = self.gather([st["lse_l"] for st in self.local[:len(shards)]])
            C.csa2_attn_combine(outs, lses, self.out[layer], self.lse[layer])
        return self.out

    def capture(self, shards, src_pos, src_blk):
        """Records one step into a CUDA graph (call ``run`` once first);
        ``graph.replay()`` then runs it as one launch with the same buffers."""
        graph = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(device=self.out.device)
        cap.wait_stream(torch.cuda.current_stream())
        with torch.cuda.graph(graph, stream=cap, capture_error_mode="thread_local"):
            self.run(shards, src_pos, src_blk)
        torch.cuda.current_stream().wait_stream(cap)
        return graph

    def device_flags(self) -> int:
        flags = 0
        for st in self.local:
            for key in ("ws_full", "ws_re", "ws_attn", "ws_score", "ws_mpool", "ws_mtop"):
                flags |= C.device_status(st[key])
        return flags


def split_caches(cache_full: dict, seq_row_off, bounds):
    """Host helper: the shards' contiguous cache arrays cut from one
    sequence-major cache dict (idx/main codes and scales, NumPy); returns per
    shard (arrays dict, row offsets [B])."""
    G = bounds.shape[0] - 1
    out = []
    for g in range(G):
        lens = bounds[g + 1] - bounds[g]
        pad = (lens + 7) // 8 * 8
        off = np.concatenate([[0], np.cumsum(pad)[:-1]]).astype(np.int64)
        rows = int(max(8, pad.sum()))
        arrs = {}
        for key, v in cache_full.items():
            if not isinstance(v, np.ndarray) or v.ndim != 2:
                continue
            a = np.zeros((rows, v.shape[1]), v.dtype)
            for b in range(len(lens)):
                s0 = int(seq_row_off[b] + bounds[g, b])
                a[off[b]:off[b] + lens[b]] = v[s0:s0 + lens[b]]
            arrs[key] = a
        out.append((arrs, off))
    return out


def to_full_cache(arrs: dict, dev) -> FullCache:
    def d(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    return FullCache(C.cache(d(arrs["idx_codes"]), d(arrs["idx_scales"])),
                     C.cache(d(arrs["main_codes"]), d(arrs["main_scales"])))
