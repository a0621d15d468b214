"""One decode step = [page metadata update] -> page scores -> page selection -> sparse attention
(the last two in one call for the top-k policy).

SparseDecoder owns the per-step device buffers (scores, selection, outputs, workspace) for a
fixed cache geometry and policy, and issues the four libekv calls on one stream. It adds no
computation of its own.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import ekv


class SparseDecoder:
    def __init__(self, cache: ekv.PagedKVCache, num_q_heads: int, policy: int, attn: int,
                 topk: int = 0, alpha: float = 1.5, delta: float = 0.0, scale: float = 1.0,
                 max_sel: Optional[int] = None):
        self.cache, self.num_q_heads, self.policy, self.attn = cache, num_q_heads, policy, attn
        self.topk, self.alpha, self.delta, self.scale = topk, alpha, delta, scale
        B, H, P, d = cache.batch, cache.num_kv_heads, cache.page_size, cache.head_dim
        mp = cache.max_pages
        if max_sel is None:
            max_sel = min(topk, mp) if policy == ekv.EKV_SEL_TOPK else mp
        self.max_sel = max_sel
        dev = cache.k_cache.device
        if policy == ekv.EKV_SEL_TOPK:
            self.scores = torch.empty((B, H, mp), dtype=torch.float32, device=dev)
        else:
            self.scores = torch.empty((B, num_q_heads, 3, mp), dtype=torch.float32, device=dev)
        self.sel_idx = torch.empty((B, H, max_sel), dtype=torch.int32, device=dev)
        self.sel_count = torch.empty((B, H), dtype=torch.int32, device=dev)
        self.tau_hat = torch.empty((B, num_q_heads), dtype=torch.float32, device=dev)
        self.out = torch.empty((B, num_q_heads, d), dtype=torch.float32, device=dev)
        self.stat = torch.empty((B, num_q_heads), dtype=torch.float32, device=dev)
        nbytes = ekv.ekv_decode_workspace_bytes(cache, num_q_heads, max_sel)
        if nbytes == 0:
            raise ValueError("unsupported decoder geometry")
        self.ws = torch.empty((nbytes,), dtype=torch.uint8, device=dev)

    def update_metadata(self, new_start: torch.Tensor, new_count: torch.Tensor, max_new: int,
                        stream=None):
        ekv.ekv_page_meta_update(self.cache, new_start, new_count, max_new, stream)

    def capture(self, q_static: torch.Tensor, pre_step=None) -> torch.cuda.CUDAGraph:
        """Capture one decode step reading `q_static` into a CUDA graph (one launch per step
        on replay instead of one host call per kernel). `pre_step`, if given, is called inside
        the capture first (e.g. a metadata update of an appended page). Run one eager step
        before capturing so that one-time set-up happens outside the capture."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            if pre_step is not None:
                pre_step()
            self.step(q_static)
        return g

    def capture_host(self, q_dev: torch.Tensor, q_host: torch.Tensor, out_host: torch.Tensor,
                     stat_host: torch.Tensor, pre_step=None) -> torch.cuda.CUDAGraph:
        """Capture a whole host-to-host step in one CUDA graph: the query copied from pinned
        host memory into `q_dev`, the decode step, and the outputs copied back into pinned host
        buffers. Replay, then synchronise the stream, to run one step."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            if pre_step is not None:
                pre_step()
            q_dev.copy_(q_host, non_blocking=True)
            self.step(q_dev)
            out_host.copy_(self.out, non_blocking=True)
            stat_host.copy_(self.stat, non_blocking=True)
        return g

    def step(self, q: torch.Tensor, stream=None, append=None):
        """One decode step. `append` = (new_start, new_count, max_new), the arguments of
        ekv_page_meta_update, refreshes the appended pages' metadata first (in the scoring call)."""
        c = self.cache
        if append is not None:
            new_start, new_count, max_new = append
            ekv.ekv_refresh_score_pages(c, new_start, new_count, max_new, q, self.num_q_heads,
                                        self.scale, self.policy, self.scores, stream)
        else:
            ekv.ekv_score_pages(c, q, self.num_q_heads, self.scale, self.policy, self.scores,
                                stream)
        if self.policy == ekv.EKV_SEL_TOPK:
            # selection and attention in one call (the decode launched behind the selection)
            ekv.ekv_select_decode(c, q, self.num_q_heads, self.scale, self.attn, self.topk,
                                  self.scores, self.sel_idx, self.sel_count, self.max_sel,
                                  self.out, self.stat, self.ws, stream)
            return self.out, self.stat
        ekv.ekv_select_pages(c, self.num_q_heads, self.policy, self.topk, self.alpha, self.delta,
                             self.scores, self.sel_idx, self.sel_count, self.max_sel,
                             self.tau_hat, stream)
        ekv.ekv_sparse_decode(c, q, self.num_q_heads, self.scale, self.attn, self.sel_idx,
                              self.sel_count, self.max_sel, self.out, self.stat, self.ws, stream)
        return self.out, self.stat
