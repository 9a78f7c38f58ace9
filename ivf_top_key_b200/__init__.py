"""Causal IVF top-k key selection on B200 (sm_100a).

`AttentionIndex` wraps one handle of the C library (one request and layer):
insert keys, seal windows, refit, and select the top-k keys of every query
of a prefill chunk by routing over cluster representatives and refining
with the exact indexer score.  Output tensors are allocated with torch on
the handle's device; everything else is forwarded to the library.
"""
from __future__ import annotations

import ctypes

import torch

from . import _capi as C
from ._capi import AiError  # noqa: F401

__all__ = ["AttentionIndex", "AiError", "quantize_fp8", "merge_topk", "C"]


class AttentionIndex:
    """One causal IVF index (see include/ai_index.h for the semantics)."""

    def __init__(self, *, d: int, H: int, key_dtype: str = "bf16", q_dtype: str = "bf16",
                 n_sinks: int = 4, window: int = 1024, clusters_per_window: int = 8,
                 cluster_cap: int = 0, refit_period: int = 16384, refit_new_seeds: int = 0,
                 refit_seed_window: int = 0, seal_iters: int = 10, async_refit: bool = True,
                 max_query_chunk: int = 8192, max_budget: int = 8192, max_k: int = 2048,
                 max_keys: int = 1 << 17, seed: int = 0, encoder_weights=None, stream=None,
                 block_routing: bool = False):
        cfg = C.AiConfig()
        cfg.d, cfg.H = d, H
        cfg.key_dtype, cfg.q_dtype = C.DTYPES[key_dtype], C.DTYPES[q_dtype]
        cfg.n_sinks, cfg.window, cfg.clusters_per_window = n_sinks, window, clusters_per_window
        cfg.cluster_cap, cfg.refit_period = cluster_cap, refit_period
        cfg.refit_new_seeds, cfg.refit_seed_window = refit_new_seeds, refit_seed_window
        cfg.seal_iters, cfg.async_refit = seal_iters, int(async_refit)
        cfg.max_query_chunk, cfg.max_budget, cfg.max_k = max_query_chunk, max_budget, max_k
        cfg.max_keys, cfg.seed = max_keys, seed
        cfg.block_routing = int(block_routing)
        self._enc = None
        if encoder_weights is not None:
            import numpy as np
            packed = np.concatenate([np.asarray(encoder_weights[k], dtype=np.float32).ravel()
                                     for k in ("A", "a", "B1", "b1", "B2", "b2")])
            self._enc = packed
            cfg.encoder_weights_host = packed.ctypes.data_as(ctypes.POINTER(ctypes.c_float))
        self.d, self.H, self.key_dtype, self.q_dtype = d, H, key_dtype, q_dtype
        self.device = torch.device("cuda", torch.cuda.current_device())
        self.stream = stream if stream is not None else torch.cuda.current_stream()
        self.h = C.ai_index_create(cfg, self.stream)

    def close(self):
        if self.h is not None:
            C.ai_index_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- maintenance
    def append_keys(self, keys: torch.Tensor, scales: torch.Tensor | None = None):
        C.ai_append_keys(self.h, keys, scales)

    def seal(self) -> int:
        return C.ai_seal(self.h)

    def refit(self, n_new_seeds: int = 0, seed_window: int = 0) -> int:
        return C.ai_refit(self.h, n_new_seeds, seed_window)

    def publish(self):
        C.ai_publish(self.h)

    # -- selection
    def route_refine(self, q, w, pos0: int, k: int, C_budget: int, out=None, out_scores=None):
        if out is None:
            out = torch.empty((q.shape[0], k), dtype=torch.int32, device=q.device)
        return C.ai_route_refine(self.h, q, w, pos0, k, C_budget, out, out_scores)

    def route_refine_shard(self, q, w, pos0: int, k: int, C_budget: int, shard: int, n_shards: int,
                           out=None, out_scores=None):
        """This shard's top k of the sharded rescore (see ai_route_refine_shard)."""
        T = q.shape[0]
        if out is None:
            out = torch.empty((T, k), dtype=torch.int32, device=q.device)
        if out_scores is None:
            out_scores = torch.empty((T, k), dtype=torch.float32, device=q.device)
        return C.ai_route_refine_shard(self.h, q, w, pos0, k, C_budget, shard, n_shards, out, out_scores)

    def select_exhaustive(self, q, w, pos0: int, k: int, out=None, out_scores=None):
        if out is None:
            out = torch.empty((q.shape[0], k), dtype=torch.int32, device=q.device)
        return C.ai_select_exhaustive(self.h, q, w, pos0, k, out, out_scores)

    # -- inspection / control
    def sync(self):
        C.ai_sync(self.h)

    def stats(self) -> dict:
        return C.ai_get_stats(self.h)

    def export_index(self) -> dict:
        return C.ai_export_index(self.h, self.d)

    def debug_candidates(self, q, w, pos0: int, C_budget: int, with_scores: bool = True):
        T = q.shape[0]
        cand = torch.empty((T, C_budget), dtype=torch.int32, device=q.device)
        nC = self.stats()["n_clusters"]
        cs = torch.empty((T, max(nC, 1)), dtype=torch.float32, device=q.device) if with_scores else None
        C.ai_debug_candidates(self.h, q, w, pos0, C_budget, cand, cs if nC > 0 else None)
        return cand, (cs[:, :nC] if cs is not None else None)

    def debug_scores(self, q, w, pos0: int):
        n = self.stats()["n_keys"]
        out = torch.empty((q.shape[0], n), dtype=torch.float32, device=q.device)
        return C.ai_debug_scores(self.h, q, w, pos0, out)

    def debug_refine_kernel(self, kernel: int):
        """Force a tensor-core refine variant (0 = by occupancy, 1 / 2 =
        one query per CTA with the list in shared / global memory, 3 =
        pipelined, 4 = pipelined with one TMEM score buffer); every variant
        computes the same result."""
        C.ai_debug_refine_kernel(self.h, kernel)

    def debug_refine_split(self, split: int):
        """Parts per query of small chunks (0 = by chunk size, 1 = never
        divide, 2..8 = at most that many); results are identical either
        way."""
        C.ai_debug_refine_split(self.h, split)

    def refine_kernel_choice(self, C_budget: int) -> int:
        """The refine kernel route_refine launches for this budget (0 = fp32
        SIMT path, 1 / 2 = one query per CTA, 3 / 4 = pipelined with two /
        one score buffers)."""
        return C.ai_refine_kernel_choice(self.h, C_budget)

    def profile(self, enable: bool = True):
        C.ai_profile_enable(self.h, enable)

    def profile_read(self) -> dict:
        """{phase: (milliseconds, timed launches)} since the last read."""
        return C.ai_profile_read(self.h)

    def checkpoint(self):
        C.ai_checkpoint(self.h)

    def rollback(self):
        C.ai_rollback(self.h)


def merge_topk(ids: torch.Tensor, scores: torch.Tensor, k: int, out=None, out_scores=None, stream=None):
    """Top k of the union of n_parts partial results [n_parts, T, k] (library kernel)."""
    T = ids.shape[1]
    if out is None:
        out = torch.empty((T, k), dtype=torch.int32, device=ids.device)
    return C.ai_merge_topk(ids, scores, k, out, out_scores, stream)


def quantize_fp8(keys_bf16: torch.Tensor, stream=None):
    """Per-key scale amax/448 and E4M3 codes (library kernel)."""
    n, d = keys_bf16.shape
    codes = torch.empty((n, d), dtype=torch.uint8, device=keys_bf16.device)
    scales = torch.empty((n,), dtype=torch.float32, device=keys_bf16.device)
    return C.ai_quantize_fp8(keys_bf16, codes, scales, stream)
