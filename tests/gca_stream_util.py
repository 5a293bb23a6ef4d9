"""Helpers for the GPU parity tests: drive a seeded stream through the C-ABI
library and keep, on the host, what the oracle needs to recompute any step.

The host mirror holds, per checked layer, the summary tokens of every frame and
the full tokens of the frames that may still be full (anchors and the recent
window), as float32 copies of the exact bf16/fp32 values."""
from __future__ import annotations

import numpy as np
import torch

from oracle import gca as ogca
from windowed_memory_attention_b200 import gca, inputs


class Mirror:
    def __init__(self, w: inputs.Workload, layers, heads=None):
        self.w = w
        self.layers = list(layers)
        self.heads = None if heads is None else list(heads)   # record only these heads
        self.summ_k = {l: {} for l in self.layers}
        self.summ_v = {l: {} for l in self.layers}
        self.full_k = {l: {} for l in self.layers}
        self.full_v = {l: {} for l in self.layers}

    def record(self, frame: int, k: torch.Tensor, v: torch.Tensor, keep_full: bool):
        """k, v: [L][S+M][H][D] on any device."""
        S = self.w.S
        for l in self.layers:
            kl = k[l].float()
            vl = v[l].float()
            if self.heads is not None:
                kl, vl = kl[:, self.heads], vl[:, self.heads]
            self.summ_k[l][frame] = kl[:S].cpu().numpy()
            self.summ_v[l][frame] = vl[:S].cpu().numpy()
            if keep_full:
                self.full_k[l][frame] = kl.cpu().numpy()
                self.full_v[l][frame] = vl.cpu().numpy()

    def drop_full(self, keep):
        for l in self.layers:
            for f in list(self.full_k[l]):
                if f not in keep:
                    del self.full_k[l][f]
                    del self.full_v[l][f]

    def frame_kv(self, layer: int):
        def get(j, summary_only):
            if summary_only:
                return self.summ_k[layer][j], self.summ_v[layer][j]
            return self.full_k[layer][j], self.full_v[layer][j]
        return get


def needed_full(w: inputs.Workload, t: int, F: int = 1):
    """Frames whose full tokens a block of F frames ending at t may read."""
    keep = set(range(min(w.n, t + 1)))
    keep |= set(range(max(0, t - F + 1 - w.k + 1), t + 1))
    return keep


def oracle_step(mirror: Mirror, layer: int, q_block: np.ndarray, last: int, F: int = 1,
                rows=None, anchor_block: bool = False, keep=None):
    """Oracle output of a query block; q_block holds all heads, the mirror's
    head subset (if any) is applied to it.  keep: special tokens a frame keeps
    after eviction (default all S)."""
    w = mirror.w
    qb = q_block if mirror.heads is None else q_block[:, :, mirror.heads]
    return ogca.stream_step(qb, last, mirror.frame_kv(layer), n=w.n, k=w.k, S=w.S,
                            scale=w.softmax_scale, anchor_block=anchor_block, rows=rows, keep=keep)


def oracle_transient(mirror: Mirror, layer: int, q: np.ndarray, k: np.ndarray, v: np.ndarray,
                     last_key: int, rows=None, anchor_block: bool = False):
    """Oracle output of a non-keyframe (q, k, v [S+M][H][D], all heads) that
    reads the cache after keyframe last_key plus its own tokens."""
    w = mirror.w
    if mirror.heads is not None:
        q, k, v = q[:, mirror.heads], k[:, mirror.heads], v[:, mirror.heads]
    return ogca.transient_step(q, k, v, last_key, mirror.frame_kv(layer), n=w.n, k=w.k, S=w.S,
                               scale=w.softmax_scale, anchor_block=anchor_block, rows=rows)


def attend_transient(cache: gca.Cache, layer: int, q: torch.Tensor, k: torch.Tensor,
                     v: torch.Tensor):
    """q, k, v: [S+M][H][D] on the GPU; returns (out, lse) on the GPU."""
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device=q.device)
    cache.attend_transient(layer, q, k, v, out, lse)
    return out, lse


def attend(cache: gca.Cache, layer: int, q: torch.Tensor, F: int = 1):
    """q: [F][S+M][H][D] on the GPU; returns (out, lse) on the GPU."""
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    cache.attend(layer, q, out, lse, num_query_frames=F)
    return out, lse


def max_err(got: torch.Tensor, want: np.ndarray) -> float:
    return float(np.abs(got.double().cpu().numpy() - want).max())


class CudaArray:
    """Wraps a raw device pointer for torch.as_tensor (CUDA array interface)."""

    def __init__(self, ptr: int, nbytes: int):
        self.__cuda_array_interface__ = {"shape": (nbytes,), "typestr": "|u1",
                                         "data": (ptr, False), "version": 2}


def pool_view(cache: gca.Cache, which: str, dtype: torch.dtype) -> torch.Tensor:
    info = cache.info()
    ptr = info.k_pool if which == "k" else info.v_pool
    raw = torch.as_tensor(CudaArray(ptr, info.pool_bytes), device="cuda")
    return raw.view(dtype)
