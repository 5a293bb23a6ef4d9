"""Seeded synthetic GCA streams: the five workloads and their input recipe.

This module holds data only — shapes and a seeded random draw per frame — and
none of the attention arithmetic.  Both the CUDA path (through ``bench.py`` and
the tests) and the CPU oracle (through the tests) receive their Q/K/V from here.

Workload shapes follow the Geometric Context Transformer pages:

* per frame M image-patch tokens plus S=6 summary tokens (1 camera, 1 anchor,
  4 register) — LingBot-Map paper digest, §2.2–2.3 (frame types, summary-token
  table);
* M = ceil(W/p) * ceil(H/p): 518x378 at patch 14 gives 37*27 = 999 — paper
  digest §1.2 and §4.3;
* the worked token-count example M~500, n=3, k=16, T=10000 — paper digest
  §2.4 (token-count table);
* default inference k=64, keyframe interval 1, bf16; windowed mode of 128
  frames overlapping by 16 — paper-to-code article §5 and code walkthrough
  §3.3.

Token order inside a frame: the S summary tokens first (camera, anchor,
register x4), then the M image tokens.  Tensors are token-major
``[L][S+M][H][D]``.

Seeding: every (workload, frame, tensor) draw has its own 64-bit seed, mixed
with SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
generators", OOPSLA 2014) from (seed0, workload id, frame, tensor id).  One draw
covers all L layers; layer l's stream is slice l of it, so layers hold
independent values.  torch's generator is device specific, so the CPU and CUDA
draws of the same seed differ; a test that compares the two paths hands both
the same tensors.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

MASK64 = (1 << 64) - 1
TENSOR_IDS = {"q": 1, "k": 2, "v": 3, "knorm": 4}


def splitmix64(x: int) -> int:
    """One SplitMix64 output step (Steele et al. 2014) on a 64-bit state."""
    x = (x + 0x9E3779B97F4A7C15) & MASK64
    z = x
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def frame_seed(workload_id: int, frame: int, tensor: str, seed0: int = 0) -> int:
    """64-bit seed of one (workload, frame, tensor) draw."""
    s = splitmix64(seed0 & MASK64)
    for field in (workload_id, frame, TENSOR_IDS[tensor]):
        s = splitmix64(s ^ (field & MASK64))
    return s


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic GCA stream.

    M image tokens + S summary tokens per frame, H heads of width D, n anchor
    frames, a k-frame pose-reference window, T frames streamed one at a time,
    L stacked layers with independent streams.
    """

    name: str
    workload_id: int
    M: int
    H: int
    n: int
    k: int
    T: int
    S: int = 6
    D: int = 64
    L: int = 1
    dtype: str = "bf16"               # "bf16" or "f32": the stored and computed input type
    key_norm_sigma: Optional[float] = None   # lognormal sigma of per-token key scaling
    page_size: int = 128
    window_frames: int = 0            # windowed (VO) mode: frames per window, 0 = direct mode
    window_overlap: int = 0
    seed0: int = 0

    @property
    def Lq(self) -> int:
        return self.M + self.S

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def windows(self):
        """Windowed (VO) mode: list of (start, length) of each window over the
        T global frames; consecutive windows overlap by ``window_overlap``."""
        if not self.window_frames:
            return [(0, self.T)]
        step = self.window_frames - self.window_overlap
        out, s = [], 0
        while True:
            ln = min(self.window_frames, self.T - s)
            out.append((s, ln))
            if s + ln >= self.T:
                return out
            s += step


# The five workloads.  Ids are part of the seed, so they never change.
TINY = Workload("tiny_M16_H2_n3_k4_T32", 1, M=16, H=2, n=3, k=4, T=32, dtype="f32")
TINY_BF16 = TINY.with_(name="tiny_M16_H2_n3_k4_T32_bf16", dtype="bf16")
WORKED_EXAMPLE = Workload("worked_M500_n3_k16_T10000", 2, M=500, H=16, n=3, k=16,
                          T=10000, key_norm_sigma=0.5)
METRIC_518x378 = Workload("gca_518x378_M999_n3_k64_T10000_L24", 3, M=999, H=16, n=3,
                          k=64, T=10000, L=24)
WINDOWED_VO = Workload("vo_M999_n3_k64_win128_ov16_T20000", 4, M=999, H=16, n=3, k=64,
                       T=20000, window_frames=128, window_overlap=16)
DENSE_CAUSAL = Workload("dense_causal_M999_T1000", 5, M=999, H=16, n=3, k=1000, T=1000)

WORKLOADS = {w.workload_id: w for w in (TINY, WORKED_EXAMPLE, METRIC_518x378,
                                        WINDOWED_VO, DENSE_CAUSAL)}


def draw(w: Workload, frame: int, tensor: str, device="cpu", layers=None) -> torch.Tensor:
    """Q, K or V of one frame for all L layers: ``[L][S+M][H][D]`` in w's dtype.

    Values are i.i.d. N(0,1) drawn in fp32 and rounded to the workload dtype.
    With ``key_norm_sigma`` set, every K token vector (per layer, per token,
    shared by the heads) is multiplied by exp(sigma * z), z ~ N(0,1), before
    rounding — lognormal key norms that make the softmax peaky.
    ``layers`` optionally selects a subset of layer indices of the draw.
    """
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(frame_seed(w.workload_id, frame, tensor, w.seed0))
    x = torch.randn((w.L, w.Lq, w.H, w.D), generator=g, device=dev, dtype=torch.float32)
    if tensor == "k" and w.key_norm_sigma:
        g2 = torch.Generator(device=dev)
        g2.manual_seed(frame_seed(w.workload_id, frame, "knorm", w.seed0))
        z = torch.randn((w.L, w.Lq), generator=g2, device=dev, dtype=torch.float32)
        x = x * torch.exp(w.key_norm_sigma * z)[:, :, None, None]
    if layers is not None:
        x = x[list(layers)]
    return x.to(w.torch_dtype())


def draw_frames(w: Workload, frames, tensor: str, layer: int = 0, device="cpu") -> torch.Tensor:
    """One layer's Q/K/V for a list of frames: ``[len(frames)][S+M][H][D]``."""
    return torch.stack([draw(w, f, tensor, device)[layer] for f in frames])
