"""Seeded synthetic streams shared by the CUDA path's tests/bench and the oracle.

This module holds only workload shapes and random-number recipes. It contains none
of the cache method's arithmetic (no attention, no paging, no scoring), so the
oracle and the CUDA library can both draw their inputs from it without sharing any
of the computation they are compared on.

Workloads follow the shapes the streaming visual-geometry pages describe:
518x378 frames at patch 14 give 37x27 = 999 patch tokens + 1 camera + 4 register
tokens = 1004 tokens per frame ("How GCTStream Implements Streaming 3D
Reconstruction with KV Cache", Implementation Example: ``patch_embed=
'dinov2_vitl14_reg'``; "Can LingBot-Map Achieve 20 FPS", opening paragraph), a
64-frame sliding window with 8 pinned scale frames ("Can LingBot-Map Achieve 20
FPS", Sliding-Window Eviction Strategy), and 518x518 frames -> 37x37 + 5 = 1374
tokens.

Recipes (all seeded, all deterministic for a given device type):
  * Q, V ~ N(0, 1) per frame.
  * K follows a per-slot random walk K_t = K_{t-1} + 0.1 * N(0, 1) held in fp32
    and rounded to the I/O dtype each frame (slow camera motion), when the
    workload is ``temporal``; otherwise K ~ N(0, 1).
  * Outlier channels (FP8 workload): a fixed seeded choice of round(0.01 * H * D)
    (head, dim) channels of K and V is multiplied by 8.
  * Residuals for the importance score: r = N(0, 1)[T, R] * exp(z)[:, None] with a
    per-(frame, token) log-normal scale z ~ N(0, 1) that is shared by all layers of
    that frame, and an independent Gaussian direction per layer.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, asdict
from typing import Dict, Optional

import torch

__all__ = ["Workload", "WORKLOADS", "FrameStream", "keyframe_schedule", "seed_for"]


@dataclass(frozen=True)
class Workload:
    name: str
    num_layers: int
    num_heads: int
    head_dim: int
    tokens_per_frame: int
    num_special_tokens: int
    page_size: int
    window_frames: int          # W (<= 0: no sliding window)
    scale_frames: int           # S pinned first frames
    keyframe_interval: int      # k
    num_frames: int
    io_dtype: str               # "f32" | "bf16"
    kv_dtype: str               # "f32" | "bf16" | "fp8_e4m3"
    softmax_scale: float
    temporal_keys: bool = False
    outlier_fraction: float = 0.0
    budget_tokens: int = 0      # B (0: no compression)
    keep_frac: float = 0.6
    lam: float = 0.5
    rank_window: int = 5
    residual_dim: int = 1024
    protect_first_frame: int = 1
    diversity_budget: int = 0
    special_frames: int = 0      # evicted frames whose special tokens stay cached (0: off)
    joint_frames: int = 0        # > 0: the stream opens with a joint phase of this many frames
    fp8_dim_adaptive: int = 0    # FP8 storage: K scales per channel, V scales per token
    description: str = ""

    def as_dict(self) -> Dict:
        return asdict(self)

    def replace(self, **kw) -> "Workload":
        d = asdict(self)
        d.update(kw)
        return Workload(**d)


WORKLOADS: Dict[str, Workload] = {
    "tiny_f32": Workload(
        name="tiny_f32", num_layers=1, num_heads=2, head_dim=32, tokens_per_frame=20,
        num_special_tokens=1, page_size=8, window_frames=4, scale_frames=1,
        keyframe_interval=1, num_frames=12, io_dtype="f32", kv_dtype="f32",
        softmax_scale=1.0 / math.sqrt(32.0),
        description="tiny fp32 case: 1 layer, 2x32 heads, 20 tok/frame, W=4, S=1, page 8, 12 frames"),
    "vggt_518x378": Workload(
        name="vggt_518x378", num_layers=1, num_heads=16, head_dim=64, tokens_per_frame=1004,
        num_special_tokens=5, page_size=16, window_frames=64, scale_frames=8,
        keyframe_interval=1, num_frames=300, io_dtype="bf16", kv_dtype="bf16",
        softmax_scale=0.125, temporal_keys=True,
        description="518x378 frames, 1004 tok/frame, 16x64 heads, W=64, S=8, page 16, bf16, 300 frames"),
    "vggt_24layer_k4": Workload(
        name="vggt_24layer_k4", num_layers=24, num_heads=16, head_dim=64, tokens_per_frame=1004,
        num_special_tokens=5, page_size=16, window_frames=64, scale_frames=8,
        keyframe_interval=4, num_frames=2000, io_dtype="bf16", kv_dtype="bf16",
        softmax_scale=0.125, temporal_keys=True,
        description="24 layers x the 518x378 shape, keyframe interval 4, 2000 frames"),
    "vggt_budget_16k": Workload(
        name="vggt_budget_16k", num_layers=24, num_heads=16, head_dim=64, tokens_per_frame=1004,
        num_special_tokens=5, page_size=16, window_frames=0, scale_frames=0,
        keyframe_interval=1, num_frames=1000, io_dtype="bf16", kv_dtype="bf16",
        softmax_scale=0.125, temporal_keys=True, budget_tokens=16384, keep_frac=0.6,
        lam=0.5, rank_window=5, residual_dim=1024, protect_first_frame=1,
        description="24 layers, budget B=16384 tokens/layer, keep/merge/drop compression, 1000 frames"),
    "vggt_518x518_fp8": Workload(
        name="vggt_518x518_fp8", num_layers=1, num_heads=16, head_dim=64, tokens_per_frame=1374,
        num_special_tokens=5, page_size=16, window_frames=128, scale_frames=8,
        keyframe_interval=1, num_frames=10000, io_dtype="bf16", kv_dtype="fp8_e4m3",
        softmax_scale=0.125, temporal_keys=False, outlier_fraction=0.01,
        description="518x518 frames, 1374 tok/frame, W=128, S=8, FP8 E4M3 K/V, 10000 frames"),
    "vggt_518x378_joint": Workload(
        name="vggt_518x378_joint", num_layers=1, num_heads=16, head_dim=64, tokens_per_frame=1004,
        num_special_tokens=5, page_size=16, window_frames=64, scale_frames=8,
        keyframe_interval=1, num_frames=8, io_dtype="bf16", kv_dtype="bf16",
        softmax_scale=0.125, temporal_keys=True, joint_frames=8,
        description="joint scale-frame phase: the first 8 frames of a 518x378 stream together, "
                    "8,032 queries over 8,032 keys per head"),
    "vggt_518x378_special": Workload(
        name="vggt_518x378_special", num_layers=1, num_heads=16, head_dim=64, tokens_per_frame=1004,
        num_special_tokens=5, page_size=16, window_frames=64, scale_frames=8,
        keyframe_interval=1, num_frames=10000, io_dtype="bf16", kv_dtype="bf16",
        softmax_scale=0.125, temporal_keys=True, special_frames=4096,
        description="518x378 stream keeping the 5 special tokens of up to 4,096 evicted frames"),
    "vggt_518x518_fp8da": Workload(
        name="vggt_518x518_fp8da", num_layers=1, num_heads=16, head_dim=64, tokens_per_frame=1374,
        num_special_tokens=5, page_size=16, window_frames=128, scale_frames=8,
        keyframe_interval=1, num_frames=10000, io_dtype="bf16", kv_dtype="fp8_e4m3",
        softmax_scale=0.125, temporal_keys=False, outlier_fraction=0.01, fp8_dim_adaptive=1,
        description="518x518 frames, W=128, dimension-adaptive FP8 storage (K per channel, V per token)"),
    "vggt_infinite_12l": Workload(
        name="vggt_infinite_12l", num_layers=12, num_heads=16, head_dim=64, tokens_per_frame=1004,
        num_special_tokens=5, page_size=16, window_frames=0, scale_frames=0,
        keyframe_interval=1, num_frames=1000, io_dtype="bf16", kv_dtype="bf16",
        softmax_scale=0.125, temporal_keys=True, diversity_budget=512,
        description="rolling diversity-pruned memory: 12 layers, 512 kept tokens per head (8,192 per "
                    "layer, ~98k total) besides the first frame, 518x378 frames, 1000 frames"),
}


def keyframe_schedule(t: int, scale_frames: int, keyframe_interval: int) -> bool:
    """Which frames persist their K/V: the first S frames, then every k-th frame.

    "Can LingBot-Map Achieve 20 FPS", Keyframe Interval Configuration, and "How
    GCTStream ...", Frame-by-Frame Causal Processing, say only every k-th frame is
    kept; the phase of that schedule is not given, so it starts at frame S.
    """
    k = max(1, int(keyframe_interval))
    return t < scale_frames or ((t - scale_frames) % k) == 0


def seed_for(base: int, layer: int, frame: int, which: int) -> int:
    """A deterministic 63-bit seed for one tensor of one frame of one layer."""
    x = (base & 0xFFFFFFFF) * 0x9E3779B1 + layer * 0x85EBCA77 + frame * 0xC2B2AE3D + which * 0x27D4EB2F
    x ^= x >> 29
    x = (x * 0xBF58476D1CE4E5B9) & ((1 << 64) - 1)
    x ^= x >> 32
    return x & ((1 << 63) - 1)


_Q, _K, _V, _K0, _RES, _Z, _OUT = range(7)

_TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


class FrameStream:
    """Generates the per-frame Q, K, V (and residuals) of one workload.

    Frames must be drawn in increasing order per layer when keys are temporal,
    because K_t depends on K_{t-1}. ``device`` may be "cpu" or a CUDA device;
    the same seed gives the same numbers on the same device type.
    """

    def __init__(self, wl: Workload, seed: int = 0, device="cpu", tokens: Optional[int] = None):
        self.wl = wl
        self.seed = int(seed)
        self.device = torch.device(device)
        self.T = int(tokens if tokens is not None else wl.tokens_per_frame)
        self.shape = (self.T, wl.num_heads, wl.head_dim)
        self.dtype = _TORCH_DTYPE[wl.io_dtype]
        self._kstate: Dict[int, torch.Tensor] = {}
        self._klast: Dict[int, int] = {}
        self._outlier_mask = None
        if wl.outlier_fraction > 0:
            n_ch = wl.num_heads * wl.head_dim
            n_out = int(round(wl.outlier_fraction * n_ch))
            g = torch.Generator(device="cpu").manual_seed(seed_for(self.seed, 0, 0, _OUT))
            perm = torch.randperm(n_ch, generator=g)[:n_out]
            m = torch.ones(n_ch, dtype=torch.float32)
            m[perm] = 8.0
            self._outlier_mask = m.view(1, wl.num_heads, wl.head_dim).to(self.device)
            self.outlier_channels = sorted(int(i) for i in perm)

    def _randn(self, shape, s):
        g = torch.Generator(device=self.device).manual_seed(s)
        return torch.randn(shape, generator=g, device=self.device, dtype=torch.float32)

    def _out(self, x: torch.Tensor) -> torch.Tensor:
        if self._outlier_mask is not None:
            x = x * self._outlier_mask
        return x.to(self.dtype)

    def frame(self, layer: int, t: int):
        """(Q, K, V) for frame t of ``layer``, each [T, H, D] in the I/O dtype."""
        wl = self.wl
        q = self._randn(self.shape, seed_for(self.seed, layer, t, _Q)).to(self.dtype)
        v = self._out(self._randn(self.shape, seed_for(self.seed, layer, t, _V)))
        if wl.temporal_keys:
            last = self._klast.get(layer, -1)
            if t == 0 or layer not in self._kstate:
                st = self._randn(self.shape, seed_for(self.seed, layer, 0, _K0))
                last = 0
                for u in range(1, t + 1):
                    st = st + 0.1 * self._randn(self.shape, seed_for(self.seed, layer, u, _K))
                last = t
            else:
                st = self._kstate[layer]
                if t < last:
                    raise ValueError("temporal keys must be drawn in increasing frame order")
                for u in range(last + 1, t + 1):
                    st = st + 0.1 * self._randn(self.shape, seed_for(self.seed, layer, u, _K))
                last = t
            self._kstate[layer] = st
            self._klast[layer] = last
            k = self._out(st)
        else:
            k = self._out(self._randn(self.shape, seed_for(self.seed, layer, t, _K)))
        return q, k, v

    def residual(self, layer: int, t: int) -> torch.Tensor:
        """Residual [T, R] fp32 whose row norms serve as the raw importance score."""
        wl = self.wl
        z = self._randn((self.T,), seed_for(self.seed, 0, t, _Z))
        r = self._randn((self.T, wl.residual_dim), seed_for(self.seed, layer, t, _RES))
        return (r * torch.exp(z)[:, None]).to(torch.float32)
