"""Brute-force cross-checks for the oracle, written independently of it.

No pages, no allocator: the retained set is rebuilt from its closed form (first S
committed keyframes, the last W committed keyframes, and the current frame), the
frames are concatenated explicitly, and the softmax is scipy's. FP8 storage goes
through torch's float8_e4m3fn cast (round-to-nearest-even for in-range values).
"""
from __future__ import annotations

import numpy as np
import scipy.special
import torch


def keyframes_before(t, S, k):
    """Committed keyframes strictly before frame t under the schedule t<S or (t-S)%k==0."""
    return [u for u in range(t) if u < S or (u - S) % max(1, k) == 0]


def retained_frames(t, S, W, k):
    """Closed form of the frames frame t attends to: pinned + window + itself."""
    prev = keyframes_before(t, S, k)
    keep = prev[:S] + [u for u in prev[-W:] if u not in prev[:S]] if W > 0 else prev
    return sorted(set(keep)) + [t]


def fp8_dequant_torch(x: np.ndarray) -> np.ndarray:
    """Absmax per-block FP8 E4M3 quantise + dequantise using torch's float8 cast."""
    x32 = torch.tensor(x, dtype=torch.float32)
    amax = x32.abs().max()
    if float(amax) == 0.0:
        return np.zeros_like(x)
    scale = amax / torch.tensor(448.0, dtype=torch.float32)
    q = (x32 / scale).to(torch.float8_e4m3fn).to(torch.float64)
    return (q * scale.double()).numpy()


def stored(K: np.ndarray, kv_dtype: str, P: int) -> np.ndarray:
    """Values the cache stores for one frame's K or V [T, H, D]."""
    if kv_dtype != "fp8_e4m3":
        return K
    T, H, D = K.shape
    out = np.zeros_like(K)
    for g in range(0, T, P):
        for h in range(H):
            out[g:g + P, h] = fp8_dequant_torch(K[g:g + P, h])
    return out


def stored_dim_adaptive(X: np.ndarray, P: int, per: str) -> np.ndarray:
    """Values the cache stores for one frame's K (per="channel": a scale per page, head and
    channel) or V (per="token": a scale per page, head and token) with dimension-adaptive
    FP8, through torch's float8 cast."""
    T, H, D = X.shape
    out = np.zeros_like(X)
    for g in range(0, T, P):
        for h in range(H):
            blk = X[g:g + P, h]
            if per == "channel":
                for d in range(D):
                    out[g:g + P, h, d] = fp8_dequant_torch(blk[:, d])
            else:
                for i in range(blk.shape[0]):
                    out[g + i, h] = fp8_dequant_torch(blk[i])
    return out


def attention(Q, K, V, scale):
    """Full softmax attention per head, fp64, scipy softmax."""
    N, H, D = K.shape
    out = np.empty((Q.shape[0], H, D))
    for h in range(H):
        z = scale * (Q[:, h] @ K[:, h].T)
        out[:, h] = scipy.special.softmax(z, axis=1) @ V[:, h]
    return out
