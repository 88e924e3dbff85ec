"""GPU parity of the joint scale-frame phase and of cross-frame special tokens (GCTStream
page: Scale-Frame Phase, Special Token Persistence) through the C ABI, against the fp64
oracle: outputs within the dtype's tolerance, page tables and stored page bytes exact."""
import numpy as np
import pytest
import torch

from kvc_gpu_util import run_parity, sample_rows
from kvc_streams import WORKLOADS

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvc():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import transformer_kv_cache_b200 as m
    return m


@pytest.mark.parametrize("base,T,H,S,W,n,frames", [
    ("vggt_518x378", 300, 4, 3, 4, 3, 9),       # 900 joint queries (7 tiles + ragged), tensor cores
    ("vggt_518x378", 37, 2, 2, 3, 1, 6),        # a one-frame joint phase, ragged pages
    ("vggt_518x518_fp8", 300, 2, 2, 3, 2, 7),   # FP8 storage
    ("tiny_f32", 37, 2, 2, 3, 2, 7),            # fp32 I/O and storage
])
def test_joint_scale_phase(kvc, base, T, H, S, W, n, frames):
    wl = WORKLOADS[base].replace(tokens_per_frame=T, num_heads=H, scale_frames=S, window_frames=W,
                                 num_special_tokens=min(5, T))
    run_parity(kvc, wl, frames, joint=n, check_pages=True)


def test_joint_scale_phase_full_size(kvc):
    """The 518x378 shape with its 8 scale frames: 8,032 queries over 8,032 keys per head,
    sampled rows, then two causal frames."""
    wl = WORKLOADS["vggt_518x378"]
    run_parity(kvc, wl, 10, joint=8, joint_rows=sample_rows(8 * wl.tokens_per_frame, 48, seed=6),
               rows=sample_rows(wl.tokens_per_frame, 32, seed=7))


@pytest.mark.parametrize("base,T,H,S,W,ns,special,k,frames", [
    ("vggt_518x378", 300, 4, 2, 3, 5, 4, 1, 14),     # one page per evicted frame, FIFO after 4
    ("vggt_518x378", 300, 2, 1, 2, 5, 3, 2, 16),     # keyframe interval 2: non-keyframes keep nothing
    ("vggt_518x378", 40, 2, 1, 2, 18, 3, 1, 10),     # specials span two pages (16 + 2)
    ("vggt_518x518_fp8", 300, 2, 1, 2, 5, 3, 1, 10), # FP8 codes zeroed past the special tokens
    ("tiny_f32", 37, 2, 1, 2, 5, 50, 1, 12),         # fp32, the cap never reached
])
def test_special_tokens_persist(kvc, base, T, H, S, W, ns, special, k, frames):
    wl = WORKLOADS[base].replace(tokens_per_frame=T, num_heads=H, scale_frames=S, window_frames=W,
                                 num_special_tokens=ns, special_frames=special, keyframe_interval=k)
    run_parity(kvc, wl, frames, check_pages=True)


def test_joint_phase_then_special_tokens(kvc):
    wl = WORKLOADS["vggt_518x378"].replace(tokens_per_frame=300, num_heads=4, scale_frames=2, window_frames=2,
                                            special_frames=3)
    run_parity(kvc, wl, 12, joint=2, check_pages=True)


def test_special_tokens_full_size_sampled(kvc):
    """The 518x378 stream (window 64, 8 scale frames) past its first evictions with the
    specials of up to 10 evicted frames kept; sampled rows on the last frames."""
    wl = WORKLOADS["vggt_518x378"].replace(special_frames=10)
    run_parity(kvc, wl, 78, check_frames={74, 77}, rows=sample_rows(wl.tokens_per_frame, 24, seed=8))


def test_scale_phase_errors(kvc):
    wl = WORKLOADS["vggt_518x378"].replace(tokens_per_frame=64, num_heads=2, scale_frames=2, window_frames=2)
    h = kvc.kvc_create(kvc.config_from_workload(wl))
    try:
        x = torch.zeros((3 * 64, 2, 64), dtype=torch.bfloat16, device="cuda")
        with pytest.raises(kvc.KVCError):
            kvc.kvc_scale_phase(h, 0, 3, x, x, x, x)             # more than scale_frames
        kvc.kvc_scale_phase(h, 0, 2, x[:128], x[:128], x[:128], x[:128])
        with pytest.raises(kvc.KVCError):
            kvc.kvc_scale_phase(h, 0, 1, x[:64], x[:64], x[:64], x[:64])   # the layer is not empty
        kvc.kvc_append_frame(h, 0, 2, x[:64], x[:64], True)           # the causal phase continues
        kvc.kvc_attend(h, 0, x[:64], x[:64])
    finally:
        kvc.kvc_destroy(h)
    for bad in (WORKLOADS["vggt_budget_16k"].replace(special_frames=2),          # no window
                WORKLOADS["vggt_infinite_12l"].replace(special_frames=2)):
        with pytest.raises(kvc.KVCError):
            kvc.kvc_create(kvc.config_from_workload(bad))
