"""GPU parity of dimension-adaptive FP8 KV storage ("XStreamVGGT" abstract: K scales per
channel, V scales per token) through the C ABI: codes and every scale bit-exact against
the fp64 oracle, attention outputs within the bf16 tolerance."""
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


@pytest.mark.parametrize("T,H,W,S,frames,splits", [
    (300, 4, 6, 2, 10, 0),     # ragged last page, eviction, automatic splits
    (300, 2, 4, 1, 8, 3),      # about three pieces per head, merged in the kernel
    (37, 2, 3, 1, 8, 0),       # one ragged query tile, last page 5 valid
])
def test_dimension_adaptive_fp8(kvc, T, H, W, S, frames, splits):
    wl = WORKLOADS["vggt_518x518_fp8"].replace(tokens_per_frame=T, num_heads=H, window_frames=W, scale_frames=S,
                                                num_special_tokens=min(5, T), fp8_dim_adaptive=1)
    run_parity(kvc, wl, frames, kv_splits=splits, check_pages=True)


def test_dimension_adaptive_fp8_with_special_tokens(kvc):
    wl = WORKLOADS["vggt_518x518_fp8"].replace(tokens_per_frame=300, num_heads=2, window_frames=2, scale_frames=1,
                                                fp8_dim_adaptive=1, special_frames=3)
    run_parity(kvc, wl, 9, check_pages=True)


def test_dimension_adaptive_fp8_full_size_sampled(kvc):
    """518x518 frames (1,374 tokens), 16 heads, the window filled past its first evictions,
    sampled query rows."""
    wl = WORKLOADS["vggt_518x518_fp8"].replace(window_frames=8, scale_frames=2, fp8_dim_adaptive=1)
    run_parity(kvc, wl, 13, check_frames={11, 12}, rows=sample_rows(wl.tokens_per_frame, 32, seed=9))


def test_dimension_adaptive_needs_fp8_storage(kvc):
    for bad in (WORKLOADS["vggt_518x378"].replace(fp8_dim_adaptive=1),
                WORKLOADS["vggt_518x518_fp8"].replace(fp8_dim_adaptive=2)):
        with pytest.raises(kvc.KVCError):
            kvc.kvc_create(kvc.config_from_workload(bad))
    wl = WORKLOADS["vggt_518x518_fp8"].replace(tokens_per_frame=64, num_heads=2)
    h = kvc.kvc_create(kvc.config_from_workload(wl))
    try:
        with pytest.raises(kvc.KVCError):
            kvc.kvc_export_fp8_group_scales(h, 0, 0, 0, 2, 64, 16)   # per-(page, head) scales only
    finally:
        kvc.kvc_destroy(h)
