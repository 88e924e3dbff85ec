"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the same
seeded inputs. Page tables and stored pages are compared bit for bit; attention outputs
within max-abs 2e-2 / mean-abs 2e-3 (bf16) or 1e-4 (fp32)."""
import numpy as np
import pytest
import torch

from kvc_gpu_util import run_parity, sample_rows, compare_out, np64
from kvc_streams import WORKLOADS, FrameStream, keyframe_schedule
from oracle import OracleConfig, StreamOracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvc():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import transformer_kv_cache_b200 as m
    return m


def test_tiny_f32_full_stream(kvc):
    wl = WORKLOADS["tiny_f32"]
    stats = run_parity(kvc, wl, wl.num_frames, check_pages=True)
    assert len(stats) == wl.num_frames


@pytest.mark.parametrize("T,H,W,S,frames,splits", [
    (300, 4, 6, 2, 12, 0),      # 3 q tiles with a ragged 44-row tail, eviction active
    (300, 4, 6, 2, 12, 1),      # no KV split
    (300, 4, 6, 2, 12, 5),      # forced split count
    (37, 2, 3, 1, 8, 0),        # one ragged q tile, 3 pages/frame, last page 5 valid
    (5, 2, 2, 0, 6, 0),         # T < P: every page partial
    (256, 2, 2, 1, 6, 3),       # T a multiple of the page size and of the q tile
    (300, 4, 20, 2, 24, 16),    # 16 split CTAs per query tile merged by the last to finish
])
def test_bf16_tensor_core_small(kvc, T, H, W, S, frames, splits):
    wl = WORKLOADS["vggt_518x378"].replace(tokens_per_frame=T, num_heads=H, window_frames=W, scale_frames=S,
                                            num_special_tokens=min(5, T))
    run_parity(kvc, wl, frames, kv_splits=splits, check_pages=True)


@pytest.mark.parametrize("kv_dtype,dim_adaptive", [("bf16", 0), ("fp8_e4m3", 0), ("fp8_e4m3", 1)])
def test_attend_all_layers_one_launch(kvc, kv_dtype, dim_adaptive):
    """kvc_attend_all on a 4-layer window cache whose layers are small (one launch for every
    layer): every layer's output against the oracle, page tables equal, keyframe interval
    2 past the window, and the library's launch count shows one attention launch per frame;
    bf16 and FP8 E4M3 storage (page scales, and dimension-adaptive scales)."""
    wl = WORKLOADS["vggt_24layer_k4"].replace(num_layers=4, tokens_per_frame=200, num_heads=4, window_frames=3,
                                              scale_frames=1, keyframe_interval=2, num_special_tokens=5,
                                              kv_dtype=kv_dtype, fp8_dim_adaptive=dim_adaptive)
    L, T, H, D = wl.num_layers, wl.tokens_per_frame, wl.num_heads, wl.head_dim
    dev = torch.device("cuda")
    h = kvc.kvc_create(kvc.config_from_workload(wl))
    try:
        st = FrameStream(wl, seed=19, device=dev)
        orc = StreamOracle(OracleConfig.from_workload(wl))
        outs = [torch.empty((T, H, D), dtype=torch.bfloat16, device=dev) for _ in range(L)]
        for t in range(11):
            key = keyframe_schedule(t, wl.scale_frames, wl.keyframe_interval)
            qkv = [st.frame(l, t) for l in range(L)]
            kvc.kvc_append_frame_all(h, t, [x[1] for x in qkv], [x[2] for x in qkv], key)
            _, before = kvc.kvc_page_table(h, 0)
            kvc.kvc_attend_all(h, [x[0] for x in qkv], outs)
            _, after = kvc.kvc_page_table(h, 0)
            attn = after["kernel_launches"] - before["kernel_launches"]
            assert attn <= 1 + L, (t, attn)              # one attention launch, at most one eviction per layer
            torch.cuda.synchronize()
            for l in range(L):
                q, k, v = qkv[l]
                orc.append(l, t, np64(k), np64(v), key)
                ref = orc.attend(l, np64(q))
                compare_out(np64(outs[l]), ref, "bf16", f"frame {t} layer {l}")
                pt, info = kvc.kvc_page_table(h, l)
                assert np.array_equal(pt, orc.page_table(l)), f"page table differs at frame {t} layer {l}"
                assert info["device_error"] == 0
    finally:
        kvc.kvc_destroy(h)


def test_bf16_keyframes_two_layers(kvc):
    wl = WORKLOADS["vggt_24layer_k4"].replace(num_layers=2, tokens_per_frame=200, num_heads=4,
                                               window_frames=4, scale_frames=2)
    run_parity(kvc, wl, 16, check_pages=True)


def test_batched_append_all_layers(kvc):
    """kvc_append_frame_all (one allocation + one append launch for all layers) gives the
    same page tables, pages and outputs as the oracle, bf16 with keyframes and FP8."""
    wl = WORKLOADS["vggt_24layer_k4"].replace(num_layers=3, tokens_per_frame=200, num_heads=4,
                                               window_frames=3, scale_frames=1)
    run_parity(kvc, wl, 12, check_pages=True, batched_append=True)
    wl8 = WORKLOADS["vggt_518x518_fp8"].replace(num_layers=2, tokens_per_frame=150, num_heads=4, window_frames=3,
                                                scale_frames=1)
    run_parity(kvc, wl8, 7, check_pages=True, batched_append=True)


def test_fp8_small_codes_and_outputs(kvc):
    wl = WORKLOADS["vggt_518x518_fp8"].replace(tokens_per_frame=150, num_heads=4, window_frames=4, scale_frames=2)
    run_parity(kvc, wl, 9, check_pages=True)


@pytest.mark.parametrize("T,H,splits", [
    (300, 3, 1),     # one piece per head: every KV tile in one softmax pass
    (300, 3, 3),     # about three pieces per head, merged in the kernel
    (37, 2, 0),      # ragged q tile, partial last page of every frame
])
def test_fp8_tensor_core(kvc, T, H, splits):
    """FP8 E4M3 storage on the tensor-core path (head dim 64, page size 16)."""
    wl = WORKLOADS["vggt_518x518_fp8"].replace(tokens_per_frame=T, num_heads=H, window_frames=5, scale_frames=2,
                                                num_special_tokens=min(5, T))
    run_parity(kvc, wl, 10, kv_splits=splits, check_pages=True)


def test_fp8_queries_beyond_the_f16_range(kvc):
    """The FP8 path feeds Q to the tensor cores as f16 (largest finite value 65,504). Query
    rows far above that range (x 2^30) and far below f16's smallest normal (x 2^-20) are
    scaled per row by a power of two, exactly, and match the oracle. The softmax scale is
    2^-30 times the usual one, so the large rows' logits are the usual well-conditioned
    ones and the other rows' logits are near zero (near-uniform weights), all resolvable in
    fp32; a split over several CTAs is included."""
    wl = WORKLOADS["vggt_518x518_fp8"].replace(tokens_per_frame=150, num_heads=4, window_frames=4, scale_frames=2,
                                                softmax_scale=0.125 * 2.0 ** -30)

    def scale_q(t, layer, q, k, v):
        q = q.clone()
        q[0:60] *= 2.0 ** 30
        q[60:80] *= 2.0 ** -20
        q[80:85, 1] *= 2.0 ** 30
        return q, k, v
    for splits in (0, 3):
        run_parity(kvc, wl, 8, transform=scale_q, kv_splits=splits)


def test_head_range_caches_rebuild_the_full_output(kvc):
    """Two caches holding heads [0, 2) and [2, 4) of a 4-head model (model_heads = 4,
    head_begin = 0 and 2) take the same full-width Q, K and V; each writes only its slice of
    O, and the two slices together equal the oracle's full output. Page tables of both
    equal the full cache's (allocation does not depend on the heads)."""
    wl = WORKLOADS["vggt_518x378"].replace(tokens_per_frame=300, num_heads=4, window_frames=3, scale_frames=1)
    half = wl.replace(num_heads=2)
    T, D = wl.tokens_per_frame, wl.head_dim
    dev = torch.device("cuda")
    hs = [kvc.kvc_create(kvc.config_from_workload(half, model_heads=4, head_begin=b)) for b in (0, 2)]
    try:
        st = FrameStream(wl, seed=17, device=dev)
        orc = StreamOracle(OracleConfig.from_workload(wl))
        for t in range(8):
            q, k, v = st.frame(0, t)
            o = torch.full((T, 4, D), float("nan"), dtype=torch.bfloat16, device=dev)
            for i, h in enumerate(hs):
                kvc.kvc_append_frame(h, 0, t, k, v, True)
                kvc.kvc_attend(h, 0, q, o)
                torch.cuda.synchronize()
                written = torch.isfinite(o.float()).all(dim=2).all(dim=0)
                assert written.tolist() == [True, True, i == 1, i == 1], (t, i)
            orc.append(0, t, np64(k), np64(v), True)
            ref = orc.attend(0, np64(q))
            compare_out(np64(o), ref, "bf16", f"frame {t}")
            for h in hs:
                pt, info = kvc.kvc_page_table(h, 0)
                assert np.array_equal(pt, orc.page_table(0)) and info["device_error"] == 0
    finally:
        for h in hs:
            kvc.kvc_destroy(h)


def test_fp8_zero_blocks(kvc):
    """All-zero K or V blocks quantise to scale 0 and codes 0; attention over them (the
    first frame's K all zero, then a zero V frame, then both zero) matches the oracle."""
    def zero(t, layer, q, k, v):
        if t in (0, 3):
            k = torch.zeros_like(k)
        if t in (2, 3):
            v = torch.zeros_like(v)
        return q, k, v
    wl = WORKLOADS["vggt_518x518_fp8"].replace(tokens_per_frame=150, num_heads=2, window_frames=4, scale_frames=1)
    run_parity(kvc, wl, 7, check_pages=True, transform=zero)


@pytest.mark.parametrize("D,P", [(32, 16), (64, 8)])
def test_fp8_simt_shapes(kvc, D, P):
    """FP8 storage with a head dim or page size the tensor-core kernel does not take."""
    wl = WORKLOADS["vggt_518x518_fp8"].replace(tokens_per_frame=100, num_heads=2, head_dim=D, page_size=P,
                                                window_frames=3, scale_frames=1, softmax_scale=D ** -0.5)
    run_parity(kvc, wl, 6, check_pages=True)


def test_fp8_full_size_steady_state_sampled(kvc):
    """The 518x518 FP8 workload at full size past the window, sampled rows."""
    wl = WORKLOADS["vggt_518x518_fp8"]
    rows = sample_rows(wl.tokens_per_frame, 48, seed=2)
    frames = wl.scale_frames + wl.window_frames + 2
    check = {0, wl.scale_frames, wl.scale_frames + wl.window_frames, frames - 1}
    stats = run_parity(kvc, wl, frames, check_frames=check, rows=rows)
    assert len(stats) == len(check)


def test_vggt_full_size_steady_state_sampled(kvc):
    """The 518x378 workload at full size past the window (eviction running), sampled rows."""
    wl = WORKLOADS["vggt_518x378"]
    rows = sample_rows(wl.tokens_per_frame, 64, seed=1)
    frames = wl.scale_frames + wl.window_frames + 4
    check = {0, 1, wl.scale_frames, wl.scale_frames + wl.window_frames - 1, wl.scale_frames + wl.window_frames,
             frames - 1}
    stats = run_parity(kvc, wl, frames, check_frames=check, rows=rows)
    assert len(stats) == len(check)


def test_split_counts_agree(kvc):
    """Different KV split counts give the same answer within fp32 reassociation."""
    wl = WORKLOADS["vggt_518x378"].replace(tokens_per_frame=500, num_heads=2, window_frames=10, scale_frames=2)
    dev = torch.device("cuda")
    outs = []
    for splits in (1, 2, 7):
        h = kvc.kvc_create(kvc.config_from_workload(wl, kv_splits=splits))
        st = FrameStream(wl, seed=3, device=dev)
        o = torch.empty((wl.tokens_per_frame, wl.num_heads, wl.head_dim), dtype=torch.bfloat16, device=dev)
        for t in range(12):
            q, k, v = st.frame(0, t)
            kvc.kvc_append_frame(h, 0, t, k, v, True)
            kvc.kvc_attend(h, 0, q, o)
        torch.cuda.synchronize()
        outs.append(np64(o))
        kvc.kvc_destroy(h)
    for o in outs[1:]:
        assert np.abs(o - outs[0]).max() <= 2 * 2 ** -8


def test_reset_replays_bit_exact(kvc):
    wl = WORKLOADS["vggt_518x378"].replace(tokens_per_frame=300, num_heads=2, window_frames=4, scale_frames=1)
    dev = torch.device("cuda")
    h = kvc.kvc_create(kvc.config_from_workload(wl))
    res = []
    for rep in range(2):
        st = FrameStream(wl, seed=4, device=dev)
        o = torch.empty((300, 2, 64), dtype=torch.bfloat16, device=dev)
        outs = []
        for t in range(8):
            q, k, v = st.frame(0, t)
            kvc.kvc_append_frame(h, 0, t, k, v, True)
            kvc.kvc_attend(h, 0, q, o)
            outs.append(o.clone())
        torch.cuda.synchronize()
        res.append(outs)
        pt, info = kvc.kvc_page_table(h, 0)
        kvc.kvc_reset(h)
        pt2, info2 = kvc.kvc_page_table(h, 0)
        assert len(pt2) == 0 and info2["tokens"] == 0
    for a, b in zip(*res):
        assert torch.equal(a, b)
    kvc.kvc_destroy(h)


def test_host_buffer_step_matches_device_path(kvc):
    wl = WORKLOADS["vggt_518x378"].replace(tokens_per_frame=300, num_heads=4, window_frames=4, scale_frames=1)
    dev = torch.device("cuda")
    h1 = kvc.kvc_create(kvc.config_from_workload(wl))
    h2 = kvc.kvc_create(kvc.config_from_workload(wl))
    st = FrameStream(wl, seed=5, device=dev)
    o = torch.empty((300, 4, 64), dtype=torch.bfloat16, device=dev)
    oh = torch.empty((300, 4, 64), dtype=torch.bfloat16).pin_memory()
    for t in range(7):
        q, k, v = st.frame(0, t)
        kvc.kvc_append_frame(h1, 0, t, k, v, True)
        kvc.kvc_attend(h1, 0, q, o)
        qh, kh, vh = (x.cpu().pin_memory() for x in (q, k, v))
        kvc.kvc_step_host(h2, 0, t, True, qh, kh, vh, oh)
        torch.cuda.synchronize()
        assert torch.equal(o.cpu(), oh)
    kvc.kvc_destroy(h1)
    kvc.kvc_destroy(h2)


def test_async_host_steps_match_device_path(kvc):
    """kvc_step_host_async: nine frames (keyframe interval 2) enqueued back to back on a
    user stream with no host sync in between, outputs downloaded into separate pinned
    buffers; after one kvc_synchronize every output equals the device path's bit for bit."""
    wl = WORKLOADS["vggt_24layer_k4"].replace(num_layers=1, tokens_per_frame=300, num_heads=4, window_frames=3,
                                               scale_frames=1, keyframe_interval=2)
    dev = torch.device("cuda")
    user = torch.cuda.Stream(device=dev)
    h1 = kvc.kvc_create(kvc.config_from_workload(wl))
    h2 = kvc.kvc_create(kvc.config_from_workload(wl), user)
    st = FrameStream(wl, seed=7, device=dev)
    frames = [st.frame(0, t) for t in range(9)]
    keys = [keyframe_schedule(t, wl.scale_frames, wl.keyframe_interval) for t in range(9)]
    want = []
    o = torch.empty((300, 4, 64), dtype=torch.bfloat16, device=dev)
    for t, (q, k, v) in enumerate(frames):
        kvc.kvc_append_frame(h1, 0, t, k, v, keys[t])
        kvc.kvc_attend(h1, 0, q, o)
        want.append(o.cpu())
    host = [tuple(x.cpu().pin_memory() for x in f) for f in frames]
    outs = [torch.full((300, 4, 64), float("nan"), dtype=torch.bfloat16).pin_memory() for _ in frames]
    for t in range(9):
        kvc.kvc_step_host_async(h2, 0, t, keys[t], *host[t], outs[t])
    kvc.kvc_synchronize(h2)
    for t in range(9):
        assert torch.equal(outs[t], want[t]), f"frame {t}"
    pt1, _ = kvc.kvc_page_table(h1, 0)
    pt2, _ = kvc.kvc_page_table(h2, 0)
    assert np.array_equal(pt1, pt2)
    kvc.kvc_destroy(h1)
    kvc.kvc_destroy(h2)


def test_memory_constant_over_long_stream(kvc):
    wl = WORKLOADS["vggt_518x378"].replace(tokens_per_frame=200, num_heads=2, window_frames=3, scale_frames=1)
    dev = torch.device("cuda")
    h = kvc.kvc_create(kvc.config_from_workload(wl))
    st = FrameStream(wl, seed=6, device=dev)
    o = torch.empty((200, 2, 64), dtype=torch.bfloat16, device=dev)
    free0 = None
    ppf = -(-200 // 16)
    for t in range(60):
        q, k, v = st.frame(0, t)
        kvc.kvc_append_frame(h, 0, t, k, v, True)
        kvc.kvc_attend(h, 0, q, o)
        if t == 10:
            torch.cuda.synchronize()
            free0 = torch.cuda.mem_get_info()[0]
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    pt, info = kvc.kvc_page_table(h, 0)
    assert info["high_water_pages"] == (1 + 3 + 1) * ppf
    assert info["frames_evicted"] == 60 - 4
    kvc.kvc_destroy(h)


def test_error_states(kvc):
    wl = WORKLOADS["vggt_518x378"].replace(tokens_per_frame=64, num_heads=2, window_frames=2, scale_frames=0)
    h = kvc.kvc_create(kvc.config_from_workload(wl))
    dev = torch.device("cuda")
    x = torch.zeros((64, 2, 64), dtype=torch.bfloat16, device=dev)
    with pytest.raises(kvc.KVCError) as e:
        kvc.kvc_attend(h, 0, x, x)
    assert e.value.status_name == "KVC_ERR_STATE"
    kvc.kvc_append_frame(h, 0, 0, x, x, True)
    with pytest.raises(kvc.KVCError) as e:
        kvc.kvc_append_frame(h, 0, 1, x, x, True)
    assert e.value.status_name == "KVC_ERR_STATE"
    with pytest.raises(kvc.KVCError) as e:
        kvc.kvc_attend(h, 5, x, x)
    assert e.value.status_name == "KVC_ERR_ARG"
    kvc.kvc_attend(h, 0, x, x)
    with pytest.raises(kvc.KVCError) as e:
        kvc.kvc_append_frame(h, 0, 0, x, x, True)       # frame index must increase
    assert e.value.status_name == "KVC_ERR_STATE"
    with pytest.raises(kvc.KVCError) as e:
        kvc.kvc_compress(h, 0, x)                        # no budget configured
    assert e.value.status_name == "KVC_ERR_ARG"
    kvc.kvc_destroy(h)
    bad = kvc.config_from_workload(wl)
    bad.head_dim = 48
    with pytest.raises(kvc.KVCError):
        kvc.kvc_create(bad)


def test_bounded_wait_reports_timeout_and_context_survives(kvc):
    wl = WORKLOADS["vggt_518x378"].replace(tokens_per_frame=64, num_heads=2, window_frames=2, scale_frames=0)
    h = kvc.kvc_create(kvc.config_from_workload(wl))
    kvc.kvc_debug_bounded_wait(h, 20000)      # 20 ms on a flag nobody sets
    with pytest.raises(kvc.KVCError) as e:
        kvc.kvc_synchronize(h)
    assert e.value.status_name == "KVC_ERR_TIMEOUT"
    kvc.kvc_reset(h)
    kvc.kvc_synchronize(h)
    x = torch.randn((64, 2, 64), device="cuda").to(torch.bfloat16)
    o = torch.empty_like(x)
    kvc.kvc_append_frame(h, 0, 0, x, x, True)
    kvc.kvc_attend(h, 0, x, o)
    kvc.kvc_synchronize(h)
    assert torch.isfinite(o.float()).all()
    kvc.kvc_destroy(h)


def test_allocation_failure_is_reported_without_leak(kvc):
    wl = WORKLOADS["vggt_518x378"].replace(tokens_per_frame=300, num_heads=4, window_frames=4, scale_frames=1)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for n in (1, 2, 4, 6):
        kvc.kvc_debug_fail_allocs(n)
        with pytest.raises(kvc.KVCError) as e:
            kvc.kvc_create(kvc.config_from_workload(wl))
        assert e.value.status_name == "KVC_ERR_OOM"
    kvc.kvc_debug_fail_allocs(0)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    h = kvc.kvc_create(kvc.config_from_workload(wl))
    kvc.kvc_destroy(h)


def test_rescale_in_some_rows_of_a_warp(kvc):
    """Rows whose running max jumps by more than 2^8 in the last KV tile rescale O while
    most rows of their warp do not; the warp must stay converged and the result exact.
    The last frame plants keys k[200] = 6 q[5] and k[230] = 6 q[70] (per head): rows 5
    and 70 then see logits near 6|q|^2/8 ~ 48 only in the final tile."""
    wl = WORKLOADS["vggt_518x378"].replace(tokens_per_frame=256, num_heads=2, window_frames=6, scale_frames=1)
    dev = torch.device("cuda")
    h = kvc.kvc_create(kvc.config_from_workload(wl, kv_splits=1))
    orc = StreamOracle(OracleConfig.from_workload(wl))
    g = torch.Generator(device=dev).manual_seed(7)
    o = torch.empty((256, 2, 64), dtype=torch.bfloat16, device=dev)
    for t in range(5):
        q, k, v = (torch.randn((256, 2, 64), generator=g, device=dev) for _ in range(3))
        if t == 4:
            k[200] = 6.0 * q[5]
            k[230] = 6.0 * q[70]
        q, k, v = (x.to(torch.bfloat16) for x in (q, k, v))
        kvc.kvc_append_frame(h, 0, t, k, v, True)
        kvc.kvc_attend(h, 0, q, o)
        orc.append(0, t, np64(k), np64(v), True)
        ref = orc.attend(0, np64(q))
        torch.cuda.synchronize()
        compare_out(np64(o), ref, "bf16", f"frame {t}")
    kvc.kvc_destroy(h)


def test_back_to_back_frames_without_host_sync(kvc):
    """Frames issued back to back with no host synchronisation (as a streaming caller
    does): no bounded wait may give up, and the last frame matches the oracle."""
    wl = WORKLOADS["vggt_518x378"]
    dev = torch.device("cuda")
    h = kvc.kvc_create(kvc.config_from_workload(wl))
    st = FrameStream(wl, seed=9, device=dev)
    orc = StreamOracle(OracleConfig.from_workload(wl))
    o = torch.empty((wl.tokens_per_frame, wl.num_heads, wl.head_dim), dtype=torch.bfloat16, device=dev)
    frames = wl.scale_frames + wl.window_frames + 40
    rows = sample_rows(wl.tokens_per_frame, 32, seed=3)
    for t in range(frames):
        q, k, v = st.frame(0, t)
        kvc.kvc_append_frame(h, 0, t, k, v, True)
        kvc.kvc_attend(h, 0, q, o)
        orc.append(0, t, np64(k), np64(v), True)
        if t < frames - 1:
            orc.commit(0)
        else:
            ref = orc.attend(0, np64(q), rows=rows)
    kvc.kvc_synchronize(h)                       # raises on a latched device error
    compare_out(np64(o)[rows], ref, "bf16", "last frame")
    kvc.kvc_destroy(h)
