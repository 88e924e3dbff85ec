"""The pages' workloads at their stated shapes and lengths on the GPU, through the C ABI,
against the fp64 oracle:

* 24 layers of the 518x378 shape with keyframe interval 4, streamed past the sliding
  window ("How GCTStream ...", Selective Frame Caching with Skip Append and Sliding
  Window Eviction), every layer attended in one launch per frame (kvc_attend_all): every
  layer's page table against the closed-form retained set at every step, three layers
  mirrored by the oracle in full (page tables bit for bit, outputs on sampled rows of late
  frames).
* 24 layers with a 16,384-token budget through two compression events per layer
  (StreamCacheVGGT page, 2.1.1-2.1.4 and 2): the rank window of 5 layers rolls over all
  24; four layers are mirrored in full, every layer is scored.
* The 518x518 FP8 stream over 10,000 frames (XStreamVGGT abstract; "Can LingBot-Map
  Achieve 20 FPS", Sliding-Window Eviction Strategy): device memory, the pool's high-water
  mark and the device error word constant at every step, page-table owners equal to the
  closed-form retained set at every step, and two late frames checked against an oracle
  fed only the frames that frame retains (codes, scales and outputs).
"""
import numpy as np
import pytest
import torch

from kvc_gpu_util import check_page_bytes, compare_out, np64, raw_score_choices, sample_rows
from kvc_streams import WORKLOADS, FrameStream, keyframe_schedule
from oracle import OracleConfig, StreamOracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvc():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import transformer_kv_cache_b200 as m
    return m


def retained(t, S, W, k):
    """Committed keyframes after frame t's step: the first S and the last W."""
    keys = [f for f in range(t + 1) if keyframe_schedule(f, S, k)]
    return sorted(set(keys[:S]) | set(keys[-W:] if W > 0 else keys))


def check_owners(pt, want, ppf, T, P):
    owners = pt[:, 0]
    assert sorted(set(owners.tolist())) == want, (sorted(set(owners.tolist())), want)
    assert len(pt) == ppf * len(want)
    for f in want:
        rows = pt[owners == f]
        assert rows[:, 1].tolist() == list(range(ppf)) and rows[:, 3].sum() == T


def test_config_24_layers_keyframe_interval_4_past_the_window(kvc):
    wl = WORKLOADS["vggt_24layer_k4"]
    L, T, H, D, P = wl.num_layers, wl.tokens_per_frame, wl.num_heads, wl.head_dim, wl.page_size
    S, W, k = wl.scale_frames, wl.window_frames, wl.keyframe_interval
    ppf = -(-T // P)
    # keyframe number S + W + 1 (the first eviction) is frame S + W * k = 264
    frames = S + W * k + 8
    mirror = (0, 11, 23)
    check = {frames - 8, frames - 3, frames - 1}          # a keyframe and non-keyframes past the window
    rows = sample_rows(T, 24, seed=5)
    dev = torch.device("cuda")
    h = kvc.kvc_create(kvc.config_from_workload(wl))
    try:
        st = FrameStream(wl, seed=31, device=dev)
        orc = StreamOracle(OracleConfig.from_workload(wl))
        outs = [torch.empty((T, H, D), dtype=torch.bfloat16, device=dev) for _ in range(L)]
        evicted = 0
        for t in range(frames):
            key = keyframe_schedule(t, S, k)
            qkv = [st.frame(l, t) for l in range(L)]
            kvc.kvc_append_frame_all(h, t, [x[1] for x in qkv], [x[2] for x in qkv], key)
            kvc.kvc_attend_all(h, [x[0] for x in qkv], outs)   # every layer in one attention launch
            want = retained(t, S, W, k)
            for l in range(L):
                q, kk, vv = qkv[l]
                o = outs[l]
                if l in mirror:
                    orc.append(l, t, np64(kk), np64(vv), key)
                    if t in check:
                        ref = orc.attend(l, np64(q), rows=rows)
                        torch.cuda.synchronize()
                        compare_out(np64(o)[rows], ref, "bf16", f"frame {t} layer {l}")
                    else:
                        orc.commit(l)
                pt, info = kvc.kvc_page_table(h, l)
                assert info["device_error"] == 0
                check_owners(pt, want, ppf, T, P)
                if l in mirror:
                    assert np.array_equal(pt, orc.page_table(l)), f"page table differs at frame {t} layer {l}"
            evicted = info["frames_evicted"]
        assert evicted >= 2
    finally:
        kvc.kvc_destroy(h)


def test_config_24_layers_budget_two_compressions(kvc):
    wl = WORKLOADS["vggt_budget_16k"]
    L, T, H, D, P = wl.num_layers, wl.tokens_per_frame, wl.num_heads, wl.head_dim, wl.page_size
    # the first compression when 17 frames exceed 16,384 tokens, the second 7 frames later
    frames = 24
    mirror = (0, 5, 11, 23)
    check = {16, 23}
    rows = sample_rows(T, 16, seed=6)
    dev = torch.device("cuda")
    h = kvc.kvc_create(kvc.config_from_workload(wl))
    events = {l: 0 for l in range(L)}
    try:
        st = FrameStream(wl, seed=41, device=dev)
        orc = StreamOracle(OracleConfig.from_workload(wl))
        o = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
        for t in range(frames):
            for l in range(L):
                q, kk, vv = st.frame(l, t)
                r = st.residual(l, t)
                kvc.kvc_append_frame(h, l, t, kk, vv, True)
                kvc.kvc_attend(h, l, q, o)
                if l in mirror:
                    orc.append(l, t, np64(kk), np64(vv), True)
                    if t in check:
                        ref = orc.attend(l, np64(q), rows=rows)
                        torch.cuda.synchronize()
                        compare_out(np64(o)[rows], ref, "bf16", f"frame {t} layer {l}")
                    else:
                        orc.commit(l)
                fired = kvc.kvc_compress(h, l, r)
                # every layer is scored: the rank window of the mirrored layers spans the others
                choice = raw_score_choices(np64(r), kvc.kvc_last_raw_scores(h))
                orc.score(l, t, np64(r), s_choice=choice)
                pt, info = kvc.kvc_page_table(h, l)
                assert info["device_error"] == 0
                if fired:
                    events[l] += 1
                    assert info["tokens"] == int(np.floor(np.float32(wl.keep_frac) * wl.budget_tokens))
                if l in mirror:
                    tc = None
                    if fired:
                        src, dst = kvc.kvc_last_merge(h, l)
                        tc = {int(a): int(b) for a, b in zip(src, dst)}
                    res = orc.compress(l, target_choice=tc)
                    assert fired == (res is not None), (t, l)
                    if res is not None:
                        assert np.array_equal(src, res["merge_src"]) and np.array_equal(dst, res["merge_dst"])
                    ids, cnt, sh = kvc.kvc_token_meta(h, l)
                    oid, ocnt, osh = orc.token_meta(l)
                    assert np.array_equal(ids, oid), f"token ids differ at frame {t} layer {l}"
                    assert np.array_equal(sh.astype(np.float64), osh), f"s_hat differs at frame {t} layer {l}"
                    assert np.array_equal(cnt, ocnt), f"counts differ at frame {t} layer {l}"
                    assert np.array_equal(pt, orc.page_table(l)), f"page table differs at frame {t} layer {l}"
                    if res is not None:
                        check_page_bytes(kvc, h, l, wl, orc)
        assert all(n >= 2 for n in events.values()), events
    finally:
        kvc.kvc_destroy(h)


def test_config_fp8_ten_thousand_frames_constant_memory(kvc):
    wl = WORKLOADS["vggt_518x518_fp8"]
    T, H, D, P = wl.tokens_per_frame, wl.num_heads, wl.head_dim, wl.page_size
    S, W, k = wl.scale_frames, wl.window_frames, wl.keyframe_interval
    ppf = -(-T // P)
    frames = wl.num_frames                                 # 10,000
    sampled = (frames // 2 + 3, frames - 1)
    rows = sample_rows(T, 16, seed=7)
    dev = torch.device("cuda")
    h = kvc.kvc_create(kvc.config_from_workload(wl))
    saved = {}
    try:
        st = FrameStream(wl, seed=51, device=dev)
        o = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
        free0 = hw0 = None
        for t in range(frames):
            q, kk, vv = st.frame(0, t)
            kvc.kvc_append_frame(h, 0, t, kk, vv, True)
            kvc.kvc_attend(h, 0, q, o)
            pt, info = kvc.kvc_page_table(h, 0)
            assert info["device_error"] == 0, t
            if t < S + W:
                check_owners(pt, list(range(t + 1)), ppf, T, P)
            else:
                assert pt[0, 0] == 0 and pt[S * ppf, 0] == t - W + 1 and pt[-1, 0] == t, t
                assert len(pt) == (S + W) * ppf, t
            if t == S + W + 1:
                torch.cuda.synchronize()
                free0, hw0 = torch.cuda.mem_get_info()[0], info["high_water_pages"]
            elif t > S + W + 1:
                assert info["high_water_pages"] == hw0, t
                if t % 250 == 0:
                    torch.cuda.synchronize()
                    assert torch.cuda.mem_get_info()[0] == free0, t
            if t in sampled:
                check_owners(pt, retained(t, S, W, k), ppf, T, P)
                pages = kvc.kvc_export_pages(h, 0, 0, len(pt), H * P * D, H, True)
                saved[t] = (np64(o)[rows], pages)
        assert torch.cuda.mem_get_info()[0] == free0
        # the late frames against an oracle fed only the frames each retains, in stream order;
        # frames are independent draws, so the stream regenerates them one by one
        for t in sampled:
            orc = StreamOracle(OracleConfig.from_workload(wl))
            for f in sorted(set(range(S)) | set(range(t - W, t))):
                _, kk, vv = st.frame(0, f)
                orc.append(0, f, np64(kk), np64(vv), True)
                orc.commit(0)
            q, kk, vv = st.frame(0, t)
            orc.append(0, t, np64(kk), np64(vv), True)
            ref = orc.attend(0, np64(q), rows=rows)
            out_t, (kb, vb, ks, vs) = saved[t]
            compare_out(out_t, ref, "bf16", f"frame {t}")
            pto = orc.page_table(0)
            assert [r[0] for r in pto[::ppf]] == retained(t, S, W, k)
            # codes and scales of every retained page, in cache order, bit for bit
            kc, vc, kso, vso = orc.fp8_pages(0)
            n = len(pto)
            assert np.array_equal(kb.reshape(n, H, P, D), kc) and np.array_equal(vb.reshape(n, H, P, D), vc)
            assert np.array_equal(ks.astype(np.float64), kso) and np.array_equal(vs.astype(np.float64), vso)
    finally:
        kvc.kvc_destroy(h)
