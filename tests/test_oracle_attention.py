"""Pins for the oracle's cache and attention: brute force over explicitly concatenated
frames, the retained-set closed form, constant memory, and attention special cases."""
import numpy as np
import pytest
import torch
from hypothesis import given, settings, strategies as st

import brute
from kvc_streams import WORKLOADS, FrameStream, keyframe_schedule
from oracle import OracleConfig, StreamOracle


def _np(x):
    return x.to(torch.float64).numpy()


def _run_and_check(wl, frames, seed=0, check_rows=None):
    st = FrameStream(wl, seed=seed, device="cpu")
    orc = StreamOracle(OracleConfig.from_workload(wl))
    hist_k, hist_v = {}, {}
    S, W, k = wl.scale_frames, wl.window_frames, wl.keyframe_interval
    steady = None
    for t in range(frames):
        q, kk, vv = st.frame(0, t)
        q, kk, vv = _np(q), _np(kk), _np(vv)
        key = keyframe_schedule(t, S, k)
        orc.append(0, t, kk, vv, key)
        if getattr(wl, "fp8_dim_adaptive", 0):
            hist_k[t] = brute.stored_dim_adaptive(kk, wl.page_size, "channel")
            hist_v[t] = brute.stored_dim_adaptive(vv, wl.page_size, "token")
        else:
            hist_k[t] = brute.stored(kk, wl.kv_dtype, wl.page_size)
            hist_v[t] = brute.stored(vv, wl.kv_dtype, wl.page_size)
        rows = check_rows
        got = orc.attend(0, q, rows=rows)
        fr = brute.retained_frames(t, S, W, k)
        Kc = np.concatenate([hist_k[u] for u in fr])
        Vc = np.concatenate([hist_v[u] for u in fr])
        qq = q if rows is None else q[rows]
        ref = brute.attention(qq, Kc, Vc, float(np.float32(wl.softmax_scale)))
        np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-12)
        # page table after the commit / eviction of step t holds exactly what frame
        # t + 1 will attend to, besides itself
        pt = orc.page_table(0)
        owners = sorted(set(pt[:, 0].tolist()))
        want = brute.retained_frames(t + 1, S, W, k)[:-1]
        assert owners == sorted(want), (t, owners, want)
        phys = pt[:, 2]
        assert len(set(phys.tolist())) == len(phys)
        ppf = -(-wl.tokens_per_frame // wl.page_size)
        assert len(pt) == ppf * len(want)
        # each frame: pages in order, last page partial
        for f in want:
            rows_f = pt[pt[:, 0] == f]
            assert rows_f[:, 1].tolist() == list(range(ppf))
            assert rows_f[:, 3].sum() == wl.tokens_per_frame
        # lowest-free allocation: ids in use are always {0..n-1} when the cache is frame-FIFO
        assert orc.pages_in_use(0) == len(pt)
        if steady is None and len(want) == S + W:
            steady = orc.high_water(0)
    return orc, steady


def test_tiny_f32_matches_brute_force():
    wl = WORKLOADS["tiny_f32"]
    orc, steady = _run_and_check(wl, wl.num_frames)
    # memory constant after S + W frames: the high-water mark stops growing
    S, W = wl.scale_frames, wl.window_frames
    ppf = -(-wl.tokens_per_frame // wl.page_size)
    assert orc.high_water(0) == (S + W + 1) * ppf


@pytest.mark.parametrize("T,P,S,W,k", [(13, 4, 2, 3, 1), (9, 8, 1, 2, 3), (16, 16, 0, 2, 2), (7, 2, 3, 1, 1),
                                       (13, 4, 2, 0, 2)])    # W = 0: no window, every keyframe stays
def test_random_small_configs_match_brute_force(T, P, S, W, k):
    wl = WORKLOADS["tiny_f32"].replace(tokens_per_frame=T, page_size=P, scale_frames=S,
                                        window_frames=W, keyframe_interval=k, num_heads=3, head_dim=8)
    _run_and_check(wl, 14, seed=T * 100 + P)


@settings(max_examples=30, deadline=None, derandomize=True)
@given(T=st.integers(1, 40), P=st.sampled_from([1, 2, 4, 8, 16]), S=st.integers(0, 3), W=st.integers(0, 4),
       k=st.integers(1, 4), H=st.integers(1, 3), D=st.sampled_from([16, 32]),
       kv=st.sampled_from(["f32", "bf16", "fp8_e4m3"]), frames=st.integers(1, 12))
def test_swept_small_configs_match_brute_force(T, P, S, W, k, H, D, kv, frames):
    """Seeded sweep over frame sizes (ragged and exact page fits, T < P), windows with and
    without scale frames, keyframe intervals, head counts and storage formats: every step's
    output and page table against brute force over the concatenated retained frames."""
    io = "bf16" if kv != "f32" else "f32"
    if kv == "fp8_e4m3" and P * D > 2048:
        P = 2048 // D
    wl = WORKLOADS["tiny_f32"].replace(tokens_per_frame=T, page_size=P, scale_frames=S, window_frames=W,
                                        keyframe_interval=k, num_heads=H, head_dim=D, io_dtype=io, kv_dtype=kv)
    _run_and_check(wl, frames, seed=T * 1000 + P * 10 + H)


def test_fp8_small_matches_brute_force():
    wl = WORKLOADS["vggt_518x518_fp8"].replace(tokens_per_frame=37, num_heads=2, head_dim=16,
                                                window_frames=3, scale_frames=2, page_size=8)
    _run_and_check(wl, 9, seed=5)


def test_fp8_dimension_adaptive_small_matches_brute_force():
    wl = WORKLOADS["vggt_518x518_fp8"].replace(tokens_per_frame=37, num_heads=2, head_dim=16,
                                                window_frames=3, scale_frames=2, page_size=8,
                                                fp8_dim_adaptive=1)
    _run_and_check(wl, 9, seed=6)


def test_bf16_temporal_small_matches_brute_force():
    wl = WORKLOADS["vggt_518x378"].replace(tokens_per_frame=45, num_heads=2, window_frames=4,
                                            scale_frames=2, keyframe_interval=2)
    _run_and_check(wl, 12, seed=7, check_rows=[0, 1, 2, 44])


def test_single_token_gives_v_and_equal_keys_give_mean_v():
    cfg = OracleConfig(num_layers=1, num_heads=2, head_dim=4, tokens_per_frame=1, num_special_tokens=0,
                       page_size=4, window_frames=2, scale_frames=0, kv_dtype="f32", softmax_scale=0.5)
    orc = StreamOracle(cfg)
    rng = np.random.default_rng(0)
    K = rng.standard_normal((1, 2, 4)); V = rng.standard_normal((1, 2, 4)); Q = rng.standard_normal((1, 2, 4))
    orc.append(0, 0, K, V, True)
    np.testing.assert_array_equal(orc.attend(0, Q), V)
    # equal keys: uniform weights -> mean of V
    cfg.tokens_per_frame = 6
    orc = StreamOracle(cfg)
    K = np.repeat(rng.standard_normal((1, 2, 4)), 6, axis=0)
    V = rng.standard_normal((6, 2, 4))
    orc.append(0, 0, K, V, True)
    np.testing.assert_allclose(orc.attend(0, rng.standard_normal((3, 2, 4))),
                               np.broadcast_to(V.mean(axis=0), (3, 2, 4)), rtol=1e-13, atol=1e-14)


def test_page_permutation_invariance():
    wl = WORKLOADS["tiny_f32"]
    st = FrameStream(wl, seed=3)
    orc = StreamOracle(OracleConfig.from_workload(wl))
    for t in range(6):
        q, k, v = (_np(x) for x in st.frame(0, t))
        orc.append(0, t, k, v, True)
        out = orc.attend(0, q, commit=False)
        L = orc.layers[0]
        L.entries = L.entries[::-1]
        out2 = orc.attend(0, q, commit=False)
        L.entries = L.entries[::-1]
        np.testing.assert_allclose(out, out2, rtol=1e-12, atol=1e-14)
        orc.commit(0)


def test_skip_append_discards_and_memory_tracks_keyframes():
    # memory before the window cap grows by one frame per keyframe (num_frames / k)
    wl = WORKLOADS["tiny_f32"].replace(window_frames=100, scale_frames=0, keyframe_interval=3)
    st = FrameStream(wl, seed=4)
    orc = StreamOracle(OracleConfig.from_workload(wl))
    ppf = -(-wl.tokens_per_frame // wl.page_size)
    for t in range(12):
        q, k, v = (_np(x) for x in st.frame(0, t))
        orc.append(0, t, k, v, keyframe_schedule(t, 0, 3))
        orc.attend(0, q)
        n_key = len([u for u in range(t + 1) if u % 3 == 0])
        assert orc.pages_in_use(0) == n_key * ppf


def test_reset_clears_everything_and_replays_identically():
    wl = WORKLOADS["tiny_f32"]
    cfg = OracleConfig.from_workload(wl)
    orc = StreamOracle(cfg)
    outs = []
    for rep in range(2):
        st = FrameStream(wl, seed=9)
        o = []
        for t in range(7):
            q, k, v = (_np(x) for x in st.frame(0, t))
            orc.append(0, t, k, v, True)
            o.append(orc.attend(0, q))
        outs.append(o)
        orc.reset()
        assert orc.page_table(0).shape[0] == 0 and orc.pages_in_use(0) == 0
    for a, b in zip(*outs):
        np.testing.assert_array_equal(a, b)


# ------------------------------------------------------------------ planted mistakes
# Dimension-adaptive FP8 misread in the oracle (on the CPU); the brute-force pin over
# torch's float8 cast must fail on each.

def _da_small():
    return WORKLOADS["vggt_518x518_fp8"].replace(tokens_per_frame=37, num_heads=2, head_dim=16,
                                                  window_frames=3, scale_frames=2, page_size=8,
                                                  fp8_dim_adaptive=1)


def test_planted_swapped_dimension_adaptive_axes_are_caught(monkeypatch):
    """K grouped per token and V per channel (KIVI's split the wrong way round)."""
    import oracle.kvcache_oracle as ko
    ch, tok = ko.fp8_quantise_channels, ko.fp8_quantise_tokens
    monkeypatch.setattr(ko, "fp8_quantise_channels", tok)
    monkeypatch.setattr(ko, "fp8_quantise_tokens", ch)
    # full pages with P = D, so that the swapped scale arrays still fit their slots and
    # only the values tell the two apart
    wl = _da_small().replace(tokens_per_frame=32, page_size=16)
    with pytest.raises(AssertionError):
        _run_and_check(wl, 5, seed=6)


def test_planted_per_page_scales_in_dimension_adaptive_mode_are_caught(monkeypatch):
    """One scale per (page, head) although the mode asks for per-channel / per-token ones."""
    import oracle.kvcache_oracle as ko

    def per_block(axis):
        def q(x):
            codes, scale, deq = ko.fp8_quantise_block(x)
            return codes, np.full(np.shape(x)[axis], scale), deq
        return q
    monkeypatch.setattr(ko, "fp8_quantise_channels", per_block(1))
    monkeypatch.setattr(ko, "fp8_quantise_tokens", per_block(0))
    with pytest.raises(AssertionError):
        _run_and_check(_da_small(), 5, seed=6)
