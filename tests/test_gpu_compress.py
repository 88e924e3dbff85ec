"""GPU parity of the budgeted-compression path: raw scores, s_hat, kept ids, merge pairs,
counts, page tables and stored K/V bit for bit against the oracle (where a rounding or a
cosine tie may go either way within the proven error of a correct fp64 evaluation, the
oracle checks the GPU's choice and follows it); attention over the compressed cache
within the bf16 tolerance."""
import numpy as np
import pytest
import torch

from kvc_gpu_util import compare_out, np64, raw_score_choices, sample_rows
from kvc_streams import WORKLOADS, FrameStream
from oracle import OracleConfig, StreamOracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvc():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import transformer_kv_cache_b200 as m
    return m


def run_budget(kvc, wl, frames, layers, rows=None, check_attn_frames=None, seed=0):
    dev = torch.device("cuda")
    h = kvc.kvc_create(kvc.config_from_workload(wl))
    events = 0
    try:
        st = FrameStream(wl, seed=seed, device=dev)
        orc = StreamOracle(OracleConfig.from_workload(wl))
        T, H, D = wl.tokens_per_frame, wl.num_heads, wl.head_dim
        o = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
        for t in range(frames):
            for l in range(layers):
                q, k, v = st.frame(l, t)
                r = st.residual(l, t)
                kvc.kvc_append_frame(h, l, t, k, v, True)
                kvc.kvc_attend(h, l, q, o)
                orc.append(l, t, np64(k), np64(v), True)
                chk = check_attn_frames is None or t in check_attn_frames
                if chk:
                    ref = orc.attend(l, np64(q), rows=rows)
                    torch.cuda.synchronize()
                    got = np64(o) if rows is None else np64(o)[rows]
                    compare_out(got, ref, "bf16", f"frame {t} layer {l}")
                else:
                    orc.commit(l)
                fired = kvc.kvc_compress(h, l, r)
                # raw scores: bit-equal to the fp32 rounding of the exact norm, except where
                # that rounding is ambiguous within a correct fp64 sum's error (then the
                # oracle follows the GPU's neighbour)
                choice = raw_score_choices(np64(r), kvc.kvc_last_raw_scores(h))
                orc.score(l, t, np64(r), s_choice=choice)
                # merge targets: the oracle's, or one whose fp64 cosine ties it within
                # StreamOracle.COS_TIE (the oracle checks and then follows it)
                tc = None
                if fired:
                    src, dst = kvc.kvc_last_merge(h, l)
                    tc = {int(a): int(b) for a, b in zip(src, dst)}
                res = orc.compress(l, target_choice=tc)
                assert fired == (res is not None), (t, l)
                ids, cnt, sh = kvc.kvc_token_meta(h, l)
                oid, ocnt, osh = orc.token_meta(l)
                assert np.array_equal(ids, oid), f"token ids differ at frame {t} layer {l}"
                assert np.array_equal(sh.astype(np.float64), osh), f"s_hat differs at frame {t} layer {l}"
                assert np.array_equal(cnt, ocnt), f"merge counts differ at frame {t} layer {l}"
                pt, info = kvc.kvc_page_table(h, l)
                assert np.array_equal(pt, orc.page_table(l)), f"page table differs at frame {t} layer {l}"
                assert info["device_error"] == 0
                if res is not None:
                    events += 1
                    assert np.array_equal(src, res["merge_src"]), f"merge sources differ at frame {t} layer {l}"
                    assert np.array_equal(dst, res["merge_dst"]), f"merge targets differ at frame {t} layer {l}"
                    # stored K and V (merged means included) bit for bit
                    n = len(pt)
                    P = wl.page_size
                    kb, vb, _, _ = kvc.kvc_export_pages(h, l, 0, n, H * P * D * 2, H)
                    L = orc.layers[l]
                    for i, (pid, owner, g, nv) in enumerate(L.entries):
                        kk = torch.from_numpy(kb[i].copy()).view(torch.bfloat16).view(H, P, D).double().numpy()
                        vv = torch.from_numpy(vb[i].copy()).view(torch.bfloat16).view(H, P, D).double().numpy()
                        assert np.array_equal(kk[:, :nv], L.pages[pid].k[:, :nv]), f"K page {i} differs"
                        assert np.array_equal(vv[:, :nv], L.pages[pid].v[:, :nv]), f"V page {i} differs"
        return events
    finally:
        kvc.kvc_destroy(h)


def test_budget_small_three_layers(kvc):
    wl = WORKLOADS["vggt_budget_16k"].replace(tokens_per_frame=64, num_heads=4, budget_tokens=300, num_layers=3,
                                               residual_dim=256)
    events = run_budget(kvc, wl, 14, 3)
    assert events >= 6


def test_budget_rank_window_rolls_over_seven_layers(kvc):
    """Seven layers per frame: from layer 5 on the 5-layer rank window drops the oldest
    layer, so the rank ring's slots of layers 0 and 1 are reused by layers 5 and 6
    (StreamCacheVGGT page, 2.1.1: a window of W = 5 layers)."""
    wl = WORKLOADS["vggt_budget_16k"].replace(tokens_per_frame=64, num_heads=4, budget_tokens=300, num_layers=7,
                                               residual_dim=256)
    events = run_budget(kvc, wl, 10, 7)
    assert events >= 14


def test_budget_ragged_pages_and_protected_growth(kvc):
    # T = 45: 3 pages per frame, the last holding 13; B = 200 -> keep 120, merge 80
    wl = WORKLOADS["vggt_budget_16k"].replace(tokens_per_frame=45, num_heads=2, budget_tokens=200, num_layers=2,
                                               residual_dim=64, num_special_tokens=3)
    events = run_budget(kvc, wl, 16, 2)
    assert events >= 5


def test_budget_full_size_one_layer(kvc):
    """Full 1004-token / 16-head / B = 16384 shape through two compression events."""
    wl = WORKLOADS["vggt_budget_16k"].replace(num_layers=1)
    rows = sample_rows(wl.tokens_per_frame, 32, seed=2)
    events = run_budget(kvc, wl, 24, 1, rows=rows, check_attn_frames={0, 16, 17, 23})
    assert events >= 2


def test_budget_error_when_protected_exceed_keep(kvc):
    wl = WORKLOADS["vggt_budget_16k"].replace(tokens_per_frame=32, num_heads=2, budget_tokens=40, num_layers=1,
                                               residual_dim=32, num_special_tokens=8)
    dev = torch.device("cuda")
    h = kvc.kvc_create(kvc.config_from_workload(wl))
    st = FrameStream(wl, seed=1, device=dev)
    o = torch.empty((32, 2, 64), dtype=torch.bfloat16, device=dev)
    with pytest.raises(kvc.KVCError) as e:
        for t in range(4):
            q, k, v = st.frame(0, t)
            kvc.kvc_append_frame(h, 0, t, k, v, True)
            kvc.kvc_attend(h, 0, q, o)
            kvc.kvc_compress(h, 0, st.residual(0, t))
    assert e.value.status_name == "KVC_ERR_BUDGET"
    kvc.kvc_destroy(h)


def test_budget_call_order_errors(kvc):
    wl = WORKLOADS["vggt_budget_16k"].replace(tokens_per_frame=32, num_heads=2, budget_tokens=400, num_layers=2,
                                               residual_dim=32)
    dev = torch.device("cuda")
    h = kvc.kvc_create(kvc.config_from_workload(wl))
    st = FrameStream(wl, seed=1, device=dev)
    o = torch.empty((32, 2, 64), dtype=torch.bfloat16, device=dev)
    q, k, v = st.frame(0, 0)
    kvc.kvc_append_frame(h, 0, 0, k, v, True)
    with pytest.raises(kvc.KVCError) as e:
        kvc.kvc_compress(h, 0, st.residual(0, 0))        # before attention
    assert e.value.status_name == "KVC_ERR_STATE"
    kvc.kvc_attend(h, 0, q, o)
    q1, k1, v1 = st.frame(1, 0)
    kvc.kvc_append_frame(h, 1, 0, k1, v1, True)
    kvc.kvc_attend(h, 1, q1, o)
    kvc.kvc_compress(h, 1, st.residual(1, 0))
    with pytest.raises(kvc.KVCError) as e:
        kvc.kvc_compress(h, 0, st.residual(0, 0))        # layer 0 after layer 1 in the same frame
    assert e.value.status_name == "KVC_ERR_STATE"
    kvc.kvc_destroy(h)


def run_pair(kvc, wl, frames, full_shape_rows=None):
    """Two caches fed the same stream: one compresses with kvc_compress on each layer in
    order, the other with kvc_compress_all (every layer scored in two launches, then the
    layers compressed side by side on the side streams). Their state must agree bit for
    bit after every frame: raw scores, token ids, merge counts, s_hat, page tables, merge
    pairs and the stored K and V. Returns the number of compression events."""
    dev = torch.device("cuda")
    L, T, H, D, P = wl.num_layers, wl.tokens_per_frame, wl.num_heads, wl.head_dim, wl.page_size
    ha = kvc.kvc_create(kvc.config_from_workload(wl))
    hb = kvc.kvc_create(kvc.config_from_workload(wl))
    events = 0
    try:
        st = FrameStream(wl, seed=5, device=dev)
        oa = [torch.empty((T, H, D), dtype=torch.bfloat16, device=dev) for _ in range(L)]
        ob = [torch.empty((T, H, D), dtype=torch.bfloat16, device=dev) for _ in range(L)]
        for t in range(frames):
            qkv = [st.frame(l, t) for l in range(L)]
            res = [st.residual(l, t) for l in range(L)]
            for h, outs in ((ha, oa), (hb, ob)):
                kvc.kvc_append_frame_all(h, t, [x[1] for x in qkv], [x[2] for x in qkv], True)
                kvc.kvc_attend_all(h, [x[0] for x in qkv], outs)
            fired_a = [kvc.kvc_compress(ha, l, res[l]) for l in range(L)]
            fired_b = kvc.kvc_compress_all(hb, res)
            assert fired_a == fired_b, (t, fired_a, fired_b)
            # the last layer's raw scores
            assert np.array_equal(kvc.kvc_last_raw_scores(ha), kvc.kvc_last_raw_scores(hb)), t
            events += sum(fired_b)
            torch.cuda.synchronize()
            for l in range(L):
                assert torch.equal(oa[l], ob[l]), f"outputs differ at frame {t} layer {l}"
                for a, b, what in zip(kvc.kvc_token_meta(ha, l, 1 << 16), kvc.kvc_token_meta(hb, l, 1 << 16),
                                      ("ids", "counts", "s_hat")):
                    assert np.array_equal(a, b), f"{what} differ at frame {t} layer {l}"
                pa, ia = kvc.kvc_page_table(ha, l)
                pb, ib = kvc.kvc_page_table(hb, l)
                assert np.array_equal(pa, pb), f"page table differs at frame {t} layer {l}"
                assert ia["device_error"] == 0 and ib["device_error"] == 0
                if fired_b[l]:
                    sa, da = kvc.kvc_last_merge(ha, l, 1 << 15)
                    sb, db = kvc.kvc_last_merge(hb, l, 1 << 15)
                    assert np.array_equal(sa, sb) and np.array_equal(da, db), f"merges differ at frame {t} layer {l}"
                    n = len(pa)
                    ka, va, _, _ = kvc.kvc_export_pages(ha, l, 0, n, H * P * D * 2, H)
                    kb, vb, _, _ = kvc.kvc_export_pages(hb, l, 0, n, H * P * D * 2, H)
                    assert np.array_equal(ka, kb) and np.array_equal(va, vb), f"pages differ at frame {t} layer {l}"
        return events
    finally:
        kvc.kvc_destroy(ha)
        kvc.kvc_destroy(hb)


def test_compress_all_matches_per_layer_calls(kvc):
    """Six layers (more than the four side streams, so two layers share a stream and its
    scratch in one call), ragged pages, special tokens, several events per layer."""
    wl = WORKLOADS["vggt_budget_16k"].replace(tokens_per_frame=45, num_heads=4, budget_tokens=300, num_layers=6,
                                               residual_dim=64, num_special_tokens=3)
    assert run_pair(kvc, wl, 16) >= 18


def test_compress_all_matches_per_layer_calls_full_shape(kvc):
    """Full 1004-token / 16-head / B = 16384 layers, 5 of them, through one compression event
    each."""
    wl = WORKLOADS["vggt_budget_16k"].replace(num_layers=5)
    assert run_pair(kvc, wl, 18) >= 5
