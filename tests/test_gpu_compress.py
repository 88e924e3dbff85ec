"""GPU parity of the budgeted-compression path: scores, kept ids, merge pairs, counts,
page tables and stored K/V bit for bit against the oracle; attention over the
compressed cache within the bf16 tolerance."""
import numpy as np
import pytest
import torch

from kvc_gpu_util import compare_out, np64, sample_rows
from kvc_streams import WORKLOADS, FrameStream
from oracle import OracleConfig, StreamOracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvc():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import transformer_kv_cache_b200 as m
    return m


def _cos_ok(orc_K, src_pos, got_pos, want_pos):
    """Merge target is the oracle's, or a different target whose fp64 cosine is equal
    within 1e-12 (a near-tie that summation order may decide either way)."""
    if got_pos == want_pos:
        return True
    a = orc_K[src_pos]
    c1 = a @ orc_K[got_pos] / (np.linalg.norm(a) * np.linalg.norm(orc_K[got_pos]))
    c2 = a @ orc_K[want_pos] / (np.linalg.norm(a) * np.linalg.norm(orc_K[want_pos]))
    return abs(c1 - c2) <= 1e-12


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
                Kb, _, ids_b = orc.gather(l)
                fired = kvc.kvc_compress(h, l, r)
                orc.score(l, t, np64(r))
                res = orc.compress(l)
                assert fired == (res is not None), (t, l)
                ids, cnt, sh = kvc.kvc_token_meta(h, l)
                oid, ocnt, osh = orc.token_meta(l)
                assert np.array_equal(ids, oid), f"token ids differ at frame {t} layer {l}"
                assert np.array_equal(sh.astype(np.float64), osh), f"s_hat differs at frame {t} layer {l}"
                pt, info = kvc.kvc_page_table(h, l)
                assert np.array_equal(pt, orc.page_table(l)), f"page table differs at frame {t} layer {l}"
                assert info["device_error"] == 0
                if res is not None:
                    events += 1
                    src, dst = kvc.kvc_last_merge(h, l)
                    assert np.array_equal(src, res["merge_src"])
                    N = ids_b.size
                    Kf = Kb.reshape(N, -1)
                    pos = {int(i): p for p, i in enumerate(ids_b)}
                    mism = [(s, g, w) for s, g, w in zip(src, dst, res["merge_dst"]) if g != w]
                    for s, g, w in mism:
                        assert _cos_ok(Kf, pos[int(s)], pos[int(g)], pos[int(w)]), (t, l, s, g, w)
                    if not mism:
                        # identical targets: counts and stored values must agree bit for bit
                        assert np.array_equal(cnt, ocnt)
                        n = len(pt)
                        P = wl.page_size
                        kb, vb, _, _ = kvc.kvc_export_pages(h, l, 0, n, H * P * D * 2, H)
                        L = orc.layers[l]
                        for i, (pid, owner, g, nv) in enumerate(L.entries):
                            kk = torch.from_numpy(kb[i].copy()).view(torch.bfloat16).view(H, P, D).double().numpy()
                            vv = torch.from_numpy(vb[i].copy()).view(torch.bfloat16).view(H, P, D).double().numpy()
                            assert np.array_equal(kk[:, :nv], L.pages[pid].k[:, :nv]), f"K page {i} differs"
                            assert np.array_equal(vv[:, :nv], L.pages[pid].v[:, :nv]), f"V page {i} differs"
                else:
                    assert np.array_equal(cnt, ocnt)
        return events
    finally:
        kvc.kvc_destroy(h)


def test_budget_small_three_layers(kvc):
    wl = WORKLOADS["vggt_budget_16k"].replace(tokens_per_frame=64, num_heads=4, budget_tokens=300, num_layers=3,
                                               residual_dim=256)
    events = run_budget(kvc, wl, 14, 3)
    assert events >= 6


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
