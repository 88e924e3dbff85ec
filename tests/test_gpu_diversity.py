"""GPU parity of the rolling diversity-pruned memory ("InfiniteVGGT" explainer page)
through the C ABI against the fp64 oracle: every head's kept token ids exactly, except
that where the Top-K is not unique within the proven rounding bound of two fp64
evaluations of the scores the GPU's choice among the tied candidates is checked and then
followed; every layer's mean diversity within that bound; attention outputs within the
bf16 tolerance."""
import numpy as np
import pytest
import torch

from kvc_gpu_util import U64, compare_out, np64, rolling_score_bound, sample_rows, top_k_valid
from kvc_streams import WORKLOADS, FrameStream
from oracle import RollingOracle, layer_budgets

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvc():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import transformer_kv_cache_b200 as m
    return m


def run_rolling(kvc, wl, frames, rows=None, budgets_at=None, check_ids=True, seed=11, prune_first=False,
                attend_all=False,
                append_all=False, adapt_at=None):
    dev = torch.device("cuda")
    L, H, D, T = wl.num_layers, wl.num_heads, wl.head_dim, wl.tokens_per_frame
    h = kvc.kvc_create(kvc.config_from_workload(wl))
    try:
        st = FrameStream(wl, seed=seed, device=dev)
        orc = RollingOracle(L, H, D, T, wl.diversity_budget, wl.softmax_scale)
        ties = [0]
        o = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
        for t in range(frames):
            if budgets_at is not None and t in budgets_at:
                kvc.kvc_set_layer_budgets(h, budgets_at[t])
                orc.set_budgets(budgets_at[t])
            if adapt_at is not None and t in adapt_at:
                # the library's layer-adaptive budgets against the oracle's rule on its own
                # means; a budget may differ only where L * k * p lies within rounding of
                # an integer (the floor of a value computed from fp64 means in another order)
                tau, kk = adapt_at[t]
                got = kvc.kvc_adapt_layer_budgets(h, L, tau, kk)
                means = [orc.layer_diversity(l) for l in range(L)]
                want = layer_budgets(means, tau, kk, lo=1, hi=wl.diversity_budget)
                z = np.array(means) / tau
                x = L * kk * np.exp(z - z.max()) / np.exp(z - z.max()).sum()
                for l in range(L):
                    if got[l] != want[l]:
                        n = np.round(x[l])
                        assert abs(x[l] - n) <= 1e-9 * max(1.0, x[l]) and got[l] in (
                            max(1, min(wl.diversity_budget, int(n) - 1)), max(1, min(wl.diversity_budget, int(n)))), \
                            (t, l, got[l], want[l], x[l])
                assert len(set(got.tolist())) > 1, "budgets did not adapt"
                orc.set_budgets(got.tolist())
            qkv = [st.frame(l, t) for l in range(L)]
            if append_all:                              # every layer's frame in one call
                kvc.kvc_append_frame_all(h, t, [x[1] for x in qkv], [x[2] for x in qkv], True)
            if attend_all:                              # every layer pruned and attended in one call
                if prune_first and t > 0:
                    kvc.kvc_prune_all(h)                # the pruning of every layer on its own; twice prunes once
                    kvc.kvc_prune_all(h)
                outs = [torch.empty_like(o) for _ in range(L)]
                kvc.kvc_attend_all(h, [x[0] for x in qkv], outs)
            for l in range(L):
                q, k, v = qkv[l]
                if not append_all:
                    kvc.kvc_append_frame(h, l, t, k, v, True)
                if attend_all:
                    o = outs[l]
                else:
                    if prune_first and t > 0:
                        kvc.kvc_prune(h, l)             # the pruning step on its own; twice prunes once
                        kvc.kvc_prune(h, l)
                    kvc.kvc_attend(h, l, q, o)
                orc.append(l, t, np64(k), np64(v))
                orc.prune(l)
                if t >= 1:
                    # kept ids: the oracle's Top-K, or a set that differs only among
                    # candidates within the proven rounding bound of the K-th score (the
                    # oracle then follows the GPU's choice)
                    for hh in range(H):
                        ids_c, Kc, _ = orc.last_cands[l][hh]
                        sc = orc.last_scores[l][hh]
                        got = kvc.kvc_head_tokens(h, l, hh)[T:]
                        bound = rolling_score_bound(Kc)
                        if not top_k_valid(got, orc.mut_ids[l][hh], ids_c, sc, bound, orc.budgets[l]):
                            orc.set_kept(l, hh, got)
                            ties[0] += 1
                    # layer mean diversity: within the bound of the scores plus the mean's own
                    # summation error
                    allsc = np.concatenate(orc.last_scores[l])
                    tol = max(float(np.max(rolling_score_bound(c[1]))) for c in orc.last_cands[l]) + \
                        4 * (allsc.size + 2) * U64 * float(np.mean(np.abs(allsc)))
                    assert abs(kvc.kvc_layer_diversity(h, l) - orc.layer_diversity(l)) <= tol, (t, l)
                ref = orc.attend(l, np64(q), rows=rows)
                torch.cuda.synchronize()
                got = np64(o) if rows is None else np64(o)[rows]
                compare_out(got, ref, "bf16", f"frame {t} layer {l}")
                if check_ids:
                    for hh in range(H):
                        ids = kvc.kvc_head_tokens(h, l, hh)
                        assert np.array_equal(ids, orc.head_ids(l, hh)), f"kept ids differ: frame {t} layer {l} head {hh}"
                _, info = kvc.kvc_page_table(h, l)
                assert info["device_error"] == 0
        return orc
    finally:
        kvc.kvc_destroy(h)


@pytest.mark.parametrize("T,H,K,frames,prune_first", [
    (150, 4, 200, 7, False),    # candidates 350 -> 200 kept per head from the second pruning on
    (150, 4, 100, 5, True),     # K not a multiple of the page size; kvc_prune before kvc_attend
    (40, 2, 400, 6, False),     # K above the candidates for several frames: nothing pruned yet
    (10, 2, 25, 6, True),       # T < P: every page partial
])
def test_rolling_memory_small(kvc, T, H, K, frames, prune_first):
    wl = WORKLOADS["vggt_infinite_12l"].replace(num_layers=2, tokens_per_frame=T, num_heads=H, diversity_budget=K,
                                                num_special_tokens=min(5, T))
    run_rolling(kvc, wl, frames, prune_first=prune_first)


def test_rolling_memory_append_all_layers(kvc):
    """kvc_append_frame_all: one allocation and one append launch for every head of every
    layer."""
    wl = WORKLOADS["vggt_infinite_12l"].replace(num_layers=3, tokens_per_frame=150, num_heads=4,
                                                diversity_budget=200)
    run_rolling(kvc, wl, 6, append_all=True)


def test_rolling_memory_attend_all_layers(kvc):
    """kvc_attend_all: every layer pruned (one launch), then every layer attended (one
    launch; the layers are small), with kept sets, layer averages and outputs checked per
    layer; the layers' budgets differ, so their page counts do too. Then kvc_prune_all
    before kvc_attend_all."""
    wl = WORKLOADS["vggt_infinite_12l"].replace(num_layers=3, tokens_per_frame=150, num_heads=4,
                                                diversity_budget=200)
    run_rolling(kvc, wl, 7, append_all=True, attend_all=True, budgets_at={3: [200, 60, 131]})
    run_rolling(kvc, wl, 5, append_all=True, attend_all=True, prune_first=True)


def test_layer_budgets_between_frames(kvc):
    """Per-layer budgets set between frames (the softmax rule on the previous frame's
    layer averages; the configured K is the largest budget a layer can take, since it
    sizes the pools) take effect at the next pruning."""
    wl = WORKLOADS["vggt_infinite_12l"].replace(num_layers=3, tokens_per_frame=120, num_heads=2,
                                                diversity_budget=160)
    b = layer_budgets([-0.2, -0.6, -0.4], 1.0, 120)     # an average of 120 per head
    assert max(b) <= 160 and min(b) < 120 < max(b)       # the configured K caps every layer
    run_rolling(kvc, wl, 6, budgets_at={3: b, 5: [160, 7, 33]})


def test_library_adapts_layer_budgets(kvc):
    """kvc_adapt_layer_budgets ("InfiniteVGGT" explainer, Layer-wise adaptive budgets): the
    softmax of the layers' mean diversity with temperature tau, computed in the library
    from its own layer means, matches the oracle's rule; the stream continues under the
    adapted budgets (twice re-adapted) with kept sets and outputs checked."""
    wl = WORKLOADS["vggt_infinite_12l"].replace(num_layers=4, tokens_per_frame=120, num_heads=4, diversity_budget=160)
    run_rolling(kvc, wl, 8, adapt_at={2: (0.02, 100), 5: (0.05, 120)})


def test_rolling_memory_full_size_sampled(kvc):
    """The page's shape on one layer: 1,004 tokens per frame, 16 heads, 512 kept per head
    (1,516 candidates per head per frame), sampled query rows."""
    wl = WORKLOADS["vggt_infinite_12l"].replace(num_layers=1)
    run_rolling(kvc, wl, 4, rows=sample_rows(wl.tokens_per_frame, 48, seed=4))


def test_rolling_memory_largest_candidate_set(kvc):
    """K = 1,040 with 1,004-token frames: 65 + 63 pages, the 2,048 candidate slots a head
    can hold (256 per CTA of the pruning cluster), sampled query rows."""
    wl = WORKLOADS["vggt_infinite_12l"].replace(num_layers=1, num_heads=4, diversity_budget=1040)
    run_rolling(kvc, wl, 4, rows=sample_rows(wl.tokens_per_frame, 32, seed=5))


def test_rolling_memory_errors(kvc):
    wl = WORKLOADS["vggt_infinite_12l"].replace(num_layers=2, tokens_per_frame=64, num_heads=2,
                                                diversity_budget=64)
    h = kvc.kvc_create(kvc.config_from_workload(wl))
    try:
        k = torch.zeros((64, 2, 64), dtype=torch.bfloat16, device="cuda")
        with pytest.raises(kvc.KVCError):
            kvc.kvc_append_frame(h, 0, 0, k, k, False)         # every frame is a candidate
        with pytest.raises(kvc.KVCError):
            kvc.kvc_set_layer_budgets(h, [64, 65])             # above the configured K
        with pytest.raises(kvc.KVCError):
            kvc.kvc_layer_diversity(h, 0)                       # never pruned
        with pytest.raises(kvc.KVCError):
            kvc.kvc_token_meta(h, 0)                            # not in this mode
        with pytest.raises(kvc.KVCError):
            kvc.kvc_prune(h, 0)                                 # no frame pending
        with pytest.raises(kvc.KVCError):
            kvc.kvc_prune(h, 2)                                 # no such layer
    finally:
        kvc.kvc_destroy(h)
    plain = WORKLOADS["vggt_518x378"].replace(num_layers=1)
    h = kvc.kvc_create(kvc.config_from_workload(plain))
    try:
        with pytest.raises(kvc.KVCError):
            kvc.kvc_prune(h, 0)                                 # not a diversity-pruned cache
    finally:
        kvc.kvc_destroy(h)
    for bad in (wl.replace(kv_dtype="fp8_e4m3"),
                WORKLOADS["vggt_infinite_12l"].replace(diversity_budget=1040 + 16)):   # 2,064 candidate slots
        with pytest.raises(kvc.KVCError):
            kvc.kvc_create(kvc.config_from_workload(bad))
    ok = WORKLOADS["vggt_infinite_12l"].replace(num_layers=1, diversity_budget=1040)  # 2,048: the largest
    kvc.kvc_destroy(kvc.kvc_create(kvc.config_from_workload(ok)))
