"""Pins for the oracle's keep / merge / drop compression: properties that any correct
implementation has, each checked with a routine other than the oracle's own."""
import math

import numpy as np
import pytest
import torch
from hypothesis import assume, given, settings, strategies as st
from scipy.spatial.distance import cdist

from kvc_streams import WORKLOADS, FrameStream
from oracle import OracleConfig, StreamOracle, bf16_round


def _small_wl(**kw):
    base = dict(tokens_per_frame=8, num_special_tokens=1, num_heads=2, head_dim=4, page_size=4,
                budget_tokens=40, num_layers=2, residual_dim=16)
    base.update(kw)
    return WORKLOADS["vggt_budget_16k"].replace(**base)


def _np(x):
    return x.to(torch.float64).numpy()


def _drive(wl, frames, seed=0, on_event=None):
    st = FrameStream(wl, seed=seed)
    orc = StreamOracle(OracleConfig.from_workload(wl))
    events = 0
    for t in range(frames):
        for l in range(wl.num_layers):
            q, k, v = (_np(x) for x in st.frame(l, t))
            orc.append(l, t, k, v, True)
            orc.attend(l, q)
            before_k, before_v, before_ids = orc.gather(l)
            ids_b, cnt_b, sh_b = orc.token_meta(l)
            orc.score(l, t, _np(st.residual(l, t)))
            ids_b, cnt_b, sh_b = orc.token_meta(l)
            res = orc.compress(l)
            if res is not None:
                events += 1
                if on_event:
                    on_event(orc, l, res, before_k, before_v, ids_b, cnt_b, sh_b)
    return orc, events


def _compression_check(frames=9, min_events=4, **kw):
    wl = _small_wl(**kw)
    n_keep = math.floor(float(np.float32(wl.keep_frac)) * wl.budget_tokens)
    n_merge = wl.budget_tokens - n_keep
    seen = []

    def check(orc, l, res, Kb, Vb, ids_b, cnt_b, sh_b):
        seen.append(1)
        N = ids_b.size
        H, D = wl.num_heads, wl.head_dim
        kept = res["kept_ids"]
        src, dst = res["merge_src"], res["merge_dst"]
        drop = res["dropped_ids"]
        # tiers partition the cache; sizes as stated
        assert len(kept) == n_keep and np.all(np.diff(kept) > 0)
        if res["n_protected"] < n_keep:
            assert len(src) == min(n_merge, N - n_keep)
        else:
            assert len(src) == 0          # no eligible target: the merge tier is dropped
        allids = np.sort(np.concatenate([kept, src, drop]))
        assert np.array_equal(allids, np.sort(ids_b))
        pos = {int(i): p for p, i in enumerate(ids_b)}
        T = wl.tokens_per_frame
        prot = {int(i) for i in ids_b if (i // T == 0) or (i % T) < wl.num_special_tokens}
        assert prot <= set(kept.tolist())
        # order by s_hat: kept (non-protected) >= merged >= dropped, ties to lower id
        key = lambda i: (-sh_b[pos[int(i)]], int(i))
        kept_np = [i for i in kept if int(i) not in prot]
        if kept_np and len(src):
            assert max(key(i) for i in kept_np) < min(key(i) for i in src)
        if len(src) and len(drop):
            assert max(key(i) for i in src) < min(key(i) for i in drop)
        # targets: kept, not protected, maximal cosine (scipy), lowest id among ties
        Kf = Kb.reshape(N, H * D)
        elig = sorted(int(i) for i in kept_np)
        E = Kf[[pos[i] for i in elig]]
        for s_id, d_id in zip(src, dst):
            assert int(d_id) in elig
            dist = cdist(Kf[[pos[int(s_id)]]], E, metric="cosine")[0]
            assert abs(dist[elig.index(int(d_id))] - dist.min()) <= 1e-12
        # counts conserved: after = keep + merged before
        Ka, Va, ids_a = orc.gather(l)
        ida, cnta, sha = orc.token_meta(l)
        assert np.array_equal(ida, kept)
        keep_merge = set(kept.tolist()) | set(src.tolist())
        assert cnta.sum() == sum(int(cnt_b[pos[i]]) for i in keep_merge)
        # protected tokens unchanged bit for bit; untargeted kept tokens unchanged
        targets = set(dst.tolist())
        for p_after, i in enumerate(ida):
            if int(i) not in targets:
                assert np.array_equal(Ka[p_after], Kb[pos[int(i)]])
                assert np.array_equal(Va[p_after], Vb[pos[int(i)]])
        # merged values = count-weighted mean (numpy average), rounded to bf16
        for j in targets:
            srcs = [int(s) for s, d in zip(src, dst) if int(d) == j]
            members = [j] + srcs
            w = np.array([cnt_b[pos[m]] for m in members], float)
            for before, after in ((Kb, Ka), (Vb, Va)):
                stack = np.stack([before[pos[m]].reshape(-1) for m in members])
                mean = np.average(stack, axis=0, weights=w)
                got = after[list(ida).index(j)].reshape(-1)
                # the cache stores bf16: the merged value is rounded once to a bf16 number
                assert np.array_equal(torch.tensor(got).to(torch.bfloat16).to(torch.float64).numpy(), got)
                ulp = np.abs(bf16_round(mean) - bf16_round(mean * (1 + 2 ** -8)))
                assert np.all(np.abs(got - bf16_round(mean)) <= ulp + 1e-300)
        # compaction packs P per page in ascending id, into the lowest free pages
        pt = orc.page_table(l)
        assert np.all(pt[:, 0] == -1)
        assert pt[:, 3].sum() == n_keep and np.all(pt[:-1, 3] == wl.page_size)

    orc, events = _drive(wl, frames, on_event=check)
    assert events >= min_events and len(seen) == events


def test_compression_properties():
    _compression_check()


@settings(max_examples=20, deadline=None, derandomize=True)
@given(T=st.integers(5, 12), P=st.sampled_from([2, 4, 8]), B=st.integers(24, 64),
       keep_frac=st.sampled_from([0.5, 0.6, 0.75]), specials=st.integers(0, 2), H=st.integers(1, 3))
def test_compression_properties_swept(T, P, B, keep_frac, specials, H):
    """The same properties over frame sizes, page sizes, budgets, keep fractions, special
    token counts and head counts; the stream runs while the protected tokens (frame 0 and
    every frame's specials) still fit the keep tier."""
    n_keep = math.floor(float(np.float32(keep_frac)) * B)
    frames = 1
    while frames < 14 and T + specials * frames <= n_keep:
        frames += 1
    assume(frames * T > B + T)            # at least one compression event
    _compression_check(frames=frames, min_events=1, tokens_per_frame=T, page_size=P, budget_tokens=B,
                       keep_frac=keep_frac, num_special_tokens=specials, num_heads=H)


def test_full_protected_keep_tier_drops_merge_tier():
    wl = _small_wl(budget_tokens=20)      # floor(0.6*20) = 12 = 8 (frame 0) + 4 specials by frame 4
    got = []
    _drive(wl, 5, on_event=lambda orc, l, res, *a: got.append(res))
    assert got and got[-1]["n_protected"] == 12 and got[-1]["merge_src"].size == 0


def test_protected_overflow_raises():
    wl = _small_wl(budget_tokens=12, tokens_per_frame=8, num_special_tokens=4)
    # frame 0 alone is 8 protected tokens > floor(0.6 * 12) = 7
    with pytest.raises(OverflowError):
        _drive(wl, 3)


def test_no_compression_below_budget():
    wl = _small_wl(budget_tokens=1000)
    orc, events = _drive(wl, 5)
    assert events == 0
    ids, cnt, sh = orc.token_meta(0)
    assert ids.size == 5 * wl.tokens_per_frame and np.all(cnt == 1)


# ------------------------------------------------------------------ planted mistakes

def test_planted_unrounded_merge_is_caught(monkeypatch):
    """The merged mean stored in fp64 without its single rounding to bf16."""
    import oracle.kvcache_oracle as ko
    monkeypatch.setattr(ko, "bf16_round", lambda x: np.asarray(x, np.float64))
    with pytest.raises(AssertionError):
        _compression_check()


def test_planted_least_similar_target_is_caught(monkeypatch):
    """Merge targets taken by the smallest cosine instead of the largest (the oracle's
    numpy is swapped for a view whose argmax is argmin; the pins use the real numpy)."""
    import oracle.kvcache_oracle as ko

    class NP:
        def __getattr__(self, name):
            return getattr(np, name)

        argmax = staticmethod(np.argmin)
    monkeypatch.setattr(ko, "np", NP())
    with pytest.raises(AssertionError):
        _compression_check()


# ------------------------------------------------------------------ validated alternatives
# A test may make the oracle follow the GPU where two correct fp64 evaluations can differ;
# the oracle accepts only what the definitions allow.

def _one_event(target_choice=None, dup=False):
    """A budget stream up to its first compression; with `dup`, frame 2's keys and
    residuals are copies of frame 1's, so the twins have equal scores and a source's
    cosines to the two copies of a target are equal."""
    wl = _small_wl(num_layers=1)
    st = FrameStream(wl, seed=3)
    orc = StreamOracle(OracleConfig.from_workload(wl))
    keep = {}
    for t in range(12):
        q, k, v = (_np(x) for x in st.frame(0, t))
        r = _np(st.residual(0, t))
        if dup and t in (1, 2):
            k = keep.setdefault("k", k)
            r = keep.setdefault("r", r)
        orc.append(0, t, k, v, True)
        orc.attend(0, q)
        orc.score(0, t, r)
        res = orc.compress(0, target_choice=target_choice)
        if res is not None:
            return orc, res
    raise AssertionError("no compression event")


def test_target_choice_refuses_a_target_that_is_not_tied():
    _, res = _one_event()
    src, dst = res["merge_src"], res["merge_dst"]
    others = [int(i) for i in res["kept_ids"] if int(i) not in set(dst.tolist()) and int(i) // 8 != 0 and int(i) % 8]
    assert others
    with pytest.raises(ValueError):
        _one_event(target_choice={int(src[0]): others[0]})


def test_target_choice_follows_an_exact_tie():
    # identical keys in frames 1 and 2: a source's cosine to the two copies of a target is
    # the same number, so either copy is a correct target
    _, res = _one_event(dup=True)
    tie = None
    for s_id, d_id in zip(res["merge_src"], res["merge_dst"]):
        twin = int(d_id) + 8 if int(d_id) // 8 == 1 else int(d_id) - 8 if int(d_id) // 8 == 2 else None
        if twin is not None and twin in set(res["kept_ids"].tolist()) and twin % 8:
            tie = (int(s_id), twin)
            break
    if tie is None:
        pytest.skip("no merge into a duplicated key on this seed")
    _, res2 = _one_event(target_choice={tie[0]: tie[1]}, dup=True)
    got = dict(zip(res2["merge_src"].tolist(), res2["merge_dst"].tolist()))
    assert got[tie[0]] == tie[1]
