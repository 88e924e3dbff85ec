"""Pins for the oracle's cross-layer consistency scoring (StreamCacheVGGT page,
sections 2.1.1 to 2.1.4): closed forms, a library variance, exact sums."""
import math
import statistics
from fractions import Fraction

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

from kvc_streams import WORKLOADS
from oracle import OracleConfig, StreamOracle, to_f32


def _orc(T, lam=0.5, window=5, layers=8):
    cfg = OracleConfig(num_layers=layers, num_heads=1, head_dim=4, tokens_per_frame=T, num_special_tokens=1,
                       page_size=4, window_frames=0, scale_frames=0, kv_dtype="bf16", softmax_scale=0.125,
                       budget_tokens=10 ** 6, lam=lam, rank_window=window, residual_dim=8)
    return StreamOracle(cfg)


def _residual_with_norms(norms, dim=8):
    r = np.zeros((len(norms), dim))
    r[:, 0] = norms
    return r


def test_constant_rank_gives_cons_one_and_fifty_percent_bonus():
    T = 12
    orc = _orc(T)
    norms = np.arange(1, T + 1, dtype=np.float64) * 0.75
    for l in range(7):
        sh = orc.score(l, 0, _residual_with_norms(norms))
        # ranks never move -> sigma = 0 -> Cons = 1 -> s_hat = fp32(s * 1.5)
        np.testing.assert_array_equal(sh, to_f32(to_f32(norms) * 1.5))


def test_raw_score_is_rounded_to_fp32_before_the_bonus():
    # norms that fp32 does not hold, in the same order at every layer: Cons = 1 and
    # s_hat = fp32(fp32(s) * 1.5), which differs from rounding s * 1.5 once for some of them
    T = 16
    norms = 1.0 + np.sort(np.random.default_rng(11).uniform(0, 1, T))
    want = to_f32(to_f32(norms) * 1.5)
    assert np.any(want != to_f32(norms * 1.5))      # the two readings differ on this input
    orc = _orc(T)
    for l in range(3):
        sh = orc.score(l, 0, _residual_with_norms(norms))
    np.testing.assert_array_equal(sh, want)


def test_lambda_zero_returns_raw_score():
    rng = np.random.default_rng(0)
    orc = _orc(50, lam=0.0)
    for l in range(6):
        r = rng.standard_normal((50, 8))
        sh = orc.score(l, 0, r)
        exact = np.array([math.sqrt(math.fsum(float(v) ** 2 for v in row)) for row in r])
        np.testing.assert_array_equal(sh, to_f32(exact))


def test_opposite_ranks_over_two_layers_give_cons_zero():
    # token 0 is best at layer 0 and worst at layer 1: normalised ranks 0 and 1,
    # population sigma = 0.5 > 1/sqrt(12) -> Cons = max(0, 1 - 0.5*sqrt(12)) = 0
    T = 10
    orc = _orc(T)
    n0 = np.linspace(1, 2, T)[::-1].copy()   # token 0 largest
    orc.score(0, 0, _residual_with_norms(n0))
    n1 = np.linspace(1, 2, T)                # token 0 smallest
    sh = orc.score(1, 0, _residual_with_norms(n1))
    assert sh[0] == float(np.float32(n1[0]))                 # no bonus for token 0
    # a middle token that keeps rank ~ (T-1)/2 on both layers gets a bonus > 0
    assert sh[T // 2] > float(np.float32(n1[T // 2]))


def test_sigma_matches_library_population_variance():
    _sigma_check(T=40, window=5, lam=0.5, layers=8, seed=1)


@settings(max_examples=25, deadline=None, derandomize=True)
@given(T=st.integers(2, 60), window=st.integers(1, 8), lam=st.sampled_from([0.0, 0.25, 0.5, 1.0]),
       layers=st.integers(1, 10), seed=st.integers(0, 1000))
def test_sigma_matches_library_population_variance_swept(T, window, lam, layers, seed):
    """The same check over frame sizes, rank windows (shorter and longer than the layer
    count), consistency weights and seeds."""
    _sigma_check(T=T, window=window, lam=lam, layers=layers, seed=seed)


def _sigma_check(T, window, lam, layers, seed):
    rng = np.random.default_rng(seed)
    orc = _orc(T, lam=lam, window=window, layers=max(layers, 1))
    ranks = []
    for l in range(layers):
        r = rng.standard_normal((T, 8))
        s = to_f32(np.sqrt((r * r).sum(axis=1)))
        # library ranking: stable argsort of -s gives ties to the lower index
        order = np.argsort(-s, kind="stable")
        R = np.empty(T, int); R[order] = np.arange(T)
        ranks.append(R)
        sh = orc.score(l, 0, r)
        win = ranks[max(0, l - window + 1): l + 1]
        for i in range(T):
            vals = [Fraction(int(w[i]), T - 1) for w in win]
            var = statistics.pvariance(vals)                       # exact rational variance
            sigma = math.sqrt(var)
            cons = max(0.0, 1.0 - sigma * math.sqrt(12.0))
            want = float(s[i]) * (1.0 + lam * cons)
            # the oracle evaluates sigma from the exact integer D in its own order;
            # agree to fp32 rounding of nearly equal fp64 values
            assert abs(sh[i] - want) <= 2 ** -22 * abs(want), (l, i, sh[i], want)


def test_ties_break_to_lower_slot_and_window_and_reset():
    T = 6
    orc = _orc(T)
    # all equal norms: ranks are the slot order at every layer -> Cons = 1
    r = np.ones((T, 8))
    for l in range(3):
        sh = orc.score(l, 0, r)
    assert np.all(sh == to_f32(to_f32(np.sqrt(8.0)) * 1.5))
    # window: two wild layers, then five constant layers -> only the last five count
    orc = _orc(T)
    rng = np.random.default_rng(5)
    orc.score(0, 1, _residual_with_norms(rng.permutation(T) + 1.0))
    orc.score(1, 1, _residual_with_norms(rng.permutation(T) + 1.0))
    base = np.arange(T, dtype=float) + 1.0
    for l in range(2, 7):
        sh = orc.score(l, 1, _residual_with_norms(base))
    np.testing.assert_array_equal(sh, to_f32(to_f32(base) * 1.5))
    # history resets at a new frame: layer 0 of frame 2 alone -> n = 1 -> Cons = 1
    sh = orc.score(0, 2, _residual_with_norms(rng.permutation(T) + 1.0))
    s = sh / 1.5
    assert np.all(np.abs(sh - to_f32(s * 1.5)) == 0)


def test_raw_score_is_fp32_of_exact_norm():
    rng = np.random.default_rng(2)
    r = (rng.standard_normal((300, 1024)) * np.exp(rng.standard_normal(300))[:, None]).astype(np.float32)
    orc = _orc(300, lam=0.0)
    sh = orc.score(0, 0, r.astype(np.float64))
    exact = np.array([math.sqrt(math.fsum(float(v) * float(v) for v in row)) for row in r])
    np.testing.assert_array_equal(sh, to_f32(exact))


# ------------------------------------------------------------------ planted mistakes

def test_planted_unrounded_raw_score_is_caught(monkeypatch):
    """s kept in fp64 instead of rounded once to fp32 (StreamCacheVGGT page, 2.1.1)."""
    import oracle.kvcache_oracle as ko
    monkeypatch.setattr(ko, "to_f32", lambda x: np.asarray(x, np.float64))
    with pytest.raises(AssertionError):
        test_raw_score_is_rounded_to_fp32_before_the_bonus()


def test_planted_sample_variance_is_caught(monkeypatch):
    """sigma from the sample variance (divide by n - 1) instead of the population one: the
    exact-rational pin must fail. Planted through the oracle's square root of D, scaled by
    n / (n - 1) inside the same expression."""
    import oracle.kvcache_oracle as ko
    real_sqrt = math.sqrt
    state = {}

    class M:
        def __getattr__(self, name):
            return getattr(math, name)

        @staticmethod
        def sqrt(x):
            n = state.get("n")
            if n is not None and n > 1 and x != 12.0:
                return real_sqrt(x * n / (n - 1))
            return real_sqrt(x)

    orig_score = ko.StreamOracle.score

    def score(self, layer, t, residual):
        # the window length the oracle will use for this call
        hist = self._rank_hist if t == self._rank_frame else {}
        state["n"] = 1 + sum(1 for l in range(layer - self.cfg.rank_window + 1, layer) if l in hist)
        return orig_score(self, layer, t, residual)
    monkeypatch.setattr(ko, "math", M())
    monkeypatch.setattr(ko.StreamOracle, "score", score)
    with pytest.raises(AssertionError):
        test_sigma_matches_library_population_variance()


def test_s_choice_takes_only_an_fp32_neighbour_of_the_norm():
    # the oracle follows another side's fp32 rounding of a norm only where it is the
    # adjacent fp32 value; two steps away is refused
    wl = WORKLOADS["vggt_budget_16k"].replace(tokens_per_frame=16, num_heads=2, residual_dim=32, num_layers=1)
    r = np.random.default_rng(4).standard_normal((16, 32)).astype(np.float32).astype(np.float64)
    exact = math.sqrt(math.fsum(float(v) * float(v) for v in r[3]))
    f = np.float32(exact)
    up1 = float(np.nextafter(f, np.float32(np.inf)))
    up2 = float(np.nextafter(np.float32(up1), np.float32(np.inf)))
    orc = StreamOracle(OracleConfig.from_workload(wl))
    sh = orc.score(0, 0, r, s_choice={3: up1})
    assert sh[3] == float(np.float32(up1 * 1.5))       # one layer: Cons = 1
    with pytest.raises(ValueError):
        StreamOracle(OracleConfig.from_workload(wl)).score(0, 0, r, s_choice={3: up2})
