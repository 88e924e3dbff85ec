"""CPU pins of the rolling diversity-pruned memory oracle ("InfiniteVGGT" explainer page):
scipy's cosine distance and softmax, brute-force Top-K, the page's worked numbers and
closed-form cases, and a planted mistake that the pins must catch."""
import numpy as np
import pytest
from hypothesis import given, settings, strategies as st
from scipy.spatial.distance import cosine
from scipy.special import softmax

import oracle.rolling_oracle as ro
from oracle import RollingOracle, diversity_scores, layer_budgets, top_k


def _scores_by_scipy(Kc):
    kh = [k / np.linalg.norm(k) for k in Kc]
    mu = np.sum(kh, axis=0)
    return np.array([-(1.0 - cosine(k, mu)) for k in Kc])


def test_scores_are_negative_cosine_to_mean_key():
    rng = np.random.default_rng(0)
    Kc = rng.standard_normal((300, 64)) * np.exp(rng.standard_normal(300))[:, None]
    np.testing.assert_allclose(diversity_scores(Kc), _scores_by_scipy(Kc), rtol=0, atol=1e-14)


def test_unique_direction_scores_highest():
    # n copies of one direction and one orthogonal key: the orthogonal key is the most
    # diverse (score -1/sqrt(n^2+1) against -n/sqrt(n^2+1) for the copies)
    n, D = 40, 16
    Kc = np.zeros((n + 1, D))
    Kc[:n, 0] = 2.0 ** np.arange(n) % 7 + 1.0       # different lengths, same direction
    Kc[n, 3] = 5.0
    sc = diversity_scores(Kc)
    assert np.argmax(sc) == n
    np.testing.assert_allclose(sc[n], -1.0 / np.sqrt(n * n + 1), rtol=1e-15)
    np.testing.assert_allclose(sc[:n], -n / np.sqrt(n * n + 1), rtol=1e-15)


def test_scores_invariant_to_positive_key_scaling():
    rng = np.random.default_rng(1)
    Kc = rng.standard_normal((50, 32))
    K2 = Kc.copy()
    K2[7] *= 8.0                                   # a power of two: the normalised key is identical
    K2[19] *= 0.25
    assert np.array_equal(diversity_scores(Kc), diversity_scores(K2))


def test_zero_key_has_no_direction():
    Kc = np.eye(4)
    Kc[2] = 0.0
    sc = diversity_scores(Kc)
    assert sc[2] == 0.0 and np.all(np.isfinite(sc))


def test_worked_example_1200_candidates_keep_512_drop_688():
    rng = np.random.default_rng(2)
    Kc = rng.standard_normal((1200, 64))
    ids = np.arange(1200) * 3 + 11
    sc = diversity_scores(Kc)
    keep = top_k(sc, ids, 512)
    assert len(keep) == 512 and 1200 - len(keep) == 688
    # brute force: the kept set is exactly the 512 largest scores (no ties here)
    want = set(np.argsort(-sc, kind="stable")[:512].tolist())
    assert set(keep.tolist()) == want
    assert np.all(np.diff(ids[keep]) > 0)           # stored in ascending id


def test_ties_go_to_lower_ids():
    Kc = np.ones((10, 8))
    ids = np.arange(10)[::-1].copy()                # ids 9..0
    keep = top_k(diversity_scores(Kc), ids, 4)
    assert sorted(ids[keep].tolist()) == [0, 1, 2, 3]


def test_budget_arithmetic_of_the_page():
    # 512 tokens per head, 16 heads -> 8,192 per layer; 12 layers -> 98,304 (~98k)
    b = layer_budgets([0.3] * 12, 1.0, 512)
    assert b == [512] * 12
    assert sum(x * 16 for x in b) == 98304
    assert layer_budgets([0.1, 0.9, 0.5], 0.0, 512) == [512, 512, 512]


def test_layer_budgets_follow_softmax_of_mean_diversity():
    d = [-0.9, -0.5, -0.7, -0.2]
    for tau in (0.05, 0.2, 1.0):
        b = layer_budgets(d, tau, 512)
        p = softmax(np.array(d) / tau)
        np.testing.assert_array_equal(b, np.floor(4 * 512 * p).astype(int))
        assert sum(b) <= 4 * 512
        assert b[3] == max(b) and b[0] == min(b)   # more diverse layer, more memory


def _stream(T=20, H=3, D=16, K=30, frames=7, seed=3):
    rng = np.random.default_rng(seed)
    orc = RollingOracle(2, H, D, T, K, 0.25)
    seen = []
    for t in range(frames):
        q = rng.standard_normal((T, H, D))
        k = rng.standard_normal((T, H, D))
        v = rng.standard_normal((T, H, D))
        seen.append((q, k, v))
        orc.append(0, t, k, v)
        out = orc.attend(0, q)
        yield t, orc, (q, k, v), out


def test_anchor_immutable_and_memory_bounded():
    T, K = 20, 30
    for t, orc, _, _ in _stream(T=T, K=K):
        for h in range(3):
            ids = orc.head_ids(0, h)
            assert np.array_equal(ids[:T], np.arange(T))              # frame 0 kept whole
            mut = orc.mut_ids[0][h]
            assert len(mut) == min(K, T * t)                         # bounded at K
            assert np.all(mut >= T) and np.all(np.diff(mut) > 0)


def _kept_set_check(T=20, H=3, D=16, K=30, frames=7, seed=3):
    # brute force on one head: candidates = previous kept + new frame, scored by scipy
    prev = {h: (np.zeros(0, int), np.zeros((0, D))) for h in range(H)}
    for t, orc, (q, k, v), _ in _stream(T=T, H=H, D=D, K=K, frames=frames, seed=seed):
        if t == 0:
            continue
        for h in range(H):
            ids = np.concatenate([prev[h][0], t * T + np.arange(T)])
            Kc = np.concatenate([prev[h][1], k[:, h, :]])
            sc = _scores_by_scipy(Kc)
            order = sorted(range(len(ids)), key=lambda i: (-round(sc[i], 12), ids[i]))[:K]
            assert set(ids[order].tolist()) == set(orc.mut_ids[0][h].tolist())
            sel = sorted(order, key=lambda i: ids[i])
            prev[h] = (ids[sel], Kc[sel])


def test_kept_set_is_top_k_of_candidates_each_frame():
    _kept_set_check()


@settings(max_examples=20, deadline=None, derandomize=True)
@given(T=st.integers(1, 24), H=st.integers(1, 3), D=st.sampled_from([4, 8, 16]), K=st.integers(1, 60),
       frames=st.integers(2, 8), seed=st.integers(0, 1000))
def test_kept_set_is_top_k_swept(T, H, D, K, frames, seed):
    """The kept set against brute-force Top-K by scipy cosine over frame sizes (a frame
    smaller and larger than K), head counts, head dims, budgets and stream lengths."""
    _kept_set_check(T=T, H=H, D=D, K=K, frames=frames, seed=seed)


def _ties_check():
    Kc = np.ones((10, 8))
    ids = np.arange(10)[::-1].copy()                # ids 9..0
    keep = ro.top_k(ro.diversity_scores(Kc), ids, 4)
    assert sorted(ids[keep].tolist()) == [0, 1, 2, 3]


def test_attention_is_softmax_over_anchor_and_kept():
    from scipy.special import softmax as sm
    for t, orc, (q, k, v), out in _stream():
        for h in range(3):
            Kh = np.concatenate([orc.anchor_k[0][h], orc.mut_k[0][h]])
            Vh = np.concatenate([orc.anchor_v[0][h], orc.mut_v[0][h]])
            want = sm(q[:, h, :] @ Kh.T * 0.25, axis=1) @ Vh
            np.testing.assert_allclose(out[:, h, :], want, rtol=0, atol=1e-12)


def test_planted_sign_mistake_is_caught(monkeypatch):
    # scoring by +cos (similarity) instead of -cos keeps the duplicates: the unique-key
    # pin must fail
    real = ro.diversity_scores
    monkeypatch.setattr(ro, "diversity_scores", lambda Kc: -real(Kc))
    n = 40
    Kc = np.zeros((n + 1, 16))
    Kc[:n, 0] = 1.0
    Kc[n, 3] = 1.0
    assert np.argmax(ro.diversity_scores(Kc)) != n


def test_layer_diversity_is_mean_of_scores():
    rng = np.random.default_rng(10)
    L, H, D, T, K = 1, 3, 16, 40, 50
    orc = RollingOracle(L, H, D, T, K, 0.25)
    for t in range(3):
        K_ = rng.standard_normal((T, H, D))
        orc.append(0, t, K_, K_)
        if t == 0:
            continue
        cands = [(orc.mut_k[0][h], K_[:, h, :]) for h in range(H)]
        orc.prune(0)
        ref = [_scores_by_scipy(np.concatenate(c)) for c in cands]
        mean = np.mean(np.concatenate(ref))
        assert abs(orc.layer_diversity(0) - mean) < 1e-13


def test_normalisation_is_division_by_the_norm():
    # |(3, 4)| = 5 exactly, so the unit key is (3/5, 4/5), each one IEEE division; a zero
    # key stays zero
    kh = ro.normalised_keys(np.array([[3.0, 4.0], [0.0, 0.0]]))
    assert kh[0, 0] == 3.0 / 5.0 and kh[0, 1] == 4.0 / 5.0
    assert np.array_equal(kh[1], [0.0, 0.0])


def test_mean_and_sum_give_the_same_scores():
    # the cosine to the mean of the unit keys equals the cosine to their sum (same
    # direction): the scores against an explicit sum-based evaluation
    rng = np.random.default_rng(12)
    Kc = rng.standard_normal((77, 64))
    kh = Kc / np.linalg.norm(Kc, axis=1, keepdims=True)
    mu = kh.sum(axis=0)
    want = -(Kc @ mu) / (np.linalg.norm(Kc, axis=1) * np.linalg.norm(mu))
    np.testing.assert_allclose(diversity_scores(Kc), want, rtol=0, atol=1e-14)


# ------------------------------------------------------------------ planted mistakes
# Plausible misreadings planted in the oracle (on the CPU), each run through a pin above.

def test_planted_similarity_instead_of_diversity_is_caught(monkeypatch):
    """Keeping the candidates most similar to the mean (+cos) instead of the most diverse."""
    real = ro.diversity_scores
    monkeypatch.setattr(ro, "diversity_scores", lambda Kc: -real(Kc))
    with pytest.raises(AssertionError):
        _kept_set_check()


def test_planted_unnormalised_keys_are_caught(monkeypatch):
    """The mean taken over raw keys (long keys dominate) instead of unit keys."""
    monkeypatch.setattr(ro, "normalised_keys", lambda Kc: np.asarray(Kc, np.float64))
    with pytest.raises(AssertionError):
        _kept_set_check()


def test_planted_new_frame_only_candidates_are_caught(monkeypatch):
    """Pruning that forgets the kept set and ranks only the new frame's tokens."""
    orig = RollingOracle.prune

    def forgetful(self, layer):
        for h in range(len(self.mut_ids[layer])):
            D = self.mut_k[layer][h].shape[1]
            self.mut_ids[layer][h] = np.zeros(0, np.int64)
            self.mut_k[layer][h] = np.zeros((0, D))
            self.mut_v[layer][h] = np.zeros((0, D))
        return orig(self, layer)
    monkeypatch.setattr(RollingOracle, "prune", forgetful)
    with pytest.raises(AssertionError):
        _kept_set_check()


def test_planted_ties_to_higher_ids_are_caught(monkeypatch):
    """Equal scores resolved towards the higher token id."""
    def top_k_high(scores, ids, k):
        order = sorted(range(len(ids)), key=lambda i: (-scores[i], -ids[i]))[:k]
        return np.array(sorted(order, key=lambda i: ids[i]), dtype=np.int64)
    monkeypatch.setattr(ro, "top_k", top_k_high)
    with pytest.raises(AssertionError):
        _ties_check()


def test_layer_budgets_clamped_to_the_pool():
    # a sharp softmax gives one layer nearly all of L * k; clamped to [1, cap] the others
    # keep one token and the favoured layer no more than its pool holds
    d = [-0.9, -0.1, -0.8]
    raw = layer_budgets(d, 0.01, 512)
    assert raw[1] > 512 and min(raw) == 0
    assert layer_budgets(d, 0.01, 512, lo=1, hi=600) == [max(1, min(600, x)) for x in raw]
    assert layer_budgets(d, 0.0, 512, lo=1, hi=300) == [300, 300, 300]
