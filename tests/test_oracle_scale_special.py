"""CPU pins of the joint scale-frame phase and of cross-frame special-token persistence
(GCTStream page: Scale-Frame Phase, Special Token Persistence), against brute force over
explicitly concatenated tokens rebuilt from the definitions, not from the oracle's pages."""
import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

import brute
from oracle import OracleConfig, StreamOracle


def _cfg(T=37, H=2, D=16, P=16, W=2, S=1, ns=5, special=3, kv="f32"):
    return OracleConfig(num_layers=1, num_heads=H, head_dim=D, tokens_per_frame=T, num_special_tokens=ns,
                        page_size=P, window_frames=W, scale_frames=S, kv_dtype=kv, softmax_scale=0.25,
                        special_frames=special)


def _frames(n, T, H, D, seed):
    rng = np.random.default_rng(seed)
    return [tuple(rng.standard_normal((T, H, D)) for _ in range(3)) for _ in range(n)]


def _joint_phase_check():
    cfg = _cfg(T=37, S=4, W=3, special=0)
    fr = _frames(4, cfg.tokens_per_frame, cfg.num_heads, cfg.head_dim, 1)
    Q = np.concatenate([f[0] for f in fr])
    K = np.concatenate([f[1] for f in fr])
    V = np.concatenate([f[2] for f in fr])
    orc = StreamOracle(cfg)
    got = orc.scale_phase(0, 4, Q, K, V)
    ref = brute.attention(Q, K, V, cfg.softmax_scale)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    # bidirectional: frame 0's queries see frame 3's keys, unlike a causal step
    causal0 = brute.attention(fr[0][0], fr[0][1], fr[0][2], cfg.softmax_scale)
    assert np.abs(got[:cfg.tokens_per_frame] - causal0).max() > 1e-3
    # the four frames are the committed scale frames: the next frame sees them all
    q4, k4, v4 = _frames(1, cfg.tokens_per_frame, cfg.num_heads, cfg.head_dim, 2)[0]
    orc.append(0, 4, k4, v4, True)
    nxt = orc.attend(0, q4)
    ref4 = brute.attention(q4, np.concatenate([K, k4]), np.concatenate([V, v4]), cfg.softmax_scale)
    np.testing.assert_allclose(nxt, ref4, rtol=0, atol=1e-12)


def test_joint_phase_is_bidirectional_attention_over_all_scale_frames():
    _joint_phase_check()


def test_joint_phase_needs_an_empty_layer_and_at_most_S_frames():
    cfg = _cfg(S=2, special=0)
    T, H, D = cfg.tokens_per_frame, cfg.num_heads, cfg.head_dim
    x = np.zeros((3 * T, H, D))
    with pytest.raises(ValueError):
        StreamOracle(cfg).scale_phase(0, 3, x, x, x)
    orc = StreamOracle(cfg)
    orc.scale_phase(0, 2, x[:2 * T], x[:2 * T], x[:2 * T])
    with pytest.raises(RuntimeError):
        orc.scale_phase(0, 1, x[:T], x[:T], x[:T])


def _expected_tokens(t, S, W, cap, T, ns):
    """Token ids frame t attends to (every frame a keyframe): scale frames and window
    frames whole, the special tokens of the last `cap` evicted frames, frame t."""
    prev = list(range(t))
    keep = set(prev[:S]) | set(prev[-W:]) if W > 0 else set(prev)
    evicted = [u for u in prev if u not in keep]
    kept_special = evicted[-cap:] if cap > 0 else []
    ids = []
    for u in prev:
        if u in keep:
            ids += [u * T + i for i in range(T)]
        elif u in kept_special:
            ids += [u * T + i for i in range(ns)]
    return ids + [t * T + i for i in range(T)]


SPECIAL_CASES = [
    (37, 16, 5, 3, 1, 2),     # one special page per evicted frame, FIFO after 3
    (40, 16, 18, 2, 2, 3),    # specials span two pages (16 + 2)
    (10, 16, 5, 50, 0, 1),    # T < P, no scale frame, cap never reached
]


def _special_tokens_check(T, P, ns, cap, S, W):
    cfg = _cfg(T=T, P=P, ns=ns, special=cap, S=S, W=W)
    H, D = cfg.num_heads, cfg.head_dim
    fr = _frames(14, T, H, D, 3)
    orc = StreamOracle(cfg)
    tokK, tokV = {}, {}
    for t, (q, k, v) in enumerate(fr):
        for i in range(T):
            tokK[t * T + i], tokV[t * T + i] = k[i], v[i]
        orc.append(0, t, k, v, True)
        ids = _expected_tokens(t, S, W, cap, T, ns)
        _, _, got_ids = orc.gather(0)
        assert sorted(got_ids.tolist()) == ids, f"frame {t}"
        out = orc.attend(0, q)
        Kc = np.stack([tokK[i] for i in ids])
        Vc = np.stack([tokV[i] for i in ids])
        np.testing.assert_allclose(out, brute.attention(q, Kc, Vc, cfg.softmax_scale), rtol=0, atol=1e-12)
    # memory: scale + window frames whole, retained frames one page per P specials
    L = orc.layers[0]
    n_ret = min(cap, 14 - S - W)
    assert len(L.retained) == n_ret
    assert sum(L.free_used) == (S + W) * -(-T // P) + n_ret * -(-ns // P)


@pytest.mark.parametrize("T,P,ns,cap,S,W", SPECIAL_CASES)
def test_special_tokens_outlive_their_frames(T, P, ns, cap, S, W):
    _special_tokens_check(T, P, ns, cap, S, W)


@settings(max_examples=25, deadline=None, derandomize=True)
@given(T=st.integers(1, 40), P=st.sampled_from([1, 2, 4, 8, 16]), ns_frac=st.floats(0.0, 1.0),
       cap=st.integers(1, 6), S=st.integers(0, 3), W=st.integers(1, 5))
def test_special_tokens_outlive_their_frames_swept(T, P, ns_frac, cap, S, W):
    """The same check over frame and page sizes (special tokens within one page, across
    pages, the whole frame), FIFO caps, scale frames and windows."""
    ns = max(1, min(T, round(ns_frac * T)))
    _special_tokens_check(T, P, ns, cap, S, W)


def test_trimmed_pages_hold_zeros_past_the_special_tokens():
    cfg = _cfg(T=37, P=16, ns=5, special=4, S=0, W=1)
    orc = StreamOracle(cfg)
    for t, (q, k, v) in enumerate(_frames(4, 37, 2, 16, 4)):
        orc.append(0, t, k, v, True)
        orc.attend(0, q)
    L = orc.layers[0]
    for pid, owner, idx, n in L.entries:
        if owner in L.retained:
            pg = L.pages[pid]
            assert idx == 0 and n == 5 and pg.valid == 5
            assert not pg.k[:, 5:].any() and not pg.v[:, 5:].any() and (pg.ids[5:] == -1).all()


def test_non_keyframes_leave_no_special_tokens():
    cfg = _cfg(T=37, P=16, ns=5, special=10, S=1, W=2)
    orc = StreamOracle(cfg)
    for t, (q, k, v) in enumerate(_frames(12, 37, 2, 16, 5)):
        orc.append(0, t, k, v, t % 2 == 0)
        orc.attend(0, q)
    assert all(f % 2 == 0 for f in orc.layers[0].retained)
    _, _, ids = orc.gather(0)
    assert all((i // 37) % 2 == 0 for i in ids.tolist())


# ------------------------------------------------------------------ planted mistakes
# Each plants one plausible misreading in the oracle (on the CPU); the pins above must
# fail on it.

def test_planted_causal_joint_phase_is_caught(monkeypatch):
    """The joint phase read as frame-by-frame causal steps over the scale frames."""
    def causal(self, layer, n, Q, K, V, rows=None):
        T = self.T
        outs = []
        for f in range(n):
            self.append(layer, f, K[f * T:(f + 1) * T], V[f * T:(f + 1) * T], True)
            outs.append(self.attend(layer, Q[f * T:(f + 1) * T]))
        return np.concatenate(outs)
    monkeypatch.setattr(StreamOracle, "scale_phase", causal)
    with pytest.raises(AssertionError):
        _joint_phase_check()


def test_planted_dropped_special_tokens_are_caught(monkeypatch):
    """Eviction that forgets the special tokens (plain sliding window)."""
    monkeypatch.setattr(StreamOracle, "_retain_special", lambda self, L, f: None)
    with pytest.raises(AssertionError):
        _special_tokens_check(*SPECIAL_CASES[0])


def test_planted_newest_first_special_cap_is_caught(monkeypatch):
    """At the special_frames cap, the newest retained frame dropped instead of the oldest."""
    orig = StreamOracle._retain_special

    def newest_first(self, L, f):
        cap = self.cfg.special_frames
        self.cfg.special_frames = 1 << 30
        try:
            orig(self, L, f)
        finally:
            self.cfg.special_frames = cap
        while len(L.retained) > cap:
            new = L.retained.pop()
            self._free(L, [e[0] for e in L.entries if e[1] == new])
            L.entries = [e for e in L.entries if e[1] != new]
    monkeypatch.setattr(StreamOracle, "_retain_special", newest_first)
    with pytest.raises(AssertionError):
        _special_tokens_check(*SPECIAL_CASES[0])


def test_planted_untrimmed_special_page_is_caught(monkeypatch):
    """The special page kept whole: the non-special tokens sharing it survive eviction."""
    def untrimmed(self, L, f):
        keep_pages = -(-min(self.cfg.num_special_tokens, self.T) // self.P)
        drop = [e[0] for e in L.entries if e[1] == f and e[2] >= keep_pages]
        self._free(L, drop)
        L.entries = [e for e in L.entries if not (e[1] == f and e[2] >= keep_pages)]
        L.retained.append(f)
        while len(L.retained) > self.cfg.special_frames:
            old = L.retained.pop(0)
            self._free(L, [e[0] for e in L.entries if e[1] == old])
            L.entries = [e for e in L.entries if e[1] != old]
    monkeypatch.setattr(StreamOracle, "_retain_special", untrimmed)
    with pytest.raises(AssertionError):
        _special_tokens_check(*SPECIAL_CASES[0])


def test_joint_phase_over_fp8_pages_matches_brute_force():
    """FP8 storage: every frame's pages quantised per (page, head) through torch's float8
    cast, then bidirectional attention over all of them."""
    import torch
    cfg = _cfg(T=37, P=8, S=3, W=2, special=0, kv="fp8_e4m3")
    T, H, D = cfg.tokens_per_frame, cfg.num_heads, cfg.head_dim
    bf = lambda x: torch.tensor(x).to(torch.bfloat16).to(torch.float64).numpy()
    fr = [tuple(bf(x) for x in f) for f in _frames(3, T, H, D, 9)]
    Q = np.concatenate([f[0] for f in fr])
    got = StreamOracle(cfg).scale_phase(0, 3, Q, np.concatenate([f[1] for f in fr]),
                                        np.concatenate([f[2] for f in fr]))
    Ks = np.concatenate([brute.stored(f[1], "fp8_e4m3", cfg.page_size) for f in fr])
    Vs = np.concatenate([brute.stored(f[2], "fp8_e4m3", cfg.page_size) for f in fr])
    np.testing.assert_allclose(got, brute.attention(Q, Ks, Vs, cfg.softmax_scale), rtol=1e-10, atol=1e-12)


def test_fp8_special_tokens_keep_their_stored_values_after_eviction():
    """Trimming keeps the page's codes and scale for the special tokens: their stored values
    after eviction are the ones the frame's quantisation gave them (no requantisation over
    the survivors), and equal torch's float8 cast of the whole page."""
    import torch
    cfg = _cfg(T=37, P=16, ns=5, special=4, S=0, W=1, kv="fp8_e4m3")
    orc = StreamOracle(cfg)
    bf = lambda x: torch.tensor(x).to(torch.bfloat16).to(torch.float64).numpy()   # the library's inputs
    fr = [tuple(bf(x) for x in f) for f in _frames(4, 37, 2, 16, 12)]
    for t, (q, k, v) in enumerate(fr):
        orc.append(0, t, k, v, True)
        orc.attend(0, q)
    L = orc.layers[0]
    assert L.retained
    for pid, owner, idx, n in L.entries:
        if owner in L.retained:
            pg = L.pages[pid]
            want_k = brute.stored(fr[owner][1], "fp8_e4m3", cfg.page_size)[:5]
            want_v = brute.stored(fr[owner][2], "fp8_e4m3", cfg.page_size)[:5]
            np.testing.assert_array_equal(pg.k[:, :5], np.transpose(want_k, (1, 0, 2)))
            np.testing.assert_array_equal(pg.v[:, :5], np.transpose(want_v, (1, 0, 2)))


def test_no_special_tokens_is_the_plain_window():
    """num_special_tokens = 0 with a special-frame cap: nothing survives an eviction, and the
    stream equals the plain sliding window bit for bit."""
    fr = _frames(9, 37, 2, 16, 13)
    outs = {}
    for special in (3, 0):
        orc = StreamOracle(_cfg(T=37, ns=0, special=special, S=1, W=2))
        outs[special] = []
        for t, (q, k, v) in enumerate(fr):
            orc.append(0, t, k, v, True)
            outs[special].append(orc.attend(0, q))
        L = orc.layers[0]
        assert all(e[1] not in L.retained for e in L.entries)   # no page kept for an evicted frame
    for a, b in zip(outs[3], outs[0]):
        np.testing.assert_array_equal(a, b)
