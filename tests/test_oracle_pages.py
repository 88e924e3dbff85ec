"""The workloads and the oracle's constants agree with numbers the pages print, and
mistakes planted in the oracle (on the CPU) are caught by the pins."""
import json
import math
import os

import numpy as np
import pytest
import torch

import brute
from kvc_streams import WORKLOADS, FrameStream
from oracle import OracleConfig, StreamOracle, to_f32
import oracle.kvcache_oracle as ko

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_constants.json")))


def test_workload_shapes_match_the_pages():
    assert WORKLOADS["vggt_518x378"].tokens_per_frame == GOLD["tokens_518x378"]["value"] == 37 * 27 + 5
    assert WORKLOADS["vggt_518x518_fp8"].tokens_per_frame == GOLD["tokens_518x518"]["value"] == 37 * 37 + 5
    assert WORKLOADS["vggt_518x378"].window_frames == GOLD["sliding_window_frames"]["value"]
    assert WORKLOADS["vggt_518x378"].scale_frames == GOLD["scale_frames"]["value"]
    wl = WORKLOADS["vggt_budget_16k"]
    assert wl.rank_window == GOLD["rank_window_layers"]["value"]
    assert wl.lam == GOLD["lambda"]["value"]
    ex = GOLD["infinitevggt_budget_example"]
    assert ex["candidates"] - ex["keep"] == ex["drop"]
    pl = GOLD["infinitevggt_per_layer"]
    assert pl["per_head"] * pl["heads"] == pl["per_layer"]
    assert abs(pl["per_layer"] * pl["layers"] - pl["total_approx"]) < 0.01 * pl["total_approx"]


def test_cons_vanishes_at_the_uniform_reference():
    # sigma = sqrt(1/12) is the uniform-null spread: Cons must be exactly 0 there
    sigma_max = math.sqrt(GOLD["uniform_variance"]["value"])
    assert max(0.0, 1.0 - sigma_max * math.sqrt(12.0)) <= 4e-16
    # any larger spread is clamped to exactly zero
    assert max(0.0, 1.0 - 0.3 * math.sqrt(12.0)) == 0.0


def _brute_frame_check(wl, frames=6):
    st = FrameStream(wl, seed=11)
    orc = StreamOracle(OracleConfig.from_workload(wl))
    hk, hv = {}, {}
    for t in range(frames):
        q, k, v = (x.to(torch.float64).numpy() for x in st.frame(0, t))
        orc.append(0, t, k, v, True)
        hk[t], hv[t] = k, v
        got = orc.attend(0, q)
        fr = brute.retained_frames(t, wl.scale_frames, wl.window_frames, 1)
        ref = brute.attention(q, np.concatenate([hk[u] for u in fr]), np.concatenate([hv[u] for u in fr]),
                              float(np.float32(wl.softmax_scale)))
        np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("mistake", ["no_max_subtract_sign", "drop_pending", "keep_wrong_end", "transpose"])
def test_planted_oracle_mistakes_are_caught(monkeypatch, mistake):
    wl = WORKLOADS["tiny_f32"]
    if mistake == "no_max_subtract_sign":
        orig = StreamOracle.attend
        def bad(self, layer, Q, rows=None, commit=True):
            self.scale = -abs(self.scale)
            return orig(self, layer, Q, rows, commit)
        monkeypatch.setattr(StreamOracle, "attend", bad)
    elif mistake == "drop_pending":
        orig_g = StreamOracle.gather
        def bad(self, layer):
            L = self.layers[layer]
            keep = L.entries
            others = [e for e in keep if e[1] != L.pending]
            L.entries = others if others else keep
            try:
                return orig_g(self, layer)
            finally:
                L.entries = keep
        monkeypatch.setattr(StreamOracle, "gather", bad)
    elif mistake == "keep_wrong_end":
        orig_c = StreamOracle.commit
        def bad(self, layer):
            L = self.layers[layer]
            orig_c(self, layer)
            # evict the newest instead of the oldest window frame
            if len(L.committed) > 2:
                f = L.committed[-1]
                self._free(L, [e[0] for e in L.entries if e[1] == f])
                L.entries = [e for e in L.entries if e[1] != f]
                L.committed = L.committed[:-1]
        monkeypatch.setattr(StreamOracle, "commit", bad)
    elif mistake == "transpose":
        orig_a = StreamOracle.append
        def bad(self, layer, t, K, V, is_key):
            return orig_a(self, layer, t, V, K, is_key)
        monkeypatch.setattr(StreamOracle, "append", bad)
    with pytest.raises(AssertionError):
        _brute_frame_check(wl)


def test_harness_keyframe_schedule_is_the_oracles_rule():
    """The streams hand both sides the same is_keyframe decision (the library takes it as an
    argument); it must be the oracle's reading of the keyframe rule, and match a hand-listed
    case: S = 2, k = 3 keeps frames 0, 1, 2, 5, 8, 11."""
    from kvc_streams import keyframe_schedule
    from oracle import is_keyframe
    for S in range(0, 5):
        for k in range(1, 6):
            for t in range(40):
                assert keyframe_schedule(t, S, k) == is_keyframe(t, S, k), (t, S, k)
    assert [t for t in range(12) if is_keyframe(t, 2, 3)] == [0, 1, 2, 5, 8, 11]
