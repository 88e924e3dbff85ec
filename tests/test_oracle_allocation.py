"""Pins of the oracle's physical page allocation (reading: the lowest free page ids, in
ascending order, for a new frame and for the block that compaction writes), with the
expected ids worked out by hand for a small window stream that evicts and reuses freed
pages and a skip-append frame, and for a budget stream that compacts twice. Allocation
orders that the reading excludes (highest free id first, never reusing a freed id) are
planted in the oracle and must fail these pins.

Pages: "Can LingBot-Map Achieve 20 FPS ...", Page-Aligned Tensor Layout (a frame's K/V
written into page-aligned storage); "How GCTStream ...", Sliding Window Eviction."""
import numpy as np
import pytest
import torch
from hypothesis import given, settings, strategies as st

from kvc_streams import WORKLOADS, FrameStream
from oracle import OracleConfig, StreamOracle
from oracle.kvcache_oracle import _Page


def _np(x):
    return x.to(torch.float64).numpy()


# T = 20, P = 8: a frame takes 3 pages (8, 8 and 4 valid slots). S = 1, W = 2.
# Keyframe flags per frame; frame 4 is a non-keyframe (attends, then its pages are freed).
WINDOW_KEYS = [True, True, True, True, False, True, True]
# Page table after each frame's step, rows (owner frame, page in frame, physical page, valid),
# derived by hand:
#   f0 -> pages 0,1,2; f1 -> 3,4,5; f2 -> 6,7,8 (3 committed = S + W, nothing evicted);
#   f3 -> 9,10,11, then f1 leaves the window: 3,4,5 free;
#   f4 -> 3,4,5 (lowest free), released after attending: 3,4,5 free again;
#   f5 -> 3,4,5, then f2 leaves: 6,7,8 free; f6 -> 6,7,8, then f3 leaves: 9,10,11 free.
def _frame_rows(f, phys):
    return [[f, 0, phys[0], 8], [f, 1, phys[1], 8], [f, 2, phys[2], 4]]


WINDOW_TABLES = [
    _frame_rows(0, [0, 1, 2]),
    _frame_rows(0, [0, 1, 2]) + _frame_rows(1, [3, 4, 5]),
    _frame_rows(0, [0, 1, 2]) + _frame_rows(1, [3, 4, 5]) + _frame_rows(2, [6, 7, 8]),
    _frame_rows(0, [0, 1, 2]) + _frame_rows(2, [6, 7, 8]) + _frame_rows(3, [9, 10, 11]),
    _frame_rows(0, [0, 1, 2]) + _frame_rows(2, [6, 7, 8]) + _frame_rows(3, [9, 10, 11]),
    _frame_rows(0, [0, 1, 2]) + _frame_rows(3, [9, 10, 11]) + _frame_rows(5, [3, 4, 5]),
    _frame_rows(0, [0, 1, 2]) + _frame_rows(5, [3, 4, 5]) + _frame_rows(6, [6, 7, 8]),
]
# the table while frame 4 (skip-append) is pending, before its release
PENDING_F4 = _frame_rows(0, [0, 1, 2]) + _frame_rows(2, [6, 7, 8]) + _frame_rows(3, [9, 10, 11]) + \
    _frame_rows(4, [3, 4, 5])


def _window_check():
    wl = WORKLOADS["tiny_f32"].replace(tokens_per_frame=20, page_size=8, window_frames=2, scale_frames=1)
    st = FrameStream(wl, seed=4, device="cpu")
    orc = StreamOracle(OracleConfig.from_workload(wl))
    for t, key in enumerate(WINDOW_KEYS):
        q, k, v = (_np(x) for x in st.frame(0, t))
        orc.append(0, t, k, v, key)
        if t == 4:
            assert orc.page_table(0).tolist() == PENDING_F4
        orc.attend(0, q)
        assert orc.page_table(0).tolist() == WINDOW_TABLES[t], t
    assert orc.high_water(0) == 12


# Budget stream: T = 8, P = 4 (2 pages per frame), one special token per frame, frame 0
# protected, B = 20: the keep tier is floor(0.6 * 20) = 12 tokens = 3 pages.
#   f0 -> 0,1; f1 -> 2,3; f2 -> 4,5: 24 > 20 tokens, compaction into the lowest free pages
#     6,7,8, then 0..5 free;  f3 -> 0,1 (20 tokens, no compaction);
#   f4 -> 2,3: 28 > 20, compaction into the lowest free 4,5,9, then 0,1,2,3,6,7,8 free;
#   f5 -> 0,1.
BLOCK = lambda phys: [[-1, g, p, 4] for g, p in enumerate(phys)]
BUDGET_TABLES = [
    [[0, 0, 0, 4], [0, 1, 1, 4]],
    [[0, 0, 0, 4], [0, 1, 1, 4], [1, 0, 2, 4], [1, 1, 3, 4]],
    BLOCK([6, 7, 8]),
    BLOCK([6, 7, 8]) + [[3, 0, 0, 4], [3, 1, 1, 4]],
    BLOCK([4, 5, 9]),
    BLOCK([4, 5, 9]) + [[5, 0, 0, 4], [5, 1, 1, 4]],
]


def _budget_check():
    wl = WORKLOADS["vggt_budget_16k"].replace(tokens_per_frame=8, num_special_tokens=1, num_heads=2, head_dim=4,
                                              page_size=4, budget_tokens=20, num_layers=1, residual_dim=16)
    st = FrameStream(wl, seed=5)
    orc = StreamOracle(OracleConfig.from_workload(wl))
    events = []
    for t in range(len(BUDGET_TABLES)):
        q, k, v = (_np(x) for x in st.frame(0, t))
        orc.append(0, t, k, v, True)
        orc.attend(0, q)
        orc.score(0, t, _np(st.residual(0, t)))
        events.append(orc.compress(0) is not None)
        assert orc.page_table(0).tolist() == BUDGET_TABLES[t], t
    assert events == [False, False, True, False, True, False]


def test_window_stream_lowest_free_pages_by_hand():
    _window_check()


def test_compaction_takes_lowest_free_pages_by_hand():
    _budget_check()


# ------------------------------------------------------------------ planted mistakes

def _highest_free(self, L, n):
    """Highest free ids of a fixed pool of 12 pages first."""
    got = [p for p in range(11, -1, -1) if p >= len(L.free_used) or not L.free_used[p]][:n]
    while len(L.free_used) < 12:
        L.free_used.append(False)
    for p in got:
        L.free_used[p] = True
        L.pages[p] = _Page(self.P, self.cfg.num_heads, self.cfg.head_dim)
    L.high_water = max(L.high_water, sum(L.free_used))
    return sorted(got)


def _never_reuse(self, L, n):
    """Fresh ids past every id handed out before, freed or not."""
    start = len(L.free_used)
    got = list(range(start, start + n))
    L.free_used.extend([True] * n)
    for p in got:
        L.pages[p] = _Page(self.P, self.cfg.num_heads, self.cfg.head_dim)
    L.high_water = max(L.high_water, sum(L.free_used))
    return got


@pytest.mark.parametrize("planted", [_highest_free, _never_reuse])
def test_planted_allocation_orders_are_caught(monkeypatch, planted):
    monkeypatch.setattr(StreamOracle, "_alloc", planted)
    with pytest.raises(AssertionError):
        _window_check()


def test_planted_never_reuse_is_caught_by_compaction(monkeypatch):
    monkeypatch.setattr(StreamOracle, "_alloc", _never_reuse)
    with pytest.raises(AssertionError):
        _budget_check()


def _window_model(T, P, S, W, keys):
    """Page tables of a window stream by a direct model of the reading: a frame takes the
    ppf lowest free ids; a committed keyframe keeps the first S and last W committed
    frames and frees the others' pages; a non-keyframe frees its own after attending."""
    ppf = -(-T // P)
    valid = [P] * (ppf - 1) + [T - (ppf - 1) * P]
    free, committed, tables = set(range(10 ** 4)), [], []
    for t, key in enumerate(keys):
        phys = sorted(free)[:ppf]
        free -= set(phys)
        if key:
            committed.append((t, phys))
            keep = committed[:S] + [c for c in committed[-W:] if c not in committed[:S]]
            for c in committed:
                if c not in keep:
                    free |= set(c[1])
            committed = [c for c in committed if c in keep]
        else:
            free |= set(phys)
        tables.append([[f, g, ph[g], valid[g]] for f, ph in sorted(committed) for g in range(ppf)])
    return tables


@settings(max_examples=25, deadline=None, derandomize=True)
@given(T=st.integers(1, 30), P=st.sampled_from([1, 2, 4, 8, 16]), S=st.integers(0, 3), W=st.integers(1, 4),
       keys=st.lists(st.booleans(), min_size=1, max_size=14))
def test_window_stream_pages_match_a_direct_model(T, P, S, W, keys):
    """The oracle's page tables over window streams with random keyframe flags (frames
    that evict, free pages that are reused, skip-append frames) against the direct model
    of the lowest-free reading."""
    wl = WORKLOADS["tiny_f32"].replace(tokens_per_frame=T, page_size=P, window_frames=W, scale_frames=S,
                                       num_heads=1, head_dim=4)
    st_ = FrameStream(wl, seed=T + 100 * P, device="cpu")
    orc = StreamOracle(OracleConfig.from_workload(wl))
    want = _window_model(T, P, S, W, keys)
    for t, key in enumerate(keys):
        q, k, v = (_np(x) for x in st_.frame(0, t))
        orc.append(0, t, k, v, key)
        orc.attend(0, q)
        assert orc.page_table(0).tolist() == want[t], t
