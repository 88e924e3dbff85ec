"""Plain fp64 CPU oracle of the streaming paged KV-cache hot path.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or execute
this module: only the tests, the smoke check and the benchmark's CPU-baseline leg
use it. It is deliberately slow and obvious: full attention matrices are
materialised, pages are Python dicts, and every quantity that decides an integer
(a rank, a tier, an FP8 code) is computed in the precision stated next to it.

What it follows (the web pages are cited by title and section):

* Frame-causal attention over a KV cache -- "How GCTStream Implements Streaming 3D
  Reconstruction with KV Cache" (GCTStream page), Frame-by-Frame Causal
  Processing; "InfiniteVGGT" explainer, Causal Attention sandwich. A frame's
  queries see the retained frames and the frame itself, with no mask inside.
* Paged storage and page-aligned append -- GCTStream page, AggregatorStream with
  Paged KV Cache; "Can LingBot-Map Achieve 20 FPS" (LingBot-Map performance
  page), Page-Aligned Tensor Layout. Each frame starts on a fresh page; the last
  page of a frame holds T mod P valid tokens.
* Sliding-window eviction with pinned scale frames -- LingBot-Map performance
  page, Sliding-Window Eviction Strategy (window 64, scale frames 8); GCTStream
  page, Sliding Window Eviction. Retained = first S committed frames plus the
  last W committed frames.
* Keyframe skip-append -- GCTStream page, Selective Frame Caching with Skip Append
  and Frame-by-Frame Causal Processing: a non-keyframe attends, then its K/V are
  discarded.
* Joint scale-frame phase -- GCTStream page, Scale-Frame Phase and the FAQ on the two
  phases: the first frames are processed together with bidirectional attention and
  share cache entries; the causal frame-by-frame phase follows.
* Cross-frame special tokens -- GCTStream page, Special Token Persistence: special
  tokens (camera / register) stay cached when their frame's other K/V are evicted.
* Reset -- GCTStream page, Cache Initialization and Cleanup.
* Cross-layer consistency scoring (CLCES) -- StreamCacheVGGT page, sections
  2.1.1 to 2.1.4: raw score = L2 norm of the FFN residual, ranks 0..N-1 over a
  window of W=5 layers, normalised rank r/(N-1), population variance against the
  uniform reference 1/12, Cons = max(0, 1 - sigma*sqrt(12)), enhanced score
  s_hat = s * (1 + lambda * Cons), rank history reset at each new frame.
* Keep / merge / drop tiers -- StreamCacheVGGT page, section 2 (core tokens kept,
  medium tokens merged into the core, lowest dropped); the page breaks off right after
  the heading of section 2.2 (hybrid compression, from dropping to merging), so tier
  sizes, the merge rule (count-weighted mean into the kept token with highest key
  cosine) and the protected set (frame 0 and the camera / register tokens) follow the
  budgeted-compression workload's statement.
* FP8 KV quantisation -- XStreamVGGT abstract (KV cache quantisation); the
  format is OCP FP8 E4M3 (bias 7, max finite 448, no infinities), one absmax
  scale per (page, head), separately for K and V. Its "dimension-adaptive" variant
  (the abstract's wording; KIVI, which it cites, quantises keys per channel and
  values per token) takes one absmax scale per (page, head, channel) for K and one
  per (page, head, token) for V.

Readings taken where the pages are silent (each is also listed in the design
notes): the order append -> attend -> commit/evict; lowest-free page allocation;
population variance; the raw score as the fp32 rounding of the exactly summed fp64 norm; ties broken by the
lower token id; protected tokens never absorb merges; merges applied
simultaneously from pre-merge values in ascending source id and rounded once to
bf16; the FP8 scale fp32(amax / 448) and codes RNE-satfinite of fp32(x / scale);
the joint phase appends its n <= S frames first, then all n*T queries attend over
all of them (no mask), then the n frames are committed; a frame's special tokens
are its first num_special_tokens tokens, and when a committed frame is evicted its
first ceil(ns / P) pages stay where they are in the page table, trimmed to those
tokens (other slots zero, page valid counts ns, P, ...), for at most
special_frames evicted frames, the oldest dropped first beyond that; a
non-keyframe is discarded whole.

Nothing here is pinned only to itself: tests/test_oracle_*.py check it against
brute force over explicitly concatenated frames, closed forms, library routines
and hand-derived format values.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Dict, List, Optional, Sequence

import numpy as np

# --------------------------------------------------------------------------------------
# Number formats
# --------------------------------------------------------------------------------------

BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127
E4M3_MAX = 448.0


def bf16_round(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value, ties to even (one rounding).

    bfloat16 keeps 8 significant bits; normals start at 2**-126 and subnormals have
    a fixed quantum of 2**-133. Results are returned as float64 holding bf16 values.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.array(x, copy=True)
    fin = np.isfinite(x) & (x != 0)
    xf = x[fin]
    _, e = np.frexp(xf)                       # |x| in [2**(e-1), 2**e)
    qe = np.maximum(e - 8, -133)              # quantum 2**(e-1-7), floor at the subnormal step
    y = np.ldexp(np.rint(np.ldexp(xf, -qe)), qe)
    y = np.where(np.abs(y) > BF16_MAX, np.copysign(np.inf, xf), y)
    out[fin] = y
    return out


def to_f32(x) -> np.ndarray:
    """Round float64 values to float32 (IEEE round-to-nearest-even), as float64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def e4m3_encode(x) -> np.ndarray:
    """OCP FP8 E4M3 code of each value: round to nearest even, saturate to +-448.

    E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; normals cover
    [2**-6, 448]; subnormals are m/8 * 2**-6; the all-ones pattern 0x7F/0xFF is NaN
    and there are no infinities. Inputs must be finite.
    """
    x = np.asarray(x, dtype=np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("e4m3_encode expects finite inputs")
    sign = np.signbit(x).astype(np.uint8)
    a = np.abs(x)
    _, e = np.frexp(a)
    unb = np.maximum(e - 1, -6)               # exponent of the binade, subnormal floor at -6
    q = np.ldexp(1.0, unb - 3)                # 3 mantissa bits
    r = np.rint(a / q) * q
    r = np.minimum(r, E4M3_MAX)               # satfinite
    _, e2 = np.frexp(r)
    unb2 = e2 - 1
    sub = r < 2.0 ** -6
    exp_field = np.where(sub, 0, unb2 + 7)
    mant = np.where(sub, r / 2.0 ** -9, (r / np.ldexp(1.0, unb2) - 1.0) * 8.0)
    code = (sign.astype(np.int64) << 7) | (exp_field.astype(np.int64) << 3) | mant.astype(np.int64)
    return code.astype(np.uint8)


def e4m3_decode(code) -> np.ndarray:
    """Value of each OCP FP8 E4M3 code, as float64 (NaN for 0x7F / 0xFF)."""
    c = np.asarray(code, dtype=np.int64)
    s = (c >> 7) & 1
    ef = (c >> 3) & 0xF
    mf = c & 7
    val = np.where(ef == 0, mf * 2.0 ** -9, (1.0 + mf / 8.0) * np.ldexp(1.0, ef - 7))
    val = np.where((ef == 15) & (mf == 7), np.nan, val)
    return np.where(s == 1, -val, val)


def fp8_quantise_block(x: np.ndarray):
    """Absmax FP8 quantisation of one (page, head) block of valid tokens.

    scale = fp32(amax / 448); code = E4M3_RNE_satfinite(fp32(x / scale)); an all-zero
    block has scale 0 and codes 0. The fp32 quotients are obtained by dividing in
    fp64 and rounding once to fp32, which equals the fp32 IEEE quotient because
    53 >= 2*24 + 2. Returns (codes uint8 like x, scale as float64, dequantised fp64).
    """
    x = np.asarray(x, dtype=np.float64)
    amax = float(np.max(np.abs(x))) if x.size else 0.0
    if amax == 0.0:
        return np.zeros(x.shape, np.uint8), 0.0, np.zeros(x.shape)
    scale = float(to_f32(amax / E4M3_MAX))
    qv = to_f32(x / scale)
    codes = e4m3_encode(qv)
    return codes, scale, e4m3_decode(codes) * scale


def fp8_quantise_channels(x: np.ndarray):
    """Dimension-adaptive FP8 of a K block [n, D] of valid tokens: each channel (column)
    quantised as its own block by fp8_quantise_block. Returns (codes [n, D], scales [D],
    dequantised fp64 [n, D])."""
    x = np.asarray(x, dtype=np.float64)
    n, D = x.shape
    codes = np.zeros((n, D), np.uint8)
    scales = np.zeros(D)
    deq = np.zeros((n, D))
    for d in range(D):
        codes[:, d], scales[d], deq[:, d] = fp8_quantise_block(x[:, d])
    return codes, scales, deq


def fp8_quantise_tokens(x: np.ndarray):
    """Dimension-adaptive FP8 of a V block [n, D] of valid tokens: each token (row)
    quantised as its own block by fp8_quantise_block. Returns (codes [n, D], scales [n],
    dequantised fp64 [n, D])."""
    x = np.asarray(x, dtype=np.float64)
    n, D = x.shape
    codes = np.zeros((n, D), np.uint8)
    scales = np.zeros(n)
    deq = np.zeros((n, D))
    for i in range(n):
        codes[i], scales[i], deq[i] = fp8_quantise_block(x[i])
    return codes, scales, deq


# --------------------------------------------------------------------------------------
# Cache configuration and state
# --------------------------------------------------------------------------------------

@dataclass
class OracleConfig:
    num_layers: int
    num_heads: int
    head_dim: int
    tokens_per_frame: int
    num_special_tokens: int
    page_size: int
    window_frames: int
    scale_frames: int
    kv_dtype: str                 # "f32" | "bf16" | "fp8_e4m3"
    softmax_scale: float          # used as its fp32 value
    budget_tokens: int = 0
    keep_frac: float = 0.6        # used as its fp32 value
    lam: float = 0.5              # used as its fp32 value
    rank_window: int = 5
    residual_dim: int = 1024
    protect_first_frame: int = 1
    special_frames: int = 0       # evicted frames whose special tokens stay (0: off)
    fp8_dim_adaptive: int = 0     # FP8: K scales per channel, V scales per token

    @staticmethod
    def from_workload(wl) -> "OracleConfig":
        return OracleConfig(
            num_layers=wl.num_layers, num_heads=wl.num_heads, head_dim=wl.head_dim,
            tokens_per_frame=wl.tokens_per_frame, num_special_tokens=wl.num_special_tokens,
            page_size=wl.page_size, window_frames=wl.window_frames, scale_frames=wl.scale_frames,
            kv_dtype=wl.kv_dtype, softmax_scale=wl.softmax_scale, budget_tokens=wl.budget_tokens,
            keep_frac=wl.keep_frac, lam=wl.lam, rank_window=wl.rank_window,
            residual_dim=wl.residual_dim, protect_first_frame=wl.protect_first_frame,
            special_frames=getattr(wl, "special_frames", 0),
            fp8_dim_adaptive=getattr(wl, "fp8_dim_adaptive", 0))


class _Page:
    """One physical page: P token slots x H heads x D dims, plus per-slot metadata."""

    def __init__(self, P, H, D):
        self.k = np.zeros((H, P, D))          # stored (dequantised) values, fp64
        self.v = np.zeros((H, P, D))
        self.k_codes = None                   # FP8 only: uint8 [H, P, D]
        self.v_codes = None
        self.k_scale = None                   # FP8 only: float64 [H] (the largest of the
        self.v_scale = None                   # channel / token scales when dimension-adaptive)
        self.k_chan_scale = None              # dimension-adaptive FP8: [H, D]
        self.v_tok_scale = None               # dimension-adaptive FP8: [H, P]
        self.ids = np.full(P, -1, np.int64)   # global token id = frame * T + slot
        self.counts = np.zeros(P, np.int64)   # merge counts (1 for an original token)
        self.shat = np.zeros(P, np.float64)   # enhanced score, fp32 value
        self.valid = 0


class _LayerState:
    def __init__(self):
        self.free_used: List[bool] = []       # page id -> in use
        self.pages: Dict[int, _Page] = {}
        # page table entries in cache order: [phys, owner, page_in_owner, valid]
        self.entries: List[List[int]] = []
        self.committed: List[int] = []        # committed frame ids in commit order
        self.retained: List[int] = []         # evicted frames whose special tokens stay
        self.pending: Optional[int] = None    # frame id appended but not yet committed
        self.pending_key: bool = False
        self.high_water = 0
        # per-frame CLCES rank history (reset at each new frame)
        self.hist_frame = -1


class StreamOracle:
    """Cache state for all layers of one stream, advanced one call at a time."""

    def __init__(self, cfg: OracleConfig):
        self.cfg = cfg
        self.layers = [_LayerState() for _ in range(cfg.num_layers)]
        self.P = cfg.page_size
        self.T = cfg.tokens_per_frame
        self.scale = float(np.float32(cfg.softmax_scale))
        # CLCES rank history of the current frame: layer -> ranks [T]
        self._rank_hist: Dict[int, np.ndarray] = {}
        self._rank_frame = -1
        self.last_merge: Dict[int, dict] = {}

    # ---------------------------------------------------------------- allocation
    def _alloc(self, L: _LayerState, n: int) -> List[int]:
        """The n lowest free physical page ids, ascending (reading: lowest free first)."""
        got = []
        pid = 0
        while len(got) < n:
            if pid >= len(L.free_used):
                L.free_used.append(False)
            if not L.free_used[pid]:
                got.append(pid)
            pid += 1
        for p in got:
            L.free_used[p] = True
            L.pages[p] = _Page(self.P, self.cfg.num_heads, self.cfg.head_dim)
        used = sum(L.free_used)
        L.high_water = max(L.high_water, used)
        return got

    def _free(self, L: _LayerState, pids: Sequence[int]):
        for p in pids:
            assert L.free_used[p]
            L.free_used[p] = False
            del L.pages[p]

    # ---------------------------------------------------------------- append
    def append(self, layer: int, t: int, K: np.ndarray, V: np.ndarray, is_key: bool):
        """Page-aligned append of frame t's K, V ([T, H, D], values of the I/O dtype)."""
        cfg, P, T = self.cfg, self.P, self.T
        L = self.layers[layer]
        if L.pending is not None:
            raise RuntimeError("append while a frame is pending")
        K = np.asarray(K, np.float64)
        V = np.asarray(V, np.float64)
        n_pages = -(-T // P)
        pids = self._alloc(L, n_pages)
        for g, pid in enumerate(pids):
            pg = L.pages[pid]
            lo, hi = g * P, min(T, (g + 1) * P)
            n = hi - lo
            pg.valid = n
            pg.ids[:n] = t * T + np.arange(lo, hi)
            pg.counts[:n] = 1
            kb = np.transpose(K[lo:hi], (1, 0, 2))   # [H, n, D]
            vb = np.transpose(V[lo:hi], (1, 0, 2))
            if cfg.kv_dtype == "fp8_e4m3":
                H = cfg.num_heads
                pg.k_codes = np.zeros((H, P, cfg.head_dim), np.uint8)
                pg.v_codes = np.zeros((H, P, cfg.head_dim), np.uint8)
                pg.k_scale = np.zeros(H)
                pg.v_scale = np.zeros(H)
                if cfg.fp8_dim_adaptive:
                    pg.k_chan_scale = np.zeros((H, cfg.head_dim))
                    pg.v_tok_scale = np.zeros((H, P))
                for h in range(H):
                    if cfg.fp8_dim_adaptive:
                        c, s, dq = fp8_quantise_channels(kb[h])
                        pg.k_codes[h, :n], pg.k_chan_scale[h], pg.k[h, :n] = c, s, dq
                        pg.k_scale[h] = s.max()
                        c, s, dq = fp8_quantise_tokens(vb[h])
                        pg.v_codes[h, :n], pg.v_tok_scale[h, :n], pg.v[h, :n] = c, s, dq
                        pg.v_scale[h] = s.max()
                        continue
                    c, s, dq = fp8_quantise_block(kb[h])
                    pg.k_codes[h, :n], pg.k_scale[h], pg.k[h, :n] = c, s, dq
                    c, s, dq = fp8_quantise_block(vb[h])
                    pg.v_codes[h, :n], pg.v_scale[h], pg.v[h, :n] = c, s, dq
            else:
                pg.k[:, :n] = kb
                pg.v[:, :n] = vb
            L.entries.append([pid, t, g, n])
        L.pending = t
        L.pending_key = bool(is_key)

    # ---------------------------------------------------------------- attention
    def gather(self, layer: int):
        """Stored K, V [N, H, D] and token ids [N] of the cache in page-table order."""
        L = self.layers[layer]
        ks, vs, ids = [], [], []
        for pid, _, _, n in L.entries:
            pg = L.pages[pid]
            ks.append(np.transpose(pg.k[:, :n], (1, 0, 2)))
            vs.append(np.transpose(pg.v[:, :n], (1, 0, 2)))
            ids.append(pg.ids[:n])
        H, D = self.cfg.num_heads, self.cfg.head_dim
        if not ks:
            return np.zeros((0, H, D)), np.zeros((0, H, D)), np.zeros(0, np.int64)
        return np.concatenate(ks), np.concatenate(vs), np.concatenate(ids)

    def attend(self, layer: int, Q: np.ndarray, rows: Optional[Sequence[int]] = None,
               commit: bool = True) -> np.ndarray:
        """O[i, h] = sum_j softmax_j(scale * q_i . k_j) v_j over every cached token.

        The full score matrix is formed per head in fp64; the row maximum is
        subtracted before exponentiation. Returns fp64 [len(rows), H, D]. With
        ``commit`` the keyframe commit / eviction (or the skip-append release)
        follows, as in the per-frame step.
        """
        Q = np.asarray(Q, np.float64)
        if rows is not None:
            Q = Q[np.asarray(rows)]
        Kc, Vc, _ = self.gather(layer)
        H = self.cfg.num_heads
        out = np.empty((Q.shape[0], H, self.cfg.head_dim))
        for h in range(H):
            z = self.scale * (Q[:, h, :] @ Kc[:, h, :].T)
            z = z - z.max(axis=1, keepdims=True)
            p = np.exp(z)
            p /= p.sum(axis=1, keepdims=True)
            out[:, h, :] = p @ Vc[:, h, :]
        if commit:
            self.commit(layer)
        return out

    # ---------------------------------------------------------------- commit / evict
    def commit(self, layer: int):
        """Keyframe: the pending frame joins the cache, then frames outside the first
        S and the last W committed frames are evicted. Non-keyframe: the pending
        frame's pages are released (skip-append)."""
        cfg = self.cfg
        L = self.layers[layer]
        t = L.pending
        if t is None:
            raise RuntimeError("commit without a pending frame")
        if L.pending_key:
            L.committed.append(t)
            if cfg.window_frames > 0:
                S, W = cfg.scale_frames, cfg.window_frames
                keep = set(L.committed[:S]) | set(L.committed[-W:])
                evict = [f for f in L.committed if f not in keep]
                if evict:
                    ev = set(evict)
                    L.committed = [f for f in L.committed if f not in ev]
                    if cfg.special_frames > 0:
                        for f in evict:
                            self._retain_special(L, f)
                        ev = set(evict) - set(L.retained)
                    self._free(L, [e[0] for e in L.entries if e[1] in ev])
                    L.entries = [e for e in L.entries if e[1] not in ev]
        else:
            self._free(L, [e[0] for e in L.entries if e[1] == t])
            L.entries = [e for e in L.entries if e[1] != t]
        L.pending = None

    def _retain_special(self, L: _LayerState, f: int):
        """Evicted frame f keeps its first ceil(ns / P) pages, trimmed to its special
        tokens (slots past them zeroed); its other pages are freed. Beyond special_frames
        retained frames the oldest is dropped whole."""
        cfg, P = self.cfg, self.P
        ns = min(cfg.num_special_tokens, self.T)
        keep_pages = -(-ns // P)
        drop = []
        for e in L.entries:
            if e[1] != f:
                continue
            if e[2] < keep_pages:
                n = min(P, ns - e[2] * P)
                pg = L.pages[e[0]]
                pg.k[:, n:] = 0.0
                pg.v[:, n:] = 0.0
                if pg.k_codes is not None:
                    pg.k_codes[:, n:] = 0
                    pg.v_codes[:, n:] = 0
                pg.ids[n:] = -1
                pg.counts[n:] = 0
                pg.valid = n
                e[3] = n
            else:
                drop.append(e[0])
        self._free(L, drop)
        L.entries = [e for e in L.entries if not (e[1] == f and e[2] >= keep_pages)]
        L.retained.append(f)
        while len(L.retained) > cfg.special_frames:
            old = L.retained.pop(0)
            self._free(L, [e[0] for e in L.entries if e[1] == old])
            L.entries = [e for e in L.entries if e[1] != old]

    # ---------------------------------------------------------------- joint scale-frame phase
    def scale_phase(self, layer: int, n: int, Q: np.ndarray, K: np.ndarray, V: np.ndarray,
                    rows: Optional[Sequence[int]] = None) -> np.ndarray:
        """The first n frames together: Q, K, V are [n*T, H, D] (frame-major). Frames
        0..n-1 are appended and committed, then all n*T queries attend over all of them
        with no mask. Returns fp64 [len(rows), H, D]."""
        L = self.layers[layer]
        if L.entries or L.committed or L.pending is not None:
            raise RuntimeError("the joint phase starts an empty layer")
        if not 1 <= n <= max(1, self.cfg.scale_frames):
            raise ValueError("the joint phase takes 1..scale_frames frames")
        T = self.T
        K = np.asarray(K, np.float64)
        V = np.asarray(V, np.float64)
        for f in range(n):
            self.append(layer, f, K[f * T:(f + 1) * T], V[f * T:(f + 1) * T], True)
            self.commit(layer)
        return self.attend_cache(layer, Q, rows)

    def attend_cache(self, layer: int, Q: np.ndarray, rows: Optional[Sequence[int]] = None) -> np.ndarray:
        """Attention of any number of queries over every cached token, nothing changed."""
        Q = np.asarray(Q, np.float64)
        if rows is not None:
            Q = Q[np.asarray(rows)]
        Kc, Vc, _ = self.gather(layer)
        H = self.cfg.num_heads
        out = np.empty((Q.shape[0], H, self.cfg.head_dim))
        for h in range(H):
            z = self.scale * (Q[:, h, :] @ Kc[:, h, :].T)
            z = z - z.max(axis=1, keepdims=True)
            p = np.exp(z)
            p /= p.sum(axis=1, keepdims=True)
            out[:, h, :] = p @ Vc[:, h, :]
        return out

    # ---------------------------------------------------------------- reset
    def reset(self):
        """Empty every layer's cache and history; the next frame starts fresh."""
        self.layers = [_LayerState() for _ in range(self.cfg.num_layers)]
        self._rank_hist = {}
        self._rank_frame = -1
        self.last_merge = {}

    # ---------------------------------------------------------------- reports
    def page_table(self, layer: int) -> np.ndarray:
        """Rows (owner, page_in_owner, phys_page, valid_tokens) in cache order; owner is
        the frame index, or -1 for pages written by compaction."""
        L = self.layers[layer]
        if not L.entries:
            return np.zeros((0, 4), np.int32)
        return np.array([[e[1], e[2], e[0], e[3]] for e in L.entries], np.int32)

    def pages_in_use(self, layer: int) -> int:
        return int(sum(self.layers[layer].free_used))

    def high_water(self, layer: int) -> int:
        return self.layers[layer].high_water

    def token_meta(self, layer: int):
        """(ids, counts, shat) of the cached tokens in page-table order."""
        L = self.layers[layer]
        ids, cnt, sh = [], [], []
        for pid, _, _, n in L.entries:
            pg = L.pages[pid]
            ids.append(pg.ids[:n]); cnt.append(pg.counts[:n]); sh.append(pg.shat[:n])
        if not ids:
            return np.zeros(0, np.int64), np.zeros(0, np.int64), np.zeros(0)
        return np.concatenate(ids), np.concatenate(cnt), np.concatenate(sh)

    def fp8_pages(self, layer: int):
        """FP8 codes [n, H, P, D] for K and V and scales [n, H] in page-table order."""
        L = self.layers[layer]
        kc = np.stack([L.pages[e[0]].k_codes for e in L.entries])
        vc = np.stack([L.pages[e[0]].v_codes for e in L.entries])
        ks = np.stack([L.pages[e[0]].k_scale for e in L.entries])
        vs = np.stack([L.pages[e[0]].v_scale for e in L.entries])
        return kc, vc, ks, vs

    def fp8_da_scales(self, layer: int):
        """Dimension-adaptive FP8 scales in page-table order: K [n, H, D], V [n, H, P]."""
        L = self.layers[layer]
        return (np.stack([L.pages[e[0]].k_chan_scale for e in L.entries]),
                np.stack([L.pages[e[0]].v_tok_scale for e in L.entries]))

    # ---------------------------------------------------------------- CLCES scoring
    def score(self, layer: int, t: int, residual: np.ndarray, s_choice: Optional[Dict[int, float]] = None) -> np.ndarray:
        """Enhanced importance s_hat of frame t's tokens at ``layer``.

        s_i: fp32 of sqrt(sum_c r_ic^2), the sum of the fp64 squares taken exactly and
        rounded once (math.fsum; the pages fix no summation order, and any order the GPU
        takes is allowed for in the tests by its error bound).
        R_i: rank of token i among the frame's T tokens, s descending, ties to the
        lower slot; history kept for the last n = min(W, number of layers scored
        this frame) layers and reset at each new frame. With N = T,
        D_i = n * sum R^2 - (sum R)^2 (exact integer), sigma_i = sqrt(D_i) / (n (N-1)),
        Cons_i = max(0, 1 - sigma_i sqrt(12)), s_hat_i = fp32(s_i (1 + lambda Cons_i)),
        each step one fp64 operation in this order. The scores are stored with the
        frame's tokens in the cache.

        s_choice (tests only) maps token slots to the other fp32 neighbour of the exact
        norm, for tokens whose rounding to fp32 another correct evaluation order may
        decide the other way; any other value is refused.
        """
        cfg = self.cfg
        r = np.asarray(residual, np.float64)
        T = r.shape[0]
        if t != self._rank_frame:
            self._rank_hist = {}
            self._rank_frame = t
        acc = np.array([math.fsum(row * row) for row in r])
        s = to_f32(np.sqrt(acc))
        for i, v in (s_choice or {}).items():
            f = np.float32(s[i])
            if float(v) not in (float(f), float(np.nextafter(f, np.float32(np.inf))),
                                float(np.nextafter(f, np.float32(-np.inf)))):
                raise ValueError(f"token {i}: {v} is not an fp32 neighbour of the norm")
            s[i] = float(v)
        order = sorted(range(T), key=lambda i: (-s[i], i))
        R = np.empty(T, np.int64)
        R[np.array(order)] = np.arange(T)
        self._rank_hist[layer] = R
        win = [l for l in range(layer - cfg.rank_window + 1, layer + 1) if l in self._rank_hist]
        n = len(win)
        Rs = np.stack([self._rank_hist[l] for l in win])          # [n, T]
        sum_r = [int(x) for x in Rs.sum(axis=0)]
        sum_r2 = [int(x) for x in (Rs * Rs).sum(axis=0)]
        lam = float(np.float32(cfg.lam))
        sqrt12 = math.sqrt(12.0)
        shat = np.empty(T)
        for i in range(T):
            Di = n * sum_r2[i] - sum_r[i] * sum_r[i]
            sigma = math.sqrt(float(Di)) / (float(n) * float(T - 1))
            cons = 1.0 - sigma * sqrt12
            if cons < 0.0:
                cons = 0.0
            shat[i] = float(np.float32(float(s[i]) * (1.0 + lam * cons)))
        # store with the frame's tokens
        L = self.layers[layer]
        for pid, owner, g, nv in L.entries:
            if owner == t:
                pg = L.pages[pid]
                pg.shat[:nv] = shat[g * self.P: g * self.P + nv]
        return shat

    # ---------------------------------------------------------------- compression
    def protected(self, ids: np.ndarray) -> np.ndarray:
        """Tokens that are always kept: every token of frame 0 (when enabled) and the
        camera / register tokens (slots 0..num_special-1) of every frame."""
        T = self.T
        frame = ids // T
        slot = ids % T
        prot = slot < self.cfg.num_special_tokens
        if self.cfg.protect_first_frame:
            prot |= frame == 0
        return prot

    # Two fp64 evaluations of one cosine of 1,024-dim keys (the dot product and the norms,
    # summed in any order) differ by at most about 2 * 1,028 * 2^-53 = 2.3e-13; targets
    # whose cosines are within COS_TIE of the best are ties that the order may decide.
    COS_TIE = 1e-12

    def compress(self, layer: int, target_choice: Optional[Dict[int, int]] = None):
        """Keep / merge / drop the committed cache of ``layer`` when it holds more than B
        tokens. Returns None when nothing happens, else a dict with the kept ids,
        the (source id, target id) merge pairs and the dropped ids.

        target_choice (tests only) maps merge-source ids to another side's target id; it is
        followed where that target's cosine ties the best within COS_TIE, and refused
        (ValueError) otherwise."""
        cfg, P = self.cfg, self.P
        L = self.layers[layer]
        if L.pending is not None:
            raise RuntimeError("compress while a frame is pending")
        B = cfg.budget_tokens
        ids, counts, shat = self.token_meta(layer)
        N = ids.size
        if B <= 0 or N <= B:
            return None
        n_keep = int(math.floor(float(np.float32(cfg.keep_frac)) * B))
        n_merge = B - n_keep
        prot = self.protected(ids)
        n_prot = int(prot.sum())
        if n_prot > n_keep:
            raise OverflowError("protected tokens exceed the keep tier")
        others = [i for i in range(N) if not prot[i]]
        others.sort(key=lambda i: (-shat[i], ids[i]))
        kept_other = others[: n_keep - n_prot]
        merged = others[n_keep - n_prot: n_keep - n_prot + n_merge]
        dropped = others[n_keep - n_prot + n_merge:]
        keep_pos = sorted([i for i in range(N) if prot[i]] + kept_other)
        Kc, Vc, _ = self.gather(layer)
        H, D = cfg.num_heads, cfg.head_dim
        Kf = Kc.reshape(N, H * D)
        Vf = Vc.reshape(N, H * D)
        eligible = sorted(kept_other)          # targets: kept tokens that are not protected
        targets = {}
        if eligible and merged:
            # cos(K_m, K_j) = K_m . K_j / (|K_j| |K_m|) for every (merge, eligible) pair, as
            # one matrix product; argmax takes the first maximum = the lowest id on ties
            E = Kf[eligible]
            En = np.sqrt((E * E).sum(axis=1))
            M = Kf[merged]
            Mn = np.sqrt((M * M).sum(axis=1))
            cos = (M @ E.T) / (En[None, :] * Mn[:, None])
            best = np.argmax(cos, axis=1)
            epos = {int(ids[j]): e for e, j in enumerate(eligible)}
            for r, m in enumerate(merged):
                b = int(best[r])
                if target_choice is not None and int(ids[m]) in target_choice:
                    alt = epos.get(int(target_choice[int(ids[m])]))
                    if alt is None or cos[r, alt] < cos[r, b] - self.COS_TIE:
                        raise ValueError(f"merge source {int(ids[m])}: target "
                                         f"{target_choice[int(ids[m])]} neither the best nor tied with it")
                    b = alt
                targets[m] = eligible[b]
        else:
            dropped = sorted(dropped + merged)
            merged = []
        # simultaneous count-weighted mean from pre-merge values, ascending source id
        newK, newV, newC = Kf.copy(), Vf.copy(), counts.copy()
        by_target: Dict[int, List[int]] = {}
        for m in sorted(merged, key=lambda i: ids[i]):
            by_target.setdefault(targets[m], []).append(m)
        for j, srcs in by_target.items():
            acck = counts[j] * Kf[j]
            accv = counts[j] * Vf[j]
            tot = int(counts[j])
            for m in srcs:
                acck = acck + counts[m] * Kf[m]
                accv = accv + counts[m] * Vf[m]
                tot += int(counts[m])
            newK[j] = bf16_round(acck / tot)
            newV[j] = bf16_round(accv / tot)
            newC[j] = tot
        # compaction: kept tokens in ascending id into the lowest free pages
        n_new = -(-len(keep_pos) // P)
        old = [e[0] for e in L.entries]
        pids = self._alloc(L, n_new)
        new_entries = []
        for g, pid in enumerate(pids):
            pg = L.pages[pid]
            sel = keep_pos[g * P: (g + 1) * P]
            n = len(sel)
            pg.valid = n
            pg.ids[:n] = ids[sel]
            pg.counts[:n] = newC[sel]
            pg.shat[:n] = shat[sel]
            pg.k[:, :n] = np.transpose(newK[sel].reshape(n, H, D), (1, 0, 2))
            pg.v[:, :n] = np.transpose(newV[sel].reshape(n, H, D), (1, 0, 2))
            new_entries.append([pid, -1, g, n])
        self._free(L, old)
        L.entries = new_entries
        L.committed = []
        res = dict(kept_ids=ids[keep_pos].copy(),
                   merge_src=np.array([ids[m] for m in sorted(merged, key=lambda i: ids[i])], np.int64),
                   merge_dst=np.array([ids[targets[m]] for m in sorted(merged, key=lambda i: ids[i])],
                                      np.int64),
                   dropped_ids=np.array(sorted(ids[dropped]), np.int64),
                   n_protected=n_prot)
        self.last_merge[layer] = res
        return res


def is_keyframe(t: int, scale_frames: int, keyframe_interval: int) -> bool:
    """First S frames, then every k-th frame from frame S on."""
    k = max(1, int(keyframe_interval))
    return t < scale_frames or ((t - scale_frames) % k) == 0
