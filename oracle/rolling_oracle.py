"""Plain fp64 CPU oracle of the rolling, diversity-pruned KV memory.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or execute
this module: only the tests and the benchmark's CPU-baseline leg use it.

What it follows ("InfiniteVGGT" explainer page, Building Blocks and the Step-by-step
recipe, with its concrete mini-example):

* Immutable anchor: every token of the first frame is kept forever, in every head.
* Rolling update, per layer and head: the candidates are the head's mutable cache plus
  the new frame's tokens; each candidate key is L2-normalised, the mean of the
  normalised candidate keys is the reference, and a candidate's diversity score is the
  negative cosine similarity of its key to that mean. The Top-K candidates by score are
  kept (K = the layer's per-head budget), the rest are discarded, so the memory stays
  bounded.
* Layer-wise adaptive budgets: each layer's average diversity, through a softmax with a
  temperature, gives the layer's share of the total budget.
* Attention of the current frame runs after the pruning, over the anchor and the kept
  tokens.

Readings taken where the page is silent (each is also listed in the design notes):
the fp64 evaluation order below (every sum over the dims -- the squares of a norm, the
terms of a dot product -- taken in blocks of 8 consecutive dims, ascending within a block,
then the block sums in ascending order; a key is normalised by multiplying it with the
correctly rounded reciprocal of its norm; every sum over candidates -- the
normalised keys for the mean, whose direction equals that of the sum, and the scores for
a head's total -- taken in blocks of 32 consecutive candidates in ascending token id,
ascending within a block, then the block sums in ascending block order); a zero key has
no direction and scores 0; ties are broken by the lower token
id; the kept tokens are stored in ascending id; pruning starts with the second frame;
the budget of layer l is floor(L * K * softmax(mean diversity / tau)_l), computed from
the previous frame's layer averages by the caller (the page gives neither the
temperature nor when budgets are recomputed).

Nothing here is pinned only to itself: tests/test_oracle_rolling.py checks it against
scipy's cosine distance and softmax, brute-force Top-K, the page's worked numbers and
closed-form cases.
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence

import numpy as np


CAND_BLOCK = 32          # candidates per block of every sum over candidates
DIM_BLOCK = 8            # dims per block of every sum over the dims


def dim_sum(terms: np.ndarray) -> np.ndarray:
    """Sum over the last axis in blocks of DIM_BLOCK entries: ascending within each block,
    then the block sums ascending. Every addition is one IEEE fp64 operation."""
    terms = np.asarray(terms, np.float64)
    D = terms.shape[-1]
    total = np.zeros(terms.shape[:-1])
    for d0 in range(0, D, DIM_BLOCK):
        part = np.zeros(terms.shape[:-1])
        for d in range(d0, min(d0 + DIM_BLOCK, D)):
            part = part + terms[..., d]
        total = total + part
    return total


def blocked_sum(x: np.ndarray) -> np.ndarray:
    """Sum over axis 0 in blocks of CAND_BLOCK rows: ascending within each block, then the
    block sums ascending. Every addition is one IEEE fp64 operation."""
    x = np.asarray(x, np.float64)
    total = np.zeros(x.shape[1:])
    for b0 in range(0, x.shape[0], CAND_BLOCK):
        part = np.zeros(x.shape[1:])
        for i in range(b0, min(b0 + CAND_BLOCK, x.shape[0])):
            part = part + x[i]
        total = total + part
    return total


def normalised_keys(Kc: np.ndarray) -> np.ndarray:
    """k_hat_i = k_i * RN(1 / |k_i|), |k_i| = sqrt of the dim_sum of the squares; a zero
    key gives k_hat = 0."""
    Kc = np.asarray(Kc, np.float64)
    N = Kc.shape[0]
    norms = np.sqrt(dim_sum(Kc * Kc))
    rcp = np.zeros(N)
    nz = norms > 0
    rcp[nz] = 1.0 / norms[nz]
    return Kc * rcp[:, None]


def diversity_scores(Kc: np.ndarray) -> np.ndarray:
    """Scores of one (layer, head)'s candidates. Kc: [N, D] keys in ascending token id.

    k_hat_i = k_i * (1 / |k_i|) (|k_i| = sqrt of the dim_sum of the squares, its
    reciprocal rounded once; a zero key gives k_hat = 0); mu = the blocked sum of the
    k_hat_i; score_i = -(k_hat_i . mu) / |mu| (dot and |mu|^2 as dim_sums of the products).
    Every step is one IEEE fp64 operation.
    """
    Kc = np.asarray(Kc, np.float64)
    N, D = Kc.shape
    khat = normalised_keys(Kc)
    mu = blocked_sum(khat) if N else np.zeros(D)
    mnorm = math.sqrt(float(dim_sum(mu * mu)))
    if mnorm == 0.0:
        return np.zeros(N)
    dot = dim_sum(khat * mu[None, :])
    return -(dot / mnorm)


def top_k(scores: np.ndarray, ids: np.ndarray, k: int) -> np.ndarray:
    """Indices (into the candidate arrays) of the k best candidates by (score descending,
    id ascending), returned in ascending id."""
    order = sorted(range(len(ids)), key=lambda i: (-scores[i], ids[i]))
    keep = order[: max(0, min(k, len(ids)))]
    return np.array(sorted(keep, key=lambda i: ids[i]), dtype=np.int64)


def layer_budgets(mean_diversity: Sequence[float], tau: float, k: int) -> List[int]:
    """Per-layer, per-head budgets floor(L * k * softmax(mean_diversity / tau)_l); tau <= 0
    gives every layer k."""
    L = len(mean_diversity)
    if tau <= 0:
        return [int(k)] * L
    z = np.asarray(mean_diversity, np.float64) / tau
    e = np.exp(z - z.max())
    p = e / e.sum()
    return [int(math.floor(L * k * float(pl))) for pl in p]


class RollingOracle:
    """Per layer: the anchor (frame 0, all heads) and, per head, the mutable kept set."""

    def __init__(self, num_layers: int, num_heads: int, head_dim: int, tokens_per_frame: int,
                 budget: int, softmax_scale: float):
        self.L, self.H, self.D, self.T = num_layers, num_heads, head_dim, tokens_per_frame
        self.budgets = [int(budget)] * num_layers
        self.scale = float(softmax_scale)
        self.reset()

    def reset(self):
        L, H, D = self.L, self.H, self.D
        self.anchor_ids = [np.zeros(0, np.int64) for _ in range(L)]
        self.anchor_k = [np.zeros((H, 0, D)) for _ in range(L)]
        self.anchor_v = [np.zeros((H, 0, D)) for _ in range(L)]
        self.mut_ids = [[np.zeros(0, np.int64) for _ in range(H)] for _ in range(L)]
        self.mut_k = [[np.zeros((0, D)) for _ in range(H)] for _ in range(L)]
        self.mut_v = [[np.zeros((0, D)) for _ in range(H)] for _ in range(L)]
        self.pending = [None] * L                 # (ids, K [T,H,D], V) of the frame appended last
        self.score_sum = [None] * L               # per head: fp64 sum of the last scores
        self.cand_count = [0] * L

    def set_budgets(self, budgets: Sequence[int]):
        self.budgets = [int(b) for b in budgets]

    def append(self, layer: int, t: int, K: np.ndarray, V: np.ndarray):
        K = np.asarray(K, np.float64)
        V = np.asarray(V, np.float64)
        ids = t * self.T + np.arange(self.T, dtype=np.int64)
        if t == 0:                                # the immutable anchor
            self.anchor_ids[layer] = ids
            self.anchor_k[layer] = np.transpose(K, (1, 0, 2)).copy()
            self.anchor_v[layer] = np.transpose(V, (1, 0, 2)).copy()
            self.pending[layer] = None
        else:
            self.pending[layer] = (ids, K, V)

    def prune(self, layer: int):
        """Score the candidates of every head and keep each head's Top-K."""
        pend = self.pending[layer]
        if pend is None:
            return
        ids_new, K, V = pend
        sums = []
        for h in range(self.H):
            ids = np.concatenate([self.mut_ids[layer][h], ids_new])
            Kc = np.concatenate([self.mut_k[layer][h], K[:, h, :]])
            Vc = np.concatenate([self.mut_v[layer][h], V[:, h, :]])
            sc = diversity_scores(Kc)
            sums.append(float(blocked_sum(sc[:, None])[0]))
            keep = top_k(sc, ids, self.budgets[layer])
            self.mut_ids[layer][h] = ids[keep]
            self.mut_k[layer][h] = Kc[keep]
            self.mut_v[layer][h] = Vc[keep]
            self.cand_count[layer] = len(ids)
        self.score_sum[layer] = sums
        self.pending[layer] = None

    def layer_diversity(self, layer: int) -> float:
        """Mean score over all heads' candidates of the layer's last pruning."""
        sums = self.score_sum[layer]
        tot = 0.0
        for s in sums:                            # heads ascending
            tot = tot + s
        return tot / float(self.H * self.cand_count[layer])

    def head_ids(self, layer: int, h: int) -> np.ndarray:
        """Token ids attended by head h (anchor, then the kept tokens), ascending."""
        return np.concatenate([self.anchor_ids[layer], self.mut_ids[layer][h]])

    def attend(self, layer: int, Q: np.ndarray, rows: Optional[Sequence[int]] = None) -> np.ndarray:
        """Prune, then fp64 attention of the frame's queries over anchor + kept, per head."""
        self.prune(layer)
        Q = np.asarray(Q, np.float64)
        rr = np.arange(Q.shape[0]) if rows is None else np.asarray(rows)
        out = np.zeros((len(rr), self.H, self.D))
        for h in range(self.H):
            Kh = np.concatenate([self.anchor_k[layer][h], self.mut_k[layer][h]])
            Vh = np.concatenate([self.anchor_v[layer][h], self.mut_v[layer][h]])
            z = (Q[rr, h, :] @ Kh.T) * self.scale
            z = z - z.max(axis=1, keepdims=True)
            p = np.exp(z)
            p = p / p.sum(axis=1, keepdims=True)
            out[:, h, :] = p @ Vh
        return out
