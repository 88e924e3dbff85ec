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

Readings taken where the page is silent (each is also listed in the design notes): a
candidate's score is the plain definition, -cos(k_i, mu) = -(k_i . mu) / (|k_i| |mu|) with
mu the mean of the normalised candidate keys k_i / |k_i|, evaluated in fp64 by numpy in
whatever order its routines take (the page fixes no order; the GPU tests allow for the
rounding of any order by a bound derived from the sums' lengths); a zero key has no
direction and scores 0, and so does every candidate when mu = 0; ties are broken by the
lower token id; the kept tokens are stored in ascending id; pruning starts with the second
frame; the budget of layer l is floor(L * K * softmax(mean diversity / tau)_l), the mean
diversity being the mean score over all heads' candidates of the layer's last pruning (the
page gives neither the temperature nor when budgets are recomputed).

Nothing here is pinned only to itself: tests/test_oracle_rolling.py checks it against
scipy's cosine distance and softmax, brute-force Top-K, the page's worked numbers and
closed-form cases.
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence

import numpy as np


def normalised_keys(Kc: np.ndarray) -> np.ndarray:
    """k_hat_i = k_i / |k_i|; a zero key has no direction and gives k_hat = 0."""
    Kc = np.asarray(Kc, np.float64)
    norms = np.linalg.norm(Kc, axis=1)
    out = np.zeros_like(Kc)
    nz = norms > 0
    out[nz] = Kc[nz] / norms[nz, None]
    return out


def diversity_scores(Kc: np.ndarray) -> np.ndarray:
    """Scores of one (layer, head)'s candidates. Kc: [N, D] keys in ascending token id.

    mu = the mean of the normalised candidate keys; score_i = -cos(k_i, mu)
    = -(k_i . mu) / (|k_i| |mu|). A zero key scores 0; every score is 0 when mu = 0.
    """
    Kc = np.asarray(Kc, np.float64)
    N, D = Kc.shape
    if N == 0:
        return np.zeros(0)
    mu = normalised_keys(Kc).mean(axis=0)
    mnorm = float(np.linalg.norm(mu))
    if mnorm == 0.0:
        return np.zeros(N)
    knorm = np.linalg.norm(Kc, axis=1)
    out = np.zeros(N)
    nz = knorm > 0
    out[nz] = -((Kc[nz] @ mu) / (knorm[nz] * mnorm))
    return out


def top_k(scores: np.ndarray, ids: np.ndarray, k: int) -> np.ndarray:
    """Indices (into the candidate arrays) of the k best candidates by (score descending,
    id ascending), returned in ascending id."""
    order = sorted(range(len(ids)), key=lambda i: (-scores[i], ids[i]))
    keep = order[: max(0, min(k, len(ids)))]
    return np.array(sorted(keep, key=lambda i: ids[i]), dtype=np.int64)


def layer_budgets(mean_diversity: Sequence[float], tau: float, k: int, lo: Optional[int] = None,
                  hi: Optional[int] = None) -> List[int]:
    """Per-layer, per-head budgets floor(L * k * softmax(mean_diversity / tau)_l); tau <= 0
    gives every layer k. With lo / hi each budget is clamped to [lo, hi] (reading: a layer
    keeps at least one token and no more than its pool holds; the page states no bound)."""
    L = len(mean_diversity)
    if tau <= 0:
        b = [int(k)] * L
    else:
        z = np.asarray(mean_diversity, np.float64) / tau
        e = np.exp(z - z.max())
        p = e / e.sum()
        b = [int(math.floor(L * k * float(pl))) for pl in p]
    if lo is not None:
        b = [max(int(lo), x) for x in b]
    if hi is not None:
        b = [min(int(hi), x) for x in b]
    return b


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
        self.last_scores = [None] * L             # per head: scores of the last pruning's candidates
        self.last_cands = [None] * L              # per head: (ids, K, V) of those candidates

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
        scores, cands = [], []
        for h in range(self.H):
            ids = np.concatenate([self.mut_ids[layer][h], ids_new])
            Kc = np.concatenate([self.mut_k[layer][h], K[:, h, :]])
            Vc = np.concatenate([self.mut_v[layer][h], V[:, h, :]])
            sc = diversity_scores(Kc)
            scores.append(sc)
            cands.append((ids, Kc, Vc))
            keep = top_k(sc, ids, self.budgets[layer])
            self.mut_ids[layer][h] = ids[keep]
            self.mut_k[layer][h] = Kc[keep]
            self.mut_v[layer][h] = Vc[keep]
        self.last_scores[layer] = scores
        self.last_cands[layer] = cands
        self.pending[layer] = None

    def set_kept(self, layer: int, h: int, kept_ids: Sequence[int]):
        """Make head h keep `kept_ids` out of its last pruning's candidates instead of its
        own Top-K. Tests use this where the Top-K is not unique within the rounding of the
        scores: the other side's choice among the tied candidates is then followed."""
        ids, Kc, Vc = self.last_cands[layer][h]
        pos = {int(x): i for i, x in enumerate(ids)}
        sel = sorted(pos[int(x)] for x in kept_ids)
        self.mut_ids[layer][h] = ids[sel]
        self.mut_k[layer][h] = Kc[sel]
        self.mut_v[layer][h] = Vc[sel]

    def layer_diversity(self, layer: int) -> float:
        """Mean score over all heads' candidates of the layer's last pruning."""
        return float(np.mean(np.concatenate(self.last_scores[layer])))

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
