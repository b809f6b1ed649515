"""Plain fp64 CPU oracle for the MoBA gate variant that also routes the top
blocks by max- and min-pooled keys.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import or call this
module: only ``tests/`` uses it.  It shares no code with the CUDA path.

Source: the paperhub.cn OpenReview discussion page of "MoBA: Mixture of Block
Attention for Long-Context LLMs", the authors' rebuttals to the reviewers' W1
(block representation, and the comparison with QUEST): besides the blocks the
mean-pooling gate selects, the ablation also selects the top blocks in terms of
max pooling and of min pooling, and reports a small but consistent LM-loss
improvement.  The page gives no formula.  Reading G1 (the plainest one the
rest supports): with the channel-wise maximum and minimum of a block's keys,
K^max_j[e] = max_u K[u, e] and K^min_j[e] = min_u K[u, e] over the block's
rows, a query at position t (current block c) attends
    the top (topk - 1) earlier blocks by <q, mean K_j>        (the MoBA gate)
  U the top `extra` earlier blocks by <q, K^max_j>
  U the top `extra` earlier blocks by <q, K^min_j>
  U {c},
every ranking over the candidates j < c with ties to the lower block index
(reading C4), and softmax attention over the union (the current block causal),
as in the plain gate.  With extra = 0 this is the plain MoBA gate.  The number
of attended blocks per row is variable: between min(topk, c + 1) and
min(topk + 2 extra, c + 1).
"""
from __future__ import annotations

from typing import List

import numpy as np

from .moba_oracle import _f64, attend_row, block_range, key_positions, mean_pool, num_blocks, select_blocks

__all__ = ["max_pool", "min_pool", "select_blocks_pooled", "moba_pooled_layer"]


def max_pool(K, B: int) -> np.ndarray:
    """K: [N, d] keys of one kv head -> [n, d], the channel-wise max of each block's rows."""
    K = _f64(K)
    N = K.shape[0]
    return np.stack([K[s:e].max(axis=0) for s, e in (block_range(j, N, B) for j in range(num_blocks(N, B)))])


def min_pool(K, B: int) -> np.ndarray:
    """K: [N, d] -> [n, d], the channel-wise min of each block's rows."""
    K = _f64(K)
    N = K.shape[0]
    return np.stack([K[s:e].min(axis=0) for s, e in (block_range(j, N, B) for j in range(num_blocks(N, B)))])


def _top(scores: np.ndarray, c: int, m: int) -> List[int]:
    """The first m of the candidates j < c ordered by (-score, j)."""
    return sorted(range(c), key=lambda j: (-float(scores[j]), j))[:m]


def select_blocks_pooled(q_row, kbar, kmax, kmin, t: int, B: int, topk: int, extra: int) -> List[int]:
    """Ascending blocks attended by the query at position t (reading G1)."""
    q = _f64(q_row)
    c = t // B
    base, _ = select_blocks(_f64(kbar) @ q, t, B, topk)      # top (topk-1) by mean, plus c
    chosen = set(base)
    chosen.update(_top(_f64(kmax) @ q, c, extra))
    chosen.update(_top(_f64(kmin) @ q, c, extra))
    return sorted(chosen)


def moba_pooled_layer(q, k, v, B: int, topk: int, extra: int, scale: float):
    """Whole layer with the pooled-gate variant: q [b,N,Hq,d], k/v [b,N,Hkv,d]
    -> (out [b,N,Hq,d], lse [b,Hq,N], sel list per (b, t, h))."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    b, N, Hq, d = q.shape
    G = Hq // k.shape[2]
    out = np.zeros((b, N, Hq, d))
    lse = np.zeros((b, Hq, N))
    sels = {}
    for bb in range(b):
        pools = [(mean_pool(k[bb, :, g], B), max_pool(k[bb, :, g], B), min_pool(k[bb, :, g], B))
                 for g in range(k.shape[2])]
        for h in range(Hq):
            g = h // G
            kbar, kmax, kmin = pools[g]
            for t in range(N):
                sel = select_blocks_pooled(q[bb, t, h], kbar, kmax, kmin, t, B, topk, extra)
                sels[(bb, t, h)] = sel
                pos = key_positions(sel, t, B, N)
                out[bb, t, h], lse[bb, h, t] = attend_row(q[bb, t, h], k[bb, pos, g], v[bb, pos, g], scale)
    return out, lse, sels
