"""Plain fp64 CPU oracle for MoBA causal prefill.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import or call this
module: only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it.  It shares no code with the
CUDA path.

Source of every step: "MoBA: Mixture of Block Attention for Long-Context LLMs"
(arXiv 2502.13189), as restated on the paper-graph summary page (cited below as
[summary], with its section names), the OpenReview discussion page ([review])
and the research-hub concept note ([note]).

Readings taken where the pages are silent or disagree (each is listed in the
design notes of the repository):
  C1  ``topk`` counts the always-selected current block: a query attends to its
      current block plus the top (topk-1) earlier blocks.
  C2  blocks are 0-indexed here; the candidates of a query at position t are the
      blocks strictly before its own block c = t // B.
  C3  with fewer than topk-1 candidates, all of them are selected.
  C4  equal scores: the lower block index wins.
  C5  the gate score is unscaled <q, mean K>; attention logits are scale*<q,k>.
  C6  GQA: query head h reads kv head h // (Hq/Hkv).
  C7  a ragged last block is pooled over its actual rows.
  C10 lse is the natural-log log-sum-exp of the attention logits.

Everything is computed in float64 from the (already rounded) inputs.
Two independent formulations are provided: a per-row gather formulation
(``moba_row`` / ``attend_row``) and a dense boolean-mask formulation
(``moba_dense``); tests check that they agree.
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "num_blocks", "block_range", "mean_pool", "gate_scores", "select_blocks",
    "key_positions", "attend_row", "moba_row", "moba_dense", "merge_partials",
    "algorithmic_pairs",
]


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):          # a torch tensor (bf16 is widened exactly)
        import torch
        x = x.detach().to("cpu")
        if x.dtype == torch.bfloat16 or x.dtype == torch.float16:
            x = x.to(torch.float32)
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# Context partitioning  ([summary] §3 "Context Partitioning": B = N/n and
# I_i = [(i-1)B+1, iB], 1-indexed; here 0-indexed and half-open)
# ---------------------------------------------------------------------------
def num_blocks(N: int, B: int) -> int:
    return (N + B - 1) // B


def block_range(j: int, N: int, B: int) -> Tuple[int, int]:
    """Positions [start, end) of block j (the last block may be shorter, C7)."""
    return j * B, min(N, (j + 1) * B)


# ---------------------------------------------------------------------------
# Block mean-pool  ([summary] §3 "Affinity Scoring": mean_pool(K[I_i]);
# Algorithm 1 Step 1: pooled keys of shape n x h x d, computed once per layer)
# ---------------------------------------------------------------------------
def mean_pool(K, B: int) -> np.ndarray:
    """K: [N, d] keys of one kv head -> [n, d], the mean of each block's rows."""
    N = K.shape[0]
    n = num_blocks(N, B)
    out = np.empty((n, K.shape[1]), dtype=np.float64)
    for j in range(n):
        s, e = block_range(j, N, B)
        out[j] = _f64(K[s:e]).mean(axis=0)
    return out


# ---------------------------------------------------------------------------
# Affinity scores  ([summary] §3 "Affinity Scoring": s_i = <q, mean_pool(K[I_i])>;
# [note] "Key math": same, no softmax scale in the gate, reading C5)
# ---------------------------------------------------------------------------
def gate_scores(q_row, kbar) -> np.ndarray:
    return _f64(kbar) @ _f64(q_row)


# ---------------------------------------------------------------------------
# Causal top-k gate  ([summary] §3 "Top-k Gating" (g_i = 1 iff s_i in Topk),
# "Current block attention" (the query's own block is always routed, as a
# shared expert) and §3 "Causality Enforcement" mechanism 1 (future blocks get
# s = -inf and g = 0); readings C1-C4)
# ---------------------------------------------------------------------------
def select_blocks(scores: Sequence[float], t: int, B: int, topk: int) -> Tuple[List[int], Optional[float]]:
    """Blocks selected by the query at position t, ascending, and the score gap.

    ``scores[j]`` is the gate score of block j.  Only j < c = t // B are
    candidates.  The top (topk-1) candidates by (-score, j) are kept and the
    current block c is added.  ``gap`` is (last selected score) - (first
    unselected score) among candidates; it is None when every candidate is
    selected (c <= topk-1), since then the selection is not a choice.
    """
    c = t // B
    cand = sorted(range(c), key=lambda j: (-float(scores[j]), j))
    m = min(topk - 1, c)
    chosen = cand[:m]
    gap = None
    if c > m:
        gap = float(scores[cand[m - 1]]) - float(scores[cand[m]]) if m > 0 else None
    return sorted(chosen + [c]), gap


# ---------------------------------------------------------------------------
# Attended positions  ([summary] §3 "Top-k Gating": I = union of selected
# blocks; §3 "Causality Enforcement" mechanism 2: causal mask inside the
# current block; Algorithm 1 Step 3: current block causal, history non-causal)
# ---------------------------------------------------------------------------
def key_positions(sel: Sequence[int], t: int, B: int, N: int) -> np.ndarray:
    c = t // B
    parts = []
    for j in sel:
        s, e = block_range(j, N, B)
        if j == c:
            e = t + 1
        parts.append(np.arange(s, e, dtype=np.int64))
    return np.concatenate(parts)


# ---------------------------------------------------------------------------
# Attention over a key set  ([summary] §3 "The Core MoBA Attention Equation":
# MoBA(q,K,V) = Softmax(q K[I]^T) V[I], with the softmax scale of reading C5)
# ---------------------------------------------------------------------------
def attend_row(q_row, Ksel, Vsel, scale: float) -> Tuple[np.ndarray, float]:
    """Returns (out [d], lse) for one query over gathered keys/values."""
    z = scale * (_f64(Ksel) @ _f64(q_row))
    m = z.max()
    w = np.exp(z - m)
    den = w.sum()
    out = (w @ _f64(Vsel)) / den
    return out, float(m + math.log(den))


def moba_row(q_row, K, V, kbar, t: int, B: int, topk: int, scale: float):
    """One query row by the gather formulation.

    q_row [d]; K, V [N, d] for the row's kv head; kbar [n, d] = mean_pool(K, B).
    Returns (out [d], lse, sel list, gap)."""
    N = K.shape[0]
    s = gate_scores(q_row, kbar)
    sel, gap = select_blocks(s, t, B, topk)
    pos = key_positions(sel, t, B, N)
    out, lse = attend_row(q_row, _f64(K[pos]), _f64(V[pos]), scale)
    return out, lse, sel, gap


# ---------------------------------------------------------------------------
# Dense-mask formulation (second, independent formulation of the same
# definition): a boolean N x N mask M[t,u] = (block(u) selected by t) and
# (u <= t), then masked softmax attention.
# ---------------------------------------------------------------------------
def moba_dense(q, k, v, B: int, topk: int, scale: float):
    """Whole layer.  q [b,N,Hq,d], k/v [b,N,Hkv,d] -> (out [b,N,Hq,d],
    lse [b,Hq,N], sel [b,N,Hq,topk] ascending and -1 padded, gap [b,N,Hq] with
    NaN where undefined).  For small N only (N x N matrices per head)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    b, N, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    n = num_blocks(N, B)
    out = np.zeros((b, N, Hq, d))
    lse = np.zeros((b, Hq, N))
    sel_out = np.full((b, N, Hq, topk), -1, dtype=np.int64)
    gap_out = np.full((b, N, Hq), np.nan)
    t_idx = np.arange(N)
    cur = t_idx // B
    blk_of = np.arange(N) // B
    for bb in range(b):
        for g in range(Hkv):
            kbar = np.stack([k[bb, s:e, g].mean(axis=0)
                             for s, e in (block_range(j, N, B) for j in range(n))])
            for hh in range(G):
                h = g * G + hh
                Q = q[bb, :, h]                                 # [N, d]
                S = Q @ kbar.T                                  # [N, n] unscaled
                cand_mask = np.arange(n)[None, :] < cur[:, None]
                Sm = np.where(cand_mask, S, -np.inf)
                order = np.argsort(-Sm, axis=1, kind="stable")  # ties: lower j first
                m = np.minimum(topk - 1, cur)                   # selected per row
                G_mask = np.zeros((N, n), dtype=bool)
                rank = np.empty_like(order)
                np.put_along_axis(rank, order, np.arange(n)[None, :].repeat(N, 0), axis=1)
                G_mask |= (rank < m[:, None]) & cand_mask
                G_mask[t_idx, cur] = True
                # gap where more candidates than selections
                srt = np.take_along_axis(Sm, order, axis=1)
                has_gap = (cur > m) & (m > 0)
                rows = np.nonzero(has_gap)[0]
                gap_out[bb, rows, h] = srt[rows, m[rows] - 1] - srt[rows, m[rows]]
                for t in range(N):
                    js = np.nonzero(G_mask[t])[0]
                    sel_out[bb, t, h, :len(js)] = js
                # token-level mask
                M = G_mask[:, blk_of] & (t_idx[None, :] <= t_idx[:, None])
                Z = scale * (Q @ k[bb, :, g].T)
                Z = np.where(M, Z, -np.inf)
                zmax = Z.max(axis=1, keepdims=True)
                W = np.exp(Z - zmax)
                den = W.sum(axis=1, keepdims=True)
                out[bb, :, h] = (W @ v[bb, :, g]) / den
                lse[bb, h] = (zmax + np.log(den))[:, 0]
    return out, lse, sel_out, gap_out


# ---------------------------------------------------------------------------
# Online-softmax merge of partial results ([summary] §3 Implementation,
# Step 4: partial outputs are combined by rescaling with their normalisers;
# Milakov & Gimelshein 2018)
# ---------------------------------------------------------------------------
def merge_partials(parts: Sequence[Tuple[np.ndarray, float]]) -> Tuple[np.ndarray, float]:
    """parts: (normalised partial output o_i, lse_i) -> (o, lse) of the union."""
    lses = np.array([p[1] for p in parts], dtype=np.float64)
    m = lses.max()
    w = np.exp(lses - m)
    o = sum(wi * _f64(p[0]) for wi, p in zip(w, parts)) / w.sum()
    return o, float(m + math.log(w.sum()))


# ---------------------------------------------------------------------------
# Algorithmic work: attended (query, key) pairs, used for FLOP accounting
# (4*d FLOPs per pair: q.k and p.v, two multiply-adds each per element)
# ---------------------------------------------------------------------------
def algorithmic_pairs(batch: int, N: int, Hq: int, B: int, topk: int) -> int:
    """Sum over (b, h, t) of |attended keys| = min(topk-1, c)*B' + (t - cB + 1),
    where B' accounts for the ragged last block (never a historical block)."""
    total = 0
    n = num_blocks(N, B)
    for c in range(n):
        s, e = block_range(c, N, B)
        L = e - s
        hist = min(topk - 1, c) * B * L          # every historical block is full
        cur = L * (L + 1) // 2
        total += hist + cur
    return total * batch * Hq
