"""Plain fp64 CPU oracle for the MoBA backward pass (gradients of the attention
output with respect to q, k and v).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import or call this
module: only ``tests/`` uses it.  It shares no code with the CUDA path.

What is differentiated: "MoBA: Mixture of Block Attention for Long-Context
LLMs", paper-graph summary §3 "The Core MoBA Attention Equation",
MoBA(q, K, V) = Softmax(q K[I]^T) V[I], with the key set I chosen by the gate
(the current block causal, "Causality Enforcement").  The pages train with
MoBA but print no backward formula.  Reading B1: the gate's selection is a
top-k of scores, piecewise constant in q and k, so its derivative is zero
almost everywhere and the gradients are those of softmax attention over the
selected keys, with the selection held fixed.  Readings C1-C6 of the forward
oracle apply.

For one query row with logits z_u = scale * <q, k_u> over its key set:
  p = softmax(z), o = sum_u p_u v_u, D = <do, o>,
  dv_u += p_u do,  dp_u = <do, v_u>,  ds_u = p_u (dp_u - D),
  dq = scale * sum_u ds_u k_u,  dk_u += scale * ds_u q.
(the standard derivative of softmax attention; the pages print no formula for
it.)  Query heads of one GQA group add into the same dk/dv of their kv head.

Everything is computed in float64 from the given inputs.  Two formulations:
a per-row gather formulation (``moba_backward``) and a dense-mask matrix
formulation (``moba_backward_dense``) for small N; tests check that they agree
and pin them against finite differences and against autograd of plain dense
attention in the special cases where MoBA is dense.
"""
from __future__ import annotations

import numpy as np

from .moba_oracle import _f64, gate_scores, key_positions, mean_pool, num_blocks, select_blocks

__all__ = ["attend_row_grad", "select_all", "moba_forward_sel", "moba_backward", "moba_backward_dense"]


def attend_row_grad(q_row, Ksel, Vsel, do_row, scale: float):
    """Gradients of one row's attention output (the formulas of the module
    docstring).  Returns (dq [d], dK [m, d], dV [m, d]) for the m gathered keys."""
    q, K, V, do = _f64(q_row), _f64(Ksel), _f64(Vsel), _f64(do_row)
    z = scale * (K @ q)
    p = np.exp(z - z.max())
    p /= p.sum()
    o = p @ V
    D = float(do @ o)
    dV = np.outer(p, do)
    dp = V @ do
    ds = p * (dp - D)
    dq = scale * (ds @ K)
    dK = scale * np.outer(ds, q)
    return dq, dK, dV


def select_all(q, k, B: int, topk: int) -> np.ndarray:
    """The gate's selection for every row: sel [b, N, Hq, topk], ascending, -1 padded."""
    q, k = _f64(q), _f64(k)
    b, N, Hq, _ = q.shape
    G = Hq // k.shape[2]
    sel = np.full((b, N, Hq, topk), -1, dtype=np.int64)
    for bb in range(b):
        kbars = [mean_pool(k[bb, :, g], B) for g in range(k.shape[2])]
        for h in range(Hq):
            kbar = kbars[h // G]
            for t in range(N):
                js, _ = select_blocks(gate_scores(q[bb, t, h], kbar), t, B, topk)
                sel[bb, t, h, :len(js)] = js
    return sel


def moba_forward_sel(q, k, v, sel, B: int, scale: float) -> np.ndarray:
    """Forward output with a given (frozen) selection: out [b, N, Hq, d]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    b, N, Hq, d = q.shape
    G = Hq // k.shape[2]
    out = np.zeros((b, N, Hq, d))
    for bb in range(b):
        for h in range(Hq):
            g = h // G
            for t in range(N):
                pos = key_positions([int(j) for j in sel[bb, t, h] if j >= 0], t, B, N)
                z = scale * (k[bb, pos, g] @ q[bb, t, h])
                p = np.exp(z - z.max())
                out[bb, t, h] = (p / p.sum()) @ v[bb, pos, g]
    return out


def moba_backward(q, k, v, dout, B: int, topk: int, scale: float, sel=None):
    """Gather formulation.  q, dout [b, N, Hq, d]; k, v [b, N, Hkv, d].
    Returns (dq, dk, dv, sel) with dk, dv [b, N, Hkv, d]."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    if sel is None:
        sel = select_all(q, k, B, topk)
    b, N, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for bb in range(b):
        for h in range(Hq):
            g = h // G
            for t in range(N):
                pos = key_positions([int(j) for j in sel[bb, t, h] if j >= 0], t, B, N)
                gq, gK, gV = attend_row_grad(q[bb, t, h], k[bb, pos, g], v[bb, pos, g], dout[bb, t, h], scale)
                dq[bb, t, h] = gq
                np.add.at(dk[bb, :, g], pos, gK)
                np.add.at(dv[bb, :, g], pos, gV)
    return dq, dk, dv, sel


def moba_backward_dense(q, k, v, dout, sel, B: int, scale: float):
    """Dense-mask formulation for small N: the token mask M[t, u] = (block of u
    selected by t) and (u <= t), then the matrix form of the same derivative
    (P = masked softmax, dV = P^T dO, dS = P * (dO V^T - rowsum(dO * O)),
    dQ = scale dS K, dK = scale dS^T Q).  Returns (dq, dk, dv)."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    b, N, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    blk = np.arange(N) // B
    tri = np.arange(N)[None, :] <= np.arange(N)[:, None]
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    n = num_blocks(N, B)
    for bb in range(b):
        for h in range(Hq):
            g = h // G
            Gm = np.zeros((N, n), dtype=bool)
            for t in range(N):
                js = [int(j) for j in sel[bb, t, h] if j >= 0]
                Gm[t, js] = True
            M = Gm[:, blk] & tri
            Q, K, V, dO = q[bb, :, h], k[bb, :, g], v[bb, :, g], dout[bb, :, h]
            Z = np.where(M, scale * (Q @ K.T), -np.inf)
            P = np.exp(Z - Z.max(axis=1, keepdims=True))
            P /= P.sum(axis=1, keepdims=True)
            O = P @ V
            dP = dO @ V.T
            dS = P * (dP - (dO * O).sum(axis=1, keepdims=True))
            dq[bb, :, h] = scale * (dS @ K)
            dk[bb, :, g] += scale * (dS.T @ Q)
            dv[bb, :, g] += P.T @ dO
    return dq, dk, dv
