"""Pins of the fp64 backward oracle (oracle/moba_backward.py) against things
other than itself: central finite differences of the forward with the
selection frozen, fp64 autograd of plain dense attention where MoBA is dense
(top-k >= n: causal; top-k = 1: block-diagonal causal), the dense-mask matrix
formulation, and invariants of softmax attention."""
import numpy as np
import pytest
import torch

from oracle import moba_backward as OB


def rand_inputs(b, N, hq, hkv, d, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((b, N, hq, d))
    k = rng.standard_normal((b, N, hkv, d))
    v = rng.standard_normal((b, N, hkv, d))
    do = rng.standard_normal((b, N, hq, d))
    return q, k, v, do


def torch_attention_grads(q, k, v, do, mask, scale):
    """Autograd of plain masked softmax attention in fp64 (mask [N, N] bool,
    True = attend); GQA by repeating kv heads."""
    tq = torch.tensor(q, requires_grad=True)
    tk = torch.tensor(k, requires_grad=True)
    tv = torch.tensor(v, requires_grad=True)
    rep = q.shape[2] // k.shape[2]
    kk = tk.repeat_interleave(rep, 2)
    vv = tv.repeat_interleave(rep, 2)
    z = torch.einsum("bthd,buhd->bhtu", tq, kk) * scale
    z = z.masked_fill(~torch.tensor(mask), float("-inf"))
    out = torch.einsum("bhtu,buhd->bthd", torch.softmax(z, dim=-1), vv)
    (out * torch.tensor(do)).sum().backward()
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


def test_finite_differences_frozen_selection():
    b, N, hq, hkv, d, B, topk, scale = 1, 40, 2, 1, 8, 8, 3, 0.4
    q, k, v, do = rand_inputs(b, N, hq, hkv, d, 0)
    dq, dk, dv, sel = OB.moba_backward(q, k, v, do, B, topk, scale)

    def loss(qq, kk, vv):
        return float((OB.moba_forward_sel(qq, kk, vv, sel, B, scale) * do).sum())

    rng = np.random.default_rng(1)
    eps = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(25):
            idx = tuple(int(rng.integers(s)) for s in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - g[idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, g[idx])


def test_dense_causal_special_case_matches_autograd():
    # top-k >= n: every earlier block is selected, so MoBA is causal attention
    b, N, hq, hkv, d, B, scale = 2, 48, 4, 2, 8, 8, 0.3
    q, k, v, do = rand_inputs(b, N, hq, hkv, d, 2)
    dq, dk, dv, _ = OB.moba_backward(q, k, v, do, B, 16, scale)
    mask = np.tril(np.ones((N, N), dtype=bool))
    rq, rk, rv = torch_attention_grads(q, k, v, do, mask, scale)
    for a, r in ((dq, rq), (dk, rk), (dv, rv)):
        assert np.abs(a - r).max() <= 1e-10


def test_topk_one_is_block_diagonal_causal():
    b, N, hq, hkv, d, B, scale = 1, 37, 2, 1, 6, 10, 0.5
    q, k, v, do = rand_inputs(b, N, hq, hkv, d, 3)
    dq, dk, dv, _ = OB.moba_backward(q, k, v, do, B, 1, scale)
    t = np.arange(N)
    mask = (t[:, None] // B == t[None, :] // B) & (t[None, :] <= t[:, None])
    rq, rk, rv = torch_attention_grads(q, k, v, do, mask, scale)
    for a, r in ((dq, rq), (dk, rk), (dv, rv)):
        assert np.abs(a - r).max() <= 1e-10


def test_gather_and_dense_mask_formulations_agree():
    b, N, hq, hkv, d, B, topk, scale = 2, 45, 4, 2, 8, 6, 3, 0.35
    q, k, v, do = rand_inputs(b, N, hq, hkv, d, 4)
    dq, dk, dv, sel = OB.moba_backward(q, k, v, do, B, topk, scale)
    rq, rk, rv = OB.moba_backward_dense(q, k, v, do, sel, B, scale)
    for a, r in ((dq, rq), (dk, rk), (dv, rv)):
        assert np.abs(a - r).max() <= 1e-10


def test_invariants():
    b, N, hq, hkv, d, B, topk, scale = 1, 50, 4, 1, 8, 7, 4, 0.3
    q, k, v, do = rand_inputs(b, N, hq, hkv, d, 5)
    dq, dk, dv, sel = OB.moba_backward(q, k, v, do, B, topk, scale)
    # every row's probabilities sum to one: the dv of a kv head sums to the do of its rows
    assert np.abs(dv.sum(axis=1)[:, 0] - do.sum(axis=(1, 2))).max() <= 1e-10
    # every row's ds sums to zero: the dk of a kv head sums to zero
    assert np.abs(dk.sum(axis=1)).max() <= 1e-10
    # a shift of every key by one vector shifts every logit of a row equally (and
    # every gate score of a row equally, so the selection stays): dq is unchanged
    shift = np.random.default_rng(6).standard_normal(d)
    dq2, _, _, sel2 = OB.moba_backward(q, k + shift, v, do, B, topk, scale)
    assert np.array_equal(sel, sel2)
    assert np.abs(dq - dq2).max() <= 1e-9


@pytest.mark.parametrize("topk", [2, 5])
def test_zero_upstream_gradient_gives_zero(topk):
    q, k, v, do = rand_inputs(1, 30, 2, 1, 4, 7)
    dq, dk, dv, _ = OB.moba_backward(q, k, v, np.zeros_like(do), 6, topk, 0.5)
    assert not dq.any() and not dk.any() and not dv.any()


def test_variable_length_selections_of_the_pooled_gate():
    # the gate variant with max/min-pooled keys gives rows different numbers of
    # blocks; the backward oracle with such a frozen selection equals fp64
    # autograd of attention under the per-head mask built from it, and its
    # dense-mask formulation
    from oracle import moba_pooled_gate as P
    b, N, hq, hkv, d, B, topk, extra, scale = 1, 48, 4, 2, 8, 6, 2, 2, 0.45
    q, k, v, do = rand_inputs(b, N, hq, hkv, d, 3)
    _, _, sels = P.moba_pooled_layer(q, k, v, B, topk, extra, scale)
    W = topk + 2 * extra
    sel = np.full((b, N, hq, W), -1, dtype=np.int64)
    mask = np.zeros((hq, N, N), dtype=bool)
    for (_, t, h), js in sels.items():
        sel[0, t, h, :len(js)] = js
        for j in js:
            mask[h, t, j * B:min(N, (j + 1) * B)] = True
    mask &= np.tril(np.ones((N, N), dtype=bool))
    assert len({len(js) for js in sels.values()}) > 2              # the row widths do vary
    dq, dk, dv, _ = OB.moba_backward(q, k, v, do, B, W, scale, sel=sel)
    rq, rk, rv = torch_attention_grads(q, k, v, do, mask, scale)
    for got, ref in ((dq, rq), (dk, rk), (dv, rv)):
        assert np.abs(got - ref).max() <= 1e-12
    for got, ref in zip((dq, dk, dv), OB.moba_backward_dense(q, k, v, do, sel, B, scale)):
        assert np.abs(got - ref).max() <= 1e-12
