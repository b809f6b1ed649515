"""Property-based cross-checks of the fp64 oracle on random small shapes
(hypothesis): the per-row gather formulation and the dense-mask formulation of
the forward agree, every selection obeys the gate's invariants, and the two
backward formulations agree.  Sizes stay tiny so the whole file runs in
seconds."""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle as O
from oracle import moba_backward as OB

shapes = st.tuples(
    st.integers(1, 2),            # batch
    st.integers(1, 40),           # seqlen
    st.sampled_from([(1, 1), (2, 1), (4, 2), (3, 3)]),   # (hq, hkv)
    st.integers(1, 9),            # block
    st.integers(1, 6),            # topk
    st.integers(0, 2 ** 31 - 1),  # seed
)


def inputs(b, N, hq, hkv, seed, d=4):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((b, N, hq, d)), rng.standard_normal((b, N, hkv, d)),
            rng.standard_normal((b, N, hkv, d)), rng.standard_normal((b, N, hq, d)))


@settings(max_examples=60, deadline=None, derandomize=True)
@given(shapes)
def test_forward_formulations_agree_and_selection_invariants(shape):
    b, N, (hq, hkv), B, topk, seed = shape
    q, k, v, _ = inputs(b, N, hq, hkv, seed)
    out, lse, sel, _ = O.moba_dense(q, k, v, B, topk, 0.5)
    G = hq // hkv
    for bb in range(b):
        for h in range(hq):
            kbar = O.mean_pool(k[bb, :, h // G], B)
            for t in range(N):
                o, l, s, _ = O.moba_row(q[bb, t, h], k[bb, :, h // G], v[bb, :, h // G], kbar, t, B, topk, 0.5)
                assert np.abs(o - out[bb, t, h]).max() <= 1e-10 and abs(l - lse[bb, h, t]) <= 1e-10
                assert s == [int(x) for x in sel[bb, t, h] if x >= 0]
                c = t // B
                assert s[-1] == c and len(s) == min(topk, c + 1) and all(j <= c for j in s)


@settings(max_examples=30, deadline=None, derandomize=True)
@given(shapes)
def test_backward_formulations_agree(shape):
    b, N, (hq, hkv), B, topk, seed = shape
    q, k, v, do = inputs(b, N, hq, hkv, seed)
    dq, dk, dv, sel = OB.moba_backward(q, k, v, do, B, topk, 0.5)
    rq, rk, rv = OB.moba_backward_dense(q, k, v, do, sel, B, 0.5)
    for a, r in ((dq, rq), (dk, rk), (dv, rv)):
        assert np.abs(a - r).max() <= 1e-9


pooled_shapes = st.tuples(
    st.integers(1, 2),            # batch
    st.integers(1, 36),           # seqlen
    st.sampled_from([(1, 1), (2, 1), (4, 2)]),   # (hq, hkv)
    st.integers(1, 7),            # block
    st.integers(1, 4),            # topk
    st.integers(0, 3),            # extra
    st.integers(0, 2 ** 31 - 1),  # seed
)


@settings(max_examples=40, deadline=None, derandomize=True)
@given(pooled_shapes)
def test_pooled_gate_layer_invariants_and_masked_attention(shape):
    # the gate variant with max/min-pooled keys: every row attends its current
    # block, a superset of the plain gate's blocks, at most topk + 2 extra blocks,
    # and its output is softmax attention under the mask of its own selection
    import torch
    from oracle import moba_pooled_gate as P
    b, N, (hq, hkv), B, topk, extra, seed = shape
    q, k, v, _ = inputs(b, N, hq, hkv, seed)
    out, lse, sels = P.moba_pooled_layer(q, k, v, B, topk, extra, 0.5)
    _, _, plain, _ = O.moba_dense(q, k, v, B, topk, 0.5)
    G = hq // hkv
    mask = np.zeros((b, hq, N, N), dtype=bool)
    for (bb, t, h), sel in sels.items():
        c = t // B
        assert sel == sorted(set(sel)) and sel[-1] == c
        assert set(int(x) for x in plain[bb, t, h] if x >= 0) <= set(sel)
        assert min(topk, c + 1) <= len(sel) <= min(topk + 2 * extra, c + 1)
        for j in sel:
            mask[bb, h, t, j * B:min(N, (j + 1) * B)] = True
    mask &= np.tril(np.ones((N, N), dtype=bool))
    tq = torch.tensor(q).transpose(1, 2)
    tk, tv = (torch.tensor(x).repeat_interleave(G, 2).transpose(1, 2) for x in (k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=torch.tensor(mask), scale=0.5)
    assert np.abs(out - ref.transpose(1, 2).numpy()).max() <= 1e-12
