"""Pins of the pooled-gate variant oracle (oracle/moba_pooled_gate.py) against
things other than itself: a hand-built example whose three rankings differ,
the plain MoBA oracle when no extra blocks are routed, pooling by NumPy's
segment reductions, a brute-force ranking by lexsort, invariants, and dense
causal attention (torch SDPA in fp64) when every earlier block is selected."""
import numpy as np
import pytest
import torch

import oracle as O
from oracle import moba_pooled_gate as P


def test_hand_built_example_where_the_three_rankings_differ():
    # q = e0, blocks of 4 keys; only coordinate 0 matters for the scores
    d, B = 4, 4
    K = np.zeros((16, d))
    K[0:4, 0] = [10, 10, 10, -5]   # block 0: mean 6.25, max 10, min -5
    K[4:8, 0] = [20, 0, 0, 0]      # block 1: mean 5,    max 20, min 0
    K[8:12, 0] = 3                 # block 2: mean 3,    max 3,  min 3
    q = np.array([1.0, 0, 0, 0])
    t = 13                         # current block 3
    pools = (O.mean_pool(K, B), P.max_pool(K, B), P.min_pool(K, B))
    # mean ranks 0 > 1 > 2, max ranks 1 > 0 > 2, min ranks 2 > 1 > 0
    assert P.select_blocks_pooled(q, *pools, t, B, topk=2, extra=0) == [0, 3]
    assert P.select_blocks_pooled(q, *pools, t, B, topk=2, extra=1) == [0, 1, 2, 3]
    assert P.select_blocks_pooled(q, *pools, t, B, topk=3, extra=1) == [0, 1, 2, 3]
    # with -q: mean ranks 2 first, max ranks 2 first (-3 > -10 > -20), min ranks 0 first (5 > 0 > -3)
    assert P.select_blocks_pooled(-q, *pools, t, B, topk=2, extra=1) == [0, 2, 3]
    # a query early in the sequence has fewer candidates: t = 5 (block 1) sees block 0 only
    assert P.select_blocks_pooled(q, *pools, 5, B, topk=2, extra=1) == [0, 1]


def test_ties_go_to_the_lower_block():
    d, B = 2, 2
    K = np.zeros((8, d))
    K[0:2, 0] = [5, 0]             # block 0: max 5, mean 2.5
    K[2:4, 0] = [5, 1]             # block 1: max 5, mean 3
    q = np.array([1.0, 0])
    pools = (O.mean_pool(K, B), P.max_pool(K, B), P.min_pool(K, B))
    # mean picks block 1; max ties 0 and 1 -> block 0; min: block 1 (1 > 0)
    assert P.select_blocks_pooled(q, *pools, t=7, B=B, topk=2, extra=1) == [0, 1, 3]


def test_pools_match_segment_reductions():
    rng = np.random.default_rng(0)
    K = rng.standard_normal((23, 5))          # ragged last block
    B = 5
    starts = np.arange(0, 23, B)
    assert np.array_equal(P.max_pool(K, B), np.maximum.reduceat(K, starts, axis=0))
    assert np.array_equal(P.min_pool(K, B), np.minimum.reduceat(K, starts, axis=0))


@pytest.mark.parametrize("seed", range(4))
def test_selection_against_lexsort_brute_force_and_invariants(seed):
    rng = np.random.default_rng(seed)
    N, d, B = 60, 6, 5
    K = rng.standard_normal((N, d)) + rng.standard_normal((N // B, d)).repeat(B, 0)
    pools = (O.mean_pool(K, B), P.max_pool(K, B), P.min_pool(K, B))
    for topk, extra in ((3, 1), (4, 2), (1, 1), (2, 0)):
        for t in range(N):
            q = rng.standard_normal(d)
            got = P.select_blocks_pooled(q, *pools, t, B, topk, extra)
            c = t // B
            want = {c}
            for pool, m in ((pools[0], topk - 1), (pools[1], extra), (pools[2], extra)):
                s = pool[:c] @ q
                order = np.lexsort((np.arange(c), -s))      # by (-score, j)
                want.update(int(j) for j in order[:m])
            assert got == sorted(want)
            plain, _ = O.select_blocks(pools[0] @ q, t, B, topk)
            assert set(plain) <= set(got) and got[-1] == c
            assert min(topk, c + 1) <= len(got) <= min(topk + 2 * extra, c + 1)


def test_extra_zero_is_the_plain_moba_layer():
    rng = np.random.default_rng(5)
    q = rng.standard_normal((1, 40, 4, 8))
    k = rng.standard_normal((1, 40, 2, 8))
    v = rng.standard_normal((1, 40, 2, 8))
    out, lse, sels = P.moba_pooled_layer(q, k, v, 6, 3, 0, 0.3)
    o_out, o_lse, o_sel, _ = O.moba_dense(q, k, v, 6, 3, 0.3)
    assert np.abs(out - o_out).max() <= 1e-12 and np.abs(lse - o_lse).max() <= 1e-12
    for (b, t, h), sel in sels.items():
        assert sel == [int(x) for x in o_sel[b, t, h] if x >= 0]


def test_every_earlier_block_selected_is_dense_causal():
    rng = np.random.default_rng(6)
    N, B, d = 30, 5, 8
    q = rng.standard_normal((1, N, 2, d))
    k = rng.standard_normal((1, N, 1, d))
    v = rng.standard_normal((1, N, 1, d))
    # extra = 5 >= the 5 earlier blocks of the last row: the max rule alone selects them all
    out, _, _ = P.moba_pooled_layer(q, k, v, B, 2, 5, 0.4)
    tq, tk, tv = (torch.tensor(x).transpose(1, 2) for x in (q, k.repeat(2, 2), v.repeat(2, 2)))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True, scale=0.4)
    assert np.abs(out - ref.transpose(1, 2).numpy()).max() <= 1e-12


@pytest.mark.parametrize("seed,N,B,Hq,Hkv,topk,extra", [
    (0, 37, 5, 4, 2, 3, 1), (1, 50, 7, 2, 1, 2, 2), (2, 64, 8, 3, 3, 1, 3), (3, 41, 6, 4, 1, 4, 1),
])
def test_layer_is_masked_attention_over_its_selections(seed, N, B, Hq, Hkv, topk, extra):
    # an independent formulation for rows with any number of selected blocks: fp64
    # SDPA (a library routine) with the boolean mask "key u is in a selected block
    # and u <= t" built from the layer's own selections
    rng = np.random.default_rng(seed)
    d = 6
    q = rng.standard_normal((1, N, Hq, d))
    k = rng.standard_normal((1, N, Hkv, d)) + rng.standard_normal((1, (N + B - 1) // B, Hkv, d)).repeat(B, 1)[:, :N]
    v = rng.standard_normal((1, N, Hkv, d))
    out, lse, sels = P.moba_pooled_layer(q, k, v, B, topk, extra, 0.35)
    G = Hq // Hkv
    mask = torch.zeros(1, Hq, N, N, dtype=torch.bool)
    for (_, t, h), sel in sels.items():
        for j in sel:
            mask[0, h, t, j * B: min(N, (j + 1) * B)] = True
    mask &= torch.ones(N, N, dtype=torch.bool).tril()
    tq = torch.tensor(q).transpose(1, 2)
    tk, tv = (torch.tensor(x).repeat_interleave(G, 2).transpose(1, 2) for x in (k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=0.35)
    assert np.abs(out - ref.transpose(1, 2).numpy()).max() <= 1e-12
    z = 0.35 * torch.einsum("bhtd,bhud->bhtu", tq, tk).masked_fill(~mask, float("-inf"))
    assert np.abs(lse - torch.logsumexp(z, -1).numpy()).max() <= 1e-12
    # some rows attend fewer blocks than the width allows (the rankings overlap)
    widths = [len(s) for (_, t, _), s in sels.items() if t // B + 1 > topk + 2 * extra]
    assert widths and min(widths) >= topk and max(widths) <= topk + 2 * extra
