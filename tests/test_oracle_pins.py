"""Pins for the fp64 oracle: each test ties the oracle to something other than
itself (a hand-derived worked example, a closed form, a library routine, brute
force, or a figure the pages print), so that a dropped term, a wrong sign or
index, or a transposed operand in the oracle fails at least one of them."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))
rng_seed = 1234


def _rand(shape, rng, scale=1.0):
    return rng.standard_normal(shape) * scale


def _sdpa(q, k, v, scale, mask=None, causal=False):
    """torch SDPA in fp64 on [N, d] single-head inputs; returns (out, lse)."""
    qt = torch.from_numpy(q)[None, None]
    kt = torch.from_numpy(k)[None, None]
    vt = torch.from_numpy(v)[None, None]
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, is_causal=causal,
                                                           scale=scale)[0, 0].numpy()
    N = q.shape[0]
    if causal:
        mask = np.tril(np.ones((N, k.shape[0]), dtype=bool))
    z = torch.from_numpy(scale * (q @ k.T))
    if mask is not None:
        z = z.masked_fill(~torch.from_numpy(mask), float("-inf"))
    lse = torch.logsumexp(z, dim=1).numpy()
    return out, lse


# --------------------------------------------------------------------------
# worked example (hand-derived, tests/golden/worked_example.json)
# --------------------------------------------------------------------------
def test_worked_example_selection_and_positions():
    ex = json.load(open(os.path.join(HERE, "golden", "worked_example.json")))
    N, B, topk, scale = ex["N"], ex["B"], ex["topk"], ex["scale"]
    K = np.array([[x, 0.0] for x in ex["x"]])
    V = np.array([[u, 1.0] for u in range(N)], dtype=np.float64)
    kbar = O.mean_pool(K, B)
    assert np.array_equal(kbar, np.array([[2, 0], [0, 0], [2, 0], [2, 0]], dtype=np.float64))
    for case in ex["cases"]:
        q = np.array(case["q"], dtype=np.float64)
        out, lse, sel, gap = O.moba_row(q, K, V, kbar, case["t"], B, topk, scale)
        assert sel == case["sel"], case
        if case["gap"] is None:
            assert gap is None
        else:
            assert gap == pytest.approx(case["gap"])
        pos = O.key_positions(sel, case["t"], B, N)
        assert pos.tolist() == case["positions"]
        # the value rows are (u, 1): the second output coordinate is exactly 1
        # and the first is the softmax-weighted mean position
        z = np.array([scale * q[0] * ex["x"][u] for u in case["positions"]])
        w = np.exp(z - z.max())
        assert out[1] == pytest.approx(1.0, abs=1e-15)
        assert out[0] == pytest.approx(float((w * np.array(case["positions"])).sum() / w.sum()), rel=1e-14)
        assert lse == pytest.approx(float(z.max() + np.log(w.sum())), rel=1e-14)


# --------------------------------------------------------------------------
# the C1 reading (topk counts the current block) against the pages' printed
# sparsity figures: 95.31% at 1M tokens with B=4096, topk=12 and 62.5% at
# 128K (paper-graph summary, section 5 'Main Quantitative Results' and the
# executive summary)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("N,B,topk,printed", [(1 << 20, 4096, 12, 95.31), (131072, 4096, 12, 62.5),
                                               (32768, 512, 3, 95.31)])
def test_sparsity_reading_matches_printed_figures(N, B, topk, printed):
    t = N - 1                                  # the last query: every earlier block is a candidate
    scores = np.arange((N + B - 1) // B, dtype=np.float64)
    sel, _ = O.select_blocks(scores, t, B, topk)
    attended = len(O.key_positions(sel, t, B, N))
    assert len(sel) == topk
    assert round(100.0 * (1.0 - attended / N), 2) == printed


# --------------------------------------------------------------------------
# mean-pool closed form, including a ragged last block (C7)
# --------------------------------------------------------------------------
def test_mean_pool_closed_form_ragged():
    N, B, d = 11, 4, 3
    K = np.array([[t, 2 * t + 1, -t] for t in range(N)], dtype=np.float64)
    kbar = O.mean_pool(K, B)
    for j, (s, e) in enumerate([(0, 4), (4, 8), (8, 11)]):
        m = (s + e - 1) / 2.0                  # mean of consecutive integers
        assert np.allclose(kbar[j], [m, 2 * m + 1, -m], rtol=0, atol=1e-15)


def test_gate_score_is_unscaled_inner_product():
    kbar = np.array([[1.0, 2.0], [-3.0, 0.5], [0.0, 4.0]])
    q = np.array([2.0, -1.0])
    assert O.gate_scores(q, kbar).tolist() == [0.0, -6.5, -4.0]


# --------------------------------------------------------------------------
# selection: invariants (T1-T3), ties (T11), brute force
# --------------------------------------------------------------------------
def test_selection_invariants_random():
    rng = np.random.default_rng(rng_seed)
    for _ in range(300):
        B = int(rng.integers(1, 6))
        N = int(rng.integers(1, 40))
        topk = int(rng.integers(1, 7))
        n = (N + B - 1) // B
        t = int(rng.integers(0, N))
        c = t // B
        s = rng.standard_normal(n)
        sel, gap = O.select_blocks(s, t, B, topk)
        assert c in sel                                  # current block always
        assert all(j <= c for j in sel)                  # never a future block
        assert len(sel) == min(topk, c + 1)              # gate count
        assert sel == sorted(sel) and len(set(sel)) == len(sel)
        hist = [j for j in sel if j != c]
        rest = [j for j in range(c) if j not in hist]
        if hist and rest:
            assert min(s[j] for j in hist) >= max(s[j] for j in rest)
            assert gap == pytest.approx(min(s[j] for j in hist) - max(s[j] for j in rest))


def test_selection_ties_lower_index_wins():
    s = np.array([1.0, 5.0, 1.0, 5.0, 1.0, 0.0])
    sel, gap = O.select_blocks(s, t=5 * 10 + 3, B=10, topk=2)      # c = 5, one slot, tie 1 vs 3
    assert sel == [1, 5] and gap == 0.0
    sel, gap = O.select_blocks(s, t=53, B=10, topk=4)              # 3 slots: 1, 3, then tie 0/2/4 -> 0
    assert sel == [0, 1, 3, 5] and gap == 0.0


def test_selection_brute_force():
    rng = np.random.default_rng(7)
    for _ in range(200):
        c = int(rng.integers(0, 8))
        topk = int(rng.integers(1, 6))
        B = 3
        t = c * B + int(rng.integers(0, B))
        s = np.round(rng.standard_normal(c + 1) * 2) / 2      # coarse values -> many ties
        m = min(topk - 1, c)
        best = None
        for comb in itertools.combinations(range(c), m):
            # key: larger score multiset first, then lexicographically smaller indices
            key = (sorted((-s[j] for j in comb)), list(comb))
            if best is None or key < best[0]:
                best = (key, comb)
        sel, _ = O.select_blocks(s, t, B, topk)
        assert sel == sorted(list(best[1]) + [c])


# --------------------------------------------------------------------------
# special cases that reduce to library routines (T4-T6)
# --------------------------------------------------------------------------
def _single_head(N, d, rng):
    return _rand((N, d), rng), _rand((N, d), rng), _rand((N, d), rng)


@pytest.mark.parametrize("N,B", [(37, 8), (64, 16), (5, 8)])
def test_topk_at_least_n_is_dense_causal(N, B):
    rng = np.random.default_rng(N + B)
    d, scale = 8, 0.3
    q, k, v = _single_head(N, d, rng)
    n = (N + B - 1) // B
    ref_out, ref_lse = _sdpa(q, k, v, scale, causal=True)
    kbar = O.mean_pool(k, B)
    for t in range(N):
        out, lse, sel, _ = O.moba_row(q[t], k, v, kbar, t, B, n + 2, scale)
        assert np.allclose(out, ref_out[t], rtol=1e-12, atol=1e-12)
        assert lse == pytest.approx(ref_lse[t], rel=1e-12)
    out, lse, _, _ = O.moba_dense(q[None, :, None], k[None, :, None], v[None, :, None], B, n, scale)
    assert np.allclose(out[0, :, 0], ref_out, rtol=1e-12, atol=1e-12)
    assert np.allclose(lse[0, 0], ref_lse, rtol=1e-12)


def test_topk_one_is_block_diagonal_causal():
    rng = np.random.default_rng(3)
    N, B, d, scale = 45, 8, 6, 0.5
    q, k, v = _single_head(N, d, rng)
    blk = np.arange(N) // B
    mask = (blk[:, None] == blk[None, :]) & (np.arange(N)[None, :] <= np.arange(N)[:, None])
    ref_out, ref_lse = _sdpa(q, k, v, scale, mask=mask)
    out, lse, sel, _ = O.moba_dense(q[None, :, None], k[None, :, None], v[None, :, None], B, 1, scale)
    assert np.allclose(out[0, :, 0], ref_out, rtol=1e-12, atol=1e-12)
    assert np.allclose(lse[0, 0], ref_lse, rtol=1e-12)
    assert (sel[0, :, 0, 0] == blk).all()


def test_single_block_is_plain_causal():
    rng = np.random.default_rng(4)
    N, d, scale = 33, 5, 1.0
    q, k, v = _single_head(N, d, rng)
    ref_out, _ = _sdpa(q, k, v, scale, causal=True)
    out, _, _, _ = O.moba_dense(q[None, :, None], k[None, :, None], v[None, :, None], N, 3, scale)
    assert np.allclose(out[0, :, 0], ref_out, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# sliding-window special case (T8): block offsets growing with the block index
# make the most recent blocks score highest, so MoBA becomes block-sliding-window
# attention (paper-graph summary, section 2.2 discussion of sliding windows as a
# special case of the gate)
# --------------------------------------------------------------------------
def test_sliding_window_special_case():
    rng = np.random.default_rng(5)
    N, B, d, topk, scale = 64, 8, 4, 3, 0.2
    q = np.abs(_rand((N, d), rng)) + 0.1           # q . u > 0 for u = (1,1,1,1)
    k = _rand((N, d), rng) * 0.01
    k += 50.0 * (np.arange(N) // B)[:, None]       # offset alpha * j * u
    v = _rand((N, d), rng)
    blk = np.arange(N) // B
    t_idx = np.arange(N)
    win = (blk[None, :] >= blk[:, None] - (topk - 1)) & (t_idx[None, :] <= t_idx[:, None])
    ref_out, ref_lse = _sdpa(q, k, v, scale, mask=win)
    out, lse, sel, _ = O.moba_dense(q[None, :, None], k[None, :, None], v[None, :, None], B, topk, scale)
    assert np.allclose(out[0, :, 0], ref_out, rtol=1e-10, atol=1e-12)
    kbar = O.mean_pool(k, B)
    for t in range(N):
        o2, l2, s2, _ = O.moba_row(q[t], k, v, kbar, t, B, topk, scale)
        c = t // B
        assert s2 == list(range(max(0, c - topk + 1), c + 1))
        assert np.allclose(o2, ref_out[t], rtol=1e-10, atol=1e-12)


# --------------------------------------------------------------------------
# two formulations agree (T9), GQA reduction and independence (T10)
# --------------------------------------------------------------------------
def _rand_layer(b, N, Hq, Hkv, d, rng):
    q = _rand((b, N, Hq, d), rng)
    k = _rand((b, N, Hkv, d), rng)
    k += np.repeat(_rand((b, (N + 3) // 4 + 1, Hkv, d), rng), 4, axis=1)[:, :N]
    v = _rand((b, N, Hkv, d), rng)
    return q, k, v


def test_gather_and_dense_formulations_agree():
    rng = np.random.default_rng(6)
    b, N, Hq, Hkv, d, B, topk, scale = 2, 29, 4, 2, 6, 4, 3, 0.4
    q, k, v = _rand_layer(b, N, Hq, Hkv, d, rng)
    out, lse, sel, gap = O.moba_dense(q, k, v, B, topk, scale)
    G = Hq // Hkv
    for bb in range(b):
        for h in range(Hq):
            g = h // G
            kbar = O.mean_pool(k[bb, :, g], B)
            for t in range(N):
                o1, l1, s1, g1 = O.moba_row(q[bb, t, h], k[bb, :, g], v[bb, :, g], kbar, t, B, topk, scale)
                assert np.allclose(o1, out[bb, t, h], rtol=1e-12, atol=1e-12)
                assert l1 == pytest.approx(lse[bb, h, t], rel=1e-12)
                row = sel[bb, t, h]
                assert row[row >= 0].tolist() == s1
                assert (row[len(s1):] == -1).all()
                if g1 is None:
                    assert np.isnan(gap[bb, t, h])
                else:
                    assert g1 == pytest.approx(gap[bb, t, h], rel=1e-12, abs=1e-14)


def test_gqa_equals_repeated_kv_and_heads_independent():
    rng = np.random.default_rng(8)
    b, N, Hq, Hkv, d, B, topk, scale = 2, 24, 6, 2, 5, 4, 3, 0.7
    q, k, v = _rand_layer(b, N, Hq, Hkv, d, rng)
    G = Hq // Hkv
    out, lse, sel, _ = O.moba_dense(q, k, v, B, topk, scale)
    out2, lse2, sel2, _ = O.moba_dense(q, np.repeat(k, G, axis=2), np.repeat(v, G, axis=2), B, topk, scale)
    assert np.allclose(out, out2, rtol=1e-13, atol=1e-13)
    assert (sel == sel2).all()
    # batch entries and heads are independent: run one (b, h) alone
    o1, l1, s1, _ = O.moba_dense(q[1:2, :, 3:4], k[1:2, :, 1:2], v[1:2, :, 1:2], B, topk, scale)
    assert np.allclose(o1[0, :, 0], out[1, :, 3], rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------------------
# merge identity (T7): softmax over a union of disjoint key sets equals the
# online-softmax merge of the per-set partials
# --------------------------------------------------------------------------
def test_merge_identity():
    rng = np.random.default_rng(9)
    d = 7
    q = _rand(d, rng)
    K = _rand((50, d), rng) * 3
    V = _rand((50, d), rng)
    full, lse_full = O.attend_row(q, K, V, 0.9)
    parts = [O.attend_row(q, K[s:e], V[s:e], 0.9) for s, e in [(0, 10), (10, 11), (11, 40), (40, 50)]]
    o, l = O.merge_partials(parts)
    assert np.allclose(o, full, rtol=1e-13, atol=1e-14)
    assert l == pytest.approx(lse_full, rel=1e-14)


# --------------------------------------------------------------------------
# FLOP accounting: closed form against a brute-force count of attended keys
# --------------------------------------------------------------------------
@pytest.mark.parametrize("N,B,topk", [(29, 4, 3), (64, 8, 12), (10, 10, 2), (7, 3, 1)])
def test_algorithmic_pairs_brute_force(N, B, topk):
    total = 0
    n = (N + B - 1) // B
    for t in range(N):
        sel, _ = O.select_blocks(np.arange(n, dtype=float), t, B, topk)
        total += len(O.key_positions(sel, t, B, N))
    assert O.algorithmic_pairs(2, N, 3, B, topk) == 2 * 3 * total


# --------------------------------------------------------------------------
# the FMA-pipe exponential used for part of the softmax (csrc/sm100.cuh,
# exp2_poly2, per lane): its fitted polynomial's relative error bound, checked in fp32
# arithmetic against the exact 2^x over the range the softmax uses
# --------------------------------------------------------------------------
def test_exp2_polynomial_error_bound():
    x = np.concatenate([np.linspace(-126.0, 8.0, 400001), -np.random.default_rng(0).random(100000) * 30])
    x = x.astype(np.float32)
    f32 = np.float32
    xc = np.maximum(x, f32(-126.0))
    r = (xc + f32(12582912.0)).astype(np.float32)
    f = (xc - (r - f32(12582912.0))).astype(np.float32)
    p = f32(0.05517206)
    for cst in (0.24261241, 0.69326101, 0.99992796):
        p = (p.astype(np.float64) * f + cst).astype(np.float32)       # fma: one rounding
    n = r.view(np.int32) - np.int32(0x4B400000)
    y = (p.view(np.int32) + (n << 23)).view(np.float32).astype(np.float64)
    ref = np.exp2(xc.astype(np.float64))
    normal = x >= -125.0
    rel = np.abs(y[normal] - ref[normal]) / ref[normal]
    assert rel.max() < 1e-4             # bf16 probabilities round at 2^-9 = 2e-3
    assert np.all((y[~normal] >= 0) & (y[~normal] < 1e-37))   # clamped tail: negligible, never negative
