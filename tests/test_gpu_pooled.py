"""The gate variant that also routes the top blocks by max- and min-pooled keys
(moba_block_maxminpool, moba_gate_pooled, moba_attn_fwd_pooled) against the
fp64 oracle (oracle/moba_pooled_gate.py) on the same seeded inputs: the pools
exactly, the selections exactly unless one of the three rankings has an fp64
score gap below GAP_TOL at its cut, the query-per-block index exactly, and the
layer's out and lse within the dtype's tolerance.  Cases cover every attention
path (tensor-core bf16 d=128, mma bf16 d=64, fp32), several passes, ragged
last blocks, GQA, topk = 1, extra = 0 and a width that selects every block."""
import numpy as np
import pytest
import torch

import moba_synth as S
import oracle as O
from oracle import moba_pooled_gate as P
from parity_util import GAP_TOL, LSE_TOL, cpu, out_tol

pytestmark = pytest.mark.gpu

CASES = {
    # tensor-core attention, five passes, GQA 2, ragged last block, W = 7
    "bf16_d128_multipass": (S.get_config("mqar").replace(batch=1, seqlen=1100, hq=4, hkv=2, block=64,
                                                         topk=3), 2, 256),
    # mma attention (head_dim 64), two batch entries, MQA, W = 4
    "bf16_d64_mqa": (S.get_config("mqar").replace(batch=2, seqlen=700, hq=4, hkv=1, head_dim=64,
                                                  block=48, topk=2), 1, 128),
    # fp32 CUDA-core attention, W = 10, GQA 2
    "f32_wide": (S.get_config("tiny").replace(batch=1, seqlen=600, hq=4, hkv=2, block=40, topk=4), 3, 0),
    # no mean slot: only the max and min rankings route earlier blocks
    "topk_one": (S.get_config("mqar").replace(batch=1, seqlen=600, hq=2, hkv=2, block=64, topk=1), 2, 128),
    # extra = 0: the plain gate computed by the variant's kernels
    "extra_zero": (S.get_config("mqar").replace(batch=1, seqlen=700, hq=2, hkv=1, block=64, topk=4), 0, 256),
    # extra >= n - 1: the max ranking alone routes every earlier block (dense causal)
    "every_block": (S.get_config("tiny").replace(batch=1, seqlen=300, hq=2, hkv=1, block=50, topk=4), 5, 128),
    # 128 blocks (four mask words per row on the tensor-core gate) and gate scores in the
    # hundreds (q std 8, key offsets of std 4), W = 12
    "bf16_many_blocks_large_scores": (S.get_config("mqar").replace(batch=1, seqlen=2048, hq=4, hkv=2, block=16,
                                                                   topk=8, q_std=8.0, offset_std=4.0), 2, 1024),
}
# outputs of the large-score case sit at |out| ~ 4, where a bf16 output's own
# rounding is 0.0156: its bound adds 2^-8 |expected| (as in test_gpu_parity.py)
REL = {"bf16_many_blocks_large_scores": 2.0 ** -8}


def run_pooled(cfg, extra, chunk):
    import long_context_prefill_moba_b200 as M
    dev = torch.device("cuda:0")
    q, k, v = S.gen_q(cfg, dev), S.gen_k(cfg, dev), S.gen_v(cfg, dev)
    layer = M.MobaPooledLayer.from_config(cfg, extra, dev, chunk)
    out = torch.empty_like(q)
    lse = torch.empty(cfg.batch, cfg.hq, cfg.seqlen, dtype=torch.float32, device=dev)
    layer.forward(q, k, v, out, lse)
    torch.cuda.synchronize()
    assert layer.device_status() == (0, 0)
    assert layer.launches > 0
    return layer, out, lse


def cut_gap(scores, m):
    """Gap between the m-th and (m+1)-th best of `scores` (None: no cut)."""
    if m <= 0 or m >= len(scores):
        return None
    s = np.sort(scores)[::-1]
    return s[m - 1] - s[m]


def check_index(layer, cfg, sel, W):
    import long_context_prefill_moba_b200 as M
    C = M.moba_query_chunk(layer.wide)
    n = cfg.nblocks
    nch = M.moba_num_chunks(layer.wide)
    b_i, t_i, h_i, slot = np.nonzero(sel >= 0)
    j = sel[b_i, t_i, h_i, slot]
    hist = j < (t_i // cfg.block)
    b_i, t_i, h_i, j = b_i[hist], t_i[hist], h_i[hist], j[hist]
    grp = (((t_i // C) * cfg.batch + b_i) * cfg.hkv + h_i // cfg.group) * n + j
    r = (b_i * cfg.seqlen + t_i) * cfg.hq + h_i
    counts = np.bincount(grp, minlength=nch * cfg.batch * cfg.hkv * n)
    off = layer.offsets.cpu().numpy().astype(np.int64)
    assert np.array_equal(off, np.concatenate([[0], np.cumsum(counts)]))
    assert off[-1] <= M.moba_rows_elems(layer.wide)
    rows = layer.rows.cpu().numpy()[: off[-1]].astype(np.int64)
    grp_of_pos = np.repeat(np.arange(len(counts)), counts)
    assert np.array_equal(np.stack([grp_of_pos, rows])[:, np.lexsort((rows, grp_of_pos))],
                          np.stack([grp, r])[:, np.lexsort((r, grp))])


@pytest.mark.parametrize("name", sorted(CASES))
def test_pooled_gate_layer_parity(cuda_device, name):
    cfg, extra, chunk = CASES[name]
    layer, out, lse = run_pooled(cfg, extra, chunk)
    W = cfg.topk + 2 * extra
    q, k, v = (x.double().numpy() for x in (cpu(S.gen_q(cfg)), cpu(S.gen_k(cfg)), cpu(S.gen_v(cfg))))

    # the pools, exactly
    mean_g, max_g, min_g = (x.cpu().numpy() for x in layer.pool_views())
    for b in range(cfg.batch):
        for g in range(cfg.hkv):
            assert np.array_equal(max_g[b, :, g].astype(np.float64), P.max_pool(k[b, :, g], cfg.block))
            assert np.array_equal(min_g[b, :, g].astype(np.float64), P.min_pool(k[b, :, g], cfg.block))
            assert np.abs(mean_g[b, :, g] - O.mean_pool(k[b, :, g], cfg.block)).max() <= 1e-5

    o_out, o_lse, o_sels = P.moba_pooled_layer(q, k, v, cfg.block, cfg.topk, extra, cfg.softmax_scale)
    sel = layer.sel_view().cpu().numpy()
    check_index(layer, cfg, sel, W)

    same = np.zeros((cfg.batch, cfg.seqlen, cfg.hq), dtype=bool)
    near = 0
    for b in range(cfg.batch):
        pools = [(O.mean_pool(k[b, :, g], cfg.block), P.max_pool(k[b, :, g], cfg.block),
                  P.min_pool(k[b, :, g], cfg.block)) for g in range(cfg.hkv)]
        for h in range(cfg.hq):
            kbar, kmax, kmin = pools[h // cfg.group]
            sa, sx, sn = q[b, :, h] @ kbar.T, q[b, :, h] @ kmax.T, q[b, :, h] @ kmin.T
            for t in range(cfg.seqlen):
                c = t // cfg.block
                row = [int(x) for x in sel[b, t, h]]
                got = [x for x in row if x >= 0]
                # structure: ascending, the current block last, -1 padding, within the width
                assert got == sorted(set(got)) and got[-1] == c, (name, t, row)
                assert all(x == -1 for x in row[len(got):])
                assert min(cfg.topk, c + 1) <= len(got) <= min(W, c + 1)
                want = o_sels[(b, t, h)]
                gaps = [cut_gap(sa[t, :c], cfg.topk - 1), cut_gap(sx[t, :c], extra),
                        cut_gap(sn[t, :c], extra)]
                tight = min([x for x in gaps if x is not None], default=np.inf) < GAP_TOL
                if got == want:
                    same[b, t, h] = True
                else:
                    assert tight, (name, b, t, h, got, want, gaps)
                    near += 1
    assert same.mean() > 0.98, (name, same.mean())
    o = cpu(out).double().numpy()
    err = (np.abs(o - o_out) - REL.get(name, 0.0) * np.abs(o_out))[same].max()
    lerr = np.abs(lse.cpu().double().numpy().transpose(0, 2, 1) - o_lse.transpose(0, 2, 1))[same].max()
    print(name, "max abs err", err, "lse err", lerr, "near-tie rows", near)
    assert err <= out_tol(cfg), (name, err)
    assert lerr <= LSE_TOL[cfg.dtype], (name, lerr)


def test_pooled_extra_zero_selects_like_the_plain_gate(cuda_device):
    # with extra = 0 the variant's selection is the plain gate's, up to near-ties
    import long_context_prefill_moba_b200 as M
    cfg, _, chunk = CASES["extra_zero"]
    layer, out, _ = run_pooled(cfg, 0, chunk)
    dev = torch.device("cuda:0")
    plain = M.MobaLayer.from_config(cfg, dev, chunk)
    q, k, v = S.gen_q(cfg, dev), S.gen_k(cfg, dev), S.gen_v(cfg, dev)
    out_p = torch.empty_like(q)
    plain.forward(q, k, v, out_p)
    torch.cuda.synchronize()
    a, b = layer.sel_view().cpu().numpy(), plain.sel_view().cpu().numpy()
    rows_same = (a == b).all(-1)
    assert rows_same.mean() > 0.98
    d = (out.float() - out_p.float()).abs().cpu().numpy()[rows_same].max()
    assert d <= out_tol(cfg)


@pytest.mark.parametrize("name", ["bf16_d128_multipass", "bf16_d64_mqa", "f32_wide"])
def test_pooled_backward_with_the_selection_fixed(cuda_device, name):
    # the variant's backward is moba_attn_bwd at the wide shape; reference: the
    # backward oracle with the GPU gate's (variable-length) selection
    from oracle import moba_backward as OB
    cfg, extra, chunk = CASES[name]
    layer, out, lse = run_pooled(cfg, extra, chunk)
    dev = torch.device("cuda:0")
    q, k, v, dout = S.gen_q(cfg, dev), S.gen_k(cfg, dev), S.gen_v(cfg, dev), S.gen_dout(cfg, dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    layer.backward(q, k, v, out, lse, dout, dq, dk, dv)
    torch.cuda.synchronize()
    assert layer.bwd_ws[:4].view(torch.int32).item() == 0 and layer.launches > 0
    sel = layer.sel_view().cpu().numpy()
    rq, rk, rv, _ = OB.moba_backward(S.gen_q(cfg), S.gen_k(cfg), S.gen_v(cfg), S.gen_dout(cfg), cfg.block,
                                     cfg.topk + 2 * extra, cfg.softmax_scale, sel=sel)
    for name_, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        err = float(np.abs(cpu(got).numpy() - ref).max())
        bound = (3e-2 if cfg.dtype == "bf16" else 2e-4) * max(1.0, float(np.abs(ref).max()))
        print(name, name_, "max abs err", err, "max |ref|", float(np.abs(ref).max()))
        assert err <= bound, (name, name_, err)
