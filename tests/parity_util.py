"""Helpers for the GPU parity tests: run the CUDA path through the binding and
compare with the fp64 oracle on the same seeded inputs (regenerated on the
CPU for the oracle, never taken from the GPU path)."""
from __future__ import annotations

import numpy as np
import torch

import moba_synth as S
import oracle as O

GAP_TOL = 1e-3          # selections may differ only where the oracle's score gap is below this


def out_tol(cfg) -> float:
    return 2e-2 if cfg.dtype == "bf16" else 1e-4


LSE_TOL = {"bf16": 2e-3, "f32": 1e-4}


def run_gpu(cfg, query_chunk=0, with_lse=True):
    import long_context_prefill_moba_b200 as M
    dev = torch.device("cuda:0")
    q, k, v = S.gen_q(cfg, dev), S.gen_k(cfg, dev), S.gen_v(cfg, dev)
    layer = M.MobaLayer.from_config(cfg, dev, query_chunk)
    out = torch.empty_like(q)
    lse = torch.empty(cfg.batch, cfg.hq, cfg.seqlen, dtype=torch.float32, device=dev) if with_lse else None
    layer.forward(q, k, v, out, lse)
    torch.cuda.synchronize()
    assert layer.device_status() == (0, 0)
    return dict(layer=layer, out=out, lse=lse, q=q, k=k, v=v)


def cpu(x):
    x = x.detach().cpu()
    return x.float() if x.dtype == torch.bfloat16 else x


def check_selection(sel_gpu_row, sel_or, gap, scores, t, B, topk):
    """Exact match unless the oracle's gap is below GAP_TOL; then the GPU set
    must still be a valid top-(topk-1) within GAP_TOL.  Returns the set to use
    for the output comparison."""
    got = [int(x) for x in sel_gpu_row if x >= 0]
    c = t // B
    assert got == sorted(got) and got[-1] == c and len(got) == min(topk, c + 1), (got, t)
    assert all(x >= 0 for x in sel_gpu_row[:len(got)]) and all(x == -1 for x in sel_gpu_row[len(got):])
    if gap is None or gap >= GAP_TOL:
        assert got == list(sel_or), (t, got, list(sel_or), gap)
        return got
    hist = [j for j in got if j != c]
    rest = [j for j in range(c) if j not in hist]
    if hist and rest:
        assert min(scores[j] for j in hist) >= max(scores[j] for j in rest) - GAP_TOL
    return got


def check_index(layer, cfg, sel):
    """offsets/rows group every (row, earlier selected block) by (pass, b, g, j)."""
    import long_context_prefill_moba_b200 as M
    s = layer.shape
    C = M.moba_query_chunk(s)
    n = cfg.nblocks
    nch = M.moba_num_chunks(s)
    sel = sel.reshape(cfg.batch, cfg.seqlen, cfg.hq, cfg.topk)
    b_i, t_i, h_i, slot = np.nonzero(sel >= 0)
    j = sel[b_i, t_i, h_i, slot]
    hist = j < (t_i // cfg.block)
    b_i, t_i, h_i, j = b_i[hist], t_i[hist], h_i[hist], j[hist]
    grp = (((t_i // C) * cfg.batch + b_i) * cfg.hkv + h_i // cfg.group) * n + j
    r = (b_i * cfg.seqlen + t_i) * cfg.hq + h_i
    counts = np.bincount(grp, minlength=nch * cfg.batch * cfg.hkv * n)
    exp_off = np.concatenate([[0], np.cumsum(counts)])
    off = layer.offsets.cpu().numpy().astype(np.int64)
    assert np.array_equal(off, exp_off)
    rows = layer.rows.cpu().numpy()[: len(r)].astype(np.int64)
    assert len(rows) == M.moba_rows_elems(s) == len(r)
    grp_of_pos = np.repeat(np.arange(len(counts)), counts)
    got = np.lexsort((rows, grp_of_pos))
    exp = np.lexsort((r, grp))
    assert np.array_equal(rows[got], r[exp])


def out_err(got, exp, cfg, rel=0.0):
    """max over elements of |got - exp| - rel * |exp| (<= out_tol(cfg) passes)."""
    return float((np.abs(got - exp) - rel * np.abs(exp)).max())


def full_parity(cfg, res, rel=0.0):
    """Whole-layer comparison with the dense-mask oracle (small configs).
    `rel` widens the output bound by rel * |expected| (see the large-score tests)."""
    q, k, v = S.gen_q(cfg), S.gen_k(cfg), S.gen_v(cfg)
    o_out, o_lse, o_sel, o_gap = O.moba_dense(q, k, v, cfg.block, cfg.topk, cfg.softmax_scale)
    layer = res["layer"]
    # mean-pool
    kbar_or = np.stack([np.stack([O.mean_pool(cpu(k[b, :, g]), cfg.block) for g in range(cfg.hkv)], 1)
                        for b in range(cfg.batch)])
    kbar = layer.meank_view().cpu().numpy()
    assert np.abs(kbar - kbar_or).max() <= 1e-5
    sel = layer.sel_view().cpu().numpy()
    out = cpu(res["out"]).numpy()
    lse = res["lse"].cpu().numpy() if res["lse"] is not None else None
    differ = np.nonzero((sel != o_sel).any(axis=-1))
    exp_out = o_out.copy()
    exp_lse = o_lse.copy()
    qd, kd, vd = (cpu(x).numpy().astype(np.float64) for x in (q, k, v))
    for b, t, h in zip(*differ):
        g = h // cfg.group
        scores = O.gate_scores(qd[b, t, h], kbar_or[b, :, g])
        used = check_selection(sel[b, t, h], [x for x in o_sel[b, t, h] if x >= 0], None
                               if np.isnan(o_gap[b, t, h]) else o_gap[b, t, h], scores, t, cfg.block,
                               cfg.topk)
        pos = O.key_positions(used, t, cfg.block, cfg.seqlen)
        exp_out[b, t, h], exp_lse[b, h, t] = O.attend_row(qd[b, t, h], kd[b, pos, g], vd[b, pos, g],
                                                          cfg.softmax_scale)
    err = out_err(out, exp_out, cfg, rel)
    assert err <= out_tol(cfg), err
    if lse is not None:
        assert np.abs(lse - exp_lse).max() <= LSE_TOL[cfg.dtype]
    check_index(layer, cfg, sel)
    return dict(max_err=float(err), n_gap_rows=len(differ[0]))


def sampled_rows(cfg, n_random, seed=0, chunk=0, max_pass_rows=16):
    """(b, h, t) rows: seeded random positions plus fixed ones: the block and
    sequence boundaries, a row of every regime with fewer earlier blocks than
    slots (c < topk - 1) and the last token of each such block, and (with the
    query pass length `chunk`) the first and last token of passes."""
    rng = np.random.default_rng(seed)
    B, N, k = cfg.block, cfg.seqlen, cfg.topk
    fixed_t = {0, B - 1, B, (k - 1) * B, N - 1, min(N - 1, (k - 2) * B + 7)}
    for c in range(min(k - 1, cfg.nblocks)):
        fixed_t |= {c * B + (37 * c + 5) % B, (c + 1) * B - 1}
    if chunk > 0:
        starts = list(range(chunk, N, chunk))
        if len(starts) > max_pass_rows // 2:
            pick = np.linspace(0, len(starts) - 1, max_pass_rows // 2).round().astype(int)
            starts = [starts[i] for i in sorted(set(pick.tolist()))]
        for p in starts:
            fixed_t |= {p - 1, p}
    rows = []
    for i, t in enumerate(sorted(x for x in fixed_t if 0 <= x < N)):
        rows.append((int(i % cfg.batch), int((7 * i) % cfg.hq), int(t)))
    for _ in range(n_random):
        rows.append((int(rng.integers(cfg.batch)), int(rng.integers(cfg.hq)), int(rng.integers(N))))
    return rows


def device_index_check(layer, exact=True):
    """moba_check_index on the layer's own gate index (every row, on the
    device); returns the status word (0 = valid)."""
    import long_context_prefill_moba_b200 as M
    status = torch.full((1,), -1, dtype=torch.int32, device=layer.device)
    M.moba_check_index(layer.shape, exact, layer.sel, layer.offsets, layer.rows, status)
    torch.cuda.synchronize()
    return int(status.item())


def sampled_parity(cfg, res, rows, rel=0.0):
    """Row-by-row comparison with the gather oracle on regenerated rows (`rel` as
    in full_parity)."""
    layer = res["layer"]
    sel_gpu = layer.sel_view()
    out_gpu = res["out"]
    lse_gpu = res["lse"]
    by_head = {}
    for b, h, t in rows:
        by_head.setdefault((b, h // cfg.group), []).append((h, t))
    worst = 0.0
    for (b, g), items in sorted(by_head.items()):
        K = S.gen_head_rows(cfg, "k", b, g)             # regenerated on the CPU
        kbar = O.mean_pool(K, cfg.block)
        kbar_gpu = layer.meank_view()[b, :, g].cpu().numpy()
        assert np.abs(kbar_gpu - kbar).max() <= 1e-5
        Vcache = {}
        for h, t in items:
            qrow = cpu(S.gen_rows(cfg, "q", b, t, t + 1, h))[0].numpy()
            scores = O.gate_scores(qrow, kbar)
            sel_or, gap = O.select_blocks(scores, t, cfg.block, cfg.topk)
            srow = sel_gpu[b, t, h].cpu().numpy()
            used = check_selection(srow, sel_or, gap, scores, t, cfg.block, cfg.topk)
            pos = O.key_positions(used, t, cfg.block, cfg.seqlen)
            for jb in used:
                if jb not in Vcache:
                    s0, e0 = O.block_range(jb, cfg.seqlen, cfg.block)
                    Vcache[jb] = cpu(S.gen_rows(cfg, "v", b, s0, e0, g)).numpy()
            c = t // cfg.block
            Vsel = np.concatenate([Vcache[jb][: t - jb * cfg.block + 1] if jb == c else Vcache[jb]
                                   for jb in used])
            Ksel = cpu(K[torch.from_numpy(pos)]).numpy()
            o, l = O.attend_row(qrow, Ksel, Vsel, cfg.softmax_scale)
            got = cpu(out_gpu[b, t, h]).numpy()
            err = out_err(got, o, cfg, rel)
            worst = max(worst, err)
            assert err <= out_tol(cfg), (b, h, t, err)
            if lse_gpu is not None:
                assert abs(float(lse_gpu[b, h, t]) - l) <= LSE_TOL[cfg.dtype], (b, h, t)
    return worst

