"""moba_check_index on the device: it accepts the gate's own index and rejects
an index with a fault planted on the host, making it inert.

The faults are made in host copies of sel/offsets/rows (never by a kernel) and
each stays inside the arrays' bounds: the checks only read the index, and read a
rows entry's sel row only after the entry has been found to be a row id of the
shape, so a corrupted index cannot make them read out of bounds."""
import numpy as np
import pytest
import torch

import moba_synth as S

pytestmark = pytest.mark.gpu

CFG = S.get_config("mqar").replace(batch=2, seqlen=1000, hq=4, hkv=2, block=96, topk=3)
CHUNK = 256


def _gate_index(dev):
    import long_context_prefill_moba_b200 as M
    layer = M.MobaLayer.from_config(CFG, dev, CHUNK)
    q, k = S.gen_q(CFG, dev), S.gen_k(CFG, dev)
    M.moba_block_meanpool(layer.shape, k, layer.meank)
    M.moba_gate_topk(layer.shape, q, layer.meank, layer.sel, layer.offsets, layer.rows, layer.gate_ws)
    torch.cuda.synchronize()
    return layer


def _check(layer, sel, off, rows, exact=True):
    import long_context_prefill_moba_b200 as M
    status = torch.full((1,), -1, dtype=torch.int32, device=sel.device)
    M.moba_check_index(layer.shape, exact, sel, off, rows, status)
    torch.cuda.synchronize()
    return int(status.item())


def test_accepts_the_gate_index(cuda_device):
    layer = _gate_index(cuda_device)
    sel, off, rows = layer.sel.clone(), layer.offsets.clone(), layer.rows.clone()
    assert _check(layer, sel, off, rows, exact=True) == 0
    assert _check(layer, sel, off, rows, exact=False) == 0
    # a passing check leaves the index as it was
    assert torch.equal(sel, layer.sel) and torch.equal(off, layer.offsets)


def _plant(name, sel, off, rows):
    """Fault `name` in host arrays sel [b, N, hq, topk], off, rows (in place)."""
    B = CFG.block
    if name == "future_block":
        t = 5 * B + 3                      # c = 5: put block 7 in its row
        sel[0, t, 1, :] = [2, 5, 7]
    elif name == "missing_current_block":
        t = 4 * B + 1
        sel[1, t, 0, :] = [0, 3, -1]
    elif name == "descending_row":
        t = 6 * B
        sel[0, t, 2, :] = [4, 1, 6]
    elif name == "row_id_out_of_range":
        rows[int(off[3]) if off[4] > off[3] else 0] = CFG.batch * CFG.seqlen * CFG.hq + 11
    elif name == "negative_row_id":
        rows[0] = -3
    elif name == "decreasing_offsets":
        i = int(np.nonzero(np.diff(off) > 0)[0][2]) + 1
        off[i] = off[i - 1] - 1
    elif name == "offsets_beyond_capacity":
        off[-1] = len(rows) + 5
    elif name == "row_in_wrong_group":
        # a rows entry whose group's block is not in the row's selection
        g0 = int(np.nonzero(np.diff(off) > 0)[0][0])
        r = int(rows[off[g0]])
        t = (r // CFG.hq) % CFG.seqlen
        j = g0 % CFG.nblocks
        h = r % CFG.hq
        b = r // (CFG.hq * CFG.seqlen)
        c = t // B
        sel[b, t, h, :] = [x for x in range(c) if x != j][:CFG.topk - 1] + [c]
    else:
        raise ValueError(name)


FAULTS = ["future_block", "missing_current_block", "descending_row", "row_id_out_of_range",
          "negative_row_id", "decreasing_offsets", "offsets_beyond_capacity", "row_in_wrong_group"]


@pytest.mark.parametrize("name", FAULTS)
def test_rejects_planted_fault_and_makes_index_inert(cuda_device, name):
    layer = _gate_index(cuda_device)
    sel = layer.sel_view().cpu().numpy().copy()
    off = layer.offsets.cpu().numpy().copy()
    rows = layer.rows.cpu().numpy().copy()
    _plant(name, sel, off, rows)
    d_sel = torch.from_numpy(sel.reshape(-1)).to(cuda_device)
    d_off = torch.from_numpy(off).to(cuda_device)
    d_rows = torch.from_numpy(rows).to(cuda_device)
    # the membership fault leaves a shorter (valid) sel row: check it with the
    # length rule relaxed so that the membership check is the one that fires
    exact = name != "row_in_wrong_group"
    assert _check(layer, d_sel, d_off, d_rows, exact) == 5   # MOBA_ERR_INTERNAL
    # inert: no group has rows, every sel row is just its own block
    assert int(d_off.abs().max().item()) == 0
    got = d_sel.view(CFG.batch, CFG.seqlen, CFG.hq, CFG.topk).cpu().numpy()
    cur = (np.arange(CFG.seqlen) // CFG.block)[None, :, None]
    assert (got[..., 0] == cur).all() and (got[..., 1:] == -1).all()
