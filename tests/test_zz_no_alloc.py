"""The allocation-free gate entry point (moba_gate_topk_noalloc).

Some callers cannot give the library device scratch memory: a plain C host
program without a device allocator, or a serving runtime that reserves all
device memory at start-up and allows no later allocation.  For them the gate
has a variant whose counters live in a fixed device array inside the library.
This test calls it through the C ABI twice in a row and checks each result
against the regular moba_gate_topk on the same inputs: identical selections and
offsets, and identical query rows in every group (their order inside a group is
unspecified for both entry points).  After each call the gate's device status
word, read back into host memory with moba_gate_noalloc_status, is 0 (no bounded
wait gave up).  The file is named to run last."""
import numpy as np
import pytest
import torch

import moba_synth as S

pytestmark = pytest.mark.gpu


def _rows_by_group(offsets, rows):
    off = offsets.cpu().numpy().astype(np.int64)
    r = rows.cpu().numpy()[: off[-1]].astype(np.int64)
    grp = np.repeat(np.arange(len(off) - 1), np.diff(off))
    order = np.lexsort((r, grp))
    return r[order]


@pytest.mark.parametrize("name,chunk", [("ragged", 256), ("mqar", 0)])
def test_gate_noalloc_matches_gate(cuda_device, name, chunk):
    import long_context_prefill_moba_b200 as M
    if name == "ragged":
        cfg = S.get_config("mqar").replace(batch=2, seqlen=1000, hq=4, hkv=2, block=96, topk=3)
    else:
        cfg = S.get_config("mqar")
    dev = cuda_device
    layer = M.MobaLayer.from_config(cfg, dev, chunk)
    s = layer.shape
    q, k = S.gen_q(cfg, dev), S.gen_k(cfg, dev)
    M.moba_block_meanpool(s, k, layer.meank)
    M.moba_gate_topk(s, q, layer.meank, layer.sel, layer.offsets, layer.rows, layer.gate_ws)
    torch.cuda.synchronize()
    ref_sel = layer.sel.clone()
    ref_off = layer.offsets.clone()
    ref_rows = _rows_by_group(layer.offsets, layer.rows)
    for call in range(2):
        sel = torch.full_like(layer.sel, -7)
        off = torch.full_like(layer.offsets, -7)
        rows = torch.full_like(layer.rows, -7)
        M.moba_gate_topk_noalloc(s, q, layer.meank, sel, off, rows)
        torch.cuda.synchronize()
        assert torch.equal(sel, ref_sel), call
        assert torch.equal(off, ref_off), call
        assert np.array_equal(_rows_by_group(off, rows), ref_rows), call
        assert M.moba_gate_noalloc_status() == 0, call


def test_gate_noalloc_rejects_oversized_shapes():
    import ctypes
    import long_context_prefill_moba_b200 as M
    s = M.make_shape(batch=64, seqlen=1 << 20, hq=8, hkv=8, head_dim=128, block=64, topk=4,
                     query_chunk=1 << 20)
    assert M.moba_check_shape(s) == 0
    assert M.moba_offsets_elems(s) - 1 > (1 << 19)
    fake = ctypes.c_void_p(1 << 20)
    assert M.lib().moba_gate_topk_noalloc(ctypes.byref(s), fake, fake, fake, fake, fake, None) == 2
