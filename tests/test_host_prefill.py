"""The whole layer from host buffers (moba_prefill_host): pass-by-pass gate and
attention with the copies overlapped.  Its outputs are checked against the
fp64 oracle with the selection and index of the device-buffer path (the gate
is deterministic, so both paths select the same blocks)."""
import pytest
import torch

import moba_synth as S
from parity_util import full_parity, out_tol, run_gpu, sampled_parity, sampled_rows

pytestmark = pytest.mark.gpu

FULL = {
    # several passes, GQA 2, a block that is not a multiple of the key tile
    "ragged_multipass": (S.get_config("mqar").replace(batch=2, seqlen=1000, hq=4, hkv=2, block=96,
                                                      topk=3), 256),
    # fp32 with head_dim 128, several passes
    "f32_d128_multipass": (S.get_config("tiny").replace(batch=1, seqlen=600, hq=2, hkv=1, head_dim=128,
                                                        block=64, topk=5), 128),
    # fp32, ragged, one pass
    "f32_ragged_gqa": (S.get_config("tiny").replace(batch=2, seqlen=333, hq=4, hkv=2, block=40, topk=4), 0),
    # no historical block at all (the gate routes only the current block)
    "topk_one": (S.get_config("mqar").replace(batch=1, seqlen=700, hq=2, hkv=2, block=64, topk=1), 256),
    # sequence shorter than one block
    "seq_shorter_than_block": (S.get_config("mqar").replace(batch=1, seqlen=100, hq=2, hkv=1, block=256,
                                                            topk=4), 0),
}


def run_host(cfg, query_chunk=0, pinned=True, with_lse=True):
    import long_context_prefill_moba_b200 as M
    q, k, v = S.gen_q(cfg), S.gen_k(cfg), S.gen_v(cfg)      # host tensors, same seeds as the device run
    out = torch.empty_like(q)
    lse = torch.empty(cfg.batch, cfg.hq, cfg.seqlen, dtype=torch.float32) if with_lse else None
    if pinned:
        q, k, v, out = (x.pin_memory() for x in (q, k, v, out))
        lse = lse.pin_memory() if lse is not None else None
    layer = M.MobaHostLayer.from_config(cfg, "cuda:0", query_chunk, with_lse=with_lse)
    layer.forward(q, k, v, out, lse)
    torch.cuda.synchronize()
    assert layer.device_status() == (0, 0)
    assert layer.launches > 0
    return out, lse


@pytest.mark.parametrize("name", sorted(FULL))
def test_host_prefill_full_parity(cuda_device, name):
    cfg, chunk = FULL[name]
    dev = run_gpu(cfg, query_chunk=chunk)
    out, lse = run_host(cfg, chunk)
    # the host run's outputs against the oracle, with the device run's gate
    info = full_parity(cfg, dict(dev, out=out, lse=lse))
    print(name, info)
    assert (out.float() - dev["out"].cpu().float()).abs().max().item() <= out_tol(cfg)
    assert (lse - dev["lse"].cpu()).abs().max().item() <= (2e-3 if cfg.dtype == "bf16" else 1e-4)


def test_host_prefill_pageable_and_without_lse(cuda_device):
    cfg, chunk = FULL["ragged_multipass"]
    out_p, _ = run_host(cfg, chunk, pinned=True)
    out_u, lse_u = run_host(cfg, chunk, pinned=False, with_lse=False)
    assert lse_u is None
    assert (out_p.float() - out_u.float()).abs().max().item() <= out_tol(cfg)


def test_host_prefill_mid_size_sampled(cuda_device):
    # five passes, GQA 4, two batch entries on the tensor-core paths
    cfg = S.get_config("1m").replace(batch=2, seqlen=20000, block=1024, topk=5)
    dev = run_gpu(cfg, query_chunk=4096)
    out, lse = run_host(cfg, 4096)
    worst = sampled_parity(cfg, dict(dev, out=out.cuda(), lse=lse.cuda()), sampled_rows(cfg, 48, seed=3))
    print("worst", worst)
