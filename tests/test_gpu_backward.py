"""GPU parity of the backward pass (moba_attn_bwd) against the fp64 oracle
(oracle/moba_backward.py) on the same seeded inputs, with the GPU gate's
selection (selection parity is covered by the forward tests)."""
import numpy as np
import pytest
import torch

import moba_synth as S
from oracle import moba_backward as OB
from parity_util import cpu, run_gpu

pytestmark = pytest.mark.gpu

CASES = {
    # bf16, several passes, GQA 2, a block that is not a multiple of 128
    "ragged_multipass": (S.get_config("mqar").replace(batch=2, seqlen=1000, hq=4, hkv=2, block=96,
                                                      topk=3), 256),
    "d64_bf16": (S.get_config("mqar").replace(batch=1, seqlen=777, hq=8, hkv=2, head_dim=64, block=128,
                                              topk=4), 0),
    "topk_one": (S.get_config("mqar").replace(batch=1, seqlen=700, hq=2, hkv=2, block=64, topk=1), 0),
    "seq_shorter_than_block": (S.get_config("mqar").replace(batch=1, seqlen=100, hq=2, hkv=1, block=256,
                                                            topk=4), 0),
    # fp32: tight tolerance
    "f32_d128_multipass": (S.get_config("tiny").replace(batch=1, seqlen=600, hq=2, hkv=1, head_dim=128,
                                                        block=64, topk=5), 128),
    "f32_ragged_gqa": (S.get_config("tiny").replace(batch=2, seqlen=333, hq=4, hkv=2, block=40, topk=4), 0),
    # tensor-core path with several row tiles per key tile and four passes
    "bf16_multitile": (S.get_config("mqar").replace(batch=1, seqlen=4096, hq=8, hkv=2, block=512, topk=4),
                       1024),
    # eight query heads on one kv head (GQA 8) on tensor cores
    "gqa8_bf16": (S.get_config("mqar").replace(batch=1, seqlen=1024, hq=8, hkv=1, block=64, topk=5), 384),
    # one-token blocks: every key tile straddles many blocks
    "block_one": (S.get_config("mqar").replace(batch=1, seqlen=200, hq=2, hkv=1, block=1, topk=3), 0),
}


def tol(cfg, ref):
    scale = max(1.0, float(np.abs(ref).max()))
    return (3e-2 if cfg.dtype == "bf16" else 2e-4) * scale


def run_backward(cfg, chunk):
    import long_context_prefill_moba_b200 as M
    res = run_gpu(cfg, query_chunk=chunk, with_lse=True)
    layer = res["layer"]
    dout = S.gen_dout(cfg, res["q"].device)
    dq, dk, dv = torch.empty_like(res["q"]), torch.empty_like(res["k"]), torch.empty_like(res["v"])
    layer.backward(res["q"], res["k"], res["v"], res["out"], res["lse"], dout, dq, dk, dv)
    torch.cuda.synchronize()
    assert layer.launches > 0
    return res, dq, dk, dv


@pytest.mark.parametrize("name", sorted(CASES))
def test_backward_parity(cuda_device, name):
    cfg, chunk = CASES[name]
    res, dq, dk, dv = run_backward(cfg, chunk)
    sel = res["layer"].sel_view().cpu().numpy()
    q, k, v, dout = S.gen_q(cfg), S.gen_k(cfg), S.gen_v(cfg), S.gen_dout(cfg)
    if cfg.seqlen > 2048:
        # the dense-mask formulation (pinned against the gather one) is the fast one at this size
        rq, rk, rv = OB.moba_backward_dense(q, k, v, dout, sel, cfg.block, cfg.softmax_scale)
    else:
        rq, rk, rv, _ = OB.moba_backward(q, k, v, dout, cfg.block, cfg.topk, cfg.softmax_scale, sel=sel)
    for name_, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        err = float(np.abs(cpu(got).numpy() - ref).max())
        print(name, name_, "max abs err", err, "max |ref|", float(np.abs(ref).max()))
        assert err <= tol(cfg, ref), (name_, err)


def test_dense_special_case_backward_matches_autograd(cuda_device):
    # top-k >= n: MoBA is dense causal attention, so its gradients are those of
    # torch's causal SDPA (autograd in fp32 on the same bf16 inputs)
    cfg = S.get_config("mqar").replace(batch=1, seqlen=640, hq=4, hkv=2, block=64, topk=16)
    res, dq, dk, dv = run_backward(cfg, 0)
    rep = cfg.hq // cfg.hkv
    q = res["q"].float().transpose(1, 2).detach().requires_grad_(True)
    k = res["k"].float().detach().requires_grad_(True)
    v = res["v"].float().detach().requires_grad_(True)
    out = torch.nn.functional.scaled_dot_product_attention(
        q, k.repeat_interleave(rep, 2).transpose(1, 2), v.repeat_interleave(rep, 2).transpose(1, 2),
        is_causal=True, scale=cfg.softmax_scale)
    dout = S.gen_dout(cfg, res["q"].device).float().transpose(1, 2)
    (out * dout).sum().backward()
    for name_, got, ref in (("dq", dq.float(), q.grad.transpose(1, 2)), ("dk", dk.float(), k.grad),
                            ("dv", dv.float(), v.grad)):
        err = (got - ref).abs().max().item()
        assert err <= 3e-2 * max(1.0, ref.abs().max().item()), (name_, err)


@pytest.mark.parametrize("name", ["ragged_multipass", "d64_bf16"])
def test_backward_is_reproducible(cuda_device, name):
    # dk, dv are written once per key: for one gate index they are bitwise the
    # same; dq too on the CUDA-core path (d64), within rounding on tensor cores
    cfg, chunk = CASES[name]
    res, dq1, dk1, dv1 = run_backward(cfg, chunk)
    dout = S.gen_dout(cfg, res["q"].device)
    dq2, dk2, dv2 = torch.empty_like(dq1), torch.empty_like(dk1), torch.empty_like(dv1)
    res["layer"].backward(res["q"], res["k"], res["v"], res["out"], res["lse"], dout, dq2, dk2, dv2)
    torch.cuda.synchronize()
    assert torch.equal(dk1, dk2) and torch.equal(dv1, dv2)
    if cfg.head_dim != 128:
        assert torch.equal(dq1, dq2)
    else:
        assert (dq1.float() - dq2.float()).abs().max().item() <= 1e-2


def test_autograd_op_matches_the_layer_backward(cuda_device):
    import long_context_prefill_moba_b200 as M
    cfg, chunk = CASES["ragged_multipass"]
    res, dq, dk, dv = run_backward(cfg, chunk)
    q, k, v = (res[x].detach().clone().requires_grad_(True) for x in ("q", "k", "v"))
    out = M.moba_attention(q, k, v, cfg.block, cfg.topk, query_chunk=chunk)
    # a fresh gate may order rows inside a group differently: equal up to rounding
    assert (out.float() - res["out"].float()).abs().max().item() <= 1e-2
    out.backward(S.gen_dout(cfg, q.device))
    torch.cuda.synchronize()
    for got, ref in ((q.grad, dq), (k.grad, dk), (v.grad, dv)):
        assert (got.float() - ref.float()).abs().max().item() <= 1e-2
