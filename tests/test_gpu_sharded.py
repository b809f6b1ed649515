"""The head-sharded layer (long_context_prefill_moba_b200/sharded.py) with the
real per-rank MobaLayer on the GPU.

Two ranks run as two processes on cuda:0 over the gloo backend (collectives on
the CPU; the layer stages its CUDA tensors through host memory).  The ranks'
kernels never wait on one another: each rank runs the ordinary single-GPU layer
on its heads once K/V have arrived, so sharing one GPU only time-slices them.
Compared with the unsharded layer in the parent process, and through it with
the fp64 oracle:
  - kv heads split over the ranks (scatter of K/V, gather of dK/dV);
  - one kv head whose query heads the ranks split (the 10M layer's pattern,
    4 query heads on 1 kv head, B = 4096, top-12, 64K tokens): broadcast of
    K/V and an fp32 sum of dK/dV.
The forward outputs are those of the unsharded layer (the same kernels compute
each row the same way) and the oracle's on sampled rows; the gradients match
the unsharded layer's within bf16 rounding (each rank rounds its dK/dV share to
bf16 before the sum) and, on the small case, the fp64 backward oracle."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import moba_synth as S
from parity_util import cpu, run_gpu, sampled_parity, sampled_rows

pytestmark = pytest.mark.gpu

CASES = {
    "kv_split": (S.get_config("mqar").replace(batch=1, seqlen=2048, hq=8, hkv=2, block=256, topk=4), 2),
    "shared_kv_head": (S.get_config("10m").replace(seqlen=65536, block=4096), 2),
}


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, name, path):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from long_context_prefill_moba_b200.sharded import ShardedMobaLayer
        cfg, _ = CASES[name]
        dev = torch.device("cuda:0")
        torch.cuda.set_device(dev)
        layer = ShardedMobaLayer.from_config(cfg, device=dev, src=0)
        h0, h1 = layer.h0, layer.h1
        q_loc = S.gen_q(cfg, dev)[:, :, h0:h1].contiguous()
        k = S.gen_k(cfg, dev) if rank == 0 else None
        v = S.gen_v(cfg, dev) if rank == 0 else None
        out_loc = torch.empty_like(q_loc)
        lse_loc = torch.empty(cfg.batch, h1 - h0, cfg.seqlen, dtype=torch.float32, device=dev)
        stream = torch.cuda.Stream(dev)          # a stream other than the current one
        stream.wait_stream(torch.cuda.current_stream(dev))   # the inputs were made on the current one
        layer.forward(q_loc, k, v, out_loc, lse_loc, stream=stream)
        dout_loc = S.gen_dout(cfg, dev)[:, :, h0:h1].contiguous()
        stream.wait_stream(torch.cuda.current_stream(dev))
        dq_loc = torch.empty_like(q_loc)
        dk = torch.empty(cfg.batch, cfg.seqlen, cfg.hkv, cfg.head_dim, dtype=q_loc.dtype, device=dev)
        dv = torch.empty_like(dk)
        layer.backward(q_loc, out_loc, lse_loc, dout_loc, dq_loc, dk, dv, stream=stream)
        stream.synchronize()
        status = layer.layer.device_status()
        got = {}
        for key, t, dim in (("out", out_loc, 2), ("lse", lse_loc, 1), ("dq", dq_loc, 2)):
            parts = [torch.empty_like(t.cpu()) for _ in range(world)]
            dist.all_gather(parts, t.cpu())
            got[key] = torch.cat(parts, dim)
        stats = [None] * world
        dist.all_gather_object(stats, status)
        if rank == 0:
            got.update(dk=dk.cpu(), dv=dv.cpu(), status=stats)
            torch.save(got, path)
    finally:
        dist.destroy_process_group()


def _unsharded(cfg):
    res = run_gpu(cfg)
    layer = res["layer"]
    dout = S.gen_dout(cfg, res["q"].device)
    dq, dk, dv = torch.empty_like(res["q"]), torch.empty_like(res["k"]), torch.empty_like(res["v"])
    layer.backward(res["q"], res["k"], res["v"], res["out"], res["lse"], dout, dq, dk, dv)
    torch.cuda.synchronize()
    return res, dq, dk, dv


def _close(a, b, rel):
    a, b = cpu(a), cpu(b)
    return float((a - b).abs().max()) <= rel * max(1.0, float(b.abs().max()))


@pytest.mark.parametrize("name", sorted(CASES))
def test_sharded_layer_on_the_gpu(cuda_device, tmp_path, name):
    cfg, world = CASES[name]
    path = str(tmp_path / "sharded.pt")
    mp.start_processes(_worker, args=(world, _free_port(), name, path), nprocs=world, join=True,
                       start_method="spawn")
    got = torch.load(path)
    assert all(s == (0, 0) for s in got["status"]), got["status"]
    res, dq, dk, dv = _unsharded(cfg)
    out_ref, lse_ref = cpu(res["out"]), res["lse"].cpu()
    identical = torch.equal(got["out"].float(), out_ref) and torch.equal(got["lse"], lse_ref)
    print(name, "sharded forward bitwise identical to the unsharded layer:", identical)
    assert _close(got["out"], out_ref, 2e-2) and _close(got["lse"], lse_ref, 2e-3)
    # the unsharded layer (and so the sharded one) against the oracle
    worst = sampled_parity(cfg, res, sampled_rows(cfg, 48, seed=7))
    print(name, "oracle worst", worst)
    assert _close(got["dq"], dq, 2e-2)
    assert _close(got["dk"], dk, 3e-2) and _close(got["dv"], dv, 3e-2)
    if cfg.seqlen <= 4096:
        from oracle import moba_backward as OB
        sel = res["layer"].sel_view().cpu().numpy()
        rq, rk, rv = OB.moba_backward_dense(S.gen_q(cfg), S.gen_k(cfg), S.gen_v(cfg), S.gen_dout(cfg), sel,
                                            cfg.block, cfg.softmax_scale)
        for g, r in ((got["dq"], rq), (got["dk"], rk), (got["dv"], rv)):
            err = float(np.abs(cpu(g).numpy() - r).max())
            assert err <= 3e-2 * max(1.0, float(np.abs(r).max())), err
