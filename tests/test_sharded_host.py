"""The head-sharded layer (long_context_prefill_moba_b200/sharded.py): the head
partition, and the whole sharded layer on 2 and 4 gloo ranks on the CPU with
the fp64 oracle standing in for the per-rank GPU layer (a test double passed
as layer_factory).  K and V exist only on the source rank before the
exchange (a scatter of disjoint kv heads, or a send to each kv head's leader
and a broadcast in its subgroup); the ranks' head-sharded outputs, gathered in rank order, must
equal the unsharded oracle layer exactly, and so must dq; dK and dV, summed
onto the source rank by the backward (gathered, or reduced per kv head), must equal the unsharded
gradients up to the order of the sum."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from long_context_prefill_moba_b200.sharded import head_shard


@pytest.mark.parametrize("hq,hkv,world", [(32, 8, 2), (32, 8, 8), (4, 1, 2), (4, 1, 4), (8, 2, 4),
                                          (16, 4, 8), (6, 3, 3), (4, 4, 1)])
def test_head_shard_partitions_heads_and_keeps_each_query_on_its_kv_head(hq, hkv, world):
    G = hq // hkv
    covered = []
    for rank in range(world):
        h0, h1, g0, g1 = head_shard(hq, hkv, world, rank)
        assert h1 - h0 == hq // world
        covered.extend(range(h0, h1))
        Gl = (h1 - h0) // (g1 - g0)
        assert (h1 - h0) % (g1 - g0) == 0
        for i in range(h1 - h0):
            # the per-rank layer maps local head i to local kv head i // G_local
            assert (h0 + i) // G == g0 + i // Gl
    assert covered == list(range(hq))


@pytest.mark.parametrize("hq,hkv,world", [(4, 1, 8), (6, 2, 4), (4, 2, 3), (12, 4, 8)])
def test_head_shard_rejects_uneven_splits(hq, hkv, world):
    with pytest.raises(ValueError):
        head_shard(hq, hkv, world, 0)


class _OracleLayer:
    """Test double of MobaLayer: the fp64 oracle on the CPU."""

    def __init__(self, batch, seqlen, hq, hkv, head_dim, block, topk, dtype, scale, query_chunk, device):
        self.block, self.topk, self.scale = block, topk, scale

    def forward(self, q, k, v, out, lse=None, stream=None):
        import oracle as O
        o, l, _, _ = O.moba_dense(q.numpy(), k.numpy(), v.numpy(), self.block, self.topk, self.scale)
        out.copy_(torch.from_numpy(o))
        if lse is not None:
            lse.copy_(torch.from_numpy(l))
        return out

    def backward(self, q, k, v, out, lse, dout, dq, dk, dv, stream=None):
        from oracle import moba_backward as OB
        gq, gk, gv, _ = OB.moba_backward(q.numpy(), k.numpy(), v.numpy(), dout.numpy(), self.block, self.topk,
                                         self.scale)
        for dst, src in ((dq, gq), (dk, gk), (dv, gv)):
            dst.copy_(torch.from_numpy(src))


def _inputs(b, N, hq, hkv, d):
    g = torch.Generator().manual_seed(5)
    return (torch.randn(b, N, hq, d, generator=g, dtype=torch.float64),
            torch.randn(b, N, hkv, d, generator=g, dtype=torch.float64),
            torch.randn(b, N, hkv, d, generator=g, dtype=torch.float64))


def _worker(rank, world, port, shape, path, src=0):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import moba_synth as S
        from long_context_prefill_moba_b200.sharded import ShardedMobaLayer
        b, N, hq, hkv, d, B, topk = shape
        q, k, v = _inputs(b, N, hq, hkv, d)
        if rank != src:                          # only the source rank holds K/V before the exchange
            k, v = None, None
        cfg = S.get_config("tiny").replace(batch=b, seqlen=N, hq=hq, hkv=hkv, head_dim=d, block=B, topk=topk,
                                           scale=0.3)
        layer = ShardedMobaLayer.from_config(cfg, device="cpu", src=src, layer_factory=_OracleLayer)
        q_loc = q[:, :, layer.h0:layer.h1].contiguous()
        out_loc = torch.empty_like(q_loc)
        lse_loc = torch.empty(b, layer.h1 - layer.h0, N, dtype=torch.float64)
        layer.forward(q_loc, k, v, out_loc, lse_loc)
        outs = [torch.empty_like(out_loc) for _ in range(world)]
        lses = [torch.empty_like(lse_loc) for _ in range(world)]
        dist.all_gather(outs, out_loc)
        dist.all_gather(lses, lse_loc)
        # backward: local dq of this rank's heads; dK, dV summed onto the source rank
        g = torch.Generator().manual_seed(9)
        dout = torch.randn(b, N, hq, d, generator=g, dtype=torch.float64)
        dq_loc = torch.empty_like(q_loc)
        dk, dv = torch.empty(b, N, hkv, d, dtype=torch.float64), torch.empty(b, N, hkv, d, dtype=torch.float64)
        layer.backward(q_loc, out_loc, lse_loc, dout[:, :, layer.h0:layer.h1].contiguous(), dq_loc, dk, dv)
        dqs = [torch.empty_like(dq_loc) for _ in range(world)]
        dist.all_gather(dqs, dq_loc)
        if rank == src:
            torch.save({"out": torch.cat(outs, 2), "lse": torch.cat(lses, 1), "dq": torch.cat(dqs, 2),
                        "dk": dk, "dv": dv, "dout": dout}, path)
    finally:
        dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.mark.parametrize("shape,world,src", [
    ((1, 70, 4, 2, 8, 16, 3), 2, 0),     # kv heads split over the ranks (scatter / gather)
    ((1, 40, 8, 4, 8, 10, 3), 4, 2),     # one kv head per rank, the source not rank 0
    ((1, 70, 4, 1, 8, 16, 3), 2, 0),     # one kv head: its query heads split (the 10M layer's case)
    ((2, 45, 8, 2, 8, 10, 2), 4, 0),     # two ranks per kv head, two batch entries
    ((2, 45, 8, 2, 8, 10, 2), 4, 1),     # the same with a source that leads no subgroup
])
def test_sharded_layer_equals_the_unsharded_layer(tmp_path, shape, world, src):
    import oracle as O
    path = str(tmp_path / "gathered.pt")
    mp.start_processes(_worker, args=(world, _free_port(), shape, path, src), nprocs=world, join=True,
                       start_method="spawn")
    got = torch.load(path)
    b, N, hq, hkv, d, B, topk = shape
    q, k, v = _inputs(b, N, hq, hkv, d)
    out, lse, _, _ = O.moba_dense(q.numpy(), k.numpy(), v.numpy(), B, topk, 0.3)
    assert np.array_equal(got["out"].numpy(), out)
    assert np.array_equal(got["lse"].numpy(), lse)
    from oracle import moba_backward as OB
    dq, dk, dv, _ = OB.moba_backward(q.numpy(), k.numpy(), v.numpy(), got["dout"].numpy(), B, topk, 0.3)
    assert np.array_equal(got["dq"].numpy(), dq)
    # dK, dV: sums over ranks in another order than the unsharded loop
    assert np.abs(got["dk"].numpy() - dk).max() <= 1e-12
    assert np.abs(got["dv"].numpy() - dv).max() <= 1e-12
