"""Head-sharded MoBA layer over the ranks of a process group (one GPU each).

"MoBA: Mixture of Block Attention for Long-Context LLMs", paper-graph summary,
Implementation, "Why this implementation is efficient" (the paper's §3.4, the
10M-token runs): tensor parallelism is extended to the query-head level, and
the key and value tensors are broadcast to the GPUs that hold the query heads,
so every GPU runs the layer for its own heads over the whole sequence.

Nothing else crosses GPUs: every query head selects its own blocks from its
own kv head's pooled keys, so once K/V are in place the per-rank layers are
independent (the same MobaLayer kernels on a slice of the heads).  The query
rows and the output stay sharded by head, as in tensor-parallel attention.

Partition (``head_shard``), P ranks, G = hq / hkv query heads per kv head:
  - hkv % P == 0: rank r owns kv heads [r hkv/P, (r+1) hkv/P) with all their
    query heads;
  - otherwise P % hkv == 0 and G % (P / hkv) == 0: the P / hkv ranks sharing a
    kv head split its G query heads into equal contiguous runs (the 10M layer,
    4 query heads on 1 kv head, runs on 2 or 4 ranks this way).
Any other (hq, hkv, P) is rejected.

K and V arrive by one broadcast each from the source rank, for the whole
[b, N, hkv, d] tensors; each rank then copies out its own kv heads.  In the
backward, each rank computes its query heads' gradients locally and the
adjoint of the broadcast, a sum-reduce onto the source rank, assembles dK and
dV (ranks that share a kv head add their contributions).  The
compute runs in the library's kernels (``MobaLayer``); ``layer_factory``
exists so the host logic can be exercised on ranks without a GPU.
"""
from __future__ import annotations

from typing import Callable, Optional, Tuple

import torch
import torch.distributed as dist

__all__ = ["head_shard", "ShardedMobaLayer"]


def head_shard(hq: int, hkv: int, world: int, rank: int) -> Tuple[int, int, int, int]:
    """(h0, h1, g0, g1): rank `rank` of `world` owns query heads [h0, h1) and kv
    heads [g0, g1); raises ValueError when the heads do not split evenly."""
    if world < 1 or not 0 <= rank < world or hq % hkv != 0:
        raise ValueError(f"bad partition request: hq={hq} hkv={hkv} world={world} rank={rank}")
    G = hq // hkv
    if hkv % world == 0:
        per = hkv // world
        return rank * per * G, (rank + 1) * per * G, rank * per, (rank + 1) * per
    if world % hkv == 0 and G % (world // hkv) == 0:
        split = world // hkv              # ranks per kv head
        g = rank // split
        run = G // split
        h0 = g * G + (rank % split) * run
        return h0, h0 + run, g, g + 1
    raise ValueError(f"{hq} query heads on {hkv} kv heads do not split over {world} ranks")


class ShardedMobaLayer:
    """One MoBA layer shape whose heads are split over the ranks of `group`.

    ``forward(q_local, k, v, out_local, lse_local=None)``: `q_local` /
    `out_local` [b, N, h1-h0, d] hold this rank's query heads; `k` and `v`
    [b, N, hkv, d] hold the layer's full K/V on the source rank and are
    receive buffers of that shape elsewhere (overwritten by the broadcast)."""

    def __init__(self, batch, seqlen, hq, hkv, head_dim, block, topk, dtype="bf16", scale=None,
                 query_chunk=0, device="cuda", group=None, src: int = 0,
                 layer_factory: Optional[Callable] = None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.src = src
        self.h0, self.h1, self.g0, self.g1 = head_shard(hq, hkv, self.world, self.rank)
        if layer_factory is None:
            from . import MobaLayer
            layer_factory = MobaLayer
        # a query head keeps its kv head: local head i reads local kv head i // G_local
        self.layer = layer_factory(batch, seqlen, self.h1 - self.h0, self.g1 - self.g0, head_dim, block,
                                   topk, dtype, scale, query_chunk, device)

    @classmethod
    def from_config(cls, cfg, device="cuda", query_chunk=0, group=None, src=0, layer_factory=None):
        return cls(cfg.batch, cfg.seqlen, cfg.hq, cfg.hkv, cfg.head_dim, cfg.block, cfg.topk, cfg.dtype,
                   cfg.scale, query_chunk, device, group, src, layer_factory)

    def broadcast_kv(self, k: torch.Tensor, v: torch.Tensor):
        """K/V of the source rank to every rank; returns this rank's kv heads."""
        dist.broadcast(k, self.src, group=self.group)
        dist.broadcast(v, self.src, group=self.group)
        return k[:, :, self.g0:self.g1].contiguous(), v[:, :, self.g0:self.g1].contiguous()

    def forward(self, q_local, k, v, out_local, lse_local=None, stream=None):
        k_loc, v_loc = self.broadcast_kv(k, v)
        self._kv = (k_loc, v_loc)
        return self.layer.forward(q_local, k_loc, v_loc, out_local, lse_local, stream)

    def backward(self, q_local, out_local, lse_local, dout_local, dq_local, dk, dv, stream=None):
        """Gradients of the last forward, its selection held fixed.  dq_local
        [b, N, h1-h0, d] receives this rank's query heads' dq.  dk, dv
        [b, N, hkv, d] receive, on the source rank, the gradients of the
        broadcast K and V: the adjoint of the broadcast sums every rank's
        contribution (its kv heads' gradients from its query heads) there,
        summed in at least fp32; elsewhere they are left as they were."""
        k_loc, v_loc = self._kv
        dk_loc, dv_loc = torch.empty_like(k_loc), torch.empty_like(v_loc)
        self.layer.backward(q_local, k_loc, v_loc, out_local, lse_local, dout_local, dq_local, dk_loc, dv_loc,
                            stream)
        # the sum runs in at least fp32 (bf16 partials would round at every add)
        acc_dtype = torch.promote_types(dk_loc.dtype, torch.float32)
        for full, part in ((dk, dk_loc), (dv, dv_loc)):
            acc = torch.zeros(full.shape, dtype=acc_dtype, device=full.device)
            acc[:, :, self.g0:self.g1] = part
            dist.reduce(acc, self.src, op=dist.ReduceOp.SUM, group=self.group)
            if self.rank == self.src:
                full.copy_(acc)
        return dq_local, dk, dv
