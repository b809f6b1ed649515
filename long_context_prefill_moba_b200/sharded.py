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

Exchange.  Each rank receives only the kv heads it reads:
  - disjoint kv heads (hkv % P == 0): one scatter of K and one of V from the
    source rank, rank r receiving [:, :, its kv heads]; the backward gathers
    the ranks' dK/dV slices onto the source rank (no sum: the slices are
    disjoint and final);
  - shared kv heads: the ranks of one kv head form a subgroup whose first rank
    leads it.  The source sends each leader its kv head's K/V slice, and each
    subgroup broadcasts the slice from its leader (with one kv head, as in the
    10M layer, this is the pages' single broadcast of K and V).  The backward
    sums the subgroup's dK/dV contributions onto the leader in at least fp32
    (the adjoint of that broadcast) and the leaders send the sums to the source.
With the gloo backend (CPU collectives) CUDA tensors are staged through host
memory.  The compute runs in the library's kernels (``MobaLayer``);
``layer_factory`` exists so the host logic can be exercised on ranks without
a GPU.  When a CUDA ``stream`` is given, every copy, collective and kernel of
a call is ordered on it.
"""
from __future__ import annotations

import contextlib
from typing import Callable, List, Optional, Tuple

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


class _Comm:
    """Collectives of one group; with gloo, CUDA tensors go through host copies."""

    def __init__(self, group):
        self.group = group
        self.stage = dist.get_backend(group) == dist.Backend.GLOO

    def host(self, t: torch.Tensor) -> torch.Tensor:
        return t.cpu() if self.stage and t.is_cuda else t

    @staticmethod
    def land(dst: torch.Tensor, src: torch.Tensor):
        if src is not dst:
            dst.copy_(src)

    def scatter(self, out: torch.Tensor, parts: Optional[List[torch.Tensor]], src: int):
        h = self.host(out)
        dist.scatter(h, [self.host(p) for p in parts] if parts is not None else None, src=src,
                     group=self.group)
        self.land(out, h)

    def gather(self, t: torch.Tensor, parts: Optional[List[torch.Tensor]], dst: int):
        hp = [self.host(p) for p in parts] if parts is not None else None
        dist.gather(self.host(t), hp, dst=dst, group=self.group)
        if parts is not None:
            for p, q in zip(parts, hp):
                self.land(p, q)

    def broadcast(self, t: torch.Tensor, src: int, group=None):
        h = self.host(t)
        dist.broadcast(h, src, group=group if group is not None else self.group)
        self.land(t, h)

    def reduce(self, t: torch.Tensor, dst: int, group):
        h = self.host(t)
        dist.reduce(h, dst, op=dist.ReduceOp.SUM, group=group)
        self.land(t, h)

    def send(self, t: torch.Tensor, dst: int):
        dist.send(self.host(t), dst)

    def recv(self, t: torch.Tensor, src: int):
        h = self.host(t)
        dist.recv(h, src)
        self.land(t, h)


class ShardedMobaLayer:
    """One MoBA layer shape whose heads are split over the ranks of `group`.

    ``forward(q_local, k, v, out_local, lse_local=None)``: `q_local` /
    `out_local` [b, N, h1-h0, d] hold this rank's query heads; `k` and `v`
    [b, N, hkv, d] hold the layer's full K/V on the source rank (`src`, a
    global rank) and are ignored elsewhere (pass None or any tensor)."""

    def __init__(self, batch, seqlen, hq, hkv, head_dim, block, topk, dtype="bf16", scale=None,
                 query_chunk=0, device="cuda", group=None, src: int = 0,
                 layer_factory: Optional[Callable] = None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.src = src
        self.dims = (batch, seqlen, hq, hkv, head_dim)
        self.h0, self.h1, self.g0, self.g1 = head_shard(hq, hkv, self.world, self.rank)
        self.comm = _Comm(group)
        self.glob = [dist.get_global_rank(group, r) if group is not None else r for r in range(self.world)]
        self.shards = [head_shard(hq, hkv, self.world, r) for r in range(self.world)]
        self.disjoint = hkv % self.world == 0
        if not self.disjoint:
            # one subgroup per kv head, created by every rank in the same order
            split = self.world // hkv
            self.leaders = [self.glob[g * split] for g in range(hkv)]
            self.subgroups = [dist.new_group([self.glob[g * split + i] for i in range(split)])
                              for g in range(hkv)]
            self.sub = self.subgroups[self.g0]
            self.leader = self.leaders[self.g0]
        if layer_factory is None:
            from . import MobaLayer
            layer_factory = MobaLayer
        # a query head keeps its kv head: local head i reads local kv head i // G_local
        self.layer = layer_factory(batch, seqlen, self.h1 - self.h0, self.g1 - self.g0, head_dim, block,
                                   topk, dtype, scale, query_chunk, device)
        self.device = torch.device(device)

    @classmethod
    def from_config(cls, cfg, device="cuda", query_chunk=0, group=None, src=0, layer_factory=None):
        return cls(cfg.batch, cfg.seqlen, cfg.hq, cfg.hkv, cfg.head_dim, cfg.block, cfg.topk, cfg.dtype,
                   cfg.scale, query_chunk, device, group, src, layer_factory)

    @property
    def me(self) -> int:
        return self.glob[self.rank]

    def _on(self, stream):
        if stream is not None and self.device.type == "cuda":
            return torch.cuda.stream(stream)
        return contextlib.nullcontext()

    def _local_kv(self, like: torch.Tensor):
        b, N, _, _, d = self.dims
        return torch.empty(b, N, self.g1 - self.g0, d, dtype=like.dtype, device=self.device)

    def exchange_kv(self, k: Optional[torch.Tensor], v: Optional[torch.Tensor], dtype):
        """This rank's kv heads of the source rank's K and V (see the module
        docstring for the exchange)."""
        like = torch.empty(0, dtype=dtype)
        out = []
        for full in (k, v):
            loc = self._local_kv(like)
            if self.disjoint:
                parts = None
                if self.me == self.src:
                    parts = [full[:, :, s[2]:s[3]].contiguous() for s in self.shards]
                self.comm.scatter(loc, parts, self.src)
            else:
                if self.me == self.src:
                    for g, lead in enumerate(self.leaders):
                        if lead != self.src:
                            self.comm.send(full[:, :, g:g + 1].contiguous(), lead)
                    if self.me == self.leader:
                        loc.copy_(full[:, :, self.g0:self.g1])
                elif self.me == self.leader:
                    self.comm.recv(loc, self.src)
                self.comm.broadcast(loc, self.leader, group=self.sub)
            out.append(loc)
        return out[0], out[1]

    def forward(self, q_local, k, v, out_local, lse_local=None, stream=None):
        with self._on(stream):
            k_loc, v_loc = self.exchange_kv(k, v, q_local.dtype)
            self._kv = (k_loc, v_loc)
            return self.layer.forward(q_local, k_loc, v_loc, out_local, lse_local)

    def backward(self, q_local, out_local, lse_local, dout_local, dq_local, dk, dv, stream=None):
        """Gradients of the last forward, its selection held fixed.  dq_local
        [b, N, h1-h0, d] receives this rank's query heads' dq.  dk, dv
        [b, N, hkv, d] receive, on the source rank, the gradients of the source
        rank's K and V: the adjoint of the exchange, which gathers disjoint kv
        heads and sums (in at least fp32) the contributions of the ranks that
        share a kv head; elsewhere they are left as they were."""
        with self._on(stream):
            k_loc, v_loc = self._kv
            if stream is not None and self.device.type == "cuda":
                for t in (k_loc, v_loc):
                    t.record_stream(stream)
            dk_loc, dv_loc = torch.empty_like(k_loc), torch.empty_like(v_loc)
            self.layer.backward(q_local, k_loc, v_loc, out_local, lse_local, dout_local, dq_local, dk_loc,
                                dv_loc)
            if self.disjoint:
                for full, part in ((dk, dk_loc), (dv, dv_loc)):
                    parts = None
                    if self.me == self.src:
                        parts = [torch.empty_like(part) for _ in range(self.world)]
                    self.comm.gather(part, parts, self.src)
                    if parts is not None:
                        for s, p in zip(self.shards, parts):
                            full[:, :, s[2]:s[3]] = p
                return dq_local, dk, dv
            # the sum runs in at least fp32 (bf16 partial sums would round at every add)
            acc_dtype = torch.promote_types(dk_loc.dtype, torch.float32)
            sums = [part.to(acc_dtype) for part in (dk_loc, dv_loc)]
            for acc in sums:
                self.comm.reduce(acc, self.leader, self.sub)
            if self.me == self.leader and self.me != self.src:
                for acc in sums:
                    self.comm.send(acc, self.src)
            if self.me == self.src:
                if self.me == self.leader:
                    for full, acc in zip((dk, dv), sums):
                        full[:, :, self.g0:self.g1] = acc.to(full.dtype)
                for g, lead in enumerate(self.leaders):
                    if lead == self.src:
                        continue
                    for full in (dk, dv):
                        buf = torch.empty_like(sums[0])
                        self.comm.recv(buf, lead)
                        full[:, :, g:g + 1] = buf.to(full.dtype)
            return dq_local, dk, dv
