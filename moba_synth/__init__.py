"""Seeded synthetic inputs for MoBA causal prefill.

This module is shared by the CPU oracle's tests, the GPU parity tests and the
benchmark.  It holds no arithmetic of the method itself (no pooling, gating or
attention): only workload shapes and a counter-based random generator.

Generator.  Every element is a pure function of (seed, tensor id, flat index):

    u   = mix32(lo32(i) ^ mix32(hi32(i) ^ salt(seed, tensor)))      (32-bit hash)
    z   = NORMAL_TABLE[u >> 16]                                     (fp32)

where ``mix32`` is a 32-bit xor-shift-multiply finaliser and NORMAL_TABLE holds
the 65536 standard-normal quantiles Phi^-1((m + 1/2) / 65536).  All hashing is
integer arithmetic kept below 2^63, the table is built once on the CPU, and the
only floating-point operations after the lookup are one multiply by an exact
power of two and one IEEE add, so the CPU and any CUDA device produce
bit-identical tensors.  Any row range of any tensor can be regenerated alone,
which lets the oracle rebuild exactly the rows it samples at 1M/10M tokens.

Workload (the pages' shapes; the pages' own data are real text and an MQAR
task that are not available, so these synthetic tensors stand in for them):

    q[b,t,h,:] ~ q_std * N(0,1)                          (q_std = 1 unless stated)
    k[b,t,g,:] ~ N(0,1) + offset_std * o[b, t // B, g, :],   o ~ N(0,1)
    v[b,t,g,:] ~ N(0,1)

The per-block key offset o makes the mean-pooled keys of different blocks
differ, as the configs ask.  q_std and offset_std are powers of two, so the
scalings are exact; q_std = 8 with offset_std = 4 gives gate scores q.meanK in
the hundreds (std ~360), the magnitude of unscaled scores in trained models.  Values are drawn in fp32 and rounded once (RNE)
to the config's dtype.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

__all__ = [
    "MobaConfig", "CONFIGS", "get_config", "normal_table",
    "gen_q", "gen_k", "gen_v", "gen_dout", "gen_rows", "TENSOR_Q", "TENSOR_K", "TENSOR_V", "TENSOR_OFF",
    "TENSOR_DOUT",
]

TENSOR_Q, TENSOR_K, TENSOR_V, TENSOR_OFF, TENSOR_DOUT = 1, 2, 3, 4, 5
_M32 = 0xFFFFFFFF
_MUL = 0x45D9F3B          # < 2^27, so (x < 2^32) * _MUL < 2^59: no int64 overflow
_CHUNK = 1 << 25          # elements per generation chunk (bounds int64 temporaries)


@dataclasses.dataclass(frozen=True)
class MobaConfig:
    name: str
    batch: int
    seqlen: int
    hq: int
    hkv: int
    head_dim: int
    block: int
    topk: int               # counts the always-selected current block
    dtype: str              # "bf16" | "f32"
    offset_std: float
    seed: int = 0
    scale: Optional[float] = None   # None -> 1/sqrt(d)
    q_std: float = 1.0              # q = q_std * N(0,1); a power of two (exact)

    def __post_init__(self):
        for name in ("q_std", "offset_std"):
            m, _ = math.frexp(getattr(self, name))
            if m != 0.5:
                raise ValueError(f"{name} must be a power of two (exact scaling)")

    @property
    def nblocks(self) -> int:
        return (self.seqlen + self.block - 1) // self.block

    @property
    def group(self) -> int:
        return self.hq // self.hkv

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.head_dim)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def replace(self, **kw) -> "MobaConfig":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    # tiny parity case: fp32, one head, d=64
    "tiny": MobaConfig("tiny", 1, 2048, 1, 1, 64, 256, 3, "f32", 1.0),
    # MQAR-shaped layer (16 MHA heads, N=2048, B=256, top-4)
    "mqar": MobaConfig("mqar", 8, 2048, 16, 16, 128, 256, 4, "bf16", 0.5),
    # Llama-3.1-8B-shaped layer at 128K tokens
    "llama8b_128k": MobaConfig("llama8b_128k", 1, 131072, 32, 8, 128, 4096, 12, "bf16", 0.5),
    # the 1M-token prefill layer (95.31% block sparsity)
    "1m": MobaConfig("1m", 1, 1048576, 32, 8, 128, 4096, 12, "bf16", 0.5),
    # 10M tokens at constant sparsity (256 blocks of 40960)
    "10m": MobaConfig("10m", 1, 10485760, 4, 1, 128, 40960, 12, "bf16", 0.5),
}


def get_config(name: str) -> MobaConfig:
    return CONFIGS[name]


_TABLE_CACHE: dict = {}


def normal_table(device="cpu") -> torch.Tensor:
    """65536 standard-normal quantiles at the cell midpoints, fp32."""
    key = str(device)
    if key not in _TABLE_CACHE:
        if "cpu" not in _TABLE_CACHE:
            p = (torch.arange(65536, dtype=torch.float64) + 0.5) / 65536.0
            _TABLE_CACHE["cpu"] = torch.special.ndtri(p).to(torch.float32)
        _TABLE_CACHE[key] = _TABLE_CACHE["cpu"].to(device)
    return _TABLE_CACHE[key]


def _mix32_int(x: int) -> int:
    x &= _M32
    x = (((x >> 16) ^ x) * _MUL) & _M32
    x = (((x >> 16) ^ x) * _MUL) & _M32
    return ((x >> 16) ^ x) & _M32


def _mix32(x: torch.Tensor) -> torch.Tensor:
    x = torch.bitwise_and(torch.bitwise_xor(x >> 16, x) * _MUL, _M32)
    x = torch.bitwise_and(torch.bitwise_xor(x >> 16, x) * _MUL, _M32)
    return torch.bitwise_xor(x >> 16, x)


def _salt(seed: int, tensor: int) -> int:
    return _mix32_int((seed * 0x2545F491) ^ _mix32_int(tensor * 0x9E3779B1))


def _normals_at(idx: torch.Tensor, seed: int, tensor: int) -> torch.Tensor:
    """N(0,1) draws (fp32) for int64 flat indices ``idx`` of one tensor."""
    salt = _salt(seed, tensor)
    hi = _mix32(torch.bitwise_xor(idx >> 32, salt))
    u = _mix32(torch.bitwise_xor(torch.bitwise_and(idx, _M32), hi))
    return normal_table(idx.device)[u >> 16]


def _flat_normals(start: int, count: int, seed: int, tensor: int, device) -> torch.Tensor:
    out = torch.empty(count, dtype=torch.float32, device=device)
    for c0 in range(0, count, _CHUNK):
        c1 = min(count, c0 + _CHUNK)
        idx = torch.arange(start + c0, start + c1, dtype=torch.int64, device=device)
        out[c0:c1] = _normals_at(idx, seed, tensor)
    return out


def _finish(x: torch.Tensor, cfg: MobaConfig) -> torch.Tensor:
    return x.to(cfg.torch_dtype)


def gen_q(cfg: MobaConfig, device="cpu") -> torch.Tensor:
    """q as [batch, seqlen, hq, head_dim] in the config dtype."""
    n = cfg.batch * cfg.seqlen * cfg.hq * cfg.head_dim
    x = _flat_normals(0, n, cfg.seed, TENSOR_Q, device)
    if cfg.q_std != 1.0:
        x = x * cfg.q_std
    return _finish(x, cfg).view(cfg.batch, cfg.seqlen, cfg.hq, cfg.head_dim)


def gen_v(cfg: MobaConfig, device="cpu") -> torch.Tensor:
    """v as [batch, seqlen, hkv, head_dim] in the config dtype."""
    n = cfg.batch * cfg.seqlen * cfg.hkv * cfg.head_dim
    x = _flat_normals(0, n, cfg.seed, TENSOR_V, device)
    return _finish(x, cfg).view(cfg.batch, cfg.seqlen, cfg.hkv, cfg.head_dim)


def gen_dout(cfg: MobaConfig, device="cpu") -> torch.Tensor:
    """An upstream gradient dL/d(out), [batch, seqlen, hq, head_dim] in the
    config dtype: standard normals of its own stream."""
    n = cfg.batch * cfg.seqlen * cfg.hq * cfg.head_dim
    x = _flat_normals(0, n, cfg.seed, TENSOR_DOUT, device)
    return _finish(x, cfg).view(cfg.batch, cfg.seqlen, cfg.hq, cfg.head_dim)


def _key_offsets(cfg: MobaConfig, device) -> torch.Tensor:
    n = cfg.batch * cfg.nblocks * cfg.hkv * cfg.head_dim
    o = _flat_normals(0, n, cfg.seed, TENSOR_OFF, device)
    return o.view(cfg.batch, cfg.nblocks, cfg.hkv, cfg.head_dim)


def gen_k(cfg: MobaConfig, device="cpu") -> torch.Tensor:
    """k as [batch, seqlen, hkv, head_dim] in the config dtype (with per-block offsets)."""
    out = torch.empty(cfg.batch, cfg.seqlen, cfg.hkv, cfg.head_dim, dtype=cfg.torch_dtype, device=device)
    off = _key_offsets(cfg, device) * cfg.offset_std   # offset_std is 1 or 0.5: exact
    rows_per_chunk = max(1, _CHUNK // (cfg.hkv * cfg.head_dim))
    row_elems = cfg.hkv * cfg.head_dim
    for b in range(cfg.batch):
        for t0 in range(0, cfg.seqlen, rows_per_chunk):
            t1 = min(cfg.seqlen, t0 + rows_per_chunk)
            start = (b * cfg.seqlen + t0) * row_elems
            z = _flat_normals(start, (t1 - t0) * row_elems, cfg.seed, TENSOR_K, device)
            z = z.view(t1 - t0, cfg.hkv, cfg.head_dim)
            blk = torch.arange(t0, t1, device=device) // cfg.block
            out[b, t0:t1] = _finish(z + off[b, blk], cfg)
    return out


def gen_rows(cfg: MobaConfig, tensor: str, b: int, t0: int, t1: int, head: int,
             device="cpu") -> torch.Tensor:
    """Rows [t0, t1) of one head of one batch entry of q, k or v: [t1-t0, head_dim].

    Bit-identical to the same slice of gen_q / gen_k / gen_v, but touches only
    the requested rows (used by the oracle to regenerate sampled rows of the
    1M and 10M workloads)."""
    d = cfg.head_dim
    t = torch.arange(t0, t1, dtype=torch.int64, device=device)
    e = torch.arange(d, dtype=torch.int64, device=device)
    if tensor == "q":
        idx = (((b * cfg.seqlen + t) * cfg.hq + head) * d)[:, None] + e[None, :]
        x = _normals_at(idx.reshape(-1), cfg.seed, TENSOR_Q).view(t1 - t0, d)
        if cfg.q_std != 1.0:
            x = x * cfg.q_std
    elif tensor == "v":
        idx = (((b * cfg.seqlen + t) * cfg.hkv + head) * d)[:, None] + e[None, :]
        x = _normals_at(idx.reshape(-1), cfg.seed, TENSOR_V).view(t1 - t0, d)
    elif tensor == "k":
        idx = (((b * cfg.seqlen + t) * cfg.hkv + head) * d)[:, None] + e[None, :]
        z = _normals_at(idx.reshape(-1), cfg.seed, TENSOR_K).view(t1 - t0, d)
        blk = t // cfg.block
        oidx = (((b * cfg.nblocks + blk) * cfg.hkv + head) * d)[:, None] + e[None, :]
        o = _normals_at(oidx.reshape(-1), cfg.seed, TENSOR_OFF).view(t1 - t0, d)
        x = z + o * cfg.offset_std
    else:
        raise ValueError(tensor)
    return _finish(x, cfg)


def gen_head_rows(cfg: MobaConfig, tensor: str, b: int, head: int, t0: int = 0,
                  t1: Optional[int] = None, device="cpu") -> torch.Tensor:
    """Like gen_rows but chunked over t so that long ranges stay within memory."""
    t1 = cfg.seqlen if t1 is None else t1
    out = torch.empty(t1 - t0, cfg.head_dim, dtype=cfg.torch_dtype, device=device)
    step = max(1, _CHUNK // cfg.head_dim)
    for a in range(t0, t1, step):
        z = min(t1, a + step)
        out[a - t0:z - t0] = gen_rows(cfg, tensor, b, a, z, head, device)
    return out
