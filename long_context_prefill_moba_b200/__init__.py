"""MoBA (Mixture of Block Attention) causal prefill on NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI in ``include/moba.h`` (``libmoba.so``, built
in-tree by ``long_context_prefill_moba_b200.build``).  Every step of the
computation runs in the library's CUDA kernels; this module only marshals
torch tensors (device memory and the current CUDA stream) into the C calls.
There is no CPU fallback: if the library is missing, importing the functions
raises.

Functions with the names of the C entry points:

    moba_block_meanpool(shape, k, meank)
    moba_gate_topk(shape, q, meank, sel, offsets, rows, ws)
    moba_attn_fwd(shape, q, k, v, sel, offsets, rows, out, lse, ws)

plus ``MobaLayer`` (owns the intermediate buffers of one shape and runs the
three steps) and ``moba_forward`` (allocating convenience call), the backward
(``moba_attn_bwd``, ``moba_attention``), the host-buffer layer
(``moba_prefill_host``, ``MobaHostLayer``) and the gate variant with max- and
min-pooled keys (``moba_block_maxminpool``, ``moba_gate_pooled``,
``moba_attn_fwd_pooled``, ``MobaPooledLayer``, ``moba_forward_pooled``).
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

__all__ = [
    "MobaShape", "MobaError", "lib", "load_library", "make_shape", "moba_check_shape",
    "moba_num_blocks", "moba_query_chunk", "moba_num_chunks", "moba_meank_elems",
    "moba_sel_elems", "moba_offsets_elems", "moba_rows_elems", "moba_gate_workspace_size",
    "moba_attn_workspace_size", "moba_block_meanpool", "moba_gate_topk", "moba_attn_fwd",
    "moba_status_string", "moba_last_launch_count", "moba_gate_topk_noalloc",
    "moba_gate_noalloc_status", "MobaLayer", "moba_forward",
    "moba_prefill_host_workspace_size", "moba_prefill_host", "MobaHostLayer",
    "moba_attn_bwd_workspace_size", "moba_attn_bwd", "moba_attention",
    "moba_pooled_wide_shape", "moba_block_maxminpool", "moba_gate_pooled", "moba_attn_fwd_pooled",
    "MobaPooledLayer", "moba_forward_pooled", "moba_workspace_size", "moba_rows_capacity",
    "moba_check_index", "MOBA_BF16", "MOBA_F32", "EXPORTED_SYMBOLS",
]

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoba.so")

MOBA_BF16, MOBA_F32 = 0, 1
MOBA_OK = 0

EXPORTED_SYMBOLS = [
    "moba_check_shape", "moba_num_blocks", "moba_query_chunk", "moba_num_chunks",
    "moba_meank_elems", "moba_sel_elems", "moba_offsets_elems", "moba_rows_elems",
    "moba_gate_workspace_size", "moba_attn_workspace_size", "moba_block_meanpool",
    "moba_gate_topk", "moba_attn_fwd", "moba_status_string", "moba_last_cuda_error",
    "moba_last_launch_count", "moba_gate_topk_noalloc", "moba_gate_noalloc_status",
    "moba_selftest_bounded_wait",
    "moba_prefill_host_workspace_size", "moba_prefill_host", "moba_attn_bwd_workspace_size",
    "moba_attn_bwd", "moba_pooled_wide_shape", "moba_block_maxminpool", "moba_gate_pooled",
    "moba_attn_fwd_pooled", "moba_workspace_size", "moba_rows_capacity", "moba_check_index",
]


class MobaShape(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("seqlen", ctypes.c_int32), ("hq", ctypes.c_int32),
        ("hkv", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("block", ctypes.c_int32),
        ("topk", ctypes.c_int32), ("dtype", ctypes.c_int32), ("scale", ctypes.c_float),
        ("query_chunk", ctypes.c_int32),
    ]

    def __repr__(self):
        return "MobaShape(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


class MobaError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = lib().moba_status_string(status).decode()
        if status == 4:
            msg += f" (cudaError {lib().moba_last_cuda_error()})"
        super().__init__(f"{where}: {msg}")
        self.status = status


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libmoba.so and declare its signatures (raises if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m long_context_prefill_moba_b200.build` (no CPU fallback exists)")
    L = ctypes.CDLL(path)
    P = ctypes.POINTER(MobaShape)
    vp, i64, sz, st = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
    for name in ("moba_num_blocks", "moba_query_chunk", "moba_num_chunks", "moba_meank_elems",
                 "moba_sel_elems", "moba_offsets_elems", "moba_rows_elems", "moba_rows_capacity"):
        getattr(L, name).argtypes = [P]
        getattr(L, name).restype = i64
    for name in ("moba_gate_workspace_size", "moba_attn_workspace_size", "moba_workspace_size"):
        getattr(L, name).argtypes = [P]
        getattr(L, name).restype = sz
    L.moba_check_shape.argtypes = [P]
    L.moba_check_shape.restype = st
    L.moba_block_meanpool.argtypes = [P, vp, vp, vp]
    L.moba_block_meanpool.restype = st
    L.moba_gate_topk.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moba_gate_topk.restype = st
    L.moba_attn_fwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moba_attn_fwd.restype = st
    L.moba_selftest_bounded_wait.argtypes = [vp, vp]
    L.moba_selftest_bounded_wait.restype = st
    L.moba_gate_topk_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp]
    L.moba_gate_topk_noalloc.restype = st
    L.moba_gate_noalloc_status.argtypes = [vp, vp]
    L.moba_gate_noalloc_status.restype = st
    L.moba_attn_bwd_workspace_size.argtypes = [P]
    L.moba_attn_bwd_workspace_size.restype = sz
    L.moba_attn_bwd.argtypes = [P] + [vp] * 13 + [sz, vp]
    L.moba_attn_bwd.restype = st
    L.moba_prefill_host_workspace_size.argtypes = [P, st]
    L.moba_prefill_host_workspace_size.restype = sz
    L.moba_prefill_host.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moba_prefill_host.restype = st
    i32 = ctypes.c_int32
    L.moba_pooled_wide_shape.argtypes = [P, i32, P]
    L.moba_pooled_wide_shape.restype = st
    L.moba_block_maxminpool.argtypes = [P, vp, vp, vp, vp]
    L.moba_block_maxminpool.restype = st
    L.moba_gate_pooled.argtypes = [P, i32] + [vp] * 8 + [sz, vp]
    L.moba_gate_pooled.restype = st
    L.moba_attn_fwd_pooled.argtypes = [P, i32] + [vp] * 9 + [sz, vp]
    L.moba_attn_fwd_pooled.restype = st
    L.moba_check_index.argtypes = [P, i32, vp, vp, vp, vp, vp]
    L.moba_check_index.restype = st
    L.moba_status_string.argtypes = [st]
    L.moba_status_string.restype = ctypes.c_char_p
    L.moba_last_cuda_error.argtypes = []
    L.moba_last_cuda_error.restype = st
    L.moba_last_launch_count.argtypes = []
    L.moba_last_launch_count.restype = st
    _lib = L
    return L


def lib():
    return load_library()


def make_shape(batch, seqlen, hq, hkv, head_dim, block, topk, dtype="bf16", scale=None,
               query_chunk=0) -> MobaShape:
    dt = {"bf16": MOBA_BF16, torch.bfloat16: MOBA_BF16, "f32": MOBA_F32, torch.float32: MOBA_F32}[dtype]
    return MobaShape(batch, seqlen, hq, hkv, head_dim, block, topk, dt,
                     0.0 if scale is None else float(scale), query_chunk)


def _s(shape):
    return ctypes.byref(shape)


def moba_check_shape(shape) -> int: return lib().moba_check_shape(_s(shape))
def moba_num_blocks(shape) -> int: return lib().moba_num_blocks(_s(shape))
def moba_query_chunk(shape) -> int: return lib().moba_query_chunk(_s(shape))
def moba_num_chunks(shape) -> int: return lib().moba_num_chunks(_s(shape))
def moba_meank_elems(shape) -> int: return lib().moba_meank_elems(_s(shape))
def moba_sel_elems(shape) -> int: return lib().moba_sel_elems(_s(shape))
def moba_offsets_elems(shape) -> int: return lib().moba_offsets_elems(_s(shape))
def moba_rows_elems(shape) -> int: return lib().moba_rows_elems(_s(shape))
def moba_gate_workspace_size(shape) -> int: return lib().moba_gate_workspace_size(_s(shape))
def moba_attn_workspace_size(shape) -> int: return lib().moba_attn_workspace_size(_s(shape))
def moba_workspace_size(shape) -> int: return lib().moba_workspace_size(_s(shape))
def moba_rows_capacity(shape) -> int: return lib().moba_rows_capacity(_s(shape))
def moba_status_string(status: int) -> str: return lib().moba_status_string(status).decode()
def moba_last_launch_count() -> int: return lib().moba_last_launch_count()


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to the MoBA library must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status: int, where: str):
    if status != MOBA_OK:
        raise MobaError(status, where)


def moba_block_meanpool(shape, k, meank, stream=None):
    _check(lib().moba_block_meanpool(_s(shape), _ptr(k), _ptr(meank), _stream(stream)),
           "moba_block_meanpool")


def moba_gate_topk(shape, q, meank, sel, offsets, rows, ws, stream=None):
    _check(lib().moba_gate_topk(_s(shape), _ptr(q), _ptr(meank), _ptr(sel), _ptr(offsets), _ptr(rows),
                                _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "moba_gate_topk")


def moba_gate_topk_noalloc(shape, q, meank, sel, offsets, rows, stream=None):
    """moba_gate_topk without caller scratch: the counters live in a fixed
    device array inside the library (for callers that cannot give the library
    device scratch memory).  Calls on one device must not overlap on the GPU."""
    _check(lib().moba_gate_topk_noalloc(_s(shape), _ptr(q), _ptr(meank), _ptr(sel), _ptr(offsets),
                                        _ptr(rows), _stream(stream)),
           "moba_gate_topk_noalloc")


def moba_gate_noalloc_status(stream=None) -> int:
    """Device status word of the last moba_gate_topk_noalloc call on the current
    device (0, or MOBA_ERR_TIMEOUT = 6); synchronises `stream`."""
    word = ctypes.c_int(-1)
    st = stream if stream is not None else torch.cuda.current_stream()
    _check(lib().moba_gate_noalloc_status(ctypes.byref(word), _stream(st)), "moba_gate_noalloc_status")
    st.synchronize()
    return int(word.value)


def moba_selftest_bounded_wait(status, stream=None):
    """Run the bounded-wait self-test kernel; `status` is a 1-element int32 CUDA tensor."""
    _check(lib().moba_selftest_bounded_wait(_ptr(status), _stream(stream)), "moba_selftest_bounded_wait")


def moba_attn_fwd(shape, q, k, v, sel, offsets, rows, out, lse, ws, stream=None):
    _check(lib().moba_attn_fwd(_s(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(sel), _ptr(offsets),
                               _ptr(rows), _ptr(out), _ptr(lse), _ptr(ws),
                               ws.numel() * ws.element_size(), _stream(stream)),
           "moba_attn_fwd")


def moba_prefill_host_workspace_size(shape, with_lse=False) -> int:
    return lib().moba_prefill_host_workspace_size(_s(shape), 1 if with_lse else 0)


def moba_prefill_host(shape, q, k, v, out, lse, status, ws, stream=None):
    """One layer from host tensors (q, k, v, out, lse: CPU, contiguous; page-locked
    for the copies to overlap the computation); `status` a 2-element CPU int32
    tensor or None; `ws` a CUDA byte tensor of moba_prefill_host_workspace_size."""
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out), ("lse", lse), ("status", status)):
        if t is not None and t.device.type != "cpu":
            raise ValueError(f"moba_prefill_host: {name} must be a host tensor")
    if ws.device.type != "cuda":
        raise ValueError("moba_prefill_host: ws must be device memory")
    _check(lib().moba_prefill_host(_s(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                   _ptr(status), _ptr(ws), ws.numel() * ws.element_size(),
                                   _stream(stream)),
           "moba_prefill_host")


def moba_attn_bwd_workspace_size(shape) -> int:
    return lib().moba_attn_bwd_workspace_size(_s(shape))


def moba_attn_bwd(shape, q, k, v, out, dout, lse, sel, offsets, rows, dq, dk, dv, ws, stream=None):
    _check(lib().moba_attn_bwd(_s(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse),
                               _ptr(sel), _ptr(offsets), _ptr(rows), _ptr(dq), _ptr(dk), _ptr(dv),
                               _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "moba_attn_bwd")


def moba_pooled_wide_shape(shape, extra) -> MobaShape:
    """The shape that sizes the pooled-gate variant's buffers: topk + 2 * extra."""
    wide = MobaShape()
    _check(lib().moba_pooled_wide_shape(_s(shape), int(extra), _s(wide)), "moba_pooled_wide_shape")
    return wide


def moba_block_maxminpool(shape, k, maxk, mink, stream=None):
    _check(lib().moba_block_maxminpool(_s(shape), _ptr(k), _ptr(maxk), _ptr(mink), _stream(stream)),
           "moba_block_maxminpool")


def moba_gate_pooled(shape, extra, q, meank, maxk, mink, sel, offsets, rows, ws, stream=None):
    _check(lib().moba_gate_pooled(_s(shape), int(extra), _ptr(q), _ptr(meank), _ptr(maxk), _ptr(mink),
                                  _ptr(sel), _ptr(offsets), _ptr(rows), _ptr(ws),
                                  ws.numel() * ws.element_size(), _stream(stream)),
           "moba_gate_pooled")


def moba_attn_fwd_pooled(shape, extra, q, k, v, sel, offsets, rows, out, lse, ws, stream=None):
    _check(lib().moba_attn_fwd_pooled(_s(shape), int(extra), _ptr(q), _ptr(k), _ptr(v), _ptr(sel),
                                      _ptr(offsets), _ptr(rows), _ptr(out), _ptr(lse), _ptr(ws),
                                      ws.numel() * ws.element_size(), _stream(stream)),
           "moba_attn_fwd_pooled")


def moba_check_index(shape, exact, sel, offsets, rows, status, stream=None):
    """Validate sel/offsets/rows on the device; `status` a 1-element int32 CUDA
    tensor that becomes 0, or MOBA_ERR_INTERNAL (5) with the index made inert."""
    _check(lib().moba_check_index(_s(shape), 1 if exact else 0, _ptr(sel), _ptr(offsets), _ptr(rows),
                                  _ptr(status), _stream(stream)),
           "moba_check_index")


class MobaHostLayer:
    """One MoBA layer shape served from host buffers (moba_prefill_host): the
    device workspace is allocated once; ``forward`` enqueues the copies and the
    three steps with the copies overlapped, on the current stream."""

    def __init__(self, batch, seqlen, hq, hkv, head_dim, block, topk, dtype="bf16", scale=None,
                 query_chunk=0, device="cuda", with_lse=False):
        self.shape = make_shape(batch, seqlen, hq, hkv, head_dim, block, topk, dtype, scale,
                                query_chunk)
        _check(moba_check_shape(self.shape), "MobaHostLayer")
        self.device = torch.device(device)
        self.with_lse = with_lse
        self.ws = torch.empty(moba_prefill_host_workspace_size(self.shape, with_lse), dtype=torch.uint8,
                              device=self.device)
        self.status = torch.zeros(2, dtype=torch.int32, pin_memory=True)
        self.launches = 0

    @classmethod
    def from_config(cls, cfg, device="cuda", query_chunk=0, with_lse=False):
        return cls(cfg.batch, cfg.seqlen, cfg.hq, cfg.hkv, cfg.head_dim, cfg.block, cfg.topk,
                   cfg.dtype, cfg.scale, query_chunk, device, with_lse)

    def forward(self, q, k, v, out, lse=None, stream=None):
        if lse is not None and not self.with_lse:
            raise ValueError("MobaHostLayer: built without an lse output")
        moba_prefill_host(self.shape, q, k, v, out, lse, self.status, self.ws, stream)
        self.launches = moba_last_launch_count()
        return out

    def device_status(self):
        """(gate, attention) status words of the last forward (synchronises)."""
        torch.cuda.synchronize(self.device)
        return int(self.status[0]), int(self.status[1])


class MobaLayer:
    """Buffers of one MoBA layer shape on one device, and the three steps.

    ``forward(q, k, v, out, lse=None)`` enqueues mean-pool, gate and attention
    on the current stream.  Intermediate results stay readable afterwards:
    ``meank``, ``sel``, ``offsets``, ``rows``."""

    def __init__(self, batch, seqlen, hq, hkv, head_dim, block, topk, dtype="bf16", scale=None,
                 query_chunk=0, device="cuda"):
        self.shape = make_shape(batch, seqlen, hq, hkv, head_dim, block, topk, dtype, scale,
                                query_chunk)
        _check(moba_check_shape(self.shape), "MobaLayer")
        dev = torch.device(device)
        self.device = dev
        i32 = torch.int32
        self.meank = torch.empty(moba_meank_elems(self.shape), dtype=torch.float32, device=dev)
        self.sel = torch.empty(moba_sel_elems(self.shape), dtype=i32, device=dev)
        self.offsets = torch.empty(moba_offsets_elems(self.shape), dtype=i32, device=dev)
        self.rows = torch.empty(max(1, moba_rows_elems(self.shape)), dtype=i32, device=dev)
        self.gate_ws = torch.empty(moba_gate_workspace_size(self.shape), dtype=torch.uint8, device=dev)
        self.attn_ws = torch.empty(moba_attn_workspace_size(self.shape), dtype=torch.uint8, device=dev)
        self.launches = 0

    @classmethod
    def from_config(cls, cfg, device="cuda", query_chunk=0):
        return cls(cfg.batch, cfg.seqlen, cfg.hq, cfg.hkv, cfg.head_dim, cfg.block, cfg.topk,
                   cfg.dtype, cfg.scale, query_chunk, device)

    def forward(self, q, k, v, out, lse=None, stream=None):
        s = self.shape
        moba_block_meanpool(s, k, self.meank, stream)
        n = moba_last_launch_count()
        moba_gate_topk(s, q, self.meank, self.sel, self.offsets, self.rows, self.gate_ws, stream)
        n += moba_last_launch_count()
        moba_attn_fwd(s, q, k, v, self.sel, self.offsets, self.rows, out, lse, self.attn_ws, stream)
        n += moba_last_launch_count()
        self.launches = n
        return out

    def backward(self, q, k, v, out, lse, dout, dq, dk, dv, stream=None):
        """dq, dk, dv of the last forward's attention given dout (the gate's
        selection, sel/offsets/rows of that forward, is held fixed); `out` and
        `lse` are that forward's outputs."""
        if getattr(self, "bwd_ws", None) is None:
            self.bwd_ws = torch.empty(moba_attn_bwd_workspace_size(self.shape), dtype=torch.uint8,
                                      device=self.device)
        moba_attn_bwd(self.shape, q, k, v, out, dout, lse, self.sel, self.offsets, self.rows, dq, dk, dv,
                      self.bwd_ws, stream)
        self.launches = moba_last_launch_count()
        return dq, dk, dv

    def device_status(self):
        """(gate, attention) device status words of the last forward (synchronises):
        0, or MOBA_ERR_TIMEOUT (6) if a bounded wait in a tensor-core kernel expired."""
        torch.cuda.synchronize(self.device)
        g = self.gate_ws[-256:-252].view(torch.int32).item()
        a = self.attn_ws[:4].view(torch.int32).item()
        return g, a

    def sel_view(self):
        s = self.shape
        return self.sel.view(s.batch, s.seqlen, s.hq, s.topk)

    def meank_view(self):
        s = self.shape
        return self.meank.view(s.batch, moba_num_blocks(s), s.hkv, s.head_dim)


class MobaPooledLayer:
    """Buffers of one layer shape for the gate variant that also routes the top
    `extra` blocks by max- and by min-pooled keys, and its four steps:
    mean-pool, max/min-pool, the three-ranking gate and the attention.  Buffers
    sized by the wide shape (topk + 2 * extra); ``rows`` holds an upper bound
    of entries, of which the gate fills ``offsets[-1]``."""

    def __init__(self, batch, seqlen, hq, hkv, head_dim, block, topk, extra, dtype="bf16", scale=None,
                 query_chunk=0, device="cuda"):
        self.shape = make_shape(batch, seqlen, hq, hkv, head_dim, block, topk, dtype, scale, query_chunk)
        self.extra = int(extra)
        self.wide = moba_pooled_wide_shape(self.shape, self.extra)
        dev = torch.device(device)
        self.device = dev
        i32, f32 = torch.int32, torch.float32
        w = self.wide
        self.meank = torch.empty(moba_meank_elems(w), dtype=f32, device=dev)
        self.maxk = torch.empty_like(self.meank)
        self.mink = torch.empty_like(self.meank)
        self.sel = torch.empty(moba_sel_elems(w), dtype=i32, device=dev)
        self.offsets = torch.empty(moba_offsets_elems(w), dtype=i32, device=dev)
        self.rows = torch.empty(max(1, moba_rows_elems(w)), dtype=i32, device=dev)
        self.gate_ws = torch.empty(moba_gate_workspace_size(w), dtype=torch.uint8, device=dev)
        self.attn_ws = torch.empty(moba_attn_workspace_size(w), dtype=torch.uint8, device=dev)
        self.launches = 0

    @classmethod
    def from_config(cls, cfg, extra, device="cuda", query_chunk=0):
        return cls(cfg.batch, cfg.seqlen, cfg.hq, cfg.hkv, cfg.head_dim, cfg.block, cfg.topk, extra,
                   cfg.dtype, cfg.scale, query_chunk, device)

    def forward(self, q, k, v, out, lse=None, stream=None):
        s, x = self.shape, self.extra
        moba_block_meanpool(s, k, self.meank, stream)
        n = moba_last_launch_count()
        moba_block_maxminpool(s, k, self.maxk, self.mink, stream)
        n += moba_last_launch_count()
        moba_gate_pooled(s, x, q, self.meank, self.maxk, self.mink, self.sel, self.offsets, self.rows,
                         self.gate_ws, stream)
        n += moba_last_launch_count()
        moba_attn_fwd_pooled(s, x, q, k, v, self.sel, self.offsets, self.rows, out, lse, self.attn_ws,
                             stream)
        n += moba_last_launch_count()
        self.launches = n
        return out

    def backward(self, q, k, v, out, lse, dout, dq, dk, dv, stream=None):
        """dq, dk, dv of the last forward's attention given dout, its selection
        held fixed: moba_attn_bwd at the wide shape (its kernels read the
        variable-length selections through sel, offsets and rows)."""
        if getattr(self, "bwd_ws", None) is None:
            self.bwd_ws = torch.empty(moba_attn_bwd_workspace_size(self.wide), dtype=torch.uint8,
                                      device=self.device)
        moba_attn_bwd(self.wide, q, k, v, out, dout, lse, self.sel, self.offsets, self.rows, dq, dk, dv,
                      self.bwd_ws, stream)
        self.launches = moba_last_launch_count()
        return dq, dk, dv

    def device_status(self):
        torch.cuda.synchronize(self.device)
        g = self.gate_ws[-256:-252].view(torch.int32).item()
        a = self.attn_ws[:4].view(torch.int32).item()
        return g, a

    def sel_view(self):
        w = self.wide
        return self.sel.view(w.batch, w.seqlen, w.hq, w.topk)

    def pool_views(self):
        s = self.shape
        shp = (s.batch, moba_num_blocks(s), s.hkv, s.head_dim)
        return self.meank.view(shp), self.maxk.view(shp), self.mink.view(shp)


def moba_forward_pooled(q, k, v, block, topk, extra, scale=None, return_lse=False, query_chunk=0):
    """out (and lse) of one layer with the pooled-gate variant."""
    b, N, hq, d = q.shape
    layer = MobaPooledLayer(b, N, hq, k.shape[2], d, block, topk, extra, q.dtype, scale, query_chunk,
                            q.device)
    out = torch.empty_like(q)
    lse = torch.empty(b, hq, N, dtype=torch.float32, device=q.device) if return_lse else None
    layer.forward(q, k, v, out, lse)
    return (out, lse) if return_lse else out


def moba_forward(q, k, v, block, topk, scale=None, return_lse=False, query_chunk=0):
    """out (and lse) of one MoBA layer; q [b,N,Hq,d], k/v [b,N,Hkv,d] CUDA tensors."""
    b, N, hq, d = q.shape
    layer = MobaLayer(b, N, hq, k.shape[2], d, block, topk, q.dtype, scale, query_chunk, q.device)
    out = torch.empty_like(q)
    lse = torch.empty(b, hq, N, dtype=torch.float32, device=q.device) if return_lse else None
    layer.forward(q, k, v, out, lse)
    return (out, lse) if return_lse else out


class _MobaAttention(torch.autograd.Function):
    """MoBA attention as a differentiable op: the forward runs the three steps,
    the backward moba_attn_bwd with the forward's selection held fixed."""

    @staticmethod
    def forward(ctx, q, k, v, block, topk, scale, query_chunk):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        b, N, hq, d = q.shape
        layer = MobaLayer(b, N, hq, k.shape[2], d, block, topk, q.dtype, scale, query_chunk, q.device)
        out = torch.empty_like(q)
        lse = torch.empty(b, hq, N, dtype=torch.float32, device=q.device)
        layer.forward(q, k, v, out, lse)
        ctx.layer = layer
        ctx.save_for_backward(q, k, v, out, lse)
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse = ctx.saved_tensors
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ctx.layer.backward(q, k, v, out, lse, dout.contiguous(), dq, dk, dv)
        return dq, dk, dv, None, None, None, None


def moba_attention(q, k, v, block, topk, scale=None, query_chunk=0):
    """Differentiable MoBA attention: q [b,N,Hq,d], k/v [b,N,Hkv,d] CUDA tensors
    -> out [b,N,Hq,d]; gradients flow to q, k, v (not through the block selection)."""
    return _MobaAttention.apply(q, k, v, block, topk, scale, query_chunk)
