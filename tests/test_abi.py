"""The C-ABI library loads, exports every symbol include/moba.h declares, and
validates its arguments on the host (no compute call needs a GPU here)."""
import ctypes
import os
import re

import pytest

import long_context_prefill_moba_b200 as M
from long_context_prefill_moba_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moba.h")


@pytest.fixture(scope="module")
def L():
    B.build()
    return M.load_library()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MOBA_API\s+[\w\s\*]*?\b(moba_\w+)\s*\(", text)))


def test_header_declares_the_binding_symbols():
    assert declared_symbols() == sorted(M.EXPORTED_SYMBOLS)


def test_every_declared_symbol_is_exported(L):
    for name in declared_symbols():
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value


def test_no_other_symbols_are_exported(L):
    out = os.popen(f"nm -D --defined-only {M.LIB_PATH}").read()
    ours = sorted({ln.split()[-1] for ln in out.splitlines() if " T " in ln and "moba" in ln})
    assert ours == declared_symbols()


def shape(**kw):
    base = dict(batch=1, seqlen=1 << 20, hq=32, hkv=8, head_dim=128, block=4096, topk=12,
                dtype="bf16", scale=None, query_chunk=0)
    base.update(kw)
    return M.make_shape(**base)


def test_sizes_of_the_1m_layer(L):
    s = shape()
    assert M.moba_check_shape(s) == 0
    assert M.moba_num_blocks(s) == 256
    C = M.moba_query_chunk(s)
    # the largest power of two whose bf16 partials (256 B + a 4-B lse each) fit 8 GiB
    assert C % 128 == 0 and C * 32 * 11 * (128 * 2 + 4) <= 8 << 30 < 2 * C * 32 * 11 * (128 * 2 + 4)
    assert C == 65536
    assert M.moba_num_chunks(s) == (1 << 20) // C
    assert M.moba_sel_elems(s) == (1 << 20) * 32 * 12
    assert M.moba_meank_elems(s) == 256 * 8 * 128
    assert M.moba_offsets_elems(s) == M.moba_num_chunks(s) * 8 * 256 + 1
    # rows: sum_t min(11, t // 4096) per head
    exact = sum(min(11, c) * 4096 for c in range(256)) * 32
    assert M.moba_rows_elems(s) == exact
    assert M.moba_attn_workspace_size(s) >= C * 32 * 11 * (128 * 2 + 4)     # bf16 partials + fp32 lse
    f = shape(dtype="f32")
    Cf = M.moba_query_chunk(f)
    assert M.moba_attn_workspace_size(f) >= Cf * 32 * 11 * 129 * 4
    assert Cf * 32 * 11 * 129 * 4 <= 8 << 30 < 2 * Cf * 32 * 11 * 129 * 4
    assert M.moba_gate_workspace_size(s) >= 2 * 4 * M.moba_num_chunks(s) * 8 * 256


def test_largest_block_count_accepted(L):
    s = shape(seqlen=65535 * 16, hq=1, hkv=1, block=16, topk=2)
    assert M.moba_check_shape(s) == 0 and M.moba_num_blocks(s) == 65535
    assert M.moba_check_shape(shape(seqlen=65535 * 16 + 1, hq=1, hkv=1, block=16, topk=2)) == 2


def test_rows_count_ragged_and_small(L):
    s = shape(batch=2, seqlen=1000, hq=4, hkv=2, block=96, topk=3)
    exact = sum(min(2, t // 96) for t in range(1000)) * 2 * 4
    assert M.moba_rows_elems(s) == exact
    s1 = shape(batch=1, seqlen=100, hq=2, hkv=1, block=128, topk=4)
    assert M.moba_rows_elems(s1) == 0 and M.moba_num_blocks(s1) == 1


@pytest.mark.parametrize("kw,status", [
    (dict(batch=0), 1), (dict(seqlen=0), 1), (dict(hq=6, hkv=4), 1), (dict(block=0), 1),
    (dict(topk=0), 1), (dict(dtype="f32", head_dim=96), 2), (dict(topk=17), 2),
    (dict(query_chunk=100), 1), (dict(scale=float("nan")), 1),
    (dict(batch=64, seqlen=1 << 20, hq=64), 2),
    (dict(seqlen=1 << 20, hq=1, hkv=1, block=8), 2),      # 131072 blocks: more than a grid axis holds
])
def test_invalid_shapes_rejected(L, kw, status):
    s = shape(**kw)
    assert M.moba_check_shape(s) == status
    assert M.moba_num_blocks(s) == -1
    assert M.moba_attn_workspace_size(s) == 0


def test_entry_points_validate_before_launching(L):
    s = shape(seqlen=4096, block=256)
    fake = ctypes.c_void_p(1 << 20)          # never dereferenced: validation fails first
    odd = ctypes.c_void_p((1 << 20) + 2)
    P = ctypes.byref(s)
    # null / misaligned pointers
    assert L.moba_block_meanpool(P, None, fake, None) == 1
    assert L.moba_block_meanpool(P, odd, fake, None) == 1
    # workspace too small
    assert L.moba_gate_topk(P, fake, fake, fake, fake, fake, fake, 16, None) == 3
    assert L.moba_attn_fwd(P, fake, fake, fake, fake, fake, fake, fake, None, fake, 16, None) == 3
    # bad shape
    bad = shape(hq=5, hkv=2)
    assert L.moba_attn_fwd(ctypes.byref(bad), fake, fake, fake, fake, fake, fake, fake, None, fake,
                           1 << 40, None) == 1
    assert L.moba_gate_topk(None, fake, fake, fake, fake, fake, fake, 1 << 40, None) == 1
    assert L.moba_last_launch_count() == 0


def test_backward_and_host_entry_points_validate_before_launching(L):
    s = shape(seqlen=4096, block=256)
    fake = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 2)
    P = ctypes.byref(s)
    big = 1 << 40
    # moba_attn_bwd(shape, q, k, v, out, dout, lse, sel, offsets, rows, dq, dk, dv, ws, ws_bytes, stream)
    args = [fake] * 13
    assert L.moba_attn_bwd(P, *args[:12], fake, 16, None) == 3                  # workspace too small
    nul = list(args)
    nul[4] = None                                                                # dout missing
    assert L.moba_attn_bwd(P, *nul[:12], fake, big, None) == 1
    mis = list(args)
    mis[9] = odd                                                                 # dq misaligned
    assert L.moba_attn_bwd(P, *mis[:12], fake, big, None) == 1
    bad = shape(hq=5, hkv=2)
    assert L.moba_attn_bwd(ctypes.byref(bad), *args[:12], fake, big, None) == 1
    # moba_prefill_host(shape, q, k, v, out, lse, status, ws, ws_bytes, stream)
    assert L.moba_prefill_host(P, fake, fake, fake, fake, None, None, fake, 16, None) == 3
    assert L.moba_prefill_host(P, None, fake, fake, fake, None, None, fake, big, None) == 1
    assert L.moba_prefill_host(P, fake, fake, fake, fake, None, None, odd, big, None) == 1
    assert L.moba_last_launch_count() == 0


def test_backward_and_host_workspace_sizes(L):
    s = shape()                                   # the 1M bf16 layer: tensor-core backward
    n_q = (1 << 20) * 32 * 128
    n_k = (1 << 20) * 8 * 128
    assert M.moba_attn_bwd_workspace_size(s) >= n_q * 4 + (1 << 20) * 32 * 4   # dq accumulator + delta
    f = shape(seqlen=4096, block=256, dtype="f32", head_dim=64)
    assert 0 < M.moba_attn_bwd_workspace_size(f) < 4096 * 32 * 64 * 4      # no dq accumulator
    no_lse = M.moba_prefill_host_workspace_size(s, False)
    with_lse = M.moba_prefill_host_workspace_size(s, True)
    assert no_lse >= 2 * (n_q + n_k) * 2 + M.moba_attn_workspace_size(s) + M.moba_gate_workspace_size(s)
    assert with_lse - no_lse >= (1 << 20) * 32 * 4 - 256      # an empty region still takes 256 B
    assert M.moba_prefill_host_workspace_size(shape(hq=5, hkv=2), False) == 0


def test_status_strings(L):
    for st in range(7):
        assert M.moba_status_string(st).startswith("MOBA_")
    assert "unknown" in M.moba_status_string(99)


def test_library_missing_fails_loudly(tmp_path):
    saved = M._lib
    try:
        M._lib = None
        with pytest.raises(RuntimeError, match="no CPU fallback"):
            M.load_library(str(tmp_path / "libmoba.so"))
    finally:
        M._lib = saved


def test_pooled_gate_wide_shape_sizes_and_validation(L):
    s = shape(batch=1, seqlen=4096, hq=4, hkv=2, block=256, topk=4)
    w = M.moba_pooled_wide_shape(s, 2)
    assert w.topk == 8
    assert [getattr(w, f) for f, _ in M.MobaShape._fields_ if f != "topk"] == \
        [getattr(s, f) for f, _ in M.MobaShape._fields_ if f != "topk"]
    assert M.moba_pooled_wide_shape(s, 0).topk == 4
    # rows: an upper bound, every row with at most min(W - 1, c) earlier blocks
    assert M.moba_rows_elems(w) == sum(min(7, t // 256) for t in range(4096)) * 4
    assert M.moba_sel_elems(w) == 4096 * 4 * 8
    for extra, status in ((-1, 1), (7, 2)):                  # 4 + 2 * 7 > MOBA_MAX_TOPK
        with pytest.raises(M.MobaError) as e:
            M.moba_pooled_wide_shape(s, extra)
        assert e.value.status == status
    assert M.moba_pooled_wide_shape(shape(topk=16), 0).topk == 16

    fake = ctypes.c_void_p(1 << 20)          # never dereferenced: validation fails first
    odd = ctypes.c_void_p((1 << 20) + 2)
    P = ctypes.byref(s)
    big = 1 << 40
    assert L.moba_block_maxminpool(P, fake, None, fake, None) == 1
    assert L.moba_block_maxminpool(P, fake, fake, odd, None) == 1
    # moba_gate_pooled(shape, extra, q, meank, maxk, mink, sel, offsets, rows, ws, ws_bytes, stream)
    assert L.moba_gate_pooled(P, 2, *[fake] * 8, 16, None) == 3
    assert L.moba_gate_pooled(P, 2, *[fake] * 8, M.moba_gate_workspace_size(w) - 1, None) == 3
    assert L.moba_gate_pooled(P, -1, *[fake] * 8, big, None) == 1
    assert L.moba_gate_pooled(P, 7, *[fake] * 8, big, None) == 2
    assert L.moba_gate_pooled(P, 2, fake, fake, None, fake, fake, fake, fake, fake, big, None) == 1
    # moba_attn_fwd_pooled(shape, extra, q, k, v, sel, offsets, rows, out, lse, ws, ws_bytes, stream)
    assert L.moba_attn_fwd_pooled(P, 2, *[fake] * 7, None, fake, 16, None) == 3
    assert L.moba_attn_fwd_pooled(P, 2, *[fake] * 7, None, fake, M.moba_attn_workspace_size(w) - 1,
                                  None) == 3
    assert L.moba_attn_fwd_pooled(P, 2, fake, fake, odd, *[fake] * 4, None, fake, big, None) == 1
    assert L.moba_attn_fwd_pooled(P, 9, *[fake] * 7, None, fake, big, None) == 2
    assert L.moba_last_launch_count() == 0
    # the attention workspace of the variant holds W - 1 partial slots per row
    assert M.moba_attn_workspace_size(w) > M.moba_attn_workspace_size(s)


def test_one_allocation_workspace_and_rows_capacity(L):
    for s in (shape(), shape(dtype="f32", head_dim=64, seqlen=4096, block=256),
              shape(batch=2, seqlen=1000, hq=4, hkv=2, block=96, topk=3)):
        g, a = M.moba_gate_workspace_size(s), M.moba_attn_workspace_size(s)
        assert M.moba_workspace_size(s) == g + a and g % 256 == 0 and a % 256 == 0
        assert M.moba_rows_capacity(s) == M.moba_rows_elems(s)
    w = M.moba_pooled_wide_shape(shape(seqlen=4096, block=256, topk=4), 3)
    assert M.moba_rows_capacity(w) == sum(min(9, t // 256) for t in range(4096)) * 32
    bad = shape(hq=5, hkv=2)
    assert M.moba_workspace_size(bad) == 0 and M.moba_rows_capacity(bad) == -1


def test_check_index_validates_before_launching(L):
    s = shape(seqlen=4096, block=256)
    fake = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 2)
    P = ctypes.byref(s)
    # moba_check_index(shape, exact, sel, offsets, rows, status, stream)
    assert L.moba_check_index(P, 1, None, fake, fake, fake, None) == 1
    assert L.moba_check_index(P, 1, fake, fake, fake, None, None) == 1
    assert L.moba_check_index(P, 1, fake, fake, None, fake, None) == 1     # rows needed: 4096 tokens
    assert L.moba_check_index(P, 1, fake, odd, fake, fake, None) == 1
    assert L.moba_check_index(ctypes.byref(shape(hq=5, hkv=2)), 1, fake, fake, fake, fake, None) == 1
    assert L.moba_last_launch_count() == 0
