"""The seeded input generator: deterministic, regenerable by row range, and
shaped like the workloads (N(0,1) entries, per-block key offsets)."""
import numpy as np
import pytest
import torch

import moba_synth as S


def test_configs_match_workload_shapes():
    c = S.get_config("1m")
    assert (c.batch, c.seqlen, c.hq, c.hkv, c.head_dim, c.block, c.topk, c.dtype) == \
        (1, 1 << 20, 32, 8, 128, 4096, 12, "bf16")
    assert c.nblocks == 256 and c.group == 4
    assert S.get_config("10m").nblocks == 256
    assert S.get_config("tiny").dtype == "f32" and S.get_config("tiny").head_dim == 64
    assert S.get_config("mqar").topk == 4 and S.get_config("mqar").hq == 16


def test_row_regeneration_matches_full_tensors():
    cfg = S.get_config("mqar").replace(batch=2, seqlen=300, block=64)
    q, k, v = S.gen_q(cfg), S.gen_k(cfg), S.gen_v(cfg)
    assert torch.equal(S.gen_rows(cfg, "q", 1, 17, 250, 9), q[1, 17:250, 9])
    assert torch.equal(S.gen_rows(cfg, "k", 0, 0, 300, 15), k[0, :, 15])
    assert torch.equal(S.gen_rows(cfg, "v", 1, 299, 300, 0), v[1, 299:300, 0])
    assert torch.equal(S.gen_head_rows(cfg, "k", 1, 4), k[1, :, 4])


def test_deterministic_and_seed_dependent():
    cfg = S.get_config("tiny")
    assert torch.equal(S.gen_q(cfg), S.gen_q(cfg))
    assert not torch.equal(S.gen_q(cfg), S.gen_q(cfg.replace(seed=1)))
    assert not torch.equal(S.gen_q(cfg)[0, :, 0], S.gen_v(cfg)[0, :, 0])


def test_distribution_and_offsets():
    cfg = S.get_config("mqar").replace(batch=1, seqlen=4096, block=256)
    q = S.gen_q(cfg).float()
    assert abs(q.mean().item()) < 0.01 and abs(q.std().item() - 1.0) < 0.01
    k = S.gen_k(cfg).float()
    # keys = N(0,1) + 0.5 * N(0,1) per-block offset: variance 1.25
    assert abs(k.var().item() - 1.25) < 0.05
    # within a block the offset is shared: block-mean spread ~ 0.5
    kb = k[0].view(16, 256, 16, 128).mean(dim=1)
    assert 0.4 < kb.std().item() < 0.6
    # values carry no offset
    v = S.gen_v(cfg).float()
    assert abs(v.var().item() - 1.0) < 0.02


def test_normal_table_quantiles():
    t = S.normal_table()
    assert t.shape == (65536,) and t.dtype == torch.float32
    assert torch.all(t[1:] > t[:-1])
    assert torch.allclose(t, -t.flip(0))
    assert abs(t.double().mean().item()) < 1e-9 and abs(t.double().var().item() - 1.0) < 1e-3


def test_bf16_rounding_is_single_rne():
    cfg = S.get_config("mqar").replace(batch=1, seqlen=64, block=16)
    k32 = S.gen_k(cfg.replace(dtype="f32"))
    k16 = S.gen_k(cfg)
    assert torch.equal(k32.to(torch.bfloat16), k16)
