"""bench.py's FLOP accounting against the oracle's pinned closed form and
against brute-force counts of attended keys: the plain layer's pairs for
every named workload, and the routed-pair count of the pooled-gate variant
(which must reduce to the plain count when every row routes min(k-1, c)
earlier blocks)."""
import os
import sys

import numpy as np
import pytest

import moba_synth as S
import oracle as O
from oracle import moba_pooled_gate as P

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


@pytest.mark.parametrize("name", sorted(S.CONFIGS))
def test_plain_pairs_match_the_oracle_closed_form(name):
    cfg = S.get_config(name)
    assert bench.algorithmic_pairs(cfg) == O.algorithmic_pairs(cfg.batch, cfg.seqlen, cfg.hq, cfg.block,
                                                               cfg.topk)


@pytest.mark.parametrize("name", sorted(S.CONFIGS))
def test_routed_flops_of_the_plain_gate_equal_the_layer_flops(name):
    cfg = S.get_config(name)
    t = np.arange(cfg.seqlen, dtype=np.int64)
    rows = int(np.minimum(cfg.topk - 1, t // cfg.block).sum()) * cfg.batch * cfg.hq
    assert bench.routed_flops(cfg, rows) == bench.attn_flops(cfg)


def test_routed_flops_of_the_pooled_gate_count_its_attended_keys():
    cfg = S.get_config("tiny").replace(seqlen=230, hq=2, hkv=1, block=24, topk=3)
    q, k, v = (x.double().numpy() for x in (S.gen_q(cfg), S.gen_k(cfg), S.gen_v(cfg)))
    _, _, sels = P.moba_pooled_layer(q, k, v, cfg.block, cfg.topk, 2, cfg.softmax_scale)
    keys = sum(len(O.key_positions(sel, t, cfg.block, cfg.seqlen)) for (_, t, _), sel in sels.items())
    routed = sum(len(sel) - 1 for sel in sels.values())
    assert bench.routed_flops(cfg, routed) == 4.0 * cfg.head_dim * keys


def test_pooled_cpu_baseline_runs_the_pooled_oracle_on_sampled_rows():
    cfg = S.get_config("mqar").replace(batch=1, seqlen=2048, hq=4, hkv=2)
    d = bench.cpu_baseline_pooled(cfg, 1, budget_s=0.5)
    assert d["kind"] == "oracle" and d["cores"] >= 1
    assert d["extrapolated_full_layer_s"] > 0 and d["sample_tflops"] > 0
    assert "pooled-gate oracle" in d["sample"]
